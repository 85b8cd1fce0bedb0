// Internal declarations shared by the host API and the kernels of libs2o.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "s2o.h"

namespace s2o {

// Derived sizes of one configuration.
struct Dims {
  int batch, Hq, Hkv, G, N, D, S, B, nB, nSeg;
  long long bhq() const { return (long long)batch * Hq; }
  long long bhkv() const { return (long long)batch * Hkv; }
};

Dims dims_of(const s2o_config &c);

// Byte offsets of the scratch arrays inside a workspace (256-byte aligned).
struct WsLayout {
  size_t qchunk, kchunk, qbar, kbar_all, kbar_top, u, kappa, rho, keys0, keys1, radix, Qbar, Kbar, r,
      ncount, flags, total;
};

WsLayout ws_layout(const Dims &d);

// Index build (s2o_index.cu). All launches on `st`; returns the first launch error.
cudaError_t launch_build_indices(const Dims &d, const s2o_config &cfg, const uint16_t *q,
                                 const uint16_t *k, const s2o_indices &out, char *ws,
                                 cudaStream_t st);
cudaError_t launch_validate(const Dims &d, const s2o_indices &idx, char *ws, uint32_t *flag_dev,
                            cudaStream_t st);
cudaError_t launch_stats(const Dims &d, const s2o_indices &idx, unsigned long long *acc_dev,
                         cudaStream_t st);
cudaError_t launch_exp64_probe(const double *x, double *y, int n, cudaStream_t st);

// Attention (s2o_attn.cu).
struct AttnArgs {
  const void *q, *k, *v;
  void *o;
  const int32_t *perm_q, *perm_k, *sel_cnt, *sel_blk, *local_tiles;
  bool dense;
  // Merge path (a workspace of s2o_prefill_workspace_size bytes): the permuted pass runs only
  // the selected blocks and writes each row's partial result and its log2-sum-exp into lse
  // [bhq, N]; the local pass then merges. Without it (merge false) the permuted pass reruns each
  // busy block's local tiles and overwrites its rows.
  bool merge = false;
  float *lse = nullptr;
  // Optional permuted copy of K and V for packed streams: row rank of copy head h at h·N + rank
  // holds the key/value row pos_sorted[h·N + rank], the keys of each block of perm_k in position
  // order. Copy heads are query heads, or KV heads when copy_per_kv is set (one key ordering per
  // KV head). Used when *copy_flag has bit 0 set; copy_flag == nullptr means no copy.
  const void *kp = nullptr, *vp = nullptr;
  const uint32_t *copy_flag = nullptr;
  bool copy_per_kv = false;
  int32_t *pos_sorted = nullptr;  // [copy heads, N]
  uint8_t *vis = nullptr;         // [copy heads, nSeg, nB] visible keys of each block per segment
  uint32_t *chunks = nullptr;     // [pairs, chunk_cap] chunk words of the packed streams
  int4 *pair_meta = nullptr;      // [pairs] tile counts {shared, unit 0 only, unit 1 only, -}
  long long chunk_cap = 0;
  // Measured-share early stop (a labelled variant, path without a workspace only): the permuted
  // pass stops a query block's list after the first block whose share of every row's running
  // normaliser is below stop_tau, and writes the listed blocks each busy query block kept.
  int32_t *stop_cnt = nullptr;
  float stop_tau = 0.f;
};
cudaError_t launch_attention(const Dims &d, const AttnArgs &a, uint64_t wait_limit_ns,
                             int max_ctas, cudaStream_t st);
// The path of a call with a workspace: a decision kernel writes *flag (bit 1 the merge path, bit 0
// packed streams from the permuted copy; see k_copy_decide for the rules per mode); then (each
// doing nothing when bit 0 is clear) the blocks of perm_k are put in position order (a.pos_sorted,
// a.vis), K and V are copied in that order (a.kp, a.vp), and each pair of units gets its chunk
// list (a.chunks, a.pair_meta).
cudaError_t launch_permuted_copy(const Dims &d, const AttnArgs &a, int mode, uint32_t *flag,
                                 cudaStream_t st);
// acc[0] += tiles the packed streams of the last call loaded, acc[1] += their tile products
// (nothing when *flag's bit 0 is clear).
cudaError_t launch_packed_counts(const Dims &d, const int4 *pair_meta, const uint32_t *flag,
                                 unsigned long long *acc, cudaStream_t st);
// acc[0] += Σ over query blocks with a selection of (local tiles + selected blocks), acc[1] += Σ
// selected blocks.
cudaError_t launch_busy_tiles(const Dims &d, const int32_t *sel_cnt, const int32_t *local_tiles,
                              unsigned long long *acc, cudaStream_t st);

// bf16 GEMM on the tensor cores (s2o_gemm.cu): row-major C[m, n] = A[m, k]·B[k, n] (+ C when
// `accumulate`), fp32 accumulation, one rounding to bf16; n and k multiples of 8 (16-byte rows).
cudaError_t launch_gemm_bf16(const void *A, const void *B, void *C, long long m, long long n,
                             long long k, bool accumulate, uint64_t limit_ns, cudaStream_t st);
cudaError_t read_and_clear_gemm_error(unsigned int *out, cudaStream_t st);

// Decoder layer (s2o_layer.cu): byte offsets of its buffers in the layer workspace (the attention's
// own workspace starts at attn_ws), and the launches before and after the attention.
struct LayerWs {
  size_t h, qkv, q, k, v, o, o_rows, gu, a, freqs, cs, perm_q, perm_k, sel_cnt, sel_blk,
      local_tiles, attn_ws;
};
LayerWs layer_ws_layout(const Dims &d, const s2o_layer_config &lc);
cudaError_t launch_layer_pre(const Dims &d, const s2o_layer_config &lc,
                             const s2o_layer_weights &w, const void *x, char *ws,
                             const LayerWs &L, uint64_t wait_limit_ns, cudaStream_t st);
cudaError_t launch_layer_post(const Dims &d, const s2o_layer_config &lc,
                              const s2o_layer_weights &w, void *x, char *ws, const LayerWs &L,
                              uint64_t wait_limit_ns, cudaStream_t st);

// Host-side count of kernel launches made by the library (all threads, all devices).
void note_launch();
unsigned long long launch_count();

// Device error record (bit 0: a bounded wait ran out).
cudaError_t read_and_clear_device_error(unsigned int *out, cudaStream_t st);

}  // namespace s2o
