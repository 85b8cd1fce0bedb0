/*
 * s2o.h — C ABI of libs2o: permuted, importance-ordered, early-stopped block-sparse causal
 * attention prefill (S2O) on one NVIDIA B200 (sm_100a).
 *
 * What the library computes is defined step by step in the project's definition file; each entry
 * point below names the passages of the pages it implements:
 *   [S2O]  "S2O: Early Stopping for Sparse Attention via Online Permutation" (research card),
 *          Summary ¶2 and Key points.
 *   [PBS]  "Sparser Block-Sparse Attention via Token Permutation" (ICML poster), lay summary.
 *   [AB]   "AB-Sparse", Eq. (1) and the Figure 2 workflow text.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors are bf16, contiguous, BHND: Q and O [batch, Hq, N, d]; K and V [batch, Hkv, N, d].
 *    Query head h reads key/value head h / (Hq/Hkv).
 *  - Tensor, index-array and workspace pointers are DEVICE pointers owned by the caller, 16-byte
 *    aligned. The structs passed by pointer (s2o_config, s2o_indices, s2o_layer_config,
 *    s2o_layer_weights) and the outputs s2o_stats, s2o_work_counts, s2o_workspace_view and the
 *    size outputs live in HOST memory (s2o_indices, s2o_layer_weights and s2o_workspace_view hold
 *    device pointers). The library never allocates device memory: scratch comes from the
 *    caller's workspace `ws` (size from s2o_workspace_size), except in
 *    s2o_build_indices_static.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream). Launching calls are
 *    asynchronous on it; argument errors are returned before anything is enqueued, and device
 *    faults surface at the caller's next synchronisation (CUDA convention).
 *  - Supported shapes: d ∈ {64, 128}; B ∈ {64, 128}; Hq % Hkv == 0; N % S == 0; S % B == 0;
 *    N/B ≤ 2048; batch·Hq·N < 2^31; 0 ≤ tau (finite). tau > 1 is legal and selects no permuted block (local window only).
 *    Anything else returns S2O_ERR_UNSUPPORTED.
 *  - Calls on different streams must not share a workspace.
 */
#ifndef S2O_H
#define S2O_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void *s2o_stream; /* a cudaStream_t */

typedef enum {
  S2O_OK = 0,
  S2O_ERR_INVALID_ARGUMENT = 1,    /* null/misaligned pointer, negative or NaN tau, ...    */
  S2O_ERR_UNSUPPORTED = 2,         /* shape outside the supported set above              */
  S2O_ERR_WORKSPACE_TOO_SMALL = 3, /* ws_bytes below s2o_workspace_size                  */
  S2O_ERR_INVALID_INDICES = 4,     /* s2o_validate_indices found a bad index array       */
  S2O_ERR_CUDA = 5,                /* a CUDA runtime call or launch failed               */
  S2O_ERR_DEVICE_TIMEOUT = 6       /* a kernel gave up a bounded wait (see below)        */
} s2o_status;

/* One attention layer. `query_perm` = 1 builds the segment-local query ordering; 0 keeps the
 * identity (the "Q perm" ablation of [S2O, Key points]). `shared_key_order` = 0 (the default)
 * builds one key ordering per query head; 1 builds one per KV head, ranked by the group's pooled
 * query, and writes it to the perm_k row of each of the group's query heads (a labelled variant:
 * the pages say "for each head" without saying which kind of head). `int4_centroids` = 1 scores
 * blocks with 4-bit key centroids and an exact integer product (a labelled variant after
 * [AB-Sparse, INT4 centroids]; 0, the default, is the fp32 centroid product). */
typedef struct {
  int batch, n_q_heads, n_kv_heads, seq_len, head_dim, segment_len, block_size;
  float tau;
  int query_perm;
  int shared_key_order;
  int int4_centroids;
} s2o_config;

/* Caller-owned index arrays (device, int32). nB = N / B.
 *  perm_q      [batch, Hq, N]      original query index at each permuted slot; slots
 *                                  [sS, (s+1)S) hold a permutation of segment s.
 *  perm_k      [batch, Hq, N]      original key index at each rank (one ordering per query head;
 *                                  with shared_key_order, each head of a KV group holds the
 *                                  group's ordering).
 *  sel_cnt     [batch, Hq, nB]     number of selected permuted key blocks of each query block.
 *  sel_blk     [batch, Hq, nB, nB] selected key-block ids (blocks of perm_k), most important
 *                                  first; entries at and after sel_cnt are not written.
 *  local_tiles [batch, Hq, nB]     original-order key tiles of the query block's own segment that
 *                                  the kernel runs (1 ≤ lt ≤ S/B). */
typedef struct {
  int32_t *perm_q, *perm_k, *sel_cnt, *sel_blk, *local_tiles;
} s2o_indices;

/* Work and sparsity counts of one index set (host struct, filled by s2o_index_stats). */
typedef struct {
  uint64_t local_tiles;    /* Σ_b lt_b                                                  */
  uint64_t selected_tiles; /* Σ_b cnt_b                                                 */
  uint64_t pairs;          /* Σ_i |K_i|: (query, key) pairs attended                   */
  uint64_t causal_pairs;   /* batch·Hq·N(N+1)/2: pairs of dense causal attention          */
} s2o_stats;

/* Device pointers into a workspace after s2o_build_indices: the intermediate values of the
 * index build (fp32 unless noted), for inspection and tests. Valid until the workspace is reused.
 *  qbar [b,Hq,d]; kbar_all [b,Hkv,d]; kbar_top, u [b,Hq,d]; kappa, rho [b,Hq,N];
 *  Qbar, Kbar [b,Hq,nB,d]; r [b,Hq,nB,nB]; n [b,Hq,nSeg,nB] (int32). */
typedef struct {
  float *qbar, *kbar_all, *kbar_top, *u, *kappa, *rho, *Qbar, *Kbar, *r;
  int32_t *n;
} s2o_workspace_view;

/* Human-readable name of a status. Never NULL. */
const char *s2o_status_string(s2o_status status);

/* Bytes of scratch that s2o_build_indices / s2o_attention_prefill / s2o_validate_indices need
 * for `cfg`, written to *bytes. Host only; no device work. */
s2o_status s2o_workspace_size(const s2o_config *cfg, size_t *bytes);

/* Element counts of the five index arrays of `cfg`, in s2o_indices field order. Host only. */
s2o_status s2o_index_sizes(const s2o_config *cfg, size_t counts[5]);

/* Steps 1–2 of the method ([S2O, Summary ¶2]: stripe-level mean pooling, the global key/value
 * ordering, the segment-local query ordering, block scores and the early stop at tau) for every
 * (batch, query head): writes the index arrays of `out`. Bit-exact with the definition: same
 * inputs give the same indices on every run. q, k: device bf16 as above. The key-side kernels
 * run on a second stream of the calling thread (created on first use, kept for the thread's
 * lifetime), forked from and joined back to `stream` with events, so the call stays ordered on
 * `stream`. */
s2o_status s2o_build_indices(const s2o_config *cfg, const void *q, const void *k,
                             const s2o_indices *out, void *ws, size_t ws_bytes,
                             s2o_stream stream);

/* Pointers to the intermediate values held in `ws` (see s2o_workspace_view). Host only. */
s2o_status s2o_workspace_views(const s2o_config *cfg, void *ws, size_t ws_bytes,
                               s2o_workspace_view *view);

/* The whole hot path ([S2O, Summary ¶2]): s2o_build_indices into `idx`, then the fused
 * gather-attention over local tiles and selected permuted blocks; O [batch, Hq, N, d] bf16 is
 * written at original positions. With ws_bytes >= s2o_prefill_workspace_size it runs the merge
 * path of s2o_attention_prefill_with_indices_ws (packed streams allowed; under shared_key_order
 * one copy per KV head); s2o_workspace_size bytes suffice without it. */
s2o_status s2o_attention_prefill(const s2o_config *cfg, const void *q, const void *k,
                                 const void *v, void *o, const s2o_indices *idx, void *ws,
                                 size_t ws_bytes, s2o_stream stream);

/* Steps 3–4 only, on caller-supplied index arrays ([S2O, Summary ¶2]: the kernel fetches the
 * scattered rows into shared memory by index and runs the blocks in list order; causality is
 * enforced on original positions). Memory-safe for any index contents (out-of-range values are
 * clamped and out-of-range output rows skipped), but the result is only defined for index arrays
 * that s2o_validate_indices accepts. */
s2o_status s2o_attention_prefill_with_indices(const s2o_config *cfg, const void *q,
                                              const void *k, const void *v,
                                              const s2o_indices *idx, void *o,
                                              s2o_stream stream);

/* Steps 3-4 with the measured-share early stop (a labelled variant of the survey's NEXT-2 row;
 * [S2O, Summary ¶2]: blocks run from most to least important and the loop "stops once a block's
 * score falls under a threshold τ", here the block's measured score; [BSFA, abstract]: pruning on
 * exact block scores). Each busy query block runs its local tiles, then its listed blocks in list
 * order; after a listed block that is not the list's last, the block's share of each row's
 * running softmax normaliser (the block's exp-sum over the sum after it) is compared with
 * cfg->tau, and the list stops when the share is below tau for every row of the block (that block
 * is kept). The rows of each query block get the attention over the local window and the kept
 * blocks. stop_cnt [batch, Hq, nB] (device int32, 16-byte aligned, owned by the caller) receives
 * the listed blocks each query block kept (0 for empty lists). tau = 0 never stops. Uses the path
 * without a workspace (local pass, then the permuted pass over list streams). Errors as
 * s2o_attention_prefill_with_indices, plus S2O_ERR_INVALID_ARGUMENT for a null stop_cnt. */
s2o_status s2o_attention_prefill_online_stop(const s2o_config *cfg, const void *q,
                                             const void *k, const void *v,
                                             const s2o_indices *idx, void *o, int32_t *stop_cnt,
                                             s2o_stream stream);

/* Bytes of scratch with which s2o_attention_prefill and s2o_attention_prefill_with_indices_ws run
 * the merge path and may use packed streams (see s2o_set_permuted_copy): s2o_workspace_size, a
 * 256-byte flag area, one fp32 log2-sum-exp per query row (batch · n_q_heads · N), the permuted
 * copy of K and V (2 · batch · n_q_heads · N · d bf16 values; one ordering per KV head uses a
 * quarter of it under GQA of four), the key positions of each key block in position order
 * (batch · n_q_heads · N int32) with their visible counts per segment (batch · n_q_heads · nSeg ·
 * nB bytes), and the packed streams' chunk lists (per pair of query blocks 2·nB·B/16 + 3·B/16
 * int32) and tile counts (16 bytes per pair). Written to *bytes. Host only; no device work. */
s2o_status s2o_prefill_workspace_size(const s2o_config *cfg, size_t *bytes);

/* As s2o_attention_prefill_with_indices, with a workspace. With ws_bytes >=
 * s2o_prefill_workspace_size (the merge path) the permuted pass runs only the selected blocks of
 * each busy query block and leaves each row's partial result and its log2-sum-exp; the local pass
 * then computes the dense local window in original order and merges the two (the attention over
 * the same key set, the fp32 accumulation split in two). When most blocks are selected, a
 * device-side decision may copy K and V into each query head's key order first, each key block's
 * rows in position order, and run packed streams (see s2o_set_permuted_copy). With a smaller
 * workspace this is s2o_attention_prefill_with_indices. ws: device, 16-byte aligned, owned by the
 * caller. */
s2o_status s2o_attention_prefill_with_indices_ws(const s2o_config *cfg, const void *q,
                                                 const void *k, const void *v,
                                                 const s2o_indices *idx, void *o, void *ws,
                                                 size_t ws_bytes, s2o_stream stream);

/* Packed streams ([S2O, Summary ¶2] fetches the scattered tokens of the selected blocks into
 * on-chip memory by index): with the permuted copy of K and V, whose key blocks hold their rows in
 * position order, the keys of block c that a query of segment s may see (position < s·S) are the
 * block's first rows; the permuted pass loads only those, in chunks of 16 rows packed into full
 * tiles, and pairs two query blocks that read one copy head and one segment so that a block both
 * selected is loaded once for both (two consecutive blocks of a query head; two query heads of a
 * KV head at one block under shared_key_order). Only the accumulation order differs from the
 * gathered form.
 * mode 1 (the default): decided on the device without synchronising: the merge path when more
 * than 1/25 of the query blocks have a selection (below that, rerunning their local tiles costs
 * less than the merge), packed streams when the selected blocks of the call outnumber twice the
 * blocks the copy writes (copying a block costs about one gather of it); 0: the merge path with
 * gathered rows (list order), never packed; 2: always packed; 3: the path without a workspace
 * even when one is given (0, 2 and 3 are for tests). Only calls given a workspace of
 * s2o_prefill_workspace_size bytes use modes 0-2. Affects calls made after it; not thread-safe
 * against concurrent calls. Other values are treated as 1. */
void s2o_set_permuted_copy(int mode);

/* Work of the attention's last call on `ws` (merge path only), for reports. */
typedef struct {
  uint64_t local_pass_tiles;      /* tile products of the local pass: every segment's triangle */
  uint64_t permuted_unit_tiles;   /* tile products (query tile × key tile) of the permuted pass */
  uint64_t permuted_loaded_tiles; /* key/value tiles the permuted pass loaded                  */
  int packed;                     /* 1 when it ran packed streams                              */
  int merged;                     /* 1 when it ran the merge path                              */
} s2o_work_counts;

/* Fills *out for the last s2o_attention_prefill / s2o_attention_prefill_with_indices_ws call that
 * used `ws` (ws_bytes >= s2o_prefill_workspace_size) with the index arrays `idx`. Uses `ws`'s
 * small scratch; SYNCHRONISES `stream`. */
s2o_status s2o_attention_work(const s2o_config *cfg, const s2o_indices *idx, void *ws,
                              size_t ws_bytes, s2o_work_counts *out, s2o_stream stream);

/* In-repo dense causal attention baseline, Eq. (1) of [AB], on the same kernel machinery
 * (contiguous tiles, no index arrays). cfg->segment_len, tau and query_perm are ignored. */
s2o_status s2o_dense_causal_prefill(const s2o_config *cfg, const void *q, const void *k,
                                    const void *v, void *o, s2o_stream stream);

/* Checks that perm_q is a segment-local permutation, perm_k a permutation of [0, N), every
 * sel_cnt in [0, nB], every listed block id in [0, nB) and unique within its list, and every
 * local_tiles value in [1, S/B] and covering its block's last query. Uses `ws`; SYNCHRONISES
 * `stream`. Returns S2O_OK or S2O_ERR_INVALID_INDICES. */
s2o_status s2o_validate_indices(const s2o_config *cfg, const s2o_indices *idx, void *ws,
                                size_t ws_bytes, s2o_stream stream);

/* Work and sparsity counts of an index set (definition: pair sparsity = 1 − pairs /
 * causal_pairs). Uses `ws`; SYNCHRONISES `stream`; writes the host struct *stats. */
s2o_status s2o_index_stats(const s2o_config *cfg, const s2o_indices *idx, void *ws,
                           size_t ws_bytes, s2o_stats *stats, s2o_stream stream);

/* Every wait inside the attention kernel and the GEMMs (on a TMA copy, a tensor-core commit, a
 * peer warp or, in the CTA-pair GEMM, the other CTA of the pair) is bounded by this many
 * nanoseconds of GPU time (default 2e9). When a wait runs out, the kernel records it, drains its
 * own copies and tensor-core work, frees its tensor memory and returns.
 * Affects launches made after the call; not thread-safe against concurrent launches. */
void s2o_set_wait_limit_ns(uint64_t ns);

/* Caps the persistent attention grid at `max_ctas` CTAs (0, the default: one CTA per SM). A smaller
 * grid gives each CTA more work items and more work-list windows, which lets small inputs exercise
 * the window turnover; results do not depend on the grid. Affects launches made after the call;
 * not thread-safe against concurrent launches. Negative values are treated as 0. */
void s2o_set_attention_max_ctas(int max_ctas);

/* Number of kernel launches the library has made in this process so far (all threads and
 * devices), for launch accounting. Host only. */
uint64_t s2o_kernel_launch_count(void);

/* Synchronises `stream`, then reports and clears the device error record: S2O_ERR_DEVICE_TIMEOUT
 * if a bounded wait ran out since the last check, S2O_ERR_CUDA if the stream holds an error,
 * else S2O_OK. */
s2o_status s2o_check_device_status(s2o_stream stream);

/* Size of the device scratch array behind s2o_build_indices_static (48 MiB: enough for a
 * 32-query-head, 8-KV-head, 32K-token layer with d = 128 and B = 128). */
#define S2O_STATIC_WORKSPACE_BYTES (48u << 20)

/* s2o_build_indices for callers that cannot allocate device memory (an operator embedded in a
 * host framework that only hands over its inputs and outputs, a serving path that must not call
 * cudaMalloc after start-up). No counterpart on the pages: it is the same index build as
 * s2o_build_indices, but its scratch is a fixed array inside the library
 * (S2O_STATIC_WORKSPACE_BYTES per GPU, held from library load until process exit) instead of a
 * caller workspace. The caller still owns and passes q, k and the index arrays.
 *  - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 *  - Configurations whose s2o_workspace_size exceeds S2O_STATIC_WORKSPACE_BYTES are rejected with
 *    S2O_ERR_WORKSPACE_TOO_SMALL before any device work.
 *  - The first call on each device (with that device current) looks up the array's device address
 *    with cudaGetSymbolAddress and keeps it with the id of the device's context; a call that finds
 *    another context on the device (after cudaDeviceReset, say) looks it up again. The first call
 *    on each host thread also creates the library's side stream and its two events for that
 *    device (as every index build does). Make those first calls before any stream capture or any
 *    region that must not create CUDA resources.
 *  - Every call on a device shares the one array and leaves its contents behind; calls whose GPU
 *    work overlaps (different streams, or different host threads) race on it and must be
 *    serialised by the caller. s2o_workspace_views does not apply to it.
 * Arguments, layouts, results and the other errors are those of s2o_build_indices. */
s2o_status s2o_build_indices_static(const s2o_config *cfg, const void *q, const void *k,
                                    const s2o_indices *out, s2o_stream stream);

/* ---- Decoder layer around the attention (end-to-end-shaped prefill with random weights) ----
 * The pages measure S2O inside Llama-3.1-8B ([S2O, Key points]: end-to-end speedup at 128K);
 * without trained weights this runs one Llama-3-architecture decoder layer with the S2O prefill
 * (or the dense causal baseline) as its attention: x += W_o·attn(RoPE(W_qkv·norm(x))), then
 * x += W_down·(silu(gate)·up) with [gate | up] = W_gu·norm(x). bf16 storage between the steps,
 * fp32 arithmetic; projections are this library's tensor-core GEMM (s2o_gemm_bf16), the rest its
 * other kernels. Heads and sizes come from the s2o_config (hidden H = n_q_heads·head_dim). */
typedef struct {
  int intermediate;            /* MLP width I (multiple of 8)                                   */
  float rms_eps;               /* RMS norm epsilon (1e-5)                                       */
  double rope_theta;           /* rotary base (500000)                                          */
  double rope_factor;          /* Llama 3.1 frequency scaling: factor (8; 0 turns it off)       */
  double rope_low_freq_factor; /* (1)                                                           */
  double rope_high_freq_factor;/* (4)                                                           */
  int rope_original_context;   /* (8192)                                                        */
  int dense_attention;         /* 1: dense causal attention instead of S2O (the baseline)       */
} s2o_layer_config;

/* Device bf16 weights, row-major, used as x·W: attn_norm [H]; w_qkv [H, (Hq + 2·Hkv)·d] (q heads,
 * then k, then v); w_o [Hq·d, H]; mlp_norm [H]; w_gu [H, 2·I] (gate columns, then up);
 * w_down [I, H]. 16-byte aligned, owned by the caller. */
typedef struct {
  const void *attn_norm, *w_qkv, *w_o, *mlp_norm, *w_gu, *w_down;
} s2o_layer_weights;

/* Bytes of scratch for s2o_layer_prefill: the layer's activations, index arrays and the
 * attention's prefill workspace (s2o_prefill_workspace_size; none for the dense baseline).
 * Host only. */
s2o_status s2o_layer_workspace_size(const s2o_config *cfg, const s2o_layer_config *lc,
                                    size_t *bytes);

/* One decoder layer in place on x [batch, N, H] bf16 (device, 16-byte aligned). The S2O path
 * builds its indices (cfg: segment_len, block_size, tau, variants) and runs the gather-attention
 * as s2o_attention_prefill does. Errors: S2O_ERR_INVALID_ARGUMENT / S2O_ERR_UNSUPPORTED for bad
 * arguments (H or I not a multiple of 8), S2O_ERR_WORKSPACE_TOO_SMALL, S2O_ERR_CUDA (a CUDA
 * failure). Asynchronous on `stream`. */
s2o_status s2o_layer_prefill(const s2o_config *cfg, const s2o_layer_config *lc,
                             const s2o_layer_weights *w, void *x, void *ws, size_t ws_bytes,
                             s2o_stream stream);

/* The decoder layer's projections: C[m, n] = A[m, k] · B[k, n] (+ C[m, n] when accumulate = 1),
 * A, B and C row-major bf16 on the device (16-byte aligned, owned by the caller), the products
 * accumulated in fp32 and the result (with the old C when accumulating) rounded to bf16 once.
 * tcgen05 kernels (256 × 256 tiles, TMEM accumulators, TMA loads; for n and k up to 8192 on pairs
 * of SMs, tcgen05 cta_group::2, launched as clusters of two CTAs); no counterpart on the
 * pages beyond the model they run the attention in ([S2O, Key points]: Llama-3.1-8B).
 * n and k must be multiples of 8 (S2O_ERR_UNSUPPORTED otherwise); any m. Every wait inside is
 * bounded like the attention kernel's (s2o_set_wait_limit_ns, reported by
 * s2o_check_device_status). Asynchronous on `stream`. */
s2o_status s2o_gemm_bf16(const void *a, const void *b, void *c, int64_t m, int64_t n, int64_t k,
                         int accumulate, s2o_stream stream);

/* Diagnostic: evaluates the library's exp64 — the binary64 exponential behind the block weights of
 * the early stop (a Cody–Waite reduction by ln 2 and a degree-13 Taylor polynomial written for
 * this library; the pages give no normalisation, see [S2O, Summary ¶2]) — on n
 * device doubles x (each ≤ 0), writing device doubles y. Asynchronous on `stream`. */
s2o_status s2o_exp64_eval(const double *x, double *y, int n, s2o_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* S2O_H */
