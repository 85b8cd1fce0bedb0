// Host side of the libs2o C ABI: argument checks, workspace layout and launches. Every check
// runs before anything is enqueued, so a returned error means no device work was started.
#include <algorithm>
#include <atomic>
#include <cmath>

#include "s2o_internal.h"

namespace s2o {

namespace {
std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};
std::atomic<int> g_attention_max_ctas{0};
std::atomic<int> g_permuted_copy{1};
std::atomic<unsigned long long> g_launches{0};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

s2o_status check_config(const s2o_config *c) {
  if (!c) return S2O_ERR_INVALID_ARGUMENT;
  if (!(c->tau >= 0.0f) || std::isinf(c->tau)) return S2O_ERR_INVALID_ARGUMENT;
  if (c->batch <= 0 || c->n_q_heads <= 0 || c->n_kv_heads <= 0 || c->seq_len <= 0 ||
      c->segment_len <= 0)
    return S2O_ERR_INVALID_ARGUMENT;
  if (c->query_perm != 0 && c->query_perm != 1) return S2O_ERR_INVALID_ARGUMENT;
  if (c->shared_key_order != 0 && c->shared_key_order != 1) return S2O_ERR_INVALID_ARGUMENT;
  if (c->int4_centroids != 0 && c->int4_centroids != 1) return S2O_ERR_INVALID_ARGUMENT;
  if (c->head_dim != 64 && c->head_dim != 128) return S2O_ERR_UNSUPPORTED;
  if (c->block_size != 64 && c->block_size != 128) return S2O_ERR_UNSUPPORTED;
  if (c->n_q_heads % c->n_kv_heads) return S2O_ERR_UNSUPPORTED;
  if (c->segment_len % c->block_size || c->seq_len % c->segment_len) return S2O_ERR_UNSUPPORTED;
  // The block scheduler keeps one warp's weights per query block: at most 2048 key blocks.
  if (c->seq_len / c->block_size > 2048) return S2O_ERR_UNSUPPORTED;
  // Flattened row coordinates of the TMA maps are 32-bit.
  if ((long long)c->batch * c->n_q_heads * c->seq_len >= (1ll << 31)) return S2O_ERR_UNSUPPORTED;
  return S2O_OK;
}

s2o_status check_dense_config(const s2o_config *c) {
  if (!c) return S2O_ERR_INVALID_ARGUMENT;
  s2o_config x = *c;
  x.segment_len = x.seq_len;
  x.tau = 0.f;
  x.query_perm = 1;
  x.shared_key_order = 0;
  x.int4_centroids = 0;
  return check_config(&x);
}

bool indices_ok(const s2o_indices *idx) {
  return idx && idx->perm_q && idx->perm_k && idx->sel_cnt && idx->sel_blk && idx->local_tiles &&
         aligned16(idx->perm_q) && aligned16(idx->perm_k) && aligned16(idx->sel_cnt) &&
         aligned16(idx->sel_blk) && aligned16(idx->local_tiles);
}

s2o_status from_cuda(cudaError_t e) { return e == cudaSuccess ? S2O_OK : S2O_ERR_CUDA; }

// Bytes of one of the permuted copies (K or V) for `heads` copy heads, 256-byte aligned.
size_t copy_bytes(const Dims &d, long long heads) {
  return align256((size_t)heads * (size_t)d.N * (size_t)d.D * 2);
}
constexpr size_t kFlagArea = 256;

// Chunk words per pair of units in the packed streams: each unit's key blocks at most B/16 chunks
// each (two units that do not share a copy head or a segment may list the same block), plus the
// padding of three groups to whole tiles.
long long chunk_cap(const Dims &d) { return 2ll * d.nB * (d.B / 16) + 3 * (d.B / 16); }
long long n_pairs(const Dims &d) { return (d.bhq() * d.nB + 1) / 2; }

// Layout of the attention's part of a prefill workspace, after the index build's part (`base`):
// the decision flag, the per-row log2-sum-exps of the merge path, the permuted copies of K and V,
// the key positions in block order and the visible counts, the packed streams' chunk lists and
// per-pair tile counts. Sized for copy heads = query heads (the largest case).
struct PrefillLayout {
  size_t flag, lse, kp, vp, pos, vis, chunks, meta, total;
};
PrefillLayout prefill_layout(const Dims &d) {
  PrefillLayout L;
  size_t off = ws_layout(d).total;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  const long long heads = d.bhq();
  L.flag = take(kFlagArea);
  L.lse = take((size_t)d.bhq() * d.N * 4);
  L.kp = take(copy_bytes(d, heads));
  L.vp = take(copy_bytes(d, heads));
  L.pos = take((size_t)heads * d.N * 4);
  L.vis = take((size_t)heads * d.nSeg * d.nB);
  L.chunks = take((size_t)n_pairs(d) * (size_t)chunk_cap(d) * 4);
  L.meta = take((size_t)n_pairs(d) * 16);
  L.total = off;
  return L;
}

// Steps 3-4. With a workspace of s2o_prefill_workspace_size bytes (and mode != 3) the device-side
// decision picks the path (the merge path, with packed streams from the permuted copy when the mode
// allows them; copy heads: KV heads when per_kv, else query heads); otherwise the path without a
// workspace.
s2o_status attention_ws(const s2o_config &c, const void *q, const void *k, const void *v,
                        const s2o_indices &idx, void *o, void *ws, size_t ws_bytes, bool per_kv,
                        cudaStream_t st) {
  const Dims d = dims_of(c);
  AttnArgs a{q, k, v, o, idx.perm_q, idx.perm_k, idx.sel_cnt, idx.sel_blk, idx.local_tiles, false};
  const int mode = g_permuted_copy.load();
  const PrefillLayout L = prefill_layout(d);
  if (mode != 3 && ws && ws_bytes >= L.total) {
    char *b = static_cast<char *>(ws);
    a.merge = true;
    a.lse = reinterpret_cast<float *>(b + L.lse);
    uint32_t *flag = reinterpret_cast<uint32_t *>(b + L.flag);
    a.kp = b + L.kp;
    a.vp = b + L.vp;
    a.pos_sorted = reinterpret_cast<int32_t *>(b + L.pos);
    a.vis = reinterpret_cast<uint8_t *>(b + L.vis);
    a.chunks = reinterpret_cast<uint32_t *>(b + L.chunks);
    a.pair_meta = reinterpret_cast<int4 *>(b + L.meta);
    a.chunk_cap = chunk_cap(d);
    a.copy_flag = flag;
    a.copy_per_kv = per_kv;
    if (launch_permuted_copy(d, a, mode, flag, st) != cudaSuccess) return S2O_ERR_CUDA;
  }
  return from_cuda(launch_attention(d, a, g_wait_limit_ns.load(), g_attention_max_ctas.load(),
                                    st));
}
}  // namespace

void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
unsigned long long launch_count() { return g_launches.load(std::memory_order_relaxed); }

Dims dims_of(const s2o_config &c) {
  Dims d;
  d.batch = c.batch;
  d.Hq = c.n_q_heads;
  d.Hkv = c.n_kv_heads;
  d.G = c.n_q_heads / c.n_kv_heads;
  d.N = c.seq_len;
  d.D = c.head_dim;
  d.S = c.segment_len;
  d.B = c.block_size;
  d.nB = c.seq_len / c.block_size;
  d.nSeg = c.seq_len / c.segment_len;
  return d;
}

WsLayout ws_layout(const Dims &d) {
  WsLayout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  const size_t bhq = (size_t)d.bhq(), bhkv = (size_t)d.bhkv();
  L.qchunk = take(bhq * d.nB * d.D * 4);
  L.kchunk = take(bhkv * d.nB * d.D * 4);
  L.qbar = take(bhq * d.D * 4);
  L.kbar_all = take(bhkv * d.D * 4);
  L.kbar_top = take(bhq * d.D * 4);
  L.u = take(bhq * d.D * 4);
  L.kappa = take(bhq * d.N * 4);
  L.rho = take(bhq * d.N * 4);
  L.keys0 = take(bhq * d.N * 8);
  L.keys1 = take(bhq * d.N * 8);
  // Radix digit counts: 256 per tile of 4096 elements of each sorted run (runs of N or of S).
  const size_t tiles_n = (size_t)(d.N + 4095) / 4096, tiles_s = (size_t)(d.S + 4095) / 4096;
  L.radix = take(bhq * 256 * std::max(tiles_n, tiles_s * (size_t)d.nSeg) * 4);
  L.Qbar = take(bhq * d.nB * d.D * 4);
  L.Kbar = take(bhq * d.nB * d.D * 4);
  L.r = take(bhq * d.nB * d.nB * 4);
  L.ncount = take(bhq * d.nSeg * d.nB * 4);
  L.flags = take(64);
  L.total = off;
  return L;
}

}  // namespace s2o

using namespace s2o;

extern "C" {

const char *s2o_status_string(s2o_status st) {
  switch (st) {
    case S2O_OK: return "S2O_OK";
    case S2O_ERR_INVALID_ARGUMENT: return "S2O_ERR_INVALID_ARGUMENT";
    case S2O_ERR_UNSUPPORTED: return "S2O_ERR_UNSUPPORTED";
    case S2O_ERR_WORKSPACE_TOO_SMALL: return "S2O_ERR_WORKSPACE_TOO_SMALL";
    case S2O_ERR_INVALID_INDICES: return "S2O_ERR_INVALID_INDICES";
    case S2O_ERR_CUDA: return "S2O_ERR_CUDA";
    case S2O_ERR_DEVICE_TIMEOUT: return "S2O_ERR_DEVICE_TIMEOUT";
  }
  return "S2O_ERR_UNKNOWN";
}

s2o_status s2o_workspace_size(const s2o_config *cfg, size_t *bytes) {
  s2o_status st = check_config(cfg);
  if (st != S2O_OK) return st;
  if (!bytes) return S2O_ERR_INVALID_ARGUMENT;
  *bytes = ws_layout(dims_of(*cfg)).total;
  return S2O_OK;
}

s2o_status s2o_index_sizes(const s2o_config *cfg, size_t counts[5]) {
  s2o_status st = check_config(cfg);
  if (st != S2O_OK) return st;
  if (!counts) return S2O_ERR_INVALID_ARGUMENT;
  const Dims d = dims_of(*cfg);
  counts[0] = (size_t)d.bhq() * d.N;
  counts[1] = (size_t)d.bhq() * d.N;
  counts[2] = (size_t)d.bhq() * d.nB;
  counts[3] = (size_t)d.bhq() * d.nB * d.nB;
  counts[4] = (size_t)d.bhq() * d.nB;
  return S2O_OK;
}

s2o_status s2o_build_indices(const s2o_config *cfg, const void *q, const void *k,
                             const s2o_indices *out, void *ws, size_t ws_bytes,
                             s2o_stream stream) {
  s2o_status st = check_config(cfg);
  if (st != S2O_OK) return st;
  if (!q || !k || !ws || !aligned16(q) || !aligned16(k) || !aligned16(ws) || !indices_ok(out))
    return S2O_ERR_INVALID_ARGUMENT;
  const Dims d = dims_of(*cfg);
  if (ws_bytes < ws_layout(d).total) return S2O_ERR_WORKSPACE_TOO_SMALL;
  return from_cuda(launch_build_indices(d, *cfg, static_cast<const uint16_t *>(q),
                                        static_cast<const uint16_t *>(k), *out,
                                        static_cast<char *>(ws), (cudaStream_t)stream));
}

s2o_status s2o_workspace_views(const s2o_config *cfg, void *ws, size_t ws_bytes,
                               s2o_workspace_view *view) {
  s2o_status st = check_config(cfg);
  if (st != S2O_OK) return st;
  if (!ws || !view) return S2O_ERR_INVALID_ARGUMENT;
  const Dims d = dims_of(*cfg);
  const WsLayout L = ws_layout(d);
  if (ws_bytes < L.total) return S2O_ERR_WORKSPACE_TOO_SMALL;
  char *b = static_cast<char *>(ws);
  view->qbar = reinterpret_cast<float *>(b + L.qbar);
  view->kbar_all = reinterpret_cast<float *>(b + L.kbar_all);
  view->kbar_top = reinterpret_cast<float *>(b + L.kbar_top);
  view->u = reinterpret_cast<float *>(b + L.u);
  view->kappa = reinterpret_cast<float *>(b + L.kappa);
  view->rho = reinterpret_cast<float *>(b + L.rho);
  view->Qbar = reinterpret_cast<float *>(b + L.Qbar);
  view->Kbar = reinterpret_cast<float *>(b + L.Kbar);
  view->r = reinterpret_cast<float *>(b + L.r);
  view->n = reinterpret_cast<int32_t *>(b + L.ncount);
  return S2O_OK;
}

s2o_status s2o_attention_prefill_with_indices(const s2o_config *cfg, const void *q,
                                              const void *k, const void *v,
                                              const s2o_indices *idx, void *o,
                                              s2o_stream stream) {
  s2o_status st = check_config(cfg);
  if (st != S2O_OK) return st;
  if (!q || !k || !v || !o || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      !indices_ok(idx))
    return S2O_ERR_INVALID_ARGUMENT;
  AttnArgs a{q, k, v, o, idx->perm_q, idx->perm_k, idx->sel_cnt, idx->sel_blk, idx->local_tiles,
             false};
  return from_cuda(launch_attention(dims_of(*cfg), a, g_wait_limit_ns.load(),
                                    g_attention_max_ctas.load(),
                                    (cudaStream_t)stream));
}

s2o_status s2o_attention_prefill_online_stop(const s2o_config *cfg, const void *q,
                                             const void *k, const void *v,
                                             const s2o_indices *idx, void *o, int32_t *stop_cnt,
                                             s2o_stream stream) {
  s2o_status st = check_config(cfg);
  if (st != S2O_OK) return st;
  if (!q || !k || !v || !o || !stop_cnt || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
      !aligned16(o) || !aligned16(stop_cnt) || !indices_ok(idx))
    return S2O_ERR_INVALID_ARGUMENT;
  const Dims d = dims_of(*cfg);
  cudaStream_t s = (cudaStream_t)stream;
  // Query blocks without a selected block keep none (the permuted pass writes the others).
  if (cudaMemsetAsync(stop_cnt, 0, (size_t)d.bhq() * d.nB * sizeof(int32_t), s) != cudaSuccess)
    return S2O_ERR_CUDA;
  AttnArgs a{q, k, v, o, idx->perm_q, idx->perm_k, idx->sel_cnt, idx->sel_blk, idx->local_tiles,
             false};
  a.stop_cnt = stop_cnt;
  a.stop_tau = cfg->tau;
  return from_cuda(launch_attention(d, a, g_wait_limit_ns.load(), g_attention_max_ctas.load(), s));
}

s2o_status s2o_attention_prefill_with_indices_ws(const s2o_config *cfg, const void *q,
                                                 const void *k, const void *v,
                                                 const s2o_indices *idx, void *o, void *ws,
                                                 size_t ws_bytes, s2o_stream stream) {
  s2o_status st = check_config(cfg);
  if (st != S2O_OK) return st;
  if (!q || !k || !v || !o || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      !indices_ok(idx) || (ws && !aligned16(ws)))
    return S2O_ERR_INVALID_ARGUMENT;
  // Caller-supplied indices: one copy per query head, each in that head's own key order.
  return attention_ws(*cfg, q, k, v, *idx, o, ws, ws_bytes, false, (cudaStream_t)stream);
}

s2o_status s2o_attention_prefill(const s2o_config *cfg, const void *q, const void *k,
                                 const void *v, void *o, const s2o_indices *idx, void *ws,
                                 size_t ws_bytes, s2o_stream stream) {
  s2o_status st = check_config(cfg);
  if (st != S2O_OK) return st;
  if (!v || !o || !aligned16(v) || !aligned16(o)) return S2O_ERR_INVALID_ARGUMENT;
  st = s2o_build_indices(cfg, q, k, idx, ws, ws_bytes, stream);
  if (st != S2O_OK) return st;
  // The indices were built here: with one key ordering per KV head the copy is made per KV head.
  return attention_ws(*cfg, q, k, v, *idx, o, ws, ws_bytes, cfg->shared_key_order != 0,
                      (cudaStream_t)stream);
}

s2o_status s2o_layer_workspace_size(const s2o_config *cfg, const s2o_layer_config *lc,
                                    size_t *bytes) {
  if (!cfg || !lc || !bytes) return S2O_ERR_INVALID_ARGUMENT;
  s2o_status st = lc->dense_attention ? check_dense_config(cfg) : check_config(cfg);
  if (st != S2O_OK) return st;
  if (lc->intermediate <= 0 || lc->intermediate % 8 || !(lc->rms_eps > 0.f))
    return S2O_ERR_INVALID_ARGUMENT;
  // The dense baseline ignores the S2O fields: size it as one segment.
  s2o_config c = *cfg;
  if (lc->dense_attention) c.segment_len = c.seq_len;
  const Dims d = dims_of(c);
  size_t attn = 0;
  if (!lc->dense_attention && (st = s2o_prefill_workspace_size(cfg, &attn)) != S2O_OK) return st;
  *bytes = layer_ws_layout(d, *lc).attn_ws + attn;
  return S2O_OK;
}

s2o_status s2o_layer_prefill(const s2o_config *cfg, const s2o_layer_config *lc,
                             const s2o_layer_weights *w, void *x, void *ws, size_t ws_bytes,
                             s2o_stream stream) {
  size_t need = 0;
  s2o_status st = s2o_layer_workspace_size(cfg, lc, &need);
  if (st != S2O_OK) return st;
  if (!w || !x || !ws || !aligned16(x) || !aligned16(ws) || !w->attn_norm || !w->w_qkv ||
      !w->w_o || !w->mlp_norm || !w->w_gu || !w->w_down || !aligned16(w->attn_norm) ||
      !aligned16(w->w_qkv) || !aligned16(w->w_o) || !aligned16(w->mlp_norm) ||
      !aligned16(w->w_gu) || !aligned16(w->w_down))
    return S2O_ERR_INVALID_ARGUMENT;
  if (ws_bytes < need) return S2O_ERR_WORKSPACE_TOO_SMALL;
  s2o_config c1 = *cfg;
  if (lc->dense_attention) c1.segment_len = c1.seq_len;
  const Dims d = dims_of(c1);
  const LayerWs L = layer_ws_layout(d, *lc);
  char *b = static_cast<char *>(ws);
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = launch_layer_pre(d, *lc, *w, x, b, L, g_wait_limit_ns.load(), s);
  if (e != cudaSuccess) return S2O_ERR_CUDA;
  void *q = b + L.q, *k = b + L.k, *v = b + L.v, *o = b + L.o;
  if (lc->dense_attention) {
    AttnArgs a{q, k, v, o, nullptr, nullptr, nullptr, nullptr, nullptr, true};
    e = launch_attention(d, a, g_wait_limit_ns.load(), g_attention_max_ctas.load(), s);
    if (e != cudaSuccess) return S2O_ERR_CUDA;
  } else {
    s2o_indices idx{reinterpret_cast<int32_t *>(b + L.perm_q), reinterpret_cast<int32_t *>(b + L.perm_k),
                    reinterpret_cast<int32_t *>(b + L.sel_cnt), reinterpret_cast<int32_t *>(b + L.sel_blk),
                    reinterpret_cast<int32_t *>(b + L.local_tiles)};
    st = s2o_attention_prefill(cfg, q, k, v, o, &idx, b + L.attn_ws, ws_bytes - L.attn_ws, stream);
    if (st != S2O_OK) return st;
  }
  e = launch_layer_post(d, *lc, *w, x, b, L, g_wait_limit_ns.load(), s);
  if (e != cudaSuccess) return S2O_ERR_CUDA;
  return S2O_OK;
}

s2o_status s2o_dense_causal_prefill(const s2o_config *cfg, const void *q, const void *k,
                                    const void *v, void *o, s2o_stream stream) {
  s2o_status st = check_dense_config(cfg);
  if (st != S2O_OK) return st;
  if (!q || !k || !v || !o || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return S2O_ERR_INVALID_ARGUMENT;
  s2o_config c = *cfg;
  c.segment_len = c.seq_len;
  AttnArgs a{q, k, v, o, nullptr, nullptr, nullptr, nullptr, nullptr, true};
  return from_cuda(launch_attention(dims_of(c), a, g_wait_limit_ns.load(),
                                    g_attention_max_ctas.load(), (cudaStream_t)stream));
}

s2o_status s2o_validate_indices(const s2o_config *cfg, const s2o_indices *idx, void *ws,
                                size_t ws_bytes, s2o_stream stream) {
  s2o_status st = check_config(cfg);
  if (st != S2O_OK) return st;
  if (!ws || !aligned16(ws) || !indices_ok(idx)) return S2O_ERR_INVALID_ARGUMENT;
  const Dims d = dims_of(*cfg);
  const WsLayout L = ws_layout(d);
  if (ws_bytes < L.total) return S2O_ERR_WORKSPACE_TOO_SMALL;
  char *b = static_cast<char *>(ws);
  uint32_t *flag = reinterpret_cast<uint32_t *>(b + L.flags);
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = launch_validate(d, *idx, b, flag, s);
  if (e != cudaSuccess) return S2O_ERR_CUDA;
  uint32_t host_flag = 0;
  if (cudaMemcpyAsync(&host_flag, flag, sizeof(host_flag), cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return S2O_ERR_CUDA;
  return host_flag ? S2O_ERR_INVALID_INDICES : S2O_OK;
}

s2o_status s2o_index_stats(const s2o_config *cfg, const s2o_indices *idx, void *ws,
                           size_t ws_bytes, s2o_stats *stats, s2o_stream stream) {
  s2o_status st = check_config(cfg);
  if (st != S2O_OK) return st;
  if (!ws || !aligned16(ws) || !stats || !indices_ok(idx)) return S2O_ERR_INVALID_ARGUMENT;
  const Dims d = dims_of(*cfg);
  const WsLayout L = ws_layout(d);
  if (ws_bytes < L.total) return S2O_ERR_WORKSPACE_TOO_SMALL;
  unsigned long long *acc = reinterpret_cast<unsigned long long *>(static_cast<char *>(ws) +
                                                                   L.flags);
  cudaStream_t s = (cudaStream_t)stream;
  if (launch_stats(d, *idx, acc, s) != cudaSuccess) return S2O_ERR_CUDA;
  unsigned long long h[3] = {0, 0, 0};
  if (cudaMemcpyAsync(h, acc, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return S2O_ERR_CUDA;
  stats->local_tiles = h[0];
  stats->selected_tiles = h[1];
  stats->pairs = h[2];
  stats->causal_pairs = (uint64_t)d.bhq() * (uint64_t)d.N * (uint64_t)(d.N + 1) / 2;
  return S2O_OK;
}

void s2o_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns.store(ns); }

s2o_status s2o_gemm_bf16(const void *a, const void *b, void *c, int64_t m, int64_t n, int64_t k,
                         int accumulate, s2o_stream stream) {
  if (!a || !b || !c || !aligned16(a) || !aligned16(b) || !aligned16(c) || m <= 0 || n <= 0 ||
      k <= 0 || (accumulate != 0 && accumulate != 1))
    return S2O_ERR_INVALID_ARGUMENT;
  if (n % 8 || k % 8 || m >= (1ll << 31) || n >= (1ll << 31) || k >= (1ll << 31))
    return S2O_ERR_UNSUPPORTED;
  return from_cuda(launch_gemm_bf16(a, b, c, m, n, k, accumulate != 0, g_wait_limit_ns.load(),
                                    (cudaStream_t)stream));
}

s2o_status s2o_prefill_workspace_size(const s2o_config *cfg, size_t *bytes) {
  s2o_status st = check_config(cfg);
  if (st != S2O_OK) return st;
  if (!bytes) return S2O_ERR_INVALID_ARGUMENT;
  *bytes = prefill_layout(dims_of(*cfg)).total;
  return S2O_OK;
}

s2o_status s2o_attention_work(const s2o_config *cfg, const s2o_indices *idx, void *ws,
                              size_t ws_bytes, s2o_work_counts *out, s2o_stream stream) {
  s2o_status st = check_config(cfg);
  if (st != S2O_OK) return st;
  if (!ws || !aligned16(ws) || !out || !indices_ok(idx)) return S2O_ERR_INVALID_ARGUMENT;
  const Dims d = dims_of(*cfg);
  const PrefillLayout L = prefill_layout(d);
  if (ws_bytes < L.total) return S2O_ERR_WORKSPACE_TOO_SMALL;
  char *b = static_cast<char *>(ws);
  cudaStream_t s = (cudaStream_t)stream;
  const long long per_seg = d.S / d.B;
  out->local_pass_tiles = (uint64_t)(d.bhq() * d.nSeg * per_seg * (per_seg + 1) / 2);
  // Selected blocks (the gathered form of the permuted pass runs each once per unit).
  unsigned long long *acc = reinterpret_cast<unsigned long long *>(b + ws_layout(d).flags);
  if (launch_stats(d, *idx, acc, s) != cudaSuccess) return S2O_ERR_CUDA;
  unsigned long long h[3] = {0, 0, 0};
  uint32_t flag = 0;
  if (cudaMemcpyAsync(h, acc, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaMemcpyAsync(&flag, b + L.flag, sizeof(flag), cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return S2O_ERR_CUDA;
  out->packed = (flag & 1u) ? 1 : 0;
  out->merged = (flag & 2u) ? 1 : 0;
  {
    // Without packed streams: the selected blocks (merge path), or each busy block's local tiles
    // and selected blocks (the path without the merge).
    unsigned long long bt[2] = {0, 0};
    if (cudaMemsetAsync(acc, 0, sizeof(bt), s) != cudaSuccess ||
        launch_busy_tiles(d, idx->sel_cnt, idx->local_tiles, acc, s) != cudaSuccess ||
        cudaMemcpyAsync(bt, acc, sizeof(bt), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
      return S2O_ERR_CUDA;
    out->permuted_unit_tiles = out->merged ? bt[1] : bt[0];
    out->permuted_loaded_tiles = out->permuted_unit_tiles;
  }
  if (out->packed) {
    unsigned long long pk[2] = {0, 0};
    if (cudaMemsetAsync(acc, 0, sizeof(pk), s) != cudaSuccess ||
        launch_packed_counts(d, reinterpret_cast<const int4 *>(b + L.meta),
                             reinterpret_cast<const uint32_t *>(b + L.flag), acc, s) !=
            cudaSuccess ||
        cudaMemcpyAsync(pk, acc, sizeof(pk), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
      return S2O_ERR_CUDA;
    out->permuted_loaded_tiles = pk[0];
    out->permuted_unit_tiles = pk[1];
  }
  return S2O_OK;
}

void s2o_set_permuted_copy(int mode) {
  g_permuted_copy.store(mode == 0 || mode == 2 || mode == 3 ? mode : 1);
}

void s2o_set_attention_max_ctas(int max_ctas) {
  g_attention_max_ctas.store(max_ctas > 0 ? max_ctas : 0);
}

uint64_t s2o_kernel_launch_count(void) { return launch_count(); }

s2o_status s2o_check_device_status(s2o_stream stream) {
  unsigned int err = 0, gerr = 0;
  cudaError_t e = read_and_clear_device_error(&err, (cudaStream_t)stream);
  if (e != cudaSuccess) return S2O_ERR_CUDA;
  if (read_and_clear_gemm_error(&gerr, (cudaStream_t)stream) != cudaSuccess) return S2O_ERR_CUDA;
  return err || gerr ? S2O_ERR_DEVICE_TIMEOUT : S2O_OK;
}

// Diagnostic: the library's exp64 (used for block weights) on n device doubles, so that tests
// can compare it bit for bit with an independent implementation.
s2o_status s2o_exp64_eval(const double *x, double *y, int n, s2o_stream stream) {
  if (!x || !y || n < 0) return S2O_ERR_INVALID_ARGUMENT;
  if (n == 0) return S2O_OK;
  return from_cuda(launch_exp64_probe(x, y, n, (cudaStream_t)stream));
}

}  // extern "C"
