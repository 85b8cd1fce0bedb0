// Decoder layer around the S2O attention: a Llama-3.1-8B-shaped prefill layer with the S2O
// prefill (or the dense causal baseline) as its attention, for end-to-end-shaped timing with
// random weights.
//
// Sources: the S2O research card names the model and its end-to-end measurement (Key points:
// Llama-3.1-8B, 3.81x end to end at 128K); the layer is the public Llama-3 decoder layer
// (pre-norm residual blocks, grouped-query attention with rotary position embedding and the
// Llama 3.1 frequency scaling, SwiGLU MLP). bf16 storage between steps, fp32 arithmetic.
//
// Steps (rows = batch·N tokens, H = Hq·d):
//   k_rmsnorm      h = bf16(g ⊙ x · (mean x² + eps)^-1/2), one warp per row
//   GEMM           qkv = h · W_qkv                       (tcgen05 GEMM, bf16 in, fp32 accumulate)
//   k_rope_split   rotate q and k by the angle table, write Q/K/V head-major [b, h, N, d]
//   attention      S2O (index build + permuted gather-attention) or dense causal
//   k_heads_to_rows O [b, Hq, N, d] -> rows [b·N, Hq·d]
//   GEMM           x += O_rows · W_o                     (the residual added before the rounding)
//   k_rmsnorm      h2 = norm(x)
//   GEMM           gu = h2 · W_gu
//   k_silu_mul     a = bf16(silu(gate) · up)
//   GEMM           x += a · W_down
// The frequency table (binary64) and the angle table (cos, sin of position·f_t from binary64
// sincos, rounded to fp32) are built per call.
#include <cmath>
#include <type_traits>

#include "s2o_internal.h"

namespace s2o {
namespace {

__device__ __forceinline__ float bf16_to_f(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

// Nearest bf16 of an fp32 value, ties to even (finite inputs).
__device__ __forceinline__ uint16_t f_to_bf16(float f) {
  const uint32_t u = __float_as_uint(f);
  return (uint16_t)((u + 0x7fffu + ((u >> 16) & 1u)) >> 16);
}

// y[row] = bf16(g ⊙ x[row] · (mean(x[row]²) + eps)^-1/2); one warp per row, 8 values per lane
// per step (H a multiple of 8).
__global__ void __launch_bounds__(256)
    k_rmsnorm(const uint16_t *__restrict__ x, const uint16_t *__restrict__ g,
              uint16_t *__restrict__ y, int H, float eps, long long rows) {
  const long long row = (long long)blockIdx.x * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= rows) return;
  const uint4 *xr = reinterpret_cast<const uint4 *>(x + row * H);
  float ss = 0.f;
  for (int c = lane; c < H / 8; c += 32) {
    const uint4 v = __ldg(xr + c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float a = bf16_to_f((uint16_t)(w[i] & 0xffffu)), b = bf16_to_f((uint16_t)(w[i] >> 16));
      ss = fmaf(a, a, ss);
      ss = fmaf(b, b, ss);
    }
  }
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float r = 1.0f / sqrtf(ss / (float)H + eps);
  const uint4 *gr = reinterpret_cast<const uint4 *>(g);
  uint4 *yr = reinterpret_cast<uint4 *>(y + row * H);
  for (int c = lane; c < H / 8; c += 32) {
    const uint4 v = __ldg(xr + c), gv = __ldg(gr + c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w}, gw[4] = {gv.x, gv.y, gv.z, gv.w};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float lo = bf16_to_f((uint16_t)(gw[i] & 0xffffu)) *
                       (bf16_to_f((uint16_t)(w[i] & 0xffffu)) * r);
      const float hi = bf16_to_f((uint16_t)(gw[i] >> 16)) * (bf16_to_f((uint16_t)(w[i] >> 16)) * r);
      o[i] = (uint32_t)f_to_bf16(lo) | ((uint32_t)f_to_bf16(hi) << 16);
    }
    yr[c] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// cs[i·(d/2) + t] = (cos, sin)(i·f_t) from the binary64 angle, rounded to fp32.
__global__ void k_rope_table(const double *__restrict__ freqs, float2 *__restrict__ cs, int N,
                             int half) {
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (long long)N * half) return;
  const int i = (int)(e / half), t = (int)(e % half);
  double s, c;
  sincos((double)i * freqs[t], &s, &c);
  cs[e] = make_float2((float)c, (float)s);
}

// One CTA per row of qkv [b·N, (Hq + 2·Hkv)·d], its warps taking the heads in turn: q and k
// heads rotated by the table (pairs t, t + d/2), v copied; written head-major to
// Q [b, Hq, N, d], K and V [b, Hkv, N, d]. Lane l takes the PER consecutive t = PER·l .. of each
// half (4-byte accesses for d = 128).
template <int D>
__global__ void __launch_bounds__(256)
    k_rope_split(const uint16_t *__restrict__ qkv, const float2 *__restrict__ cs,
                 uint16_t *__restrict__ Q, uint16_t *__restrict__ K, uint16_t *__restrict__ V,
                 int N, int Hq, int Hkv) {
  constexpr int HALF = D / 2, PER = HALF / 32;
  static_assert(PER == 1 || PER == 2, "d = 64 or 128");
  using W = typename std::conditional<PER == 2, uint32_t, uint16_t>::type;
  const int heads = Hq + 2 * Hkv;
  const long long row = blockIdx.x;
  const int b = (int)(blockIdx.x / (unsigned)N), i = (int)(blockIdx.x % (unsigned)N);
  const int lane = threadIdx.x % 32, t0 = PER * lane;
  const float2 *csr = cs + (long long)i * HALF + t0;
  float2 r[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) r[e] = __ldg(csr + e);
  for (int h = threadIdx.x / 32; h < heads; h += blockDim.x / 32) {
    const uint16_t *src = qkv + (row * heads + h) * D;
    uint16_t *dst;
    if (h < Hq)
      dst = Q + (((long long)b * Hq + h) * N + i) * D;
    else if (h < Hq + Hkv)
      dst = K + (((long long)b * Hkv + (h - Hq)) * N + i) * D;
    else
      dst = V + (((long long)b * Hkv + (h - Hq - Hkv)) * N + i) * D;
    const W lo = *reinterpret_cast<const W *>(src + t0);
    const W hi = *reinterpret_cast<const W *>(src + HALF + t0);
    if (h >= Hq + Hkv) {
      *reinterpret_cast<W *>(dst + t0) = lo;
      *reinterpret_cast<W *>(dst + HALF + t0) = hi;
      continue;
    }
    W olo = 0, ohi = 0;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      const float a = bf16_to_f((uint16_t)(lo >> (16 * e)));
      const float bb = bf16_to_f((uint16_t)(hi >> (16 * e)));
      olo |= (W)f_to_bf16(a * r[e].x - bb * r[e].y) << (16 * e);
      ohi |= (W)f_to_bf16(bb * r[e].x + a * r[e].y) << (16 * e);
    }
    *reinterpret_cast<W *>(dst + t0) = olo;
    *reinterpret_cast<W *>(dst + HALF + t0) = ohi;
  }
}

// rows[b·N + i][h·d + c] = O[b][h][i][c], 16-byte pieces.
template <int D>
__global__ void __launch_bounds__(256)
    k_heads_to_rows(const uint4 *__restrict__ O, uint4 *__restrict__ rows, int N, int Hq,
                    long long n_pieces) {
  constexpr int P = D / 8;  // pieces per head row
  const long long x = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (x >= n_pieces) return;
  const int c = (int)(x % P);
  const long long r = x / P;  // (b, i, h) with h fastest
  const int h = (int)(r % Hq);
  const long long bi = r / Hq;
  const long long b = bi / N;
  const int i = (int)(bi % N);
  rows[x] = __ldg(O + ((b * Hq + h) * N + i) * P + c);
}

// a[row][j] = bf16(silu(gate) · up), gate = gu[row][j], up = gu[row][I + j]; one CTA per row,
// 8 values a thread per step.
__global__ void __launch_bounds__(256)
    k_silu_mul(const uint16_t *__restrict__ gu, uint16_t *__restrict__ a, int I) {
  const long long row = blockIdx.x;
  const uint4 *g4 = reinterpret_cast<const uint4 *>(gu + row * 2LL * I);
  const uint4 *u4 = reinterpret_cast<const uint4 *>(gu + row * 2LL * I + I);
  uint4 *a4 = reinterpret_cast<uint4 *>(a + row * (long long)I);
  for (int c = threadIdx.x; c < I / 8; c += blockDim.x) {
    const uint4 g = __ldg(g4 + c), u = __ldg(u4 + c);
    const uint32_t gw[4] = {g.x, g.y, g.z, g.w}, uw[4] = {u.x, u.y, u.z, u.w};
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float r[2];
#pragma unroll
      for (int hlf = 0; hlf < 2; ++hlf) {
        const float z = bf16_to_f((uint16_t)(gw[k] >> (16 * hlf)));
        const float up = bf16_to_f((uint16_t)(uw[k] >> (16 * hlf)));
        r[hlf] = __fdividef(z, 1.0f + __expf(-z)) * up;
      }
      o[k] = (uint32_t)f_to_bf16(r[0]) | ((uint32_t)f_to_bf16(r[1]) << 16);
    }
    a4[c] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

unsigned grid_for(long long n, int per) { return (unsigned)((n + per - 1) / per); }

}  // namespace

namespace {
// f_t = θ^(-2t/d) with the Llama 3.1 scaling of long wavelengths (one thread per t), binary64.
__global__ void k_rope_freqs(double *__restrict__ f, int d, double theta, double factor,
                             double lo, double hi, double orig) {
  const int t = threadIdx.x;
  if (t >= d / 2) return;
  const double base = pow(theta, -2.0 * t / d);
  double v = base;
  if (factor > 0) {
    const double lam = 2.0 * 3.14159265358979323846 / base;
    if (lam < orig / hi) {
      v = base;
    } else if (lam > orig / lo) {
      v = base / factor;
    } else {
      const double s = (orig / lam - lo) / (hi - lo);
      v = (1.0 - s) * base / factor + s * base;
    }
  }
  f[t] = v;
}
}  // namespace

LayerWs layer_ws_layout(const Dims &d, const s2o_layer_config &lc) {
  LayerWs L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = (off + bytes + 255) & ~size_t(255);
    return at;
  };
  const size_t rows = (size_t)d.batch * d.N, H = (size_t)d.Hq * d.D;
  const size_t qkvw = (size_t)(d.Hq + 2 * d.Hkv) * d.D, I = (size_t)lc.intermediate;
  L.h = take(rows * H * 2);
  L.qkv = take(rows * qkvw * 2);
  L.q = take(rows * H * 2);
  L.k = take((size_t)d.bhkv() * d.N * d.D * 2);
  L.v = take((size_t)d.bhkv() * d.N * d.D * 2);
  L.o = take(rows * H * 2);
  L.o_rows = take(rows * H * 2);
  L.gu = take(rows * 2 * I * 2);
  L.a = take(rows * I * 2);
  L.freqs = take((size_t)d.D / 2 * 8);
  L.cs = take((size_t)d.N * d.D / 2 * 8);
  L.perm_q = take((size_t)d.bhq() * d.N * 4);
  L.perm_k = take((size_t)d.bhq() * d.N * 4);
  L.sel_cnt = take((size_t)d.bhq() * d.nB * 4);
  L.sel_blk = take((size_t)d.bhq() * d.nB * d.nB * 4);
  L.local_tiles = take((size_t)d.bhq() * d.nB * 4);
  L.attn_ws = off;
  return L;
}

cudaError_t launch_layer_pre(const Dims &d, const s2o_layer_config &lc,
                             const s2o_layer_weights &w, const void *x, char *ws,
                             const LayerWs &L, uint64_t wait_limit_ns, cudaStream_t st) {
  cudaError_t e;
  const long long rows = (long long)d.batch * d.N, H = (long long)d.Hq * d.D;
  const long long qkvw = (long long)(d.Hq + 2 * d.Hkv) * d.D;
  uint16_t *h = reinterpret_cast<uint16_t *>(ws + L.h);
  k_rmsnorm<<<grid_for(rows, 8), 256, 0, st>>>(static_cast<const uint16_t *>(x),
                                               static_cast<const uint16_t *>(w.attn_norm), h,
                                               (int)H, lc.rms_eps, rows);
  note_launch();
  if ((e = launch_gemm_bf16(h, w.w_qkv, ws + L.qkv, rows, qkvw, H, false, wait_limit_ns, st)) !=
      cudaSuccess)
    return e;
  k_rope_freqs<<<1, 64, 0, st>>>(reinterpret_cast<double *>(ws + L.freqs), d.D, lc.rope_theta,
                                 lc.rope_factor, lc.rope_low_freq_factor, lc.rope_high_freq_factor,
                                 (double)lc.rope_original_context);
  note_launch();
  const long long n_cs = (long long)d.N * (d.D / 2);
  k_rope_table<<<grid_for(n_cs, 256), 256, 0, st>>>(reinterpret_cast<const double *>(ws + L.freqs),
                                                     reinterpret_cast<float2 *>(ws + L.cs), d.N,
                                                     d.D / 2);
  note_launch();
  auto *qkv = reinterpret_cast<const uint16_t *>(ws + L.qkv);
  auto *cs = reinterpret_cast<const float2 *>(ws + L.cs);
  auto *Q = reinterpret_cast<uint16_t *>(ws + L.q), *K = reinterpret_cast<uint16_t *>(ws + L.k),
       *V = reinterpret_cast<uint16_t *>(ws + L.v);
  if (d.D == 128)
    k_rope_split<128><<<(unsigned)rows, 256, 0, st>>>(qkv, cs, Q, K, V, d.N, d.Hq, d.Hkv);
  else
    k_rope_split<64><<<(unsigned)rows, 256, 0, st>>>(qkv, cs, Q, K, V, d.N, d.Hq, d.Hkv);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_layer_post(const Dims &d, const s2o_layer_config &lc,
                              const s2o_layer_weights &w, void *x, char *ws, const LayerWs &L,
                              uint64_t wait_limit_ns, cudaStream_t st) {
  cudaError_t e;
  const long long rows = (long long)d.batch * d.N, H = (long long)d.Hq * d.D;
  const long long I = lc.intermediate;
  const long long pieces = rows * H / 8;
  if (d.D == 128)
    k_heads_to_rows<128><<<grid_for(pieces, 256), 256, 0, st>>>(
        reinterpret_cast<const uint4 *>(ws + L.o), reinterpret_cast<uint4 *>(ws + L.o_rows), d.N,
        d.Hq, pieces);
  else
    k_heads_to_rows<64><<<grid_for(pieces, 256), 256, 0, st>>>(
        reinterpret_cast<const uint4 *>(ws + L.o), reinterpret_cast<uint4 *>(ws + L.o_rows), d.N,
        d.Hq, pieces);
  note_launch();
  if ((e = launch_gemm_bf16(ws + L.o_rows, w.w_o, x, rows, H, H, true, wait_limit_ns, st)) !=
      cudaSuccess)
    return e;
  uint16_t *h = reinterpret_cast<uint16_t *>(ws + L.h);
  k_rmsnorm<<<grid_for(rows, 8), 256, 0, st>>>(static_cast<const uint16_t *>(x),
                                               static_cast<const uint16_t *>(w.mlp_norm), h,
                                               (int)H, lc.rms_eps, rows);
  note_launch();
  if ((e = launch_gemm_bf16(h, w.w_gu, ws + L.gu, rows, 2 * I, H, false, wait_limit_ns, st)) !=
      cudaSuccess)
    return e;
  k_silu_mul<<<(unsigned)rows, 256, 0, st>>>(reinterpret_cast<const uint16_t *>(ws + L.gu),
                                             reinterpret_cast<uint16_t *>(ws + L.a), (int)I);
  note_launch();
  if ((e = launch_gemm_bf16(ws + L.a, w.w_down, x, rows, H, I, true, wait_limit_ns, st)) !=
      cudaSuccess)
    return e;
  return cudaGetLastError();
}

}  // namespace s2o
