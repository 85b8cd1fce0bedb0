// Index construction of S2O on sm_100a: stripe mean pooling, the global key/value ordering, the
// segment-local query ordering, block scores and the importance-ordered early stop.
//
// Sources: "S2O: Early Stopping for Sparse Attention via Online Permutation" (research card),
// Summary ¶2 (stripe-level mean pooling; a segment-local query ordering and a global key/value
// ordering kept as index arrays; blocks processed from most to least important, stopping once a
// block's score falls under τ) and "AB-Sparse", Figure 2 workflow text (block score r = q·cᵀ
// against mean-pooled centroids). The formulas where the pages are silent are this project's
// readings, fixed in its definition file.
//
// Every floating-point step below is an explicitly rounded IEEE operation (__fadd_rn, __fmaf_rn,
// __fdiv_rn, __dadd_rn, __ddiv_rn, ...) in the order the definition fixes, so the index arrays are
// bit-exact and reproducible. These kernels are bandwidth- or latency-bound; none is a dense
// contraction worth tensor cores (the block-score product needs a fixed fp32 FMA order).
#include <algorithm>
#include <climits>
#include <cmath>
#include <type_traits>

#include "s2o_internal.h"

namespace s2o {
namespace {

constexpr int kWarp = 32;

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }
__device__ __forceinline__ float bf16_at(const uint16_t *p) {
  return __uint_as_float((uint32_t)__ldg(p) << 16);
}

// DOT(row, vec) of a bf16 row (D values, 16-byte aligned) against an fp32 vector: the
// definition's sequential FMA chain over t = 0..D-1. The whole row is loaded first (D/8 16-byte
// loads in flight per thread).
template <int D>
__device__ __forceinline__ float dot_row(const uint16_t *row, const float *vec) {
  uint4 v[D / 8];
  const uint4 *p = reinterpret_cast<const uint4 *>(row);
#pragma unroll
  for (int c = 0; c < D / 8; ++c) v[c] = __ldg(p + c);
  float acc = 0.f;
#pragma unroll
  for (int c = 0; c < D / 8; ++c) {
    const uint32_t w[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      acc = __fmaf_rn(bf16_lo(w[x]), vec[c * 8 + 2 * x], acc);
      acc = __fmaf_rn(bf16_hi(w[x]), vec[c * 8 + 2 * x + 1], acc);
    }
  }
  return acc;
}

// DOT(row, vec) for a row already in registers (D bf16 values as D/8 16-byte words) against an
// fp32 vector in shared memory read four values at a time: the same sequential FMA chain over
// t = 0..D-1.
template <int D>
__device__ __forceinline__ float dot_regs(const uint4 (&v)[D / 8], const float4 *vec4) {
  float acc = 0.f;
#pragma unroll
  for (int c = 0; c < D / 8; ++c) {
    const float4 a = vec4[2 * c], b = vec4[2 * c + 1];
    acc = __fmaf_rn(bf16_lo(v[c].x), a.x, acc);
    acc = __fmaf_rn(bf16_hi(v[c].x), a.y, acc);
    acc = __fmaf_rn(bf16_lo(v[c].y), a.z, acc);
    acc = __fmaf_rn(bf16_hi(v[c].y), a.w, acc);
    acc = __fmaf_rn(bf16_lo(v[c].z), b.x, acc);
    acc = __fmaf_rn(bf16_hi(v[c].z), b.y, acc);
    acc = __fmaf_rn(bf16_lo(v[c].w), b.z, acc);
    acc = __fmaf_rn(bf16_hi(v[c].w), b.w, acc);
  }
  return acc;
}

// 16-byte asynchronous copy global -> shared (cached in L2 only), and the wait for all of this
// thread's copies. A CTA stages contiguous rows this way with no registers held per load, so many
// loads are in flight.
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(smem_dst)),
               "l"(gsrc)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// Sort key of an fp32 score: monotone in the value, −0 folded onto +0, NaN below everything.
__device__ __forceinline__ uint32_t sort_key(float x) {
  uint32_t b = __float_as_uint(x);
  if ((b & 0x7fffffffu) > 0x7f800000u) return 0u;
  if ((b & 0x7fffffffu) == 0u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// exp64: Cody–Waite reduction by ln 2 with a two-part constant, then the degree-13 Taylor
// polynomial of e^t by Horner's rule with fused multiply-adds, then an exact scaling by 2^k.
// Written for this project from the mathematics; defined for x <= 0 (all block-weight arguments).
// k = rint(x/ln 2) is taken by adding and subtracting 1.5·2^52 (round half to even, as rint),
// which also leaves k in the low word of the sum: no conversion instruction is needed.
__device__ __forceinline__ double exp64(double x_in) {
  // Branch-free: arguments below -700 (results that underflow) run the same steps on -700 and are
  // replaced by 0 at the end, so that independent calls interleave.
  const double x = x_in < -700.0 ? -700.0 : x_in;
  const double kInvLn2 = 0x1.71547652b82fep+0;  // nearest binary64 to 1/ln 2
  const double kLn2Hi = 0x1.62e42fefa39efp-1;   // nearest binary64 to ln 2
  const double kLn2Lo = 0x1.abc9e3b39803fp-56;  // nearest binary64 to ln 2 − kLn2Hi
  const double kRound = 0x1.8p52;
  // 1/j! for j = 0..13, each the correctly rounded quotient (j! is exact in binary64).
  const double c[14] = {1.0 / 1.0,         1.0 / 1.0,          1.0 / 2.0,
                        1.0 / 6.0,         1.0 / 24.0,         1.0 / 120.0,
                        1.0 / 720.0,       1.0 / 5040.0,       1.0 / 40320.0,
                        1.0 / 362880.0,    1.0 / 3628800.0,    1.0 / 39916800.0,
                        1.0 / 479001600.0, 1.0 / 6227020800.0};
  const double y = __dadd_rn(__dmul_rn(x, kInvLn2), kRound);
  const double k = __dsub_rn(y, kRound);
  double t = __fma_rn(-k, kLn2Hi, x);
  t = __fma_rn(-k, kLn2Lo, t);
  double p = c[13];
#pragma unroll
  for (int j = 12; j >= 0; --j) p = __fma_rn(p, t, c[j]);
  // k in [-1010, 0]: 2^k is a normal binary64 number, so the product is exact.
  const int ki = __double2loint(y);
  const double e = __dmul_rn(p, __hiloint2double((ki + 1023) << 20, 0));
  return x_in < -700.0 ? 0.0 : e;
}

// An integer 0 <= n < 2^31 as binary64, exactly, without a conversion instruction.
__device__ __forceinline__ double int_to_double(int n) {
  return __dsub_rn(__hiloint2double(0x43300000, n), 0x1p52);
}

// ------------------------------------------------------------------ pooling (step 1a)

// Chunk sums of the MEAN rule: one thread per (chunk of B rows, two columns), rows summed
// sequentially from +0 in row order.
template <int D>
__global__ void __launch_bounds__(256)
    k_pool_chunks(const uint16_t *__restrict__ src, float *__restrict__ out, int B,
                  long long n_chunks) {
  constexpr int P = D / 2;
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long chunk = tid / P;
  const int t = (int)(tid % P) * 2;
  if (chunk >= n_chunks) return;
  const uint32_t *p = reinterpret_cast<const uint32_t *>(src + (size_t)chunk * B * D + t);
  float a0 = 0.f, a1 = 0.f;
#pragma unroll 8
  for (int e = 0; e < B; ++e) {
    const uint32_t v = __ldg(p + (size_t)e * P);
    a0 = __fadd_rn(a0, bf16_lo(v));
    a1 = __fadd_rn(a1, bf16_hi(v));
  }
  *reinterpret_cast<float2 *>(out + (size_t)chunk * D + t) = make_float2(a0, a1);
}

// Chunk sums added sequentially in chunk order, then divided by the list length. One CTA per
// (head, 32 columns): all threads stage up to 1024 chunk sums at once in shared memory (many loads
// in flight), then one warp adds them in chunk order.
template <int D>
__global__ void __launch_bounds__(256)
    k_pool_finish(const float *__restrict__ chunks, float *__restrict__ out, int n_chunks,
                  float len) {
  constexpr int kStage = 1024;
  extern __shared__ float4 stage4[];  // [kStage][32]
  float *stage = reinterpret_cast<float *>(stage4);
  const long long head = blockIdx.y;
  const int col0 = blockIdx.x * 32;
  const float *base = chunks + (size_t)head * n_chunks * D + col0;
  float acc = 0.f;
  for (int c0 = 0; c0 < n_chunks; c0 += kStage) {
    const int n = min(kStage, n_chunks - c0);
    // Eight loads in flight per thread before their stores (a load-store loop would wait for
    // each load in turn).
    for (int x0 = threadIdx.x; x0 < n * 8; x0 += 8 * blockDim.x) {
      float4 v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int x = x0 + i * blockDim.x;
        if (x < n * 8)
          v[i] = __ldg(reinterpret_cast<const float4 *>(base + (size_t)(c0 + x / 8) * D) + x % 8);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int x = x0 + i * blockDim.x;
        if (x < n * 8) stage4[x] = v[i];
      }
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      int c = 0;
      for (; c + 8 <= n; c += 8) {
        float v[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) v[x] = stage[(c + x) * 32 + threadIdx.x];
#pragma unroll
        for (int x = 0; x < 8; ++x) acc = __fadd_rn(acc, v[x]);
      }
      for (; c < n; ++c) acc = __fadd_rn(acc, stage[c * 32 + threadIdx.x]);
    }
    __syncthreads();
  }
  if (threadIdx.x < 32) out[head * D + col0 + threadIdx.x] = __fdiv_rn(acc, len);
}

// One pass over K, one CTA per chunk of B key rows of a KV head. The chunk's rows (contiguous in
// memory) are staged in shared memory with coalesced asynchronous copies (rows padded by 16 bytes,
// so that per-row reads are free of bank conflicts), then:
//   kappa_j = DOT(qbar_h, k_j) for the G query heads of the group (one thread per key row, qbar
//   read four values at a time), and the chunk sum of the MEAN rule for kbar_all (one thread per
//   two columns adding the rows in order).
template <int D>
__global__ void __launch_bounds__(128)
    k_kpass(const uint16_t *__restrict__ k, const float *__restrict__ qbar,
            float *__restrict__ kappa, float *__restrict__ kchunk, int N, int B, int Hq, int Hkv,
            int G, int shared_order) {
  constexpr int RS = D * 2 + 16;  // staged row stride in bytes
  extern __shared__ float4 sm4[];
  float *qb = reinterpret_cast<float *>(sm4);                                     // [G][D]
  unsigned char *rows = reinterpret_cast<unsigned char *>(sm4 + (size_t)G * D / 4);  // [B][RS]
  const long long kh = blockIdx.y;
  const int chunk = blockIdx.x, r = threadIdx.x;
  const long long beta = kh / Hkv;
  const int g = (int)(kh % Hkv);
  const size_t qh0 = (size_t)beta * Hq + (size_t)g * G;
  const unsigned char *src =
      reinterpret_cast<const unsigned char *>(k + ((size_t)kh * N + (size_t)chunk * B) * D);
  for (int x = threadIdx.x; x < B * (D / 8); x += blockDim.x)
    cp_async16(rows + (x / (D / 8)) * RS + (x % (D / 8)) * 16, src + (size_t)x * 16);
  for (int x = threadIdx.x; x < G * D; x += blockDim.x) qb[x] = qbar[qh0 * D + x];
  cp_async_wait_all();
  __syncthreads();
  if (shared_order) {
    // One ordering per KV head: the group's pooled query (the G mean queries added in head
    // order, divided by G) replaces the first head's; column t is read and written by thread t.
    for (int t = threadIdx.x; t < D; t += blockDim.x) {
      float acc = qb[t];
      for (int hi = 1; hi < G; ++hi) acc = __fadd_rn(acc, qb[hi * D + t]);
      qb[t] = __fdiv_rn(acc, (float)G);
    }
    __syncthreads();
  }
  const int n_heads = shared_order ? 1 : G;
  const int j = chunk * B + r;
  if (r < B) {
    // Up to four query heads at a time: their chains interleave (each still runs over t in
    // order) and the row is read once per group of heads.
    const uint4 *row = reinterpret_cast<const uint4 *>(rows + r * RS);
    for (int h0 = 0; h0 < n_heads; h0 += 4) {
      const int nh = min(4, n_heads - h0);
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 2
      for (int c = 0; c < D / 8; ++c) {
        const uint4 v = row[c];
        const float x[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                            bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) {
          if (hh < nh) {
            const float4 *qv = sm4 + (size_t)(h0 + hh) * D / 4;
            const float4 a = qv[2 * c], b = qv[2 * c + 1];
            float t = acc[hh];
            t = __fmaf_rn(x[0], a.x, t);
            t = __fmaf_rn(x[1], a.y, t);
            t = __fmaf_rn(x[2], a.z, t);
            t = __fmaf_rn(x[3], a.w, t);
            t = __fmaf_rn(x[4], b.x, t);
            t = __fmaf_rn(x[5], b.y, t);
            t = __fmaf_rn(x[6], b.z, t);
            t = __fmaf_rn(x[7], b.w, t);
            acc[hh] = t;
          }
        }
      }
#pragma unroll
      for (int hh = 0; hh < 4; ++hh)
        if (hh < nh) kappa[(qh0 + h0 + hh) * N + j] = acc[hh];
      if (shared_order)  // the group's score, in every query head's row
        for (int hi = 1; hi < G; ++hi) kappa[(qh0 + hi) * N + j] = acc[0];
    }
  }
  if (r < D / 2) {
    float a0 = 0.f, a1 = 0.f;
    for (int e = 0; e < B; ++e) {
      const uint32_t w = *reinterpret_cast<const uint32_t *>(rows + e * RS + r * 4);
      a0 = __fadd_rn(a0, bf16_lo(w));
      a1 = __fadd_rn(a1, bf16_hi(w));
    }
    *reinterpret_cast<float2 *>(kchunk + ((size_t)kh * (N / B) + chunk) * D + 2 * r) =
        make_float2(a0, a1);
  }
}

// kbar_top = MEAN of the B top-ranked keys (rank order); u = kbar_top − kbar_all.
__global__ void k_kbar_top(const uint16_t *__restrict__ k, const int32_t *__restrict__ perm_k,
                           const float *__restrict__ kbar_all, float *__restrict__ kbar_top,
                           float *__restrict__ u, int N, int D, int B, int Hq, int Hkv, int G) {
  const long long qh = blockIdx.x;
  const long long kh = (qh / Hq) * Hkv + (qh % Hq) / G;
  const int t = threadIdx.x;
  // Rows in rank order, sixteen loads in flight, added sequentially.
  float acc = 0.f;
  for (int e0 = 0; e0 < B; e0 += 16) {
    float v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int j = __ldg(perm_k + qh * N + e0 + i);
      v[i] = bf16_at(k + ((size_t)kh * N + j) * D + t);
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) acc = __fadd_rn(acc, v[i]);
  }
  const float top = __fdiv_rn(acc, (float)B);
  kbar_top[qh * D + t] = top;
  u[qh * D + t] = __fsub_rn(top, kbar_all[kh * D + t]);
}

// rho_i = DOT(q_i, u_h), one thread per query row. A CTA's 128 rows (contiguous) are staged in
// shared memory with coalesced asynchronous copies (rows padded by 16 bytes), then each thread
// reads its row and runs the chain with u read four values at a time.
template <int D>
__global__ void __launch_bounds__(128)
    k_rho(const uint16_t *__restrict__ q, const float *__restrict__ u, float *__restrict__ rho,
          int N) {
  constexpr int RS = D * 2 + 16;
  __shared__ __align__(16) unsigned char rows[128 * RS];
  __shared__ float4 us4[D / 4];
  const long long qh = blockIdx.y;
  const int i0 = blockIdx.x * 128;
  const int nrows = min(128, N - i0);
  const unsigned char *src =
      reinterpret_cast<const unsigned char *>(q + ((size_t)qh * N + i0) * D);
  for (int x = threadIdx.x; x < nrows * (D / 8); x += blockDim.x)
    cp_async16(rows + (x / (D / 8)) * RS + (x % (D / 8)) * 16, src + (size_t)x * 16);
  if (threadIdx.x < D / 4) us4[threadIdx.x] = reinterpret_cast<const float4 *>(u + qh * D)[threadIdx.x];
  cp_async_wait_all();
  __syncthreads();
  if (threadIdx.x >= nrows) return;
  uint4 v[D / 8];
#pragma unroll
  for (int c = 0; c < D / 8; ++c)
    v[c] = *reinterpret_cast<const uint4 *>(rows + threadIdx.x * RS + c * 16);
  rho[qh * N + i0 + threadIdx.x] = dot_regs<D>(v, us4);
}

// ------------------------------------------------------------------ ordering (step 2)

// ------------------------------------------------------------------ stable radix sorting
//
// Orderings are stable least-significant-digit radix sorts of 32-bit keys, 8 bits per pass, with
// the original index as the value: key = ~(sort key), so ascending keys are descending scores and
// equal keys keep index order (the lower index first), exactly the ordering the definition fixes.

__device__ __forceinline__ uint32_t desc_key(float score) { return ~sort_key(score); }

// Lanes of the warp holding the same 8-bit digit (eight ballots).
__device__ __forceinline__ unsigned match_digit(uint32_t d) {
  unsigned peers = 0xffffffffu;
#pragma unroll
  for (int b = 0; b < 8; ++b) {
    const unsigned bb = __ballot_sync(0xffffffffu, (d >> b) & 1u);
    peers &= ((d >> b) & 1u) ? bb : ~bb;
  }
  return peers;
}

// One counting pass inside a CTA: the destination, in stable order by digit, of R elements per
// lane (element r of lane l of warp w is w·32R + r·32 + l). Scratch: hist[warps·256],
// dbase[256]. Also returns, in dbase, each digit's first destination.
template <int R, int NW>
__device__ __forceinline__ void radix_ranks(const uint32_t (&digit)[R], int (&dest)[R],
                                            int *hist, int *dbase) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const unsigned full = 0xffffffffu, below = (1u << lane) - 1u;
  int *wh = hist + warp * 256;
  for (int d = lane; d < 256; d += 32) wh[d] = 0;
  __syncwarp();
  int rank[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const unsigned peers = match_digit(digit[r]);
    rank[r] = wh[digit[r]] + __popc(peers & below);
    __syncwarp();
    if (lane == __ffs(peers) - 1) wh[digit[r]] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // Per digit: exclusive prefix over the NW warps (in place) and the digit's total; the NW
  // counts are loaded together.
  for (int d = threadIdx.x; d < 256; d += blockDim.x) {
    int c[NW];
#pragma unroll
    for (int w = 0; w < NW; ++w) c[w] = hist[w * 256 + d];
    int run = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      hist[w * 256 + d] = run;
      run += c[w];
    }
    dbase[d] = run;
  }
  __syncthreads();
  if (warp == 0) {  // exclusive scan of the 256 digit totals, 8 per lane
    int v[8], sum = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[i] = dbase[lane * 8 + i];
      sum += v[i];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(full, incl, o);
      if (lane >= o) incl += t;
    }
    int run = incl - sum;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      dbase[lane * 8 + i] = run;
      run += v[i];
    }
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < R; ++r) dest[r] = dbase[digit[r]] + wh[digit[r]] + rank[r];
}

// Segment-local query ordering, one CTA per (query head, segment) of at most 32·R·(blockDim/32)
// queries: four counting passes over the keys of the segment's rho values in shared memory, then
// perm_q (the identity when the query ordering is off).
template <int R>
__global__ void __launch_bounds__(512)
    k_segment_sort(const float *__restrict__ rho, int32_t *__restrict__ perm_q, int N, int S,
                   int query_perm) {
  extern __shared__ int sm_i[];
  const int n = blockDim.x * R;
  uint32_t *skey = reinterpret_cast<uint32_t *>(sm_i);  // [n]
  uint32_t *sval = skey + n;                            // [n]
  int *hist = reinterpret_cast<int *>(sval + n);        // [warps·256]
  int *dbase = hist + (blockDim.x / 32) * 256;          // [256]
  const long long qh = blockIdx.y;
  const int s0 = blockIdx.x * S;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (!query_perm) {
    for (int r = threadIdx.x; r < S; r += blockDim.x) perm_q[qh * N + s0 + r] = s0 + r;
    return;
  }
  uint32_t key[R], val[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int e = warp * 32 * R + r * 32 + lane;
    key[r] = e < S ? desc_key(__ldg(rho + qh * N + s0 + e)) : 0xffffffffu;
    val[r] = (uint32_t)e;
  }
  for (int pass = 0; pass < 4; ++pass) {
    uint32_t dig[R];
    int dest[R];
#pragma unroll
    for (int r = 0; r < R; ++r) dig[r] = (key[r] >> (8 * pass)) & 255u;
    radix_ranks<R, 16>(dig, dest, hist, dbase);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      skey[dest[r]] = key[r];
      sval[dest[r]] = val[r];
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int e = warp * 32 * R + r * 32 + lane;
      key[r] = skey[e];
      val[r] = sval[e];
    }
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int e = warp * 32 * R + r * 32 + lane;
    if (e < S) perm_q[qh * N + s0 + e] = s0 + (int32_t)val[r];
  }
  (void)n;
}

// Step 2b fused per (query head, segment), one CTA of 256 threads: rho_i = DOT(q_i, u_h) for the
// segment's rows (also stored), their segment-local order (perm_q) and the means Qbar of the
// ordered query blocks. The arithmetic is k_rho's, k_segment_sort's and k_block_means's step for
// step; fused, the segment's rows come from HBM once (for rho) and the block means read them
// again right after the ordering, from L2 while the segment is still resident (with every SM's
// two segments in flight at 128K tokens, about a third of those re-reads hit), where three
// launches read Q twice and sort in between. Two groups of 128 threads stage
// chunks of 128 contiguous rows with asynchronous copies (rows padded by 16 bytes) and take one
// row per thread; the ordering is k_segment_sort's four counting passes over R keys per thread;
// then each warp forms the means of every eighth block of the segment.
// Threads of k_rho_order_means (two CTAs per SM; 512 threads and one CTA per SM measured the same).
constexpr int kFuseNT = 256;
template <int D, int NT>
constexpr size_t fused_order_smem(int R) {
  return (size_t)(NT / 128) * 128 * (D * 2 + 16) + D * 4 + (size_t)2 * NT * R * 4 +
         (size_t)(NT / 32) * 256 * 4 + 256 * 4;
}
__device__ __forceinline__ void group_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
template <int D, int R, int NT>
__global__ void __launch_bounds__(NT, NT == 256 ? 2 : 1)
    k_rho_order_means(const uint16_t *__restrict__ q, const float *__restrict__ u,
                      float *__restrict__ rho, int32_t *__restrict__ perm_q,
                      float *__restrict__ qbar, int N, int S, int B, int nB) {
  constexpr int NW = NT / 32, NG = NT / 128, RS = D * 2 + 16;
  constexpr int CPL = D / 32;  // block-mean columns per lane (4 or 2)
  using Vec = typename std::conditional<CPL == 4, uint2, uint32_t>::type;
  extern __shared__ __align__(16) unsigned char smem_f[];
  float4 *us4 = reinterpret_cast<float4 *>(smem_f + NG * 128 * RS);  // [D/4]
  uint32_t *skey = reinterpret_cast<uint32_t *>(us4 + D / 4);       // [NT·R]
  uint32_t *sval = skey + NT * R;                                    // [NT·R]
  int *hist = reinterpret_cast<int *>(sval + NT * R);                // [NW·256]
  int *dbase = hist + NW * 256;                                      // [256]
  const long long qh = blockIdx.y;
  const int s0 = blockIdx.x * S;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x < D / 4)
    us4[threadIdx.x] = reinterpret_cast<const float4 *>(u + qh * D)[threadIdx.x];
  __syncthreads();
  // rho: group g stages chunks g, g + NG, ... of the segment (named barrier 1 + g).
  {
    const int g = threadIdx.x / 128, t = threadIdx.x % 128;
    unsigned char *stage = smem_f + g * 128 * RS;
    const unsigned char *seg =
        reinterpret_cast<const unsigned char *>(q + ((size_t)qh * N + s0) * D);
    for (int c = g; c * 128 < S; c += NG) {
      const int nrows = min(128, S - c * 128);
      const unsigned char *src = seg + (size_t)c * 128 * D * 2;
      for (int x = t; x < nrows * (D / 8); x += 128)
        cp_async16(stage + (x / (D / 8)) * RS + (x % (D / 8)) * 16, src + (size_t)x * 16);
      cp_async_wait_all();
      group_sync(1 + g, 128);
      if (t < nrows) {
        uint4 v[D / 8];
#pragma unroll
        for (int c2 = 0; c2 < D / 8; ++c2)
          v[c2] = *reinterpret_cast<const uint4 *>(stage + t * RS + c2 * 16);
        const float r_i = dot_regs<D>(v, us4);
        rho[qh * N + s0 + c * 128 + t] = r_i;  // kept in the workspace (an intermediate)
        skey[c * 128 + t] = desc_key(r_i);
      }
      group_sync(1 + g, 128);  // the stage may be refilled
    }
  }
  __syncthreads();
  // perm_q: stable descending order of rho inside the segment (as k_segment_sort).
  uint32_t key[R], val[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int e = warp * 32 * R + r * 32 + lane;
    key[r] = e < S ? skey[e] : 0xffffffffu;
    val[r] = (uint32_t)e;
  }
  for (int pass = 0; pass < 4; ++pass) {
    uint32_t dig[R];
    int dest[R];
#pragma unroll
    for (int r = 0; r < R; ++r) dig[r] = (key[r] >> (8 * pass)) & 255u;
    radix_ranks<R, NW>(dig, dest, hist, dbase);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      skey[dest[r]] = key[r];
      sval[dest[r]] = val[r];
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int e = warp * 32 * R + r * 32 + lane;
      key[r] = skey[e];
      val[r] = sval[e];
    }
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int e = warp * 32 * R + r * 32 + lane;
    if (e < S) perm_q[qh * N + s0 + e] = s0 + (int32_t)val[r];
  }
  // Qbar of the segment's ordered blocks (sval holds the order): as k_block_means, one warp per
  // block, the rows (from L2) added in slot order.
  const Vec *base = reinterpret_cast<const Vec *>(q + (size_t)qh * N * D) + lane;
  for (int bl = warp; bl * B < S; bl += NW) {
    const uint32_t *pp = sval + bl * B;
    float acc[CPL];
#pragma unroll
    for (int x = 0; x < CPL; ++x) acc[x] = 0.f;
    for (int e0 = 0; e0 < B; e0 += 32) {
      const int my_row = s0 + (int)pp[e0 + lane];
#pragma unroll
      for (int h = 0; h < 32; h += 16) {
        Vec v[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int row = __shfl_sync(0xffffffffu, my_row, h + e);
          v[e] = __ldg(base + (size_t)row * (D / CPL));
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          if constexpr (CPL == 4) {
            const uint2 w = *reinterpret_cast<const uint2 *>(&v[e]);
            acc[0] = __fadd_rn(acc[0], bf16_lo(w.x));
            acc[1] = __fadd_rn(acc[1], bf16_hi(w.x));
            acc[2] = __fadd_rn(acc[2], bf16_lo(w.y));
            acc[3] = __fadd_rn(acc[3], bf16_hi(w.y));
          } else {
            const uint32_t w = *reinterpret_cast<const uint32_t *>(&v[e]);
            acc[0] = __fadd_rn(acc[0], bf16_lo(w));
            acc[1] = __fadd_rn(acc[1], bf16_hi(w));
          }
        }
      }
    }
    const float len = (float)B;
    float *dst = qbar + ((size_t)qh * nB + s0 / B + bl) * D + lane * CPL;
#pragma unroll
    for (int x = 0; x < CPL; ++x) dst[x] = __fdiv_rn(acc[x], len);
  }
}

// Copies the first row of each group of G rows (row_len int32, a multiple of 4, 16-byte aligned
// rows) to the group's other G - 1 rows. Grid: (any, groups).
__global__ void k_replicate_group_rows(int32_t *__restrict__ a, long long row_len, int G) {
  int32_t *grp = a + (long long)blockIdx.y * G * row_len;
  for (long long x = (long long)blockIdx.x * blockDim.x + threadIdx.x; x < row_len / 4;
       x += (long long)gridDim.x * blockDim.x) {
    const int4 v = reinterpret_cast<const int4 *>(grp)[x];
    for (int hi = 1; hi < G; ++hi) reinterpret_cast<int4 *>(grp + hi * row_len)[x] = v;
  }
}

// Multi-CTA stable radix sort of runs of run_len elements (one run per query head), tiles of
// kRadixTile elements: per pass a digit count per tile, then a scatter per tile that derives its
// offsets from the run's counts.
constexpr int kRadixR = 8, kRadixThreads = 512, kRadixTile = kRadixR * kRadixThreads;
static_assert(kRadixThreads == 2 * 256, "the scatter reads each digit's counts with two threads");

// Element e of a tile, for thread (warp, lane) and round r.
__device__ __forceinline__ int radix_elem(int r) {
  return (threadIdx.x / 32) * 32 * kRadixR + r * 32 + threadIdx.x % 32;
}

// Keys and values of pass 0 come from the scores (read at score_base): key = desc_key(score),
// value = the index in the run (idx0 = index of the tile's first element); later passes read the
// keys and values at base.
__device__ __forceinline__ void radix_load(const float *score, const uint32_t *keys,
                                           const uint32_t *vals, long long score_base,
                                           long long base, int idx0, int n,
                                           uint32_t (&key)[kRadixR], uint32_t (&val)[kRadixR]) {
#pragma unroll
  for (int r = 0; r < kRadixR; ++r) {
    const int e = radix_elem(r);
    if (e < n) {
      key[r] = score ? desc_key(__ldg(score + score_base + e)) : __ldg(keys + base + e);
      val[r] = score ? (uint32_t)(idx0 + e) : __ldg(vals + base + e);
    } else {
      key[r] = 0xffffffffu;
      val[r] = 0u;
    }
  }
}

// counts[(run·256 + digit)·tiles + tile] for one pass.
__global__ void __launch_bounds__(kRadixThreads)
    k_radix_count(const float *__restrict__ score, const uint32_t *__restrict__ keys,
                  long long run_len, long long score_stride, int tiles, int shift,
                  int *__restrict__ counts) {
  __shared__ int h[256];
  const long long run = blockIdx.x / tiles;
  const int tile = blockIdx.x % tiles;
  const long long base = (score ? run * score_stride : run * run_len) + (long long)tile * kRadixTile;
  const int n = (int)min((long long)kRadixTile, run_len - (long long)tile * kRadixTile);
  for (int d = threadIdx.x; d < 256; d += blockDim.x) h[d] = 0;
  __syncthreads();
  // All of a thread's keys are loaded before they are counted (kRadixR loads in flight).
  uint32_t kv[kRadixR];
#pragma unroll
  for (int r = 0; r < kRadixR; ++r) {
    const int e = r * kRadixThreads + (int)threadIdx.x;
    kv[r] = e < n ? (score ? desc_key(__ldg(score + base + e)) : __ldg(keys + base + e)) : 0u;
  }
#pragma unroll
  for (int r = 0; r < kRadixR; ++r)
    if (r * kRadixThreads + (int)threadIdx.x < n) atomicAdd(&h[(kv[r] >> shift) & 255u], 1);
  __syncthreads();
  for (int d = threadIdx.x; d < 256; d += blockDim.x)
    counts[(run * 256 + d) * tiles + tile] = h[d];
}

// Scatter of one pass: each tile derives its output offset per digit from the per-tile counts
// (the run's elements with a smaller digit plus those with the same digit in earlier tiles), ranks
// its elements by digit (stable), groups them in shared memory and writes each digit's run to its
// offset. The last pass writes only the values, as the permutation.
__global__ void __launch_bounds__(kRadixThreads)
    k_radix_scatter(const float *__restrict__ score, const uint32_t *__restrict__ keys_in,
                    const uint32_t *__restrict__ vals_in, uint32_t *__restrict__ keys_out,
                    uint32_t *__restrict__ vals_out, int32_t *__restrict__ perm_out,
                    long long run_len, long long head_len, long long score_stride,
                    long long perm_stride, int tiles, int shift,
                    const int *__restrict__ counts) {
  extern __shared__ int sm_r[];
  uint32_t *skey = reinterpret_cast<uint32_t *>(sm_r);   // [tile]
  uint32_t *sval = skey + kRadixTile;                     // [tile]
  int *hist = reinterpret_cast<int *>(sval + kRadixTile);  // [warps·256]
  int *dbase = hist + (kRadixThreads / 32) * 256;          // [256]
  int *goff = dbase + 256;                                 // [256]
  int *dtot = goff + 256;                                  // [256]
  const long long run = blockIdx.x / tiles;
  const int tile = blockIdx.x % tiles;
  const long long base = run * run_len + (long long)tile * kRadixTile;
  const int n = (int)min((long long)kRadixTile, run_len - (long long)tile * kRadixTile);
  uint32_t key[kRadixR], val[kRadixR], dig[kRadixR];
  int dest[kRadixR];
  radix_load(score, keys_in, vals_in, run * score_stride + (long long)tile * kRadixTile, base,
             tile * kRadixTile, n, key, val);
  // Per digit d (threads 2d and 2d + 1, half of the tiles each): the run's total and the count in
  // tiles before this one; then the exclusive scan of the 256 totals.
  const unsigned full = 0xffffffffu;
  {
    const int d = threadIdx.x >> 1, half = threadIdx.x & 1;
    const int *c = counts + (run * 256 + d) * tiles;
    int tot = 0, pre = 0;
    if ((tiles & 7) == 0 && tiles <= 64) {  // 16-byte aligned halves of at most 32 counts
      const int per = tiles / 2, t0 = half * per;
      const int4 *c4 = reinterpret_cast<const int4 *>(c + t0);
      int4 v[8];
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (4 * k < per) v[k] = __ldg(c4 + k);
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (4 * k < per) {
          const int t = t0 + 4 * k;
          tot += v[k].x + v[k].y + v[k].z + v[k].w;
          pre += (t < tile ? v[k].x : 0) + (t + 1 < tile ? v[k].y : 0) +
                 (t + 2 < tile ? v[k].z : 0) + (t + 3 < tile ? v[k].w : 0);
        }
    } else {
      for (int t0 = half; t0 < tiles; t0 += 16) {  // eight loads in flight
        int v[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = t0 + 2 * k < tiles ? __ldg(c + t0 + 2 * k) : 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          tot += v[k];
          pre += t0 + 2 * k < tile ? v[k] : 0;
        }
      }
    }
    tot += __shfl_xor_sync(full, tot, 1);
    pre += __shfl_xor_sync(full, pre, 1);
    if (!half) {
      goff[d] = pre;
      dtot[d] = tot;
    }
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int v[8], s8 = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[i] = dtot[lane * 8 + i];
      s8 += v[i];
    }
    int incl = s8;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(full, incl, o);
      if (lane >= o) incl += t;
    }
    int run_sum = incl - s8;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      goff[lane * 8 + i] += run_sum;
      run_sum += v[i];
    }
  }
  // (radix_ranks synchronises the CTA before goff is read.)
#pragma unroll
  for (int r = 0; r < kRadixR; ++r) dig[r] = (key[r] >> shift) & 255u;
  radix_ranks<kRadixR, kRadixThreads / 32>(dig, dest, hist, dbase);
#pragma unroll
  for (int r = 0; r < kRadixR; ++r) {
    skey[dest[r]] = key[r];
    sval[dest[r]] = val[r];
  }
  __syncthreads();
  const long long out0 = run * run_len;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const uint32_t k = skey[i];
    const int d = (int)((k >> shift) & 255u);
    const long long at = goff[d] + (i - dbase[d]);
    if (perm_out)  // positions within the head: a run's first element sits at run·run_len mod N
      perm_out[run * perm_stride + at] = (int32_t)((run * run_len) % head_len + sval[i]);
    else {
      keys_out[out0 + at] = k;
      vals_out[out0 + at] = sval[i];
    }
  }
}

// ------------------------------------------------------------------ blocks and scores

// Block means over permuted blocks: out[(qh·nB + blk)] = MEAN(rows perm[blk·B .. blk·B+B-1]) of
// source head src_head(qh) (the query head itself, or its KV head when kv_map is set). One warp
// per block, D/32 columns per lane, the rows added in list order; row loads go out 16 at a time.
template <int D>
__global__ void __launch_bounds__(256)
    k_block_means(const uint16_t *__restrict__ src, const int32_t *__restrict__ perm,
                  float *__restrict__ out, int N, int B, int nB, long long n_blocks, int Hq,
                  int Hkv, int G, int kv_map) {
  constexpr int CPL = D / 32;  // columns per lane (4 or 2)
  using Vec = typename std::conditional<CPL == 4, uint2, uint32_t>::type;
  const long long blk = (long long)blockIdx.x * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (blk >= n_blocks) return;
  const long long qh = blk / nB;
  const int b = (int)(blk % nB);
  const long long sh = kv_map ? (qh / Hq) * Hkv + (qh % Hq) / G : qh;
  const int32_t *pp = perm + qh * N + (size_t)b * B;
  const Vec *base = reinterpret_cast<const Vec *>(src + (size_t)sh * N * D) + lane;
  float acc[CPL];
#pragma unroll
  for (int x = 0; x < CPL; ++x) acc[x] = 0.f;
  for (int e0 = 0; e0 < B; e0 += 32) {
    const int my_row = min(max(__ldg(pp + e0 + lane), 0), N - 1);
#pragma unroll
    for (int h = 0; h < 32; h += 16) {
      Vec v[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int row = __shfl_sync(0xffffffffu, my_row, h + e);
        v[e] = __ldg(base + (size_t)row * (D / CPL));
      }
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        if constexpr (CPL == 4) {
          const uint2 w = *reinterpret_cast<const uint2 *>(&v[e]);
          acc[0] = __fadd_rn(acc[0], bf16_lo(w.x));
          acc[1] = __fadd_rn(acc[1], bf16_hi(w.x));
          acc[2] = __fadd_rn(acc[2], bf16_lo(w.y));
          acc[3] = __fadd_rn(acc[3], bf16_hi(w.y));
        } else {
          const uint32_t w = *reinterpret_cast<const uint32_t *>(&v[e]);
          acc[0] = __fadd_rn(acc[0], bf16_lo(w));
          acc[1] = __fadd_rn(acc[1], bf16_hi(w));
        }
      }
    }
  }
  const float len = (float)B;
  float *dst = out + (size_t)blk * D + lane * CPL;
#pragma unroll
  for (int x = 0; x < CPL; ++x) dst[x] = __fdiv_rn(acc[x], len);
}

// n[qh][s][c] = number of keys of permuted key block c whose original index is below s·S.
__global__ void __launch_bounds__(256)
    k_ncount(const int32_t *__restrict__ perm_k, int32_t *__restrict__ n, int N, int B, int S,
             int nB, int nSeg) {
  extern __shared__ int seg_of[];  // [32][B + 1]
  const long long qh = blockIdx.y;
  const int c0 = blockIdx.x * 32;
  for (int x = threadIdx.x; x < 32 * B; x += blockDim.x) {
    const int cl = x / B, e = x % B, c = c0 + cl;
    seg_of[cl * (B + 1) + e] = c < nB ? __ldg(perm_k + qh * N + (size_t)c * B + e) / S : INT_MAX;
  }
  __syncthreads();
  const int cl = threadIdx.x % 32, c = c0 + cl;
  if (c >= nB) return;
  const int *mine = seg_of + cl * (B + 1);
  for (int s = threadIdx.x / 32; s < nSeg; s += blockDim.x / 32) {
    int cnt = 0;
    for (int e = 0; e < B; ++e) cnt += mine[e] < s;
    n[((size_t)qh * nSeg + s) * nB + c] = cnt;
  }
}

// r[qh][b][c] = DOT(Qbar_b, Kbar_c) × σ_d: a register-tiled fp32 product whose accumulators
// each run the definition's sequential FMA chain over t = 0..D-1. A 128×128 tile per CTA, 8×8
// accumulators per thread (paired FMAs); the operands go through shared memory transposed, 32
// values of t at a time. Two CTAs per SM overlap one's operand loads with the other's products
// (loading the next 32 values during the products instead measured slower: at 128 registers the
// extra live operands spill).
template <int D>
__global__ void __launch_bounds__(256, 2)
    k_block_scores(const float *__restrict__ Qbar, const float *__restrict__ Kbar,
                   float *__restrict__ r, int nB, float sigma) {
  __shared__ __align__(16) float As[32][128 + 4];
  __shared__ __align__(16) float Bs[32][128 + 4];
  const long long qh = blockIdx.z;
  const int b0 = blockIdx.y * 128, c0 = blockIdx.x * 128;
  const int tr = threadIdx.x / 16, tc = threadIdx.x % 16;
  const float *A = Qbar + (size_t)qh * nB * D;
  const float *Bm = Kbar + (size_t)qh * nB * D;
  // Loader mapping: 4 float4 per matrix per thread: row = x / 8, t = (x % 8) * 4.
  float4 pa[4], pb[4];
  auto fetch = [&](int t0) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int x = threadIdx.x + k * 256, row = x / 8, t = (x % 8) * 4;
      pa[k] = b0 + row < nB ? __ldg(reinterpret_cast<const float4 *>(A + (size_t)(b0 + row) * D + t0 + t))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
      pb[k] = c0 + row < nB ? __ldg(reinterpret_cast<const float4 *>(Bm + (size_t)(c0 + row) * D + t0 + t))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  auto stash = [&]() {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int x = threadIdx.x + k * 256, row = x / 8, t = (x % 8) * 4;
      As[t + 0][row] = pa[k].x;
      As[t + 1][row] = pa[k].y;
      As[t + 2][row] = pa[k].z;
      As[t + 3][row] = pa[k].w;
      Bs[t + 0][row] = pb[k].x;
      Bs[t + 1][row] = pb[k].y;
      Bs[t + 2][row] = pb[k].z;
      Bs[t + 3][row] = pb[k].w;
    }
  };
  float2 acc[8][4];  // acc[i][jj] holds columns 2jj and 2jj+1
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = make_float2(0.f, 0.f);
  for (int t0 = 0; t0 < D; t0 += 32) {
    fetch(t0);
    __syncthreads();  // the previous chunk has been consumed
    stash();
    __syncthreads();
#pragma unroll 8
    for (int tt = 0; tt < 32; ++tt) {
      const float4 a0 = *reinterpret_cast<const float4 *>(&As[tt][tr * 8]);
      const float4 a1 = *reinterpret_cast<const float4 *>(&As[tt][tr * 8 + 4]);
      const float4 v0 = *reinterpret_cast<const float4 *>(&Bs[tt][tc * 8]);
      const float4 v1 = *reinterpret_cast<const float4 *>(&Bs[tt][tc * 8 + 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float2 v[4] = {make_float2(v0.x, v0.y), make_float2(v0.z, v0.w),
                           make_float2(v1.x, v1.y), make_float2(v1.z, v1.w)};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j].x = __fmaf_rn(a[i], v[j].x, acc[i][j].x);
          acc[i][j].y = __fmaf_rn(a[i], v[j].y, acc[i][j].y);
        }
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int b = b0 + tr * 8 + i;
    if (b >= nB) continue;
    float *dst = r + ((size_t)qh * nB + b) * nB + c0 + tc * 8;
    // 16-byte stores need 16-byte aligned rows, i.e. nB a multiple of 4 (N/B need not be).
    if ((nB & 3) == 0 && c0 + tc * 8 + 8 <= nB) {
      reinterpret_cast<float4 *>(dst)[0] =
          make_float4(__fmul_rn(acc[i][0].x, sigma), __fmul_rn(acc[i][0].y, sigma),
                      __fmul_rn(acc[i][1].x, sigma), __fmul_rn(acc[i][1].y, sigma));
      reinterpret_cast<float4 *>(dst)[1] =
          make_float4(__fmul_rn(acc[i][2].x, sigma), __fmul_rn(acc[i][2].y, sigma),
                      __fmul_rn(acc[i][3].x, sigma), __fmul_rn(acc[i][3].y, sigma));
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float x = (j & 1) ? acc[i][j >> 1].y : acc[i][j >> 1].x;
        if (c0 + tc * 8 + j < nB) dst[j] = __fmul_rn(x, sigma);
      }
    }
  }
}

// ------------------------------------------------------------------ 4-bit key centroids (variant)

// Key-centroid codes per query head and channel t: lo = min_c K̄, step = (max − lo)/15 (1 if 0),
// code = clamp(rint((K̄ − lo)/step), 0, 15). One CTA per (query head, 32 channels): lane = channel,
// the 32 warps split the blocks for the min/max (exact in any order) and write the codes.
template <int D>
__global__ void __launch_bounds__(1024)
    k_kbar_codes(const float *__restrict__ Kbar, int8_t *__restrict__ kcode,
                 float *__restrict__ kstep, int nB) {
  __shared__ float smin[32][33], smax[32][33];
  const long long qh = blockIdx.y;
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  const int t = blockIdx.x * 32 + lane;
  const float *kb = Kbar + (size_t)qh * nB * D + t;
  float mn = kb[0], mx = kb[0];
  for (int c = warp; c < nB; c += 32) {
    const float x = kb[(size_t)c * D];
    mn = x < mn ? x : mn;
    mx = x > mx ? x : mx;
  }
  smin[warp][lane] = mn;
  smax[warp][lane] = mx;
  __syncthreads();
  mn = smin[0][lane];
  mx = smax[0][lane];
  for (int w = 1; w < 32; ++w) {
    mn = smin[w][lane] < mn ? smin[w][lane] : mn;
    mx = smax[w][lane] > mx ? smax[w][lane] : mx;
  }
  float step = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
  if (step == 0.0f) step = 1.0f;
  if (warp == 0) kstep[qh * D + t] = step;
  for (int c = warp; c < nB; c += 32) {
    const int code = __float2int_rn(__fdiv_rn(__fsub_rn(kb[(size_t)c * D], mn), step));
    kcode[((size_t)qh * nB + c) * D + t] = (int8_t)min(max(code, 0), 15);
  }
}

// Query-centroid codes per query block: a_t = Q̄_t × step_t, sq = max_t |a_t| / 127 (1 if 0),
// code = clamp(rint(a_t / sq), −127, 127). One warp per block.
template <int D>
__global__ void __launch_bounds__(256)
    k_qbar_codes(const float *__restrict__ Qbar, const float *__restrict__ kstep,
                 int8_t *__restrict__ qcode, float *__restrict__ qstep, int nB,
                 long long n_blocks) {
  const long long blk = (long long)blockIdx.x * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (blk >= n_blocks) return;
  const long long qh = blk / nB;
  float a[D / 32], m = 0.0f;
#pragma unroll
  for (int k = 0; k < D / 32; ++k) {
    const int t = lane + 32 * k;
    a[k] = __fmul_rn(Qbar[(size_t)blk * D + t], kstep[qh * D + t]);
    m = fmaxf(m, fabsf(a[k]));
  }
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float sq = __fdiv_rn(m, 127.0f);
  if (sq == 0.0f) sq = 1.0f;
  if (lane == 0) qstep[blk] = sq;
#pragma unroll
  for (int k = 0; k < D / 32; ++k) {
    const int code = __float2int_rn(__fdiv_rn(a[k], sq));
    qcode[(size_t)blk * D + lane + 32 * k] = (int8_t)min(max(code, -127), 127);
  }
}

// r[qh][b][c] = fp32(fp32(Σ_t qa_{b,t}·qK_{c,t}) × sq_b) × σ_d, the sum an exact integer (four
// codes per dp4a). A 128×128 tile per CTA, 8×8 outputs per thread; the code words are staged
// word-major (word w of every row of the tile contiguous) so that a thread reads its 8 rows' or
// columns' words with two 16-byte loads.
template <int D>
__global__ void __launch_bounds__(256)
    k_block_scores_i8(const int8_t *__restrict__ qcode, const int8_t *__restrict__ kcode,
                      const float *__restrict__ qstep, float *__restrict__ r, int nB,
                      float sigma) {
  constexpr int W = D / 4;  // 32-bit words per row
  __shared__ __align__(16) int As[W][128];
  __shared__ __align__(16) int Bs[W][128];
  const long long qh = blockIdx.z;
  const int b0 = blockIdx.y * 128, c0 = blockIdx.x * 128;
  const int tr = threadIdx.x / 16, tc = threadIdx.x % 16;
  const int *qa = reinterpret_cast<const int *>(qcode + (size_t)qh * nB * D);
  const int *qk = reinterpret_cast<const int *>(kcode + (size_t)qh * nB * D);
  for (int x = threadIdx.x; x < 128 * (W / 4); x += blockDim.x) {
    const int row = x / (W / 4), w0 = (x % (W / 4)) * 4;
    const int4 va = b0 + row < nB
                        ? *reinterpret_cast<const int4 *>(qa + (size_t)(b0 + row) * W + w0)
                        : make_int4(0, 0, 0, 0);
    const int4 vb = c0 + row < nB
                        ? *reinterpret_cast<const int4 *>(qk + (size_t)(c0 + row) * W + w0)
                        : make_int4(0, 0, 0, 0);
    As[w0][row] = va.x;
    As[w0 + 1][row] = va.y;
    As[w0 + 2][row] = va.z;
    As[w0 + 3][row] = va.w;
    Bs[w0][row] = vb.x;
    Bs[w0 + 1][row] = vb.y;
    Bs[w0 + 2][row] = vb.z;
    Bs[w0 + 3][row] = vb.w;
  }
  __syncthreads();
  int acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0;
#pragma unroll 4
  for (int w = 0; w < W; ++w) {
    const int4 a0 = *reinterpret_cast<const int4 *>(&As[w][tr * 8]);
    const int4 a1 = *reinterpret_cast<const int4 *>(&As[w][tr * 8 + 4]);
    const int4 v0 = *reinterpret_cast<const int4 *>(&Bs[w][tc * 8]);
    const int4 v1 = *reinterpret_cast<const int4 *>(&Bs[w][tc * 8 + 4]);
    const int a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    const int v[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = __dp4a(a[i], v[j], acc[i][j]);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int b = b0 + tr * 8 + i;
    if (b >= nB) continue;
    const float sq = qstep[(size_t)qh * nB + b];
    float *dst = r + ((size_t)qh * nB + b) * nB + c0 + tc * 8;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (c0 + tc * 8 + j < nB)
        dst[j] = __fmul_rn(__fmul_rn(__int2float_rn(acc[i][j]), sq), sigma);
  }
}

// ------------------------------------------------------------------ scheduling (step 4 order)

__device__ __forceinline__ bool goes_before(double pa, int ca, double pb, int cb) {
  return pa > pb || (pa == pb && ca < cb);
}

// a[i] for a register array and a run-time index, by a tree of selects (no local memory).
__device__ __forceinline__ double pick32(const double (&a)[32], int i) {
  double l1[16], l2[8], l3[4], l4[2];
#pragma unroll
  for (int j = 0; j < 16; ++j) l1[j] = (i & 1) ? a[2 * j + 1] : a[2 * j];
#pragma unroll
  for (int j = 0; j < 8; ++j) l2[j] = (i & 2) ? l1[2 * j + 1] : l1[2 * j];
#pragma unroll
  for (int j = 0; j < 4; ++j) l3[j] = (i & 4) ? l2[2 * j + 1] : l2[2 * j];
#pragma unroll
  for (int j = 0; j < 2; ++j) l4[j] = (i & 8) ? l3[2 * j + 1] : l3[2 * j];
  return (i & 16) ? l4[1] : l4[0];
}

// Block scheduling: for each query block the local tile count, the normalised block scores p
// over its candidate blocks, the selection p >= τ, and the selected list sorted by
// (p descending, block ascending).
// A group of GL lanes (a power of two; 32/GL query blocks per warp) serves one query block. Lane l
// of the group owns the chunks k = l + GL·h (h < CPL) of 32 consecutive blocks: it sums a chunk's
// weights sequentially in block order, keeping them in registers until the selection (they are
// recomputed when it owns two chunks), and Z adds the chunk sums in chunk order. Shared memory per
// query block holds only the selected list (cap2 entries; cap2 bounds the list length: at most
// floor(1/τ) + 1 blocks can reach p >= τ since the p sum to one).
template <int CPL>
__global__ void __launch_bounds__(128)
    k_schedule(const float *__restrict__ r, const int32_t *__restrict__ ncount,
               const int32_t *__restrict__ perm_q, int32_t *__restrict__ sel_cnt,
               int32_t *__restrict__ sel_blk, int32_t *__restrict__ local_tiles, int N, int B,
               int S, int nB, int nSeg, int cap2, int GL, double tau, long long n_qblocks) {
  extern __shared__ unsigned char smem_raw[];
  const int lane = threadIdx.x % kWarp, li = lane & (GL - 1), gi = threadIdx.x / GL;
  const long long per_cta = blockDim.x / GL;
  const long long qb = (long long)blockIdx.x * per_cta + gi;
  // A warp whose first query block is past the end has nothing to do; inside a warp every lane
  // takes part in the shuffles, and a group past the end works on block 0 and writes nothing.
  if ((long long)blockIdx.x * per_cta + (threadIdx.x & ~(kWarp - 1)) / GL >= n_qblocks) return;
  const bool real = qb < n_qblocks;
  const long long q0 = real ? qb : 0;
  const size_t per_q = ((size_t)cap2 * 12 + 15) & ~(size_t)15;
  double *lp = reinterpret_cast<double *>(smem_raw + per_q * gi);
  int *lc = reinterpret_cast<int *>(lp + cap2);
  const unsigned full = 0xffffffffu;

  const long long qh = q0 / nB;
  const int b = (int)(q0 % nB);
  const int s = (int)((long long)b * B / S);

  int mx = -1;
  for (int e = li; e < B; e += GL) mx = max(mx, __ldg(perm_q + qh * N + (size_t)b * B + e));
  for (int o = GL / 2; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(full, mx, o, GL));
  if (real && li == 0) local_tiles[qb] = (mx - s * S) / B + 1;

  const float *rr = r + (size_t)q0 * nB;
  const int32_t *nn = ncount + ((size_t)qh * nSeg + s) * nB;
  // Rows start 16-byte aligned when nB is a multiple of 4 (the arrays themselves are).
  const bool vec = (nB & 3) == 0;
  const int n_chunks = (nB + 31) / 32;
  int nv[32];
  float rv[32];
  // Counts and scores of this lane's chunk h (zeros past nB).
  auto load_chunk = [&](int h) {
    const int c0 = 32 * (li + GL * h);
    if (vec && c0 + 32 <= nB) {
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        const int4 n4 = __ldg(reinterpret_cast<const int4 *>(nn + c0) + v);
        const float4 r4 = __ldg(reinterpret_cast<const float4 *>(rr + c0) + v);
        nv[4 * v] = n4.x, nv[4 * v + 1] = n4.y, nv[4 * v + 2] = n4.z, nv[4 * v + 3] = n4.w;
        rv[4 * v] = r4.x, rv[4 * v + 1] = r4.y, rv[4 * v + 2] = r4.z, rv[4 * v + 3] = r4.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int c = c0 + i;
        nv[i] = c < nB ? __ldg(nn + c) : 0;
        rv[i] = c < nB ? __ldg(rr + c) : 0.f;
      }
    }
  };

  // M = max block score over the candidates (blocks with a visible key). A query block with no
  // candidate runs the steps below with no weights and ends with an empty list.
  float M = 0.f;
  bool any = false;
#pragma unroll
  for (int h = 0; h < CPL; ++h) {
    load_chunk(h);
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (nv[i] > 0) {
        M = any ? fmaxf(M, rv[i]) : rv[i];
        any = true;
      }
  }
  for (int o = GL / 2; o > 0; o >>= 1) {
    const float other = __shfl_xor_sync(full, M, o, GL);
    const bool other_any = __shfl_xor_sync(full, any ? 1 : 0, o, GL) != 0;
    if (other_any) M = any ? fmaxf(M, other) : other;
    any = any || other_any;
  }
  const double Md = (double)M;

  // Weights of the loaded chunk (-1 marks a block that is not a candidate).
  double wk[32];
  auto weights = [&]() {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const double e =
          __dmul_rn(int_to_double(max(nv[i], 0)), exp64(__dsub_rn((double)rv[i], Md)));
      wk[i] = nv[i] > 0 ? e : -1.0;
    }
  };
  // Z: each chunk summed sequentially from +0 in block order (a non-candidate adds +0), then the
  // chunk sums in chunk order.
  double part[CPL];
#pragma unroll
  for (int h = 0; h < CPL; ++h) {
    if (CPL > 1) load_chunk(h);
    weights();
    double acc = 0.0;
#pragma unroll
    for (int i = 0; i < 32; ++i) acc = __dadd_rn(acc, wk[i] < 0.0 ? 0.0 : wk[i]);
    part[h] = acc;
  }
  double Z = 0.0;
#pragma unroll
  for (int h = 0; h < CPL; ++h)
    for (int k = 0; k < GL && GL * h + k < n_chunks; ++k)
      Z = __dadd_rn(Z, __shfl_sync(full, part[h], k, GL));

  // Selection p_c = w_c / Z >= τ. A weight below (τ·Z)(1 − 2^-48) gives p < τ whatever the
  // rounding, so its division is skipped; every other candidate's p is computed exactly. The
  // selected blocks go to the list in block order (the lanes of a group own consecutive chunks),
  // their p computed again when written.
  const double t_lo = __dmul_rn(__dmul_rn(tau, Z), 1.0 - 0x1p-48);
  int cnt = 0;
#pragma unroll
  for (int h = 0; h < CPL; ++h) {
    if (CPL > 1) {
      load_chunk(h);
      weights();
    }
    unsigned near = 0, mine = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (wk[i] >= 0.0 && (tau == 0.0 || !(wk[i] < t_lo))) near |= 1u << i;
    for (unsigned m = near; m; m &= m - 1) {
      const int i = __ffs(m) - 1;
      if (__ddiv_rn(pick32(wk, i), Z) >= tau) mine |= 1u << i;
    }
    const int n_mine = __popc(mine);
    int incl = n_mine;
    for (int o = 1; o < GL; o <<= 1) {
      const int t = __shfl_up_sync(full, incl, o, GL);
      if (li >= o) incl += t;
    }
    int slot = cnt + incl - n_mine;
    cnt += __shfl_sync(full, incl, GL - 1, GL);
    for (unsigned m = mine; m; m &= m - 1, ++slot) {
      const int i = __ffs(m) - 1;
      if (slot < cap2) {
        lp[slot] = __ddiv_rn(pick32(wk, i), Z);
        lc[slot] = 32 * (li + GL * h) + i;
      }
    }
  }
  __syncwarp();
  cnt = min(cnt, cap2);
  // Bitonic network over the warp's largest power of two Pw >= every group's count (lists padded
  // with entries that go after every block), order "goes_before".
  int Pw = 1;
  while (Pw < cnt) Pw <<= 1;
  for (int o = 16; o > 0; o >>= 1) Pw = max(Pw, __shfl_xor_sync(full, Pw, o));
  for (int e = cnt + li; e < Pw; e += GL) {
    lp[e] = -1.0;
    lc[e] = INT_MAX;
  }
  __syncwarp();
  for (int k = 2; k <= Pw; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = li; i < Pw; i += GL) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const bool up = (i & k) == 0;
          const bool after = goes_before(lp[ixj], lc[ixj], lp[i], lc[i]);
          if (after == up) {
            const double tp = lp[i];
            const int tcb = lc[i];
            lp[i] = lp[ixj];
            lc[i] = lc[ixj];
            lp[ixj] = tp;
            lc[ixj] = tcb;
          }
        }
      }
      __syncwarp();
    }
  }
  if (real) {
    int32_t *dst = sel_blk + (size_t)qb * nB;
    for (int e = li; e < cnt; e += GL) dst[e] = lc[e];
    if (li == 0) sel_cnt[qb] = cnt;
  }
}

// ------------------------------------------------------------------ validation and stats

__global__ void k_validate_perms(const int32_t *__restrict__ perm_q,
                                 const int32_t *__restrict__ perm_k,
                                 unsigned *__restrict__ seen_q, unsigned *__restrict__ seen_k,
                                 int N, int S, long long total, unsigned *__restrict__ flag) {
  const long long x = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (x >= total) return;
  const long long qh = x / N;
  const int slot = (int)(x % N);
  const int s0 = (slot / S) * S;
  const int iq = perm_q[x], ik = perm_k[x];
  if (iq < s0 || iq >= s0 + S) {
    atomicOr(flag, 1u);
  } else {
    const long long bit = qh * N + iq;
    if (atomicOr(seen_q + bit / 32, 1u << (bit % 32)) & (1u << (bit % 32))) atomicOr(flag, 2u);
  }
  if (ik < 0 || ik >= N) {
    atomicOr(flag, 4u);
  } else {
    const long long bit = qh * N + ik;
    if (atomicOr(seen_k + bit / 32, 1u << (bit % 32)) & (1u << (bit % 32))) atomicOr(flag, 8u);
  }
}

// One warp per query block: list length, block ids in range and unique, local tile count in
// range and covering the block's last query (when perm_q is in range).
__global__ void __launch_bounds__(128)
    k_validate_lists(const int32_t *__restrict__ perm_q, const int32_t *__restrict__ sel_cnt,
                     const int32_t *__restrict__ sel_blk, const int32_t *__restrict__ local_tiles,
                     int N, int B, int S, int nB, long long n_qblocks, unsigned *__restrict__ flag) {
  extern __shared__ unsigned bits[];  // per warp: (nB + 31) / 32 words
  const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
  const long long qb = (long long)blockIdx.x * (blockDim.x / kWarp) + warp;
  if (qb >= n_qblocks) return;
  const int words = (nB + 31) / 32;
  unsigned *mine = bits + warp * words;
  for (int e = lane; e < words; e += kWarp) mine[e] = 0u;
  __syncwarp();
  const long long qh = qb / nB;
  const int b = (int)(qb % nB);
  const int s0 = (int)((long long)b * B / S) * S;
  const int cnt = sel_cnt[qb];
  if (cnt < 0 || cnt > nB) {
    if (lane == 0) atomicOr(flag, 16u);
  } else {
    for (int e = lane; e < cnt; e += kWarp) {
      const int c = sel_blk[qb * nB + e];
      if (c < 0 || c >= nB) {
        atomicOr(flag, 32u);
      } else if (atomicOr(mine + c / 32, 1u << (c % 32)) & (1u << (c % 32))) {
        atomicOr(flag, 64u);
      }
    }
  }
  int mx = -1;
  for (int e = lane; e < B; e += kWarp) mx = max(mx, perm_q[qh * N + (size_t)b * B + e]);
  for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) {
    const int lt = local_tiles[qb];
    if (lt < 1 || lt > S / B) atomicOr(flag, 128u);
    if (mx >= s0 && mx < s0 + S && lt < (mx - s0) / B + 1) atomicOr(flag, 256u);
  }
}

// acc[0] += Σ lt, acc[1] += Σ cnt, acc[2] += Σ_i |K_i| (local keys plus visible keys of the
// listed blocks), one warp per query block.
__global__ void __launch_bounds__(128)
    k_stats(const int32_t *__restrict__ perm_q, const int32_t *__restrict__ perm_k,
            const int32_t *__restrict__ sel_cnt, const int32_t *__restrict__ sel_blk,
            const int32_t *__restrict__ local_tiles, int N, int B, int S, int nB,
            long long n_qblocks, unsigned long long *__restrict__ acc) {
  const int warp = threadIdx.x / kWarp, lane = threadIdx.x % kWarp;
  const long long qb = (long long)blockIdx.x * (blockDim.x / kWarp) + warp;
  if (qb >= n_qblocks) return;
  const long long qh = qb / nB;
  const int b = (int)(qb % nB);
  const int s0 = (int)((long long)b * B / S) * S;
  const int cnt = min(max(sel_cnt[qb], 0), nB);
  unsigned long long local_pairs = 0, visible = 0;
  for (int e = lane; e < B; e += kWarp) local_pairs += perm_q[qh * N + (size_t)b * B + e] - s0 + 1;
  for (int x = 0; x < cnt; ++x) {
    const int c = min(max(sel_blk[qb * nB + x], 0), nB - 1);
    for (int e = lane; e < B; e += kWarp) visible += perm_k[qh * N + (size_t)c * B + e] < s0;
  }
  for (int o = 16; o > 0; o >>= 1) {
    local_pairs += __shfl_xor_sync(0xffffffffu, local_pairs, o);
    visible += __shfl_xor_sync(0xffffffffu, visible, o);
  }
  if (lane == 0) {
    atomicAdd(acc + 0, (unsigned long long)local_tiles[qb]);
    atomicAdd(acc + 1, (unsigned long long)cnt);
    atomicAdd(acc + 2, local_pairs + visible * (unsigned long long)B);
  }
}

__global__ void k_exp64_probe(const double *x, double *y, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) y[i] = exp64(x[i]);
}

inline unsigned blocks_for(long long n, int per) { return (unsigned)((n + per - 1) / per); }

// Stable radix sort of runs of run_len scores each (descending, ties to the lower index), the
// permutation written to perm_out as positions within a head of head_len elements (a run of
// segment length S starts at its segment's first position). Run r's scores start at
// score + r·score_stride and its permutation at perm_out + r·perm_stride (both default to
// run_len). Keys and values ping-pong between (k0, v0) and (k1, v1).
cudaError_t radix_sort_runs(const float *score, uint32_t *k0, uint32_t *v0, uint32_t *k1,
                            uint32_t *v1, int *counts, long long total, long long run_len,
                            long long head_len, int32_t *perm_out, cudaStream_t st,
                            long long score_stride = 0, long long perm_stride = 0) {
  if (score_stride <= 0) score_stride = run_len;
  if (perm_stride <= 0) perm_stride = run_len;
  const int tiles = (int)((run_len + kRadixTile - 1) / kRadixTile);
  const long long runs = total / run_len;
  const unsigned grid = (unsigned)(runs * tiles);
  const size_t smem = (size_t)2 * kRadixTile * 4 + (size_t)(kRadixThreads / 32) * 256 * 4 + 768 * 4;
  cudaError_t e = cudaFuncSetAttribute(k_radix_scatter, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const uint32_t *kin = nullptr, *vin = nullptr;
  uint32_t *kout = k0, *vout = v0;
  for (int pass = 0; pass < 4; ++pass) {
    const float *sc = pass == 0 ? score : nullptr;
    k_radix_count<<<grid, kRadixThreads, 0, st>>>(sc, kin, run_len, score_stride, tiles,
                                                  8 * pass, counts);
    note_launch();
    k_radix_scatter<<<grid, kRadixThreads, smem, st>>>(sc, kin, vin, kout, vout,
                                                       pass == 3 ? perm_out : nullptr, run_len,
                                                       head_len, score_stride, perm_stride,
                                                       tiles, 8 * pass, counts);
    note_launch();
    kin = kout;
    vin = vout;
    kout = kout == k0 ? k1 : k0;
    vout = vout == v0 ? v1 : v0;
  }
  return cudaGetLastError();
}

// A second stream of the calling thread on the current device, for kernels that are independent
// of the caller's stream between a fork and a join (both by events). Created on first use, kept
// for the thread's lifetime.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork_ev = nullptr, join_ev = nullptr;
};

cudaError_t side_stream(SideStream **out) {
  thread_local SideStream cache[16];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 16) return cudaErrorInvalidDevice;
  SideStream &ss = cache[dev];
  if (!ss.s) {
    if ((e = cudaStreamCreateWithFlags(&ss.s, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&ss.fork_ev, cudaEventDisableTiming)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&ss.join_ev, cudaEventDisableTiming)) != cudaSuccess) return e;
  }
  *out = &ss;
  return cudaSuccess;
}

template <int D>
cudaError_t build_d(const Dims &d, const s2o_config &cfg, const uint16_t *q, const uint16_t *k,
                    const s2o_indices &out, char *ws, cudaStream_t st) {
  const WsLayout L = ws_layout(d);
  float *qchunk = reinterpret_cast<float *>(ws + L.qchunk);
  float *kchunk = reinterpret_cast<float *>(ws + L.kchunk);
  float *qbar = reinterpret_cast<float *>(ws + L.qbar);
  float *kbar_all = reinterpret_cast<float *>(ws + L.kbar_all);
  float *kbar_top = reinterpret_cast<float *>(ws + L.kbar_top);
  float *u = reinterpret_cast<float *>(ws + L.u);
  float *kappa = reinterpret_cast<float *>(ws + L.kappa);
  float *rho = reinterpret_cast<float *>(ws + L.rho);
  // Radix sort buffers: keys and values of two ping-pong copies, digit counts.
  uint32_t *rk0 = reinterpret_cast<uint32_t *>(ws + L.keys0), *rv0 = rk0 + d.bhq() * d.N;
  uint32_t *rk1 = reinterpret_cast<uint32_t *>(ws + L.keys1), *rv1 = rk1 + d.bhq() * d.N;
  int *rcount = reinterpret_cast<int *>(ws + L.radix);
  float *Qbar = reinterpret_cast<float *>(ws + L.Qbar);
  float *Kbar = reinterpret_cast<float *>(ws + L.Kbar);
  float *r = reinterpret_cast<float *>(ws + L.r);
  int32_t *ncount = reinterpret_cast<int32_t *>(ws + L.ncount);

  const long long bhq = d.bhq(), bhkv = d.bhkv();
  const long long nq = bhq * d.N;
  cudaError_t e;

  // Step 1a: mean query per query head; one pass over K for kappa and the mean key per KV head.
  k_pool_chunks<D><<<blocks_for(nq / d.B * (D / 2), 256), 256, 0, st>>>(q, qchunk, d.B, nq / d.B);
  note_launch();
  const size_t fin_smem = (size_t)1024 * 32 * sizeof(float);
  if ((e = cudaFuncSetAttribute(k_pool_finish<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)fin_smem)) != cudaSuccess)
    return e;
  k_pool_finish<D><<<dim3(D / 32, (unsigned)bhq), 256, fin_smem, st>>>(qchunk, qbar, d.nB,
                                                                       (float)d.N);
  note_launch();
  const size_t kpass_smem = (size_t)d.G * D * sizeof(float) + (size_t)d.B * (D * 2 + 16);
  if ((e = cudaFuncSetAttribute(k_kpass<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kpass_smem)) != cudaSuccess)
    return e;
  const int shared_order = cfg.shared_key_order && d.G > 1 ? 1 : 0;
  k_kpass<D><<<dim3((unsigned)d.nB, (unsigned)bhkv), 128, kpass_smem, st>>>(
      k, qbar, kappa, kchunk, d.N, d.B, d.Hq, d.Hkv, d.G, shared_order);
  note_launch();
  k_pool_finish<D><<<dim3(D / 32, (unsigned)bhkv), 256, fin_smem, st>>>(kchunk, kbar_all, d.nB,
                                                                         (float)d.N);
  note_launch();
  // Step 2a: global key/value ordering.
  if (shared_order) {
    // One ordering per KV head (sorted from the group's first query-head rows), copied to the
    // other rows of the group.
    const long long gstride = (long long)d.G * d.N;
    if ((e = radix_sort_runs(kappa, rk0, rv0, rk1, rv1, rcount, bhkv * d.N, d.N, d.N, out.perm_k,
                             st, gstride, gstride)) != cudaSuccess)
      return e;
    const unsigned rep_x = std::min(blocks_for(d.N / 4, 256), 64u);
    k_replicate_group_rows<<<dim3(rep_x, (unsigned)bhkv), 256, 0, st>>>(out.perm_k, d.N, d.G);
    note_launch();
  } else if ((e = radix_sort_runs(kappa, rk0, rv0, rk1, rv1, rcount, nq, d.N, d.N, out.perm_k,
                                  st)) != cudaSuccess) {
    return e;
  }
  // Key side of step 2c (block means K̄ and visibility counts): they depend only on perm_k and
  // run on a side stream next to the query-side kernels, joined before the block scores.
  const long long nblk = bhq * d.nB;
  SideStream *side = nullptr;
  if ((e = side_stream(&side)) != cudaSuccess) return e;
  if ((e = cudaEventRecord(side->fork_ev, st)) != cudaSuccess) return e;
  if ((e = cudaStreamWaitEvent(side->s, side->fork_ev, 0)) != cudaSuccess) return e;
  k_block_means<D><<<blocks_for(nblk, 8), 256, 0, side->s>>>(k, out.perm_k, Kbar, d.N, d.B, d.nB,
                                                             nblk, d.Hq, d.Hkv, d.G, 1);
  note_launch();
  const size_t nc_smem = (size_t)32 * (d.B + 1) * sizeof(int);
  k_ncount<<<dim3((d.nB + 31) / 32, (unsigned)bhq), 256, nc_smem, side->s>>>(
      out.perm_k, ncount, d.N, d.B, d.S, d.nB, d.nSeg);
  note_launch();
  if ((e = cudaEventRecord(side->join_ev, side->s)) != cudaSuccess) return e;
  // The caller's stream waits for the side stream on every path out of this function.
  struct Join {
    cudaStream_t st;
    cudaEvent_t ev;
    bool pending = true;
    cudaError_t now() {
      pending = false;
      return cudaStreamWaitEvent(st, ev, 0);
    }
    ~Join() {
      if (pending) cudaStreamWaitEvent(st, ev, 0);
    }
  } join{st, side->join_ev};
  // Step 1b: query scores against the top stripe block.
  k_kbar_top<<<(unsigned)bhq, D, 0, st>>>(k, out.perm_k, kbar_all, kbar_top, u, d.N, D, d.B, d.Hq,
                                          d.Hkv, d.G);
  note_launch();
  // Step 2b: query scores, segment-local query ordering, query block means.
  const int qp = cfg.query_perm ? 1 : 0;
  const dim3 seg_grid((unsigned)d.nSeg, (unsigned)bhq);
  if (qp && d.S <= 16 * kFuseNT) {
    // One fused launch per (query head, segment).
    auto fused = [&](auto kernel, int R) -> cudaError_t {
      const size_t smem = fused_order_smem<D, kFuseNT>(R);
      cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
      if (err != cudaSuccess) return err;
      kernel<<<seg_grid, kFuseNT, smem, st>>>(q, u, rho, out.perm_q, Qbar, d.N, d.S, d.B, d.nB);
      return cudaSuccess;
    };
    if ((e = d.S <= kFuseNT       ? fused(k_rho_order_means<D, 1, kFuseNT>, 1)
             : d.S <= 2 * kFuseNT ? fused(k_rho_order_means<D, 2, kFuseNT>, 2)
             : d.S <= 4 * kFuseNT ? fused(k_rho_order_means<D, 4, kFuseNT>, 4)
             : d.S <= 8 * kFuseNT ? fused(k_rho_order_means<D, 8, kFuseNT>, 8)
                                  : fused(k_rho_order_means<D, 16, kFuseNT>, 16)) != cudaSuccess)
      return e;
    note_launch();
  } else {
    if (qp) {
      k_rho<D><<<dim3((d.N + 127) / 128, (unsigned)bhq), 128, 0, st>>>(q, u, rho, d.N);
      note_launch();
    }
    if (d.S <= 4096 || !qp) {
      auto seg = [&](auto kernel, int R) -> cudaError_t {
        const size_t smem = (size_t)2 * 512 * R * 4 + 16 * 256 * 4 + 256 * 4;
        cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)smem);
        if (err != cudaSuccess) return err;
        kernel<<<seg_grid, 512, smem, st>>>(rho, out.perm_q, d.N, d.S, qp);
        return cudaSuccess;
      };
      if ((e = d.S <= 512    ? seg(k_segment_sort<1>, 1)
               : d.S <= 1024 ? seg(k_segment_sort<2>, 2)
               : d.S <= 2048 ? seg(k_segment_sort<4>, 4)
                             : seg(k_segment_sort<8>, 8)) != cudaSuccess)
        return e;
      note_launch();
    } else {
      // Segments longer than one CTA's sort: the multi-CTA radix sort over runs of S.
      if ((e = radix_sort_runs(rho, rk0, rv0, rk1, rv1, rcount, nq, d.S, d.N, out.perm_q, st)) !=
          cudaSuccess)
        return e;
    }
    k_block_means<D><<<blocks_for(nblk, 8), 256, 0, st>>>(q, out.perm_q, Qbar, d.N, d.B, d.nB,
                                                          nblk, d.Hq, d.Hkv, d.G, 0);
    note_launch();
  }
  // Block scores (after the key side joins).
  if ((e = join.now()) != cudaSuccess) return e;
  const float sigma = D == 64 ? 0x1p-3f : 0x1.6a09e6p-4f;  // nearest fp32 to 1/sqrt(D)
  const unsigned tiles = (unsigned)((d.nB + 127) / 128);
  if (cfg.int4_centroids) {
    // Codes in the radix key buffer (free once the orderings are built).
    int8_t *kcode = reinterpret_cast<int8_t *>(rk0);
    int8_t *qcode = kcode + (size_t)bhq * d.nB * D;
    float *kstep = reinterpret_cast<float *>(qcode + (size_t)bhq * d.nB * D);
    float *qstep = kstep + (size_t)bhq * D;
    k_kbar_codes<D><<<dim3(D / 32, (unsigned)bhq), 1024, 0, st>>>(Kbar, kcode, kstep, d.nB);
    note_launch();
    k_qbar_codes<D><<<blocks_for(nblk, 8), 256, 0, st>>>(Qbar, kstep, qcode, qstep, d.nB, nblk);
    note_launch();
    k_block_scores_i8<D><<<dim3(tiles, tiles, (unsigned)bhq), 256, 0, st>>>(qcode, kcode, qstep,
                                                                             r, d.nB, sigma);
    note_launch();
  } else {
    k_block_scores<D><<<dim3(tiles, tiles, (unsigned)bhq), 256, 0, st>>>(Qbar, Kbar, r, d.nB,
                                                                         sigma);
    note_launch();
  }
  // Scheduling. The selected list of a query block holds at most floor(1/τ) + 1 entries.
  int cap = d.nB;
  if (cfg.tau > 0.f) {
    const double bound = std::floor(1.0 / (double)cfg.tau) + 2.0;
    if (bound < (double)cap) cap = (int)bound;
  }
  int cap2 = 1;
  while (cap2 < cap) cap2 <<= 1;
  // Lanes per query block: the chunks of 32 blocks rounded up to a power of two, at most 32 (two
  // chunks per lane beyond 1024 blocks; check_config caps nB at 2048).
  const int n_chunks = (d.nB + 31) / 32;
  int GL = 1;
  while (GL < n_chunks && GL < 32) GL <<= 1;
  const size_t per_q = ((size_t)cap2 * 12 + 15) & ~(size_t)15;
  const int sched_threads = 128;
  const size_t sched_smem = per_q * (size_t)(sched_threads / GL);
  auto sched = n_chunks <= 32 ? k_schedule<1> : k_schedule<2>;
  if ((e = cudaFuncSetAttribute(sched, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)sched_smem)) != cudaSuccess)
    return e;
  sched<<<blocks_for(nblk, sched_threads / GL), sched_threads, sched_smem, st>>>(
      r, ncount, out.perm_q, out.sel_cnt, out.sel_blk, out.local_tiles, d.N, d.B, d.S, d.nB,
      d.nSeg, cap2, GL, (double)cfg.tau, nblk);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_build_indices(const Dims &d, const s2o_config &cfg, const uint16_t *q,
                                 const uint16_t *k, const s2o_indices &out, char *ws,
                                 cudaStream_t st) {
  return d.D == 64 ? build_d<64>(d, cfg, q, k, out, ws, st) : build_d<128>(d, cfg, q, k, out, ws, st);
}

cudaError_t launch_validate(const Dims &d, const s2o_indices &idx, char *ws, uint32_t *flag_dev,
                            cudaStream_t st) {
  const WsLayout L = ws_layout(d);
  const long long total = d.bhq() * d.N;
  const size_t words = (size_t)((total + 31) / 32);
  unsigned *seen_q = reinterpret_cast<unsigned *>(ws + L.keys0);
  unsigned *seen_k = seen_q + words;
  cudaError_t e;
  if ((e = cudaMemsetAsync(seen_q, 0, 2 * words * sizeof(unsigned), st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(flag_dev, 0, sizeof(uint32_t), st)) != cudaSuccess) return e;
  k_validate_perms<<<blocks_for(total, 256), 256, 0, st>>>(idx.perm_q, idx.perm_k, seen_q, seen_k,
                                                           d.N, d.S, total, flag_dev);
  note_launch();
  const long long nblk = d.bhq() * d.nB;
  const size_t smem = (size_t)4 * ((d.nB + 31) / 32) * sizeof(unsigned);
  k_validate_lists<<<blocks_for(nblk, 4), 128, smem, st>>>(idx.perm_q, idx.sel_cnt, idx.sel_blk,
                                                           idx.local_tiles, d.N, d.B, d.S, d.nB,
                                                           nblk, flag_dev);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_stats(const Dims &d, const s2o_indices &idx, unsigned long long *acc_dev,
                         cudaStream_t st) {
  cudaError_t e;
  if ((e = cudaMemsetAsync(acc_dev, 0, 3 * sizeof(unsigned long long), st)) != cudaSuccess)
    return e;
  const long long nblk = d.bhq() * d.nB;
  k_stats<<<blocks_for(nblk, 4), 128, 0, st>>>(idx.perm_q, idx.perm_k, idx.sel_cnt, idx.sel_blk,
                                               idx.local_tiles, d.N, d.B, d.S, d.nB, nblk,
                                               acc_dev);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_exp64_probe(const double *x, double *y, int n, cudaStream_t st) {
  k_exp64_probe<<<blocks_for(n, 256), 256, 0, st>>>(x, y, n);
  note_launch();
  return cudaGetLastError();
}

}  // namespace s2o
