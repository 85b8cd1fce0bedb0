// bf16 GEMM with fp32 accumulation on the 5th-generation tensor cores (tcgen05 + TMEM + TMA), for
// the projections of the decoder layer around the attention (the end-to-end-shaped prefill of the
// S2O card's Key points: Llama-3.1-8B at 128K).
//
// C[m, n] = A[m, k] · B[k, n] (+ C[m, n] when accumulating), all row-major bf16, the sum in fp32
// and rounded to bf16 once (the residual adds into the same rounding). Two kernels; the call takes
// the CTA-pair kernel further below for n and k up to 8192, this one otherwise (and for a single
// tile). One persistent CTA per SM, 192 threads, 256 × 256 output tiles:
//   warp 0      TMA producer: per K step of 64, the A tile (256 rows × 64, K-major, one 128-byte
//               swizzled box) and the B tile (64 × 256, N-major: four {64, 64} boxes, one per
//               64-column atom) into a 3-stage ring.
//   warp 1      MMA issuer (one elected thread): per stage, four tcgen05.mma kind::f16 (M = 128,
//               N = 256, K = 16) for each 128-row half of the tile, both halves reading the same
//               B tile, into two TMEM accumulators of 256 fp32 columns (all 512 columns). A tile's
//               first products of a half wait until the epilogue has read that half of the previous
//               tile.
//   warps 2-5   epilogue: the thread of TMEM lane r owns row r of each half, reads 32 columns at a
//               time with tcgen05.ld, adds the old C when accumulating, rounds to bf16 and stores
//               64 bytes per row and chunk; it frees each half as soon as it has read it.
// Per stage the two halves share the B tile: 64 KB of loads per 8.4 MFLOP (131 FLOP per byte from
// L2), against 87 with a single 128-row half.
// Tiles are walked in groups of 32 row tiles per column tile, so a group's A panels and the B
// panel in use stay in L2. Every wait is bounded by %globaltimer (the same limit as the attention
// kernel); on a timeout the kernel records it in its error word, drains its copies and products,
// frees TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "s2o_internal.h"

namespace s2o {

__device__ unsigned int g_gemm_error;

namespace {

constexpr int kBM = 256, kHalf = 128, kBN = 256, kBK = 64, kStages = 3, kThreadsG = 192,
              kGroupM = 16;
constexpr uint32_t kABytes = kBM * kBK * 2;     // 32 KB: 256 rows × 128 bytes
constexpr uint32_t kAHalf = kHalf * kBK * 2;    // 16 KB: one 128-row half
constexpr uint32_t kBAtom = kBK * 128;          // 8 KB: 64 k-rows × 64 columns
constexpr uint32_t kBBytes = (kBN / 64) * kBAtom;  // 32 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t kOffBar = kStages * kStageBytes;  // 192 KB of stages
constexpr uint32_t kSmem = kOffBar + 256 + 1024;    // barriers + alignment slack
constexpr uint32_t kTmemCols = 512;                 // one accumulator of 256 columns per half
constexpr uint64_t kDrainNs = 2000000000ull;

// Barrier slots: full[3], empty[3], acc_full, acc_empty[2] (one per half), drain.
enum { kFull = 0, kEmpty = 3, kAccFull = 6, kAccEmpty = 7, kDrainBar = 9, kBars = 10 };

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint32_t a, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(a), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t a, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(a), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t a) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(a) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t a, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(a), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __noinline__ bool mbar_wait_slow(uint32_t a, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(a, parity)) return true;
    if (globaltimer_ns() - t0 > limit_ns) {
      atomicOr(&g_gemm_error, 1u);
      return false;
    }
  }
}
// True once the phase of the given parity has completed; false (recorded in the error word) if it
// has not after limit_ns nanoseconds.
__device__ __forceinline__ bool mbar_wait(uint32_t a, uint32_t parity, uint64_t limit_ns) {
  return mbar_try_wait(a, parity) || mbar_wait_slow(a, parity, limit_ns);
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *tm, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
// Four K = 16 products of one stage into one accumulator (A and B from shared memory); the first
// accumulates only if `acc0` is set.
__device__ __forceinline__ void mma4(uint32_t d, uint32_t idesc, const uint64_t (&a)[4],
                                     const uint64_t (&b)[4], uint32_t acc0) {
  asm volatile(
      "{\n\t.reg .pred p0, p1;\n\t"
      "setp.ne.b32 p0, %10, 0;\n\t"
      "setp.eq.b32 p1, %0, %0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %2, %6, %1, p0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %7, %1, p1;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %4, %8, %1, p1;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %5, %9, %1, p1;\n\t}\n" ::"r"(d),
      "r"(idesc), "l"(a[0]), "l"(a[1]), "l"(a[2]), "l"(a[3]), "l"(b[0]), "l"(b[1]), "l"(b[2]),
      "l"(b[3]), "r"(acc0)
      : "memory");
}
// 32 TMEM lanes × 32 consecutive 32-bit columns; thread t of the warp receives lane (base + t).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
        "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
        "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]),
        "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]),
        "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])::"memory");
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// UMMA shared-memory descriptor, 128-byte swizzle (as in the attention kernel): start address,
// leading byte offset (atom stride along the contiguous dimension for MN-major operands), stride
// byte offset 1024 (eight 128-byte rows), version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo_bytes) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)(1024u >> 4) << 32) | (1ull << 46) | (2ull << 61);
}
__host__ __device__ constexpr uint32_t idesc_bf16(int m, int n, int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

struct GemmParams {
  uint16_t *c;
  int m, n, k;
  int m_tiles, n_tiles, k_steps;
  long long tiles;
  int accumulate;
  unsigned long long limit_ns;
};

// Tile t in grouped order: kGroupM row tiles per column tile, the column tile fastest within a
// group's rows... (row tile, column tile).
__device__ __forceinline__ void tile_coords(const GemmParams &g, long long t, int &tm, int &tn) {
  const long long per_group = (long long)kGroupM * g.n_tiles;
  const long long grp = t / per_group;
  const int first = (int)(grp * kGroupM);
  const int rows = min(kGroupM, g.m_tiles - first);
  const long long r = t - grp * per_group;
  tn = (int)(r / rows);
  tm = first + (int)(r % rows);
}

__global__ void __launch_bounds__(kThreadsG, 1)
    k_gemm_bf16(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                const GemmParams g) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem), sBar = sbase + kOffBar;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffBar + kBars * 8);
  auto bar = [&](int i) { return sBar + 8u * (uint32_t)i; };
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(kFull + s), 1);
      mbar_init(bar(kEmpty + s), 1);
    }
    mbar_init(bar(kAccFull), 1);
    for (int h = 0; h < 2; ++h) mbar_init(bar(kAccEmpty + h), 4);  // one arrival per epilogue warp
    mbar_init(bar(kDrainBar), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint64_t lim = g.limit_ns;
  bool ok = true;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    long long it = 0;  // stages filled so far
    for (long long t = blockIdx.x; ok && t < g.tiles; t += gridDim.x) {
      int tm, tn;
      tile_coords(g, t, tm, tn);
      for (int ks = 0; ks < g.k_steps; ++ks, ++it) {
        const int st = (int)(it % kStages);
        if (it >= kStages) {
          bool got = true;
          if (lane == 0) got = mbar_wait(bar(kEmpty + st), (uint32_t)(((it / kStages) - 1) & 1), lim);
          if (!__shfl_sync(0xffffffffu, got, 0)) {
            ok = false;
            break;
          }
        }
        if (lane == 0) {
          const uint32_t a_dst = sbase + st * kStageBytes, b_dst = a_dst + kABytes;
          mbar_expect_tx(bar(kFull + st), kStageBytes);
          tma_load_2d(a_dst, &tm_a, ks * kBK, tm * kBM, bar(kFull + st));
          for (int at = 0; at < kBN / 64; ++at)
            tma_load_2d(b_dst + at * kBAtom, &tm_b, tn * kBN + at * 64, ks * kBK, bar(kFull + st));
        }
        __syncwarp();
      }
    }
    // Drain: the last fill of each stage lands before the CTA exits.
    if (lane == 0)
      for (int st = 0; st < kStages; ++st) {
        if (it <= st) continue;
        const long long last = st + ((it - 1 - st) / kStages) * kStages;
        mbar_wait(bar(kFull + st), (uint32_t)((last / kStages) & 1), kDrainNs);
      }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdesc = idesc_bf16(kHalf, kBN, 0, 1);
      long long it = 0;
      int tcount = 0;
      for (long long t = blockIdx.x; ok && t < g.tiles; t += gridDim.x, ++tcount) {
        for (int ks = 0; ks < g.k_steps; ++ks, ++it) {
          const int st = (int)(it % kStages);
          if (!mbar_wait(bar(kFull + st), (uint32_t)((it / kStages) & 1), lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_s = sbase + st * kStageBytes, b_s = a_s + kABytes;
          const uint64_t bd = sw128_desc(b_s, kBAtom);
          // K steps of 16: A advances 32 bytes inside its 128-byte rows, B 16 rows of 128 bytes.
          const uint64_t b4[4] = {bd, bd + 128, bd + 256, bd + 384};
          for (int h = 0; h < 2; ++h) {
            // A half's first products of a tile wait until the epilogue has read that half of
            // the previous tile.
            if (ks == 0 && tcount > 0) {
              if (!mbar_wait(bar(kAccEmpty + h), (uint32_t)((tcount - 1) & 1), lim)) {
                ok = false;
                break;
              }
              tc_fence_after();
            }
            const uint64_t ad = sw128_desc(a_s + h * kAHalf, 16);
            const uint64_t a4[4] = {ad, ad + 2, ad + 4, ad + 6};
            mma4(tmem + (uint32_t)(h * kBN), kIdesc, a4, b4, ks > 0 ? 1u : 0u);
          }
          if (!ok) break;
          tc_commit(bar(kEmpty + st));
        }
        if (!ok) break;
        tc_commit(bar(kAccFull));
      }
      // Drain: every product issued above completes before TMEM is freed.
      tc_commit(bar(kDrainBar));
      mbar_wait(bar(kDrainBar), 0, kDrainNs);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue
    const int quad = warp & 3;  // TMEM lane quarter this warp may read
    const int row = quad * 32 + lane;
    int tcount = 0;
    for (long long t = blockIdx.x; ok && t < g.tiles; t += gridDim.x, ++tcount) {
      int tm, tn;
      tile_coords(g, t, tm, tn);
      if (!__all_sync(0xffffffffu, mbar_wait(bar(kAccFull), (uint32_t)(tcount & 1), lim))) {
        ok = false;
        break;
      }
      tc_fence_after();
      for (int h = 0; h < 2; ++h) {
        const long long grow = (long long)tm * kBM + h * kHalf + row;
        const bool in_row = grow < g.m;
        uint16_t *crow = g.c + grow * g.n + (long long)tn * kBN;
        const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(h * kBN);
#pragma unroll 1
        for (int c0 = 0; c0 < kBN; c0 += 32) {
          uint32_t v[32];
          tmem_ld32(taddr + c0, v);
          const int col = tn * kBN + c0;
          uint32_t ow[16];  // the old C values of the chunk as bf16 pairs (accumulating)
          const bool full = in_row && col + 32 <= g.n;
          if (g.accumulate && full) {
            const uint4 *src = reinterpret_cast<const uint4 *>(crow + c0);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 o4 = src[q];
              ow[4 * q] = o4.x;
              ow[4 * q + 1] = o4.y;
              ow[4 * q + 2] = o4.z;
              ow[4 * q + 3] = o4.w;
            }
          }
          tmem_wait_ld(v);
          if (full) {
            uint4 outv[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                float lo = __uint_as_float(v[q * 8 + 2 * e]), hi = __uint_as_float(v[q * 8 + 2 * e + 1]);
                if (g.accumulate) {
                  lo += __uint_as_float(ow[4 * q + e] << 16);
                  hi += __uint_as_float(ow[4 * q + e] & 0xffff0000u);
                }
                w[e] = pack_bf16(lo, hi);
              }
              outv[q] = make_uint4(w[0], w[1], w[2], w[3]);
            }
            uint4 *dst = reinterpret_cast<uint4 *>(crow + c0);
#pragma unroll
            for (int q = 0; q < 4; ++q) dst[q] = outv[q];
          } else if (in_row) {
            // Ragged column tail: element by element.
            for (int e = 0; e < 32 && col + e < g.n; ++e) {
              float x = __uint_as_float(v[e]);
              if (g.accumulate) x += __uint_as_float((uint32_t)crow[c0 + e] << 16);
              crow[c0 + e] = (uint16_t)(pack_bf16(x, 0.f) & 0xffffu);
            }
          }
        }
        // This warp has read its lanes of this half's accumulator: the issuer may reuse it.
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kAccEmpty + h));
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

// ------------------------------------------------------------------ the CTA-pair kernel
//
// The same product on pairs of SMs (a cluster of two CTAs, tcgen05 cta_group::2): a pair computes
// 256 × 256 output tiles with M = 256, N = 256 products; CTA r of the pair holds rows 128r..128r+127
// of the A tile and columns 128r..128r+127 of the B tile in its shared memory (the tensor core reads
// both CTAs' halves), and accumulates its 128 rows × 256 columns in its own TMEM. Each CTA loads
// 32 KB per K step of 64 (131 FLOP per byte, as the single-CTA tile), and the accumulator takes 256
// of the 512 TMEM columns, so two alternate: the epilogue of one tile overlaps the next tile's
// products. Roles per CTA (192 threads): warp 0 loads the CTA's halves (TMA, 128-byte swizzle,
// no multicast) into a 6-stage ring; warp 1 of the first CTA (the leader) issues the products;
// warps 2-5 run the epilogue of the CTA's rows. Between the two CTAs: the peer's tile loads
// complete on the leader's stage barrier (the cta_group::2 form of the TMA load); the leader's
// commits of a stage release and of a finished accumulator arrive on the barrier at the same
// offset in both CTAs (the commit's cluster form; no load is multicast); every epilogue warp of
// both CTAs releases an accumulator with a plain arrival on the leader's barrier. Every wait is
// bounded by %globaltimer.
constexpr int kPH = 128, kPNh = 128, kPStages = 6;
constexpr uint32_t kPA = kPH * kBK * 2;         // 16 KB: this CTA's 128 rows of A
constexpr uint32_t kPB = (kPNh / 64) * kBAtom;  // 16 KB: this CTA's 128 columns of B
constexpr uint32_t kPStage = kPA + kPB;
constexpr uint32_t kPOffBar = kPStages * kPStage;  // 192 KB of stages
constexpr uint32_t kPSmem = kPOffBar + 256 + 1024;
// Barrier slots: full[stages] (used on the leader), empty[stages], acc_full[2], acc_empty[2]
// (leader), drain.
constexpr int kPFull = 0, kPEmpty = kPStages, kPAccFull = 2 * kPStages,
              kPAccEmpty = 2 * kPStages + 2, kPDrain = 2 * kPStages + 4, kPBars = 2 * kPStages + 5;
static_assert(kPBars * 8 + 4 <= 256, "barrier area");

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// The address in CTA `rank` of the cluster of the shared-memory word at local address a.
__device__ __forceinline__ uint32_t map_to_cta(uint32_t a, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t a, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(a), "r"(parity)
      : "memory");
  return ok != 0;
}
// A wait that also orders with arrivals from the other CTA of the pair; false (recorded in the
// error word) after limit_ns.
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t a, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait_cluster(a, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait_cluster(a, parity)) return true;
    if (globaltimer_ns() - t0 > limit_ns) {
      atomicOr(&g_gemm_error, 1u);
      return false;
    }
  }
}
// TMA tile load into this CTA's shared memory whose completion is counted on a barrier of either
// CTA of the pair (cluster address).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *tm, int x, int y,
                                                 uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(bar_cluster)
      : "memory");
}
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
// The same completion signalled on the barrier at this offset in both CTAs of the pair (a commit,
// not a memory load).
__device__ __forceinline__ void tc_commit_pair_both(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"((uint16_t)3)
      : "memory");
}
// Four K = 16 products of one stage, M = 256 over the CTA pair; the first accumulates only if
// `acc0` is set.
__device__ __forceinline__ void mma4_pair(uint32_t d, uint32_t idesc, const uint64_t (&a)[4],
                                          const uint64_t (&b)[4], uint32_t acc0) {
  asm volatile(
      "{\n\t.reg .pred p0, p1;\n\t"
      "setp.ne.b32 p0, %10, 0;\n\t"
      "setp.eq.b32 p1, %0, %0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %2, %6, %1, p0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %3, %7, %1, p1;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %4, %8, %1, p1;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %5, %9, %1, p1;\n\t}\n" ::"r"(d),
      "r"(idesc), "l"(a[0]), "l"(a[1]), "l"(a[2]), "l"(a[3]), "l"(b[0]), "l"(b[1]), "l"(b[2]),
      "l"(b[3]), "r"(acc0)
      : "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

__global__ void __launch_bounds__(kThreadsG, 1)
    k_gemm_bf16_pair(const __grid_constant__ CUtensorMap tm_a,
                     const __grid_constant__ CUtensorMap tm_b, const GemmParams g) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem), sBar = sbase + kPOffBar;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kPOffBar + kPBars * 8);
  auto bar = [&](int i) { return sBar + 8u * (uint32_t)i; };
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const long long pair = blockIdx.x / 2, n_pairs = gridDim.x / 2;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kPStages; ++s) {
      mbar_init(bar(kPFull + s), 1);
      mbar_init(bar(kPEmpty + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(kPAccFull + b), 1);
      mbar_init(bar(kPAccEmpty + b), 8);  // one arrival per epilogue warp of both CTAs
    }
    mbar_init(bar(kPDrain), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    // Both CTAs of the pair allocate together (the same columns in each).
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync_all();  // barriers initialised and TMEM allocated in both CTAs
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint64_t lim = g.limit_ns;
  bool ok = true;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA loads (both CTAs)
    long long it = 0;
    if (lane == 0) {
      for (long long t = pair; ok && t < g.tiles; t += n_pairs) {
        int tm, tn;
        tile_coords(g, t, tm, tn);
        for (int ks = 0; ks < g.k_steps; ++ks, ++it) {
          const int st = (int)(it % kPStages);
          if (it >= kPStages) {
            if (!mbar_wait_cluster(bar(kPEmpty + st), (uint32_t)(((it / kPStages) - 1) & 1), lim)) {
              ok = false;
              break;
            }
          }
          const uint32_t a_dst = sbase + st * kPStage, b_dst = a_dst + kPA;
          const int row = tm * kBM + (int)rank * kPH, col = tn * kBN + (int)rank * kPNh;
          if (leader) {
            mbar_expect_tx(bar(kPFull + st), 2 * kPStage);  // both CTAs' halves
            tma_load_2d(a_dst, &tm_a, ks * kBK, row, bar(kPFull + st));
            for (int at = 0; at < kPNh / 64; ++at)
              tma_load_2d(b_dst + at * kBAtom, &tm_b, col + at * 64, ks * kBK, bar(kPFull + st));
          } else {
            const uint32_t fb = map_to_cta(bar(kPFull + st), 0);
            tma_load_2d_pair(a_dst, &tm_a, ks * kBK, row, fb);
            for (int at = 0; at < kPNh / 64; ++at)
              tma_load_2d_pair(b_dst + at * kBAtom, &tm_b, col + at * 64, ks * kBK, fb);
          }
        }
      }
      // Drain (leader): the last fill of each stage, both halves, lands before the pair exits.
      if (leader)
        for (int st = 0; st < kPStages; ++st) {
          if (it <= st) continue;
          const long long last = st + ((it - 1 - st) / kPStages) * kPStages;
          mbar_wait_cluster(bar(kPFull + st), (uint32_t)((last / kPStages) & 1), kDrainNs);
        }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (leader)
    if (leader && lane == 0) {
      constexpr uint32_t kIdesc = idesc_bf16(2 * kPH, kBN, 0, 1);
      long long it = 0;
      int tc = 0;
      for (long long t = pair; ok && t < g.tiles; t += n_pairs, ++tc) {
        const int b = tc & 1;
        if (tc >= 2) {
          if (!mbar_wait_cluster(bar(kPAccEmpty + b), (uint32_t)(((tc >> 1) - 1) & 1), lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        const uint32_t d = tmem + (uint32_t)(b * kBN);
        for (int ks = 0; ks < g.k_steps; ++ks, ++it) {
          const int st = (int)(it % kPStages);
          if (!mbar_wait_cluster(bar(kPFull + st), (uint32_t)((it / kPStages) & 1), lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_s = sbase + st * kPStage, b_s = a_s + kPA;
          const uint64_t ad = sw128_desc(a_s, 16), bd = sw128_desc(b_s, kBAtom);
          const uint64_t a4[4] = {ad, ad + 2, ad + 4, ad + 6};
          const uint64_t b4[4] = {bd, bd + 128, bd + 256, bd + 384};
          mma4_pair(d, kIdesc, a4, b4, ks > 0 ? 1u : 0u);
          tc_commit_pair_both(bar(kPEmpty + st));  // frees the stage in both CTAs
        }
        if (!ok) break;
        tc_commit_pair_both(bar(kPAccFull + b));  // both CTAs' epilogues
      }
      tc_commit_pair(bar(kPDrain));
      mbar_wait_cluster(bar(kPDrain), 0, kDrainNs);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue (both CTAs)
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t acc_empty_leader = map_to_cta(bar(kPAccEmpty), 0);
    int tc = 0;
    for (long long t = pair; ok && t < g.tiles; t += n_pairs, ++tc) {
      const int b = tc & 1;
      int tm, tn;
      tile_coords(g, t, tm, tn);
      if (!__all_sync(0xffffffffu,
                      mbar_wait_cluster(bar(kPAccFull + b), (uint32_t)((tc >> 1) & 1), lim))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const long long grow = (long long)tm * kBM + (long long)rank * kPH + row;
      const bool in_row = grow < g.m;
      uint16_t *crow = g.c + grow * g.n + (long long)tn * kBN;
      const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(b * kBN);
#pragma unroll 1
      for (int c0 = 0; c0 < kBN; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(taddr + c0, v);
        const int col = tn * kBN + c0;
        uint32_t ow[16];
        const bool full = in_row && col + 32 <= g.n;
        if (g.accumulate && full) {
          const uint4 *src = reinterpret_cast<const uint4 *>(crow + c0);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 o4 = src[q];
            ow[4 * q] = o4.x;
            ow[4 * q + 1] = o4.y;
            ow[4 * q + 2] = o4.z;
            ow[4 * q + 3] = o4.w;
          }
        }
        tmem_wait_ld(v);
        if (c0 + 32 == kBN) {
          // The whole accumulator of this warp's lanes is read: release it to the issuer.
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(acc_empty_leader + 8u * (uint32_t)b);
        }
        if (full) {
          uint4 outv[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float lo = __uint_as_float(v[q * 8 + 2 * e]), hi = __uint_as_float(v[q * 8 + 2 * e + 1]);
              if (g.accumulate) {
                lo += __uint_as_float(ow[4 * q + e] << 16);
                hi += __uint_as_float(ow[4 * q + e] & 0xffff0000u);
              }
              w[e] = pack_bf16(lo, hi);
            }
            outv[q] = make_uint4(w[0], w[1], w[2], w[3]);
          }
          uint4 *dst = reinterpret_cast<uint4 *>(crow + c0);
#pragma unroll
          for (int q = 0; q < 4; ++q) dst[q] = outv[q];
        } else if (in_row) {
          for (int e = 0; e < 32 && col + e < g.n; ++e) {
            float x = __uint_as_float(v[e]);
            if (g.accumulate) x += __uint_as_float((uint32_t)crow[c0 + e] << 16);
            crow[c0 + e] = (uint16_t)(pack_bf16(x, 0.f) & 0xffffu);
          }
        }
      }
    }
  }
  // Neither CTA leaves while the other may still signal its barriers or read its shared memory.
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

PFN_cuTensorMapEncodeTiled_v12000 gemm_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D bf16 map over a row-major [rows, cols] matrix with a {64, box_rows} box, 128-byte swizzle.
bool gemm_map(CUtensorMap *m, const void *base, long long rows, long long cols, int box_rows) {
  auto fn = gemm_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int gemm_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

}  // namespace

cudaError_t launch_gemm_bf16(const void *A, const void *B, void *C, long long m, long long n,
                             long long k, bool accumulate, uint64_t limit_ns, cudaStream_t st) {
  if (m <= 0 || n <= 0 || k <= 0 || n % 8 || k % 8 || m >= (1ll << 31) || n >= (1ll << 31) ||
      k >= (1ll << 31))
    return cudaErrorInvalidValue;
  static_assert(kSmem <= 232448 && kPSmem <= 232448, "shared memory budget");
  GemmParams g;
  g.c = static_cast<uint16_t *>(C);
  g.m = (int)m;
  g.n = (int)n;
  g.k = (int)k;
  g.m_tiles = (int)((m + kBM - 1) / kBM);
  g.n_tiles = (int)((n + kBN - 1) / kBN);
  g.k_steps = (int)((k + kBK - 1) / kBK);
  g.tiles = (long long)g.m_tiles * g.n_tiles;
  g.accumulate = accumulate ? 1 : 0;
  g.limit_ns = limit_ns;
  cudaError_t e;
  // The CTA pair measured faster for N and K up to 8192 (1.29-1.34 against 1.04-1.29 PFLOP/s at
  // the decoder layer's q/k/v and output shapes); above that (N = 28672, K = 14336) its 74
  // concurrent tiles span more row panels than L2 holds and the single-CTA kernel is faster.
  if (n <= 8192 && k <= 8192 && g.tiles >= 2) {
    CUtensorMap ta, tb;
    if (!gemm_map(&ta, A, m, k, kPH) || !gemm_map(&tb, B, k, n, kBK)) return cudaErrorInvalidValue;
    if ((e = cudaFuncSetAttribute(k_gemm_bf16_pair, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kPSmem)) != cudaSuccess)
      return e;
    // A persistent grid of CTA pairs: as many pairs as fit at once (one CTA per SM), at most one
    // per tile.
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(kThreadsG);
    cfg.dynamicSmemBytes = kPSmem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3((unsigned)(2 * (gemm_sm_count() / 2)));
    int max_pairs = 0;
    if ((e = cudaOccupancyMaxActiveClusters(&max_pairs, k_gemm_bf16_pair, &cfg)) != cudaSuccess)
      return e;
    if (max_pairs <= 0) return cudaErrorLaunchOutOfResources;
    const long long pairs = std::min<long long>(g.tiles, max_pairs);
    cfg.gridDim = dim3((unsigned)(2 * pairs));
    e = cudaLaunchKernelEx(&cfg, k_gemm_bf16_pair, ta, tb, g);
    note_launch();
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  CUtensorMap ta, tb;
  if (!gemm_map(&ta, A, m, k, kBM) || !gemm_map(&tb, B, k, n, kBK)) return cudaErrorInvalidValue;
  if ((e = cudaFuncSetAttribute(k_gemm_bf16, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kSmem)) != cudaSuccess)
    return e;
  const long long grid = std::min<long long>(g.tiles, gemm_sm_count());
  k_gemm_bf16<<<(unsigned)grid, kThreadsG, kSmem, st>>>(ta, tb, g);
  note_launch();
  return cudaGetLastError();
}

cudaError_t read_and_clear_gemm_error(unsigned int *out, cudaStream_t st) {
  cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_gemm_error, sizeof(unsigned int), 0,
                                            cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return e;
  if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return e;
  if (*out) {
    const unsigned int zero = 0;
    if ((e = cudaMemcpyToSymbolAsync(g_gemm_error, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice,
                                     st)) != cudaSuccess)
      return e;
    e = cudaStreamSynchronize(st);
  }
  return e;
}

}  // namespace s2o
