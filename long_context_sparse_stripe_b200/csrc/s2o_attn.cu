// Fused gather-attention of S2O on sm_100a (tcgen05 tensor cores, TMEM accumulators, TMA).
//
// Sources: "S2O: Early Stopping for Sparse Attention via Online Permutation" (research card),
// Summary ¶2: the kernel fetches scattered tokens into on-chip memory through the index arrays
// and runs key blocks from most to least important, stopping at τ (the stop is already folded
// into the per-query-block list length); causality stays on original positions. The attention
// itself is Eq. (1) of "AB-Sparse" restricted to the selected key set, computed flash-style with
// an online softmax (the normaliser of Milakov & Gimelshein, cited by the S2O paper).
//
// One CTA owns one (batch, query head, query block) work item: 128 query rows (the block's B rows
// gathered by perm_q; rows B..127 are zero when B = 64). It runs lt local tiles (contiguous keys of
// the block's own segment, mask key <= query) and then the cnt selected key blocks (keys gathered
// by perm_k, mask key < segment start). Warp roles (256 threads):
//   warp 0  K producer: Q once, then K tiles into a 3-deep ring (TMA tile loads for contiguous
//           tiles, TMA tile::gather4 for gathered rows; 128-byte swizzle).
//   warp 1  MMA issuer: owns TMEM; S = Q·Kᵀ into one of two TMEM S buffers, O += P·V into TMEM.
//   warp 2  V producer: V tiles into a 2-deep ring.
//   warp 3  idle.
//   warps 4-7 softmax: thread r owns query row r (TMEM lane r): masks, online max/sum in the exp2
//           domain, conditional rescale of O (only when the running max grows by more than 2^8),
//           P as bf16 into a 128B-swizzled shared tile, and the final O/ℓ store at original rows.
// Every wait is bounded (globaltimer); on a timeout the kernel records it, drains its own TMA
// copies and tensor-core work, frees TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "s2o_internal.h"

namespace s2o {

__device__ unsigned int g_device_error;

namespace {

constexpr int kThreads = 256;
constexpr int kM = 128;  // query rows per CTA (UMMA M)
constexpr uint64_t kDrainNs = 2000000000ull;

// ------------------------------------------------------------------ PTX wrappers

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
      atomicOr(&g_device_error, 1u);
      return false;
    }
  }
}
// True once the phase of the given parity has completed; false (recorded in the device error
// word) if it has not after limit_ns nanoseconds.
__device__ __forceinline__ bool mbar_wait(uint32_t a, uint32_t parity, uint64_t limit_ns) {
  return mbar_try_wait(a, parity) || mbar_wait_slow(a, parity, limit_ns);
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tma_load_tile(uint32_t dst, const CUtensorMap *tm, int x, int y,
                                              uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tma_gather4(uint32_t dst, const CUtensorMap *tm, int x, int y0,
                                            int y1, int y2, int y3, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y0), "r"(y1), "r"(y2), "r"(y3), "r"(bar)
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
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
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
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
// Waits for this thread's tcgen05.ld results; the register operands make every later use of
// the loaded values depend on the wait.
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
        "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
        "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]),
        "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]),
        "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])::"memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// UMMA shared-memory descriptor for a 128-byte-swizzled operand: start address, leading byte
// offset (atom stride along the contiguous dimension for MN-major operands; unused for K-major),
// stride byte offset 1024 (eight 128-byte rows), descriptor version 1, layout SWIZZLE_128B.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo_bytes) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)(1024u >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of tcgen05.mma kind::f16: bf16 A and B, fp32 accumulate, M×N tile,
// A and B K-major unless the MN-major flag is set.
__host__ __device__ constexpr uint32_t idesc_bf16(int m, int n, int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

// ------------------------------------------------------------------ layout

template <int D, int BN>
struct Layout {
  static constexpr int KST = 3, VST = 2;
  static constexpr uint32_t ATOM_Q = kM * 128;  // bytes of one 64-column atom of a 128-row tile
  static constexpr uint32_t ATOM_KV = BN * 128;
  static constexpr uint32_t Q_BYTES = kM * D * 2;
  static constexpr uint32_t KV_BYTES = BN * D * 2;
  static constexpr uint32_t P_BYTES = kM * BN * 2;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + KST * KV_BYTES;
  static constexpr uint32_t OFF_P = OFF_V + VST * KV_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_P + P_BYTES;
  static constexpr uint32_t BAR_BYTES = 256;
  static constexpr uint32_t SMEM = OFF_BAR + BAR_BYTES + 1024;  // + alignment slack
  static constexpr uint32_t COLS_NEEDED = 2 * BN + D;
  static constexpr uint32_t TMEM_COLS = COLS_NEEDED <= 256 ? 256 : 512;
  static constexpr uint32_t S_COL = 0, O_COL = 2 * BN;
};

// Barrier slots (8 bytes each) inside the barrier area.
enum Bar {
  kQFull = 0,
  kKFull = 1,    // 3
  kKEmpty = 4,   // 3
  kVFull = 7,    // 2
  kVEmpty = 9,   // 2
  kSFull = 11,   // 2
  kSFree = 13,   // 2
  kPFull = 15,
  kPVDone = 16,
  kDrain = 17,
  kNumBars = 18
};

struct Params {
  const int32_t *perm_q, *perm_k, *sel_cnt, *sel_blk, *local_tiles;
  uint16_t *o;
  int N, S, nB, nSeg, Hq, Hkv, G;
  int dense;
  float scale_log2;  // log2(e) / sqrt(d)
  unsigned long long limit_ns;
};

struct Work {
  long long qh, kh;  // flat (batch, query head) and (batch, kv head)
  int b, s, lt, cnt;
  const int32_t *sel;  // the query block's selected list (sel_blk row)
};

// Work item order: S2O groups the CTAs of one (batch, KV head, segment) together so that the
// segment's K/V tiles and the group's gathered rows stay in L2; the dense baseline runs the
// longest query blocks first.
template <int BN>
__device__ __forceinline__ Work decode_work(const Params &p) {
  Work w;
  long long item = blockIdx.x;
  const int hi = (int)(item % p.G);
  item /= p.G;
  const int per_seg = p.S / BN;
  int b, g;
  long long beta;
  if (p.dense) {
    b = p.nB - 1 - (int)(item % p.nB);
    item /= p.nB;
  } else {
    const int bl = (int)(item % per_seg);
    item /= per_seg;
    const int s = (int)(item % p.nSeg);
    item /= p.nSeg;
    b = s * per_seg + bl;
  }
  g = (int)(item % p.Hkv);
  beta = item / p.Hkv;
  w.qh = beta * p.Hq + (long long)g * p.G + hi;
  w.kh = beta * p.Hkv + g;
  w.b = b;
  w.s = (int)((long long)b * BN / p.S);
  if (p.dense) {
    w.lt = b + 1;
    w.cnt = 0;
    w.sel = nullptr;
  } else {
    const long long qb = w.qh * p.nB + b;
    w.lt = min(max(__ldg(p.local_tiles + qb), 1), per_seg);
    w.cnt = p.sel_cnt ? min(max(__ldg(p.sel_cnt + qb), 0), p.nB) : 0;
    w.sel = p.sel_blk + qb * p.nB;
  }
  return w;
}

__device__ __forceinline__ int selected_block(const Work &w, const Params &p, int j) {
  return min(max(__ldg(w.sel + (j - w.lt)), 0), p.nB - 1);
}

// ------------------------------------------------------------------ the kernel

template <int D, int BN>
__global__ void __launch_bounds__(kThreads, 1)
    s2o_attention_kernel(const __grid_constant__ CUtensorMap tm_q_tile,
                         const __grid_constant__ CUtensorMap tm_q_row,
                         const __grid_constant__ CUtensorMap tm_k_tile,
                         const __grid_constant__ CUtensorMap tm_k_row,
                         const __grid_constant__ CUtensorMap tm_v_tile,
                         const __grid_constant__ CUtensorMap tm_v_row, const Params p) {
  using L = Layout<D, BN>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + L::OFF_Q, sK = sbase + L::OFF_K, sV = sbase + L::OFF_V,
                 sP = sbase + L::OFF_P, sBar = sbase + L::OFF_BAR;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::OFF_BAR + kNumBars * 8);
  auto bar = [&](int i) { return sBar + 8u * (uint32_t)i; };

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const Work w = decode_work<BN>(p);
  const int T = w.lt + w.cnt;
  const int seg0 = w.s * p.S;  // first original position of the block's segment

  if (threadIdx.x == 0) {
    mbar_init(bar(kQFull), 1);
    for (int i = 0; i < L::KST; ++i) {
      mbar_init(bar(kKFull + i), 1);
      mbar_init(bar(kKEmpty + i), 1);
    }
    for (int i = 0; i < L::VST; ++i) {
      mbar_init(bar(kVFull + i), 1);
      mbar_init(bar(kVEmpty + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kSFull + i), 1);
      mbar_init(bar(kSFree + i), 128);
    }
    mbar_init(bar(kPFull), 128);
    mbar_init(bar(kPVDone), 1);
    mbar_init(bar(kDrain), 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(L::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (BN < kM && warp >= 4) {
    // Rows BN..127 of the Q tile are padding: zero them (the TMA writes rows 0..BN-1).
    const int row = threadIdx.x - 128;
    if (row >= BN) {
      for (int a = 0; a < D / 64; ++a) {
        uint4 *dst = reinterpret_cast<uint4 *>(smem + L::OFF_Q + a * L::ATOM_Q + row * 128);
        for (int c = 0; c < 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
      }
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const uint64_t lim = p.limit_ns;
  bool ok = true;

  if (warp == 0) {
    // ---------------------------------------------------------------- K producer (+ Q)
    int issued = 0;
    if (lane == 0) mbar_expect_tx(bar(kQFull), BN * D * 2);
    __syncwarp();
    const int q_row0 = (int)(w.qh * p.N);
    if (p.dense || p.perm_q == nullptr) {
      if (lane == 0)
        for (int a = 0; a < D / 64; ++a)
          tma_load_tile(sQ + a * L::ATOM_Q, &tm_q_tile, a * 64, q_row0 + w.b * BN, bar(kQFull));
    } else if (lane < BN / 4) {
      const int4 r4 = __ldg(reinterpret_cast<const int4 *>(p.perm_q + w.qh * p.N +
                                                          (size_t)w.b * BN) + lane);
      const int hiq = p.N - 1;
      const int y0 = q_row0 + min(max(r4.x, 0), hiq), y1 = q_row0 + min(max(r4.y, 0), hiq),
                y2 = q_row0 + min(max(r4.z, 0), hiq), y3 = q_row0 + min(max(r4.w, 0), hiq);
      for (int a = 0; a < D / 64; ++a)
        tma_gather4(sQ + a * L::ATOM_Q + lane * 4 * 128, &tm_q_row, a * 64, y0, y1, y2, y3,
                    bar(kQFull));
    }
    const int kv_row0 = (int)(w.kh * p.N);
    for (int j = 0; j < T; ++j) {
      const int st = j % L::KST;
      if (j >= L::KST) {
        bool got = true;
        if (lane == 0) got = mbar_wait(bar(kKEmpty + st), ((j / L::KST) - 1) & 1, lim);
        if (!__shfl_sync(0xffffffffu, got, 0)) {
          ok = false;
          break;
        }
      }
      if (lane == 0) mbar_expect_tx(bar(kKFull + st), L::KV_BYTES);
      __syncwarp();
      const uint32_t dst = sK + st * L::KV_BYTES;
      if (j < w.lt) {
        if (lane == 0)
          for (int a = 0; a < D / 64; ++a)
            tma_load_tile(dst + a * L::ATOM_KV, &tm_k_tile, a * 64, kv_row0 + seg0 + j * BN,
                          bar(kKFull + st));
      } else if (lane < BN / 4) {
        const int c = selected_block(w, p, j);
        const int4 r4 = __ldg(reinterpret_cast<const int4 *>(p.perm_k + w.qh * p.N +
                                                            (size_t)c * BN) + lane);
        const int hik = p.N - 1;
        const int y0 = kv_row0 + min(max(r4.x, 0), hik), y1 = kv_row0 + min(max(r4.y, 0), hik),
                  y2 = kv_row0 + min(max(r4.z, 0), hik), y3 = kv_row0 + min(max(r4.w, 0), hik);
        for (int a = 0; a < D / 64; ++a)
          tma_gather4(dst + a * L::ATOM_KV + lane * 4 * 128, &tm_k_row, a * 64, y0, y1, y2, y3,
                      bar(kKFull + st));
      }
      issued = j + 1;
    }
    // Drain: the last copy issued into each slot must have landed before the CTA exits.
    if (lane == 0) {
      mbar_wait(bar(kQFull), 0, kDrainNs);
      for (int st = 0; st < L::KST; ++st) {
        int last = -1;
        for (int j = st; j < issued; j += L::KST) last = j;
        if (last >= 0) mbar_wait(bar(kKFull + st), (last / L::KST) & 1, kDrainNs);
      }
    }
    __syncwarp();
  } else if (warp == 2) {
    // ---------------------------------------------------------------- V producer
    int issued = 0;
    const int kv_row0 = (int)(w.kh * p.N);
    for (int j = 0; j < T; ++j) {
      const int st = j % L::VST;
      if (j >= L::VST) {
        bool got = true;
        if (lane == 0) got = mbar_wait(bar(kVEmpty + st), ((j / L::VST) - 1) & 1, lim);
        if (!__shfl_sync(0xffffffffu, got, 0)) {
          ok = false;
          break;
        }
      }
      if (lane == 0) mbar_expect_tx(bar(kVFull + st), L::KV_BYTES);
      __syncwarp();
      const uint32_t dst = sV + st * L::KV_BYTES;
      if (j < w.lt) {
        if (lane == 0)
          for (int a = 0; a < D / 64; ++a)
            tma_load_tile(dst + a * L::ATOM_KV, &tm_v_tile, a * 64, kv_row0 + seg0 + j * BN,
                          bar(kVFull + st));
      } else if (lane < BN / 4) {
        const int c = selected_block(w, p, j);
        const int4 r4 = __ldg(reinterpret_cast<const int4 *>(p.perm_k + w.qh * p.N +
                                                            (size_t)c * BN) + lane);
        const int hik = p.N - 1;
        const int y0 = kv_row0 + min(max(r4.x, 0), hik), y1 = kv_row0 + min(max(r4.y, 0), hik),
                  y2 = kv_row0 + min(max(r4.z, 0), hik), y3 = kv_row0 + min(max(r4.w, 0), hik);
        for (int a = 0; a < D / 64; ++a)
          tma_gather4(dst + a * L::ATOM_KV + lane * 4 * 128, &tm_v_row, a * 64, y0, y1, y2, y3,
                      bar(kVFull + st));
      }
      issued = j + 1;
    }
    if (lane == 0) {
      for (int st = 0; st < L::VST; ++st) {
        int last = -1;
        for (int j = st; j < issued; j += L::VST) last = j;
        if (last >= 0) mbar_wait(bar(kVFull + st), (last / L::VST) & 1, kDrainNs);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescQK = idesc_bf16(kM, BN, 0, 0);
      constexpr uint32_t kIdescPV = idesc_bf16(kM, D, 0, 1);
      auto issue_qk = [&](int j) -> bool {
        const int st = j % L::KST;
        if (!mbar_wait(bar(kKFull + st), (j / L::KST) & 1, lim)) return false;
        if (j >= 2 && !mbar_wait(bar(kSFree + (j & 1)), ((j >> 1) - 1) & 1, lim)) return false;
        tc_fence_after();
        const uint32_t d_tmem = tmem + L::S_COL + (uint32_t)(j & 1) * BN;
        const uint32_t kst = sK + st * L::KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t a = sw128_desc(sQ + (kk / 4) * L::ATOM_Q + (kk % 4) * 32, 16);
          const uint64_t bd = sw128_desc(kst + (kk / 4) * L::ATOM_KV + (kk % 4) * 32, 16);
          tc_mma(d_tmem, a, bd, kIdescQK, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(kKEmpty + st));
        tc_commit(bar(kSFull + (j & 1)));
        return true;
      };
      auto issue_pv = [&](int j) -> bool {
        const int st = j % L::VST;
        if (!mbar_wait(bar(kVFull + st), (j / L::VST) & 1, lim)) return false;
        if (!mbar_wait(bar(kPFull), j & 1, lim)) return false;
        tc_fence_after();
        const uint32_t vst = sV + st * L::KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t a = sw128_desc(sP + (kk / 4) * L::ATOM_Q + (kk % 4) * 32, 16);
          const uint64_t bd = sw128_desc(vst + kk * 16 * 128, L::ATOM_KV);
          tc_mma(tmem + L::O_COL, a, bd, kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(bar(kVEmpty + st));
        tc_commit(bar(kPVDone));
        return true;
      };
      ok = mbar_wait(bar(kQFull), 0, lim);
      if (ok) ok = issue_qk(0);
      if (ok && T > 1) ok = issue_qk(1);
      for (int j = 0; ok && j < T; ++j) {
        ok = issue_pv(j);
        if (ok && j + 2 < T) ok = issue_qk(j + 2);
      }
      // Drain: every tensor-core operation issued above completes before TMEM is freed.
      tc_commit(bar(kDrain));
      mbar_wait(bar(kDrain), 0, kDrainNs);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- softmax + epilogue
    const int quad = warp - 4;
    const int row = quad * 32 + lane;
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    const unsigned full = 0xffffffffu;
    // Original position of this row's query (padding rows: the segment's last position).
    int i_orig = seg0 + p.S - 1;
    bool store_row = false;
    if (row < BN) {
      const int v = (p.dense || p.perm_q == nullptr)
                        ? w.b * BN + row
                        : __ldg(p.perm_q + w.qh * p.N + (size_t)w.b * BN + row);
      store_row = v >= seg0 && v < seg0 + p.S;
      i_orig = store_row ? v : seg0;
    }
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    uint32_t s[BN];
    for (int j = 0; j < T; ++j) {
      const int buf = j & 1;
      // Warp-uniform outcome: the tcgen05.ld below is a warp-collective instruction.
      if (!__all_sync(full, mbar_wait(bar(kSFull + buf), (j >> 1) & 1, lim))) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int c0 = 0; c0 < BN / 32; ++c0) {
        uint32_t(&chunk)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[c0 * 32]);
        tmem_ld32(trow + L::S_COL + buf * BN + c0 * 32, chunk);
        tmem_wait_ld(chunk);
      }
      tc_fence_before();
      mbar_arrive(bar(kSFree + buf));

      // Masks on original positions.
      if (j < w.lt) {
        const int limit = i_orig - (seg0 + j * BN);  // keys col <= limit are causal
        if (__any_sync(full, limit < BN - 1)) {
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (c > limit) s[c] = __float_as_uint(-INFINITY);
        }
      } else {
        const int c = selected_block(w, p, j);
        const int32_t *keys = p.perm_k + w.qh * p.N + (size_t)c * BN;
        uint32_t mw[BN / 32];
        bool all = true;
#pragma unroll
        for (int x = 0; x < BN / 32; ++x) {
          const int key = __ldg(keys + x * 32 + lane);
          mw[x] = __ballot_sync(full, key >= 0 && key < seg0);
          all = all && mw[x] == full;
        }
        if (!all) {
#pragma unroll
          for (int cc = 0; cc < BN; ++cc)
            if (!((mw[cc / 32] >> (cc % 32)) & 1u)) s[cc] = __float_as_uint(-INFINITY);
        }
      }
      // Row max and (below) row sum with 8 independent partial results: no 128-long dependency
      // chain on a single accumulator.
      float mp[8];
#pragma unroll
      for (int x = 0; x < 8; ++x) mp[x] = __uint_as_float(s[x]);
#pragma unroll
      for (int c = 8; c < BN; ++c) mp[c % 8] = fmaxf(mp[c % 8], __uint_as_float(s[c]));
      const float mt = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])),
                             fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7])));
      const float m_new = fmaxf(m_run, mt * sl2);
      const bool rescale = m_new > m_run + 8.0f;
      float m_use = rescale ? m_new : m_run;
      if (m_use == -INFINITY) m_use = 0.f;
      const float alpha = rescale ? ex2(m_run - m_use) : 1.f;
      float sp[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < BN; ++c) {
        const float pv = ex2(fmaf(__uint_as_float(s[c]), sl2, -m_use));
        sp[c % 8] += pv;
        s[c] = __float_as_uint(pv);
      }
      const float rs = ((sp[0] + sp[1]) + (sp[2] + sp[3])) + ((sp[4] + sp[5]) + (sp[6] + sp[7]));
      if (j > 0) {
        if (!__all_sync(full, mbar_wait(bar(kPVDone), (j - 1) & 1, lim))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(full, rescale)) {
#pragma unroll
          for (int c0 = 0; c0 < D / 32; ++c0) {
            uint32_t o[32];
            tmem_ld32(trow + L::O_COL + c0 * 32, o);
            tmem_wait_ld(o);
#pragma unroll
            for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * alpha);
            tmem_st32(trow + L::O_COL + c0 * 32, o);
          }
          tmem_wait_st();
        }
      }
      l_run = l_run * alpha + rs;
      m_run = m_use;
      // P (bf16) into the K-major 128B-swizzled A tile: row `row`, 16-byte chunk ch of the
      // 64-column atom ch / 8 lands at physical chunk (ch % 8) ^ (row % 8).
      unsigned char *prow = smem + L::OFF_P + row * 128;
#pragma unroll
      for (int ch = 0; ch < BN / 8; ++ch) {
        uint4 v;
        v.x = pack_bf16(__uint_as_float(s[ch * 8 + 0]), __uint_as_float(s[ch * 8 + 1]));
        v.y = pack_bf16(__uint_as_float(s[ch * 8 + 2]), __uint_as_float(s[ch * 8 + 3]));
        v.z = pack_bf16(__uint_as_float(s[ch * 8 + 4]), __uint_as_float(s[ch * 8 + 5]));
        v.w = pack_bf16(__uint_as_float(s[ch * 8 + 6]), __uint_as_float(s[ch * 8 + 7]));
        *reinterpret_cast<uint4 *>(prow + (ch / 8) * L::ATOM_Q + (((ch % 8) ^ (row % 8)) * 16)) =
            v;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(kPFull));
    }
    if (ok && __all_sync(full, mbar_wait(bar(kPVDone), (T - 1) & 1, lim))) {
      tc_fence_after();
      const float inv_l = 1.f / l_run;
      uint16_t *orow = p.o + ((size_t)w.qh * p.N + i_orig) * D;
#pragma unroll
      for (int c0 = 0; c0 < D / 32; ++c0) {
        uint32_t o[32];
        tmem_ld32(trow + L::O_COL + c0 * 32, o);
        tmem_wait_ld(o);
        if (store_row) {
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            uint4 v;
            v.x = pack_bf16(__uint_as_float(o[x * 8 + 0]) * inv_l,
                            __uint_as_float(o[x * 8 + 1]) * inv_l);
            v.y = pack_bf16(__uint_as_float(o[x * 8 + 2]) * inv_l,
                            __uint_as_float(o[x * 8 + 3]) * inv_l);
            v.z = pack_bf16(__uint_as_float(o[x * 8 + 4]) * inv_l,
                            __uint_as_float(o[x * 8 + 5]) * inv_l);
            v.w = pack_bf16(__uint_as_float(o[x * 8 + 6]) * inv_l,
                            __uint_as_float(o[x * 8 + 7]) * inv_l);
            *reinterpret_cast<uint4 *>(orow + c0 * 32 + x * 8) = v;
          }
        }
      }
    }
    tc_fence_before();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(L::TMEM_COLS)
                 : "memory");
  }
}

// ------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D bf16 tensor map over a [rows, D] row-major matrix, box {64 columns, box_rows}, 128-byte
// swizzle (one 64-column atom per box row is exactly one 128-byte swizzle span).
bool make_map(CUtensorMap *m, const void *base, long long rows, int D, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int BN>
cudaError_t launch_t(const Dims &d, const AttnArgs &a, uint64_t limit_ns, cudaStream_t st) {
  using L = Layout<D, BN>;
  static_assert(L::SMEM <= 232448, "shared memory budget");
  CUtensorMap tq, tqr, tk, tkr, tv, tvr;
  const long long q_rows = d.bhq() * d.N, kv_rows = d.bhkv() * d.N;
  if (!make_map(&tq, a.q, q_rows, D, BN) || !make_map(&tqr, a.q, q_rows, D, 1) ||
      !make_map(&tk, a.k, kv_rows, D, BN) || !make_map(&tkr, a.k, kv_rows, D, 1) ||
      !make_map(&tv, a.v, kv_rows, D, BN) || !make_map(&tvr, a.v, kv_rows, D, 1))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(s2o_attention_kernel<D, BN>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::SMEM);
  if (e != cudaSuccess) return e;
  Params p;
  p.perm_q = a.perm_q;
  p.perm_k = a.perm_k;
  p.sel_cnt = a.sel_cnt;
  p.sel_blk = a.sel_blk;
  p.local_tiles = a.local_tiles;
  p.o = static_cast<uint16_t *>(a.o);
  p.N = d.N;
  p.S = a.dense ? d.N : d.S;
  p.nB = d.nB;
  p.nSeg = a.dense ? 1 : d.nSeg;
  p.Hq = d.Hq;
  p.Hkv = d.Hkv;
  p.G = d.G;
  p.dense = a.dense ? 1 : 0;
  p.scale_log2 = (float)(1.4426950408889634 / __builtin_sqrt((double)D));
  p.limit_ns = limit_ns;
  const unsigned grid = (unsigned)(d.bhq() * d.nB);
  s2o_attention_kernel<D, BN><<<grid, kThreads, L::SMEM, st>>>(tq, tqr, tk, tkr, tv, tvr, p);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const Dims &d, const AttnArgs &a, uint64_t wait_limit_ns,
                             cudaStream_t st) {
  if (d.D == 128 && d.B == 128) return launch_t<128, 128>(d, a, wait_limit_ns, st);
  if (d.D == 128 && d.B == 64) return launch_t<128, 64>(d, a, wait_limit_ns, st);
  if (d.D == 64 && d.B == 128) return launch_t<64, 128>(d, a, wait_limit_ns, st);
  return launch_t<64, 64>(d, a, wait_limit_ns, st);
}

cudaError_t read_and_clear_device_error(unsigned int *out, cudaStream_t st) {
  cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_device_error, sizeof(unsigned int), 0,
                                            cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return e;
  if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return e;
  if (*out) {
    const unsigned int zero = 0;
    if ((e = cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof(zero), 0,
                                     cudaMemcpyHostToDevice, st)) != cudaSuccess)
      return e;
    e = cudaStreamSynchronize(st);
  }
  return e;
}

}  // namespace s2o
