// Fused gather-attention of S2O on sm_100a (tcgen05 tensor cores, TMEM accumulators, TMA).
//
// Sources: "S2O: Early Stopping for Sparse Attention via Online Permutation" (research card),
// Summary ¶2: the kernel fetches scattered tokens into on-chip memory through the index arrays
// and runs key blocks from most to least important, stopping at τ (the stop is already folded
// into the per-query-block list length); causality stays on original positions. The attention
// itself is Eq. (1) of "AB-Sparse" restricted to the selected key set, computed flash-style with
// an online softmax (the normaliser of Milakov & Gimelshein, cited by the S2O paper).
//
// Work decomposition. A unit is one (batch, query head, query block) of 128 query rows (rows
// B..127 are zero when B = 64). S2O runs in two launches of the same kernel:
//   local pass     every original-order query block runs the causal triangle of its own segment
//                  (the dense local window; masks on the diagonal tile only) and writes its rows;
//   permuted pass  only the query blocks whose selected list is not empty, rows gathered by
//                  perm_q: lt local tiles (contiguous keys of the block's segment, mask key <=
//                  query on original positions), then the cnt selected key blocks (keys gathered
//                  by perm_k, mask key < segment start); it overwrites their rows.
// Each row ends with the attention over exactly its key set. The dense baseline is a third mode
// (original-order blocks over all earlier keys). Units are ordered (batch, KV head, segment,
// block, query head of the group) — the dense mode longest blocks first — so consecutive units
// usually read the same local key tiles. A work item is two units, Q0 and Q1, with one stream of
// key/value tiles: the local tiles once for both when they share them, then the two selected
// lists interleaved. The grid is persistent (one CTA per SM); each CTA walks windows of a work
// list that warp 0 fills between two CTA-wide barriers (the permuted pass lists only units with
// selected blocks). With a workspace, a decision kernel picks the path on the device: when many
// query blocks are busy, the permuted pass runs only the selected blocks and leaves partial rows
// that the local pass merges (the merge path); when most blocks are selected, K and V are first
// copied into key order, each block's rows by position, and the permuted pass streams only the
// visible rows of a pair of units' selected blocks in 16-row chunks of the copy, a block both
// units selected loaded once (packed streams). The contiguous modes, the forms of the permuted
// pass and the merging local pass are separate instantiations of the kernel.
//
// Warp roles (384 threads):
//   warps 0, 11 K and V producers: K (warp 0) and V (warp 11) tiles of the stream into two rings
//               (TMA tile loads for contiguous tiles, TMA tile::gather4 for gathered rows; 128-byte
//               swizzle). Gathers are issued from two warps because one warp's stream of gather4
//               instructions limits the permuted pass when lists are long.
//   warp 1      MMA issuer: owns TMEM (512 columns: S0, S1, O0, O1). S_x = Q_x·Kᵀ, then
//               O_x += P_x·V with P_x read from TMEM (bf16 pairs written over S_x). The two query
//               tiles ping-pong: while one softmax group works on S0, the tensor core runs Q1's
//               products.
//   warp 2      Q producer: Q0 and Q1 of the next work item as soon as the last Q·Kᵀ of the
//               current one has finished.
//   warps 3-6   softmax of Q0, warps 7-10 softmax of Q1: the thread of TMEM lane r owns query row
//               r (a warp reaches the lane quarter warp % 4):
//               masks on original positions, online max/sum in the exp2 domain, conditional
//               rescale of O (only when the running max grows by more than 2^8, exact in real
//               arithmetic), P as bf16 into TMEM, and the final O/ℓ store at the original rows.
// Every wait is bounded (globaltimer); on a timeout the kernel records it in a device error word,
// drains its own TMA copies and tensor-core work, frees TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>
#include <type_traits>

#include "s2o_internal.h"

namespace s2o {

__device__ unsigned int g_device_error;

namespace {

constexpr int kThreads = 384;
constexpr int kM = 128;  // query rows per tile (UMMA M)
constexpr int kList = 256;  // units per work-list window
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

// D (TMEM) = A·B (+ D): A read from TMEM (128 lanes, bf16 pairs along K), B from shared memory.
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// ------------------------------------------------------------------ layout

template <int D, int BN>
struct Layout {
  static constexpr uint32_t ATOM_Q = kM * 128;  // bytes of one 64-column atom of a 128-row tile
  static constexpr uint32_t ATOM_KV = BN * 128;
  static constexpr uint32_t Q_BYTES = kM * D * 2;
  static constexpr uint32_t KV_BYTES = BN * D * 2;
  static constexpr int KST = KV_BYTES >= 32768 ? 2 : 4;  // K ring depth
  static constexpr int VST = KV_BYTES >= 32768 ? 2 : 4;  // V ring depth
  static constexpr uint32_t OFF_Q = 0;                   // Q0, then Q1
  static constexpr uint32_t OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + KST * KV_BYTES;
  // Output staging: one 64-column atom of a 128-row tile per softmax group (TMA tile stores).
  static constexpr uint32_t OFF_OST = OFF_V + VST * KV_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_OST + 2 * ATOM_Q;
  static constexpr uint32_t BAR_BYTES = 256;
  static constexpr uint32_t OFF_LIST = OFF_BAR + BAR_BYTES;  // work list: kList units + count
  static constexpr uint32_t SMEM = OFF_LIST + kList * 4 + 16 + 1024;  // + alignment slack
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t S_COL = 0;    // S_x at S_COL + 128·x (P_x over its first BN/2 columns)
  static constexpr uint32_t O_COL = 256;  // O_x at O_COL + D·x
};

// Barrier slots (8 bytes each) inside the barrier area; rings use up to four slots.
enum Bar {
  kQFull = 0,    // 2: Q_x landed (TMA transaction count)
  kQEmpty = 2,   // 2: the last Q_x·Kᵀ of a work item finished
  kKFull = 4,    // 4
  kKEmpty = 8,   // 4
  kVFull = 12,   // 4
  kVEmpty = 16,  // 4
  kSFull = 20,   // 2: S_x = Q_x·Kᵀ finished (and every earlier product of the CTA)
  kPFull = 22,   // 2: P_x written to TMEM and O_x rescaled (one arrival per softmax warp)
  kOFull = 24,   // 2: the last O_x += P_x·V of a work item finished
  kDrain = 26,
  kOSel = 27,    // 2: an atom of the permuted pass's partial rows landed in the output stage
  kNumBars = 29
};
// Byte offset in the barrier area of the two early-stop flags (after the barriers and the TMEM
// address).
constexpr int kStopFlagAt = 240;

// Unit sets of a launch.
enum Mode {
  kPermuted = 0,  // query blocks of perm_q: local tiles then the selected list
  kDense = 1,     // dense causal attention (Eq. 1): original-order blocks, all earlier keys
  kLocal = 2      // the dense local window only: original-order blocks, keys of their segment
};

// Division of n < 2^31 by a fixed divisor d ≥ 1 as a multiply-high and a shift (division by
// invariant integers using multiplication, Granlund and Montgomery): with L = ⌈log2 d⌉, p = 31 + L
// and m = ⌈2^p / d⌉ (m < 2^32), m = (2^p + e)/d with 0 ≤ e < d ≤ 2^L, so n·e < 2^p and
// ⌊n·m / 2^p⌋ = ⌊n/d⌋. d = 1 is passed through.
struct FastDiv {
  uint32_t d, m, s;  // divisor, multiplier, p − 32 (d > 1)
  void init(int divisor) {
    d = (uint32_t)divisor;
    int L = 0;
    while ((1ull << L) < d) ++L;
    m = d > 1 ? (uint32_t)(((1ull << (31 + L)) + d - 1) / d) : 0u;
    s = d > 1 ? (uint32_t)(L - 1) : 0u;
  }
  __device__ __forceinline__ uint32_t div(uint32_t n) const {
    return d > 1 ? __umulhi(n, m) >> s : n;
  }
  // Quotient, and n − q·d into r.
  __device__ __forceinline__ uint32_t divmod(uint32_t n, uint32_t &r) const {
    const uint32_t q = div(n);
    r = n - q * d;
    return q;
  }
};

// Kernel instantiations (a launch's mode picks one):
//   kKindContig  the contiguous modes: the dense local window (local pass) and the dense baseline;
//   kKindList    the permuted pass over list streams: query blocks gathered by perm_q, selected
//                blocks gathered row by row by perm_k, in list order (with or without the block's
//                local tiles, see Params::sel_only);
//   kKindPacked  the permuted pass over packed streams from the permuted copy of K and V (see
//                below);
//   kKindMerge   the local pass that also merges each row with the permuted pass's partial result;
//   kKindOnline  the permuted pass over list streams with the measured-share early stop (a
//                labelled variant): a query block's list ends after the first selected block
//                whose share of every row's running normaliser is below τ.
enum Kind { kKindContig = 0, kKindList = 1, kKindPacked = 2, kKindMerge = 3, kKindOnline = 4 };

struct Params {
  const int32_t *perm_q, *perm_k, *sel_cnt, *sel_blk, *local_tiles;
  uint16_t *o;
  int N, S, nB, nSeg, Hq, Hkv, G;
  int mode;
  int skip_empty;  // permuted mode: only blocks with a non-empty selected list
  int o_v8;        // O is 32-byte aligned: rows are written with 32-byte stores
  long long n_units, n_items;
  float scale_log2;  // log2(e) / sqrt(d)
  unsigned long long limit_ns;
  FastDiv div_G, div_seg, div_nB, div_nSeg, div_Hkv;  // unit-id decoding (S/B blocks a segment)
  // Permuted pass: 1 when it runs only the selected blocks and leaves the local window to the
  // local pass (merge path): it writes each row's partial result O_sel (bf16, at the row's place
  // in O) and its log2-sum-exp into lse_out; 0 when it also reruns the block's local tiles and
  // writes the final rows (the path without a workspace).
  int sel_only;
  float *lse_out;        // permuted pass, sel_only: [b, Hq, N] log2 Σ 2^(s·log2e/√d) per row
  const float *lse_in;   // kKindMerge: the same array (−inf where no selected block ran)
  // Device-side decision word (see k_copy_decide): bit 0 packed streams from the permuted copy,
  // bit 1 the merge path. A launch given it runs only when (word & run_mask) == run_value.
  const uint32_t *copy_flag;
  uint32_t run_mask, run_value;
  int copy_per_kv;            // copy rows per KV head (else per query head)
  // Packed streams (kKindPacked): per pair of units, chunk words at chunks + pair·chunk_cap (see
  // k_pack_pairs) and the tile counts {both, only unit 0, only unit 1, -} in pair_meta; pairs
  // are two heads of one KV head at one block when pair_heads is set, else two consecutive blocks
  // of one query head.
  const uint32_t *chunks;
  const int4 *pair_meta;
  long long chunk_cap;
  int pair_heads;
  // Measured-share early stop (kKindOnline): the listed blocks each busy query block kept.
  int32_t *stop_cnt;
  float stop_tau;
};

struct Unit {
  long long qh, kh;  // flat (batch, query head) and (batch, kv head)
  int b, seg0, lt, cnt;
  const int32_t *sel;  // the query block's selected list (sel_blk row)
};

// Unit order. The contiguous modes and list streams keep the units of one (batch, KV head,
// segment) together, query heads of the group fastest, so that the segment's K/V tiles stay in L2
// and paired units share local tiles; the dense baseline runs the longest query blocks first.
// Packed streams pair two units that read one copy head and one segment: with a copy per query
// head the order is (batch, KV head, query head of the group, segment, block), blocks fastest, so
// that a pair is two consecutive blocks of one query head; with a copy per KV head (pair_heads)
// it is the list-stream order, so that a pair is two query heads of one KV head at one block.
template <int BN, int KIND>
__device__ __forceinline__ Unit decode_unit(const Params &p, uint32_t u) {
  constexpr bool PERM = KIND == kKindList || KIND == kKindPacked || KIND == kKindOnline;
  constexpr bool PACKED = KIND == kKindPacked;
  // Unit ids are below 2^31 (the host checks): divisions by multiply-high.
  Unit r;
  uint32_t rem;
  int hi, b, bl;  // query head of the group, block, and the block's index inside its segment
  if (PACKED && !p.pair_heads) {
    u = p.div_seg.divmod(u, rem);
    bl = (int)rem;
    u = p.div_nSeg.divmod(u, rem);
    b = (int)rem * (int)p.div_seg.d + bl;
    r.seg0 = (int)rem * p.S;
    u = p.div_G.divmod(u, rem);
    hi = (int)rem;
  } else {
    u = p.div_G.divmod(u, rem);
    hi = (int)rem;
    if (!PERM && p.mode == kDense) {
      u = p.div_nB.divmod(u, rem);
      b = p.nB - 1 - (int)rem;
      bl = b;
      r.seg0 = 0;
    } else {
      u = p.div_seg.divmod(u, rem);
      bl = (int)rem;
      u = p.div_nSeg.divmod(u, rem);
      b = (int)rem * (int)p.div_seg.d + bl;
      r.seg0 = (int)rem * p.S;
    }
  }
  const uint32_t beta_u = p.div_Hkv.divmod(u, rem);
  const int g = (int)rem;
  const long long beta = beta_u;
  r.qh = beta * p.Hq + (long long)g * p.G + hi;
  r.kh = beta * p.Hkv + g;
  r.b = b;
  if (!PERM) {
    r.lt = bl + 1;  // the causal triangle of the block's segment (or sequence)
    r.cnt = 0;
    r.sel = nullptr;
  } else if (PACKED) {
    r.lt = 0;
    r.cnt = 0;  // set from the pair's tile counts
    r.sel = nullptr;
  } else {
    const long long qb = r.qh * p.nB + b;
    r.lt = p.sel_only ? 0 : min(max(__ldg(p.local_tiles + qb), 1), (int)p.div_seg.d);
    r.cnt = p.sel_cnt ? min(max(__ldg(p.sel_cnt + qb), 0), p.nB) : 0;
    r.sel = p.sel_blk + qb * p.nB;
  }
  return r;
}

struct Pair {
  Unit u0, u1;
  int valid1;  // the second unit exists and has work (the last work item may hold one)
  int valid0;  // the first unit has work (always, except in a packed pair whose unit 0 has none)
  int shared;  // both units read the same local key tiles
  int L;       // local items of the stream
  int total;   // stream length
  // Packed streams: tiles both units use, then tiles of unit 0 only and of unit 1 only
  // (interleaved), the pair's chunk list, and each unit's copy head.
  int tb, t0, t1;
  long long chunk0;
  long long ch0, ch1;
};

// Work item i of the current window. List streams and the contiguous modes: units list[2i] and
// list[2i+1] (the second may be absent past the list's end). Packed streams: the pair index is
// list[2i]; its units are 2·pair and 2·pair + 1.
constexpr uint32_t kNoUnit = 0xffffffffu;
template <int BN, int KIND>
__device__ __forceinline__ Pair decode_pair(const Params &p, const uint32_t *list, int n_list,
                                            int i) {
  constexpr bool PACKED = KIND == kKindPacked;
  Pair P;
  if (PACKED) {
    const uint32_t w = list[2 * i];
    const int4 m = __ldg(p.pair_meta + w);
    P.tb = m.x;
    P.t0 = m.y;
    P.t1 = m.z;
    P.chunk0 = (long long)w * p.chunk_cap;
    P.u0 = decode_unit<BN, KIND>(p, 2 * w);
    const bool has1 = 2ll * w + 1 < p.n_units;
    P.u1 = has1 ? decode_unit<BN, KIND>(p, 2 * w + 1) : P.u0;
    P.u0.cnt = P.tb + P.t0;
    P.u1.cnt = has1 ? P.tb + P.t1 : 0;
    P.valid0 = P.u0.cnt > 0;
    P.valid1 = P.u1.cnt > 0;
    P.shared = 0;
    P.L = 0;
    P.total = P.tb + P.t0 + P.t1;
    P.ch0 = (p.copy_per_kv ? P.u0.kh : P.u0.qh) * p.N;
    P.ch1 = (p.copy_per_kv ? P.u1.kh : P.u1.qh) * p.N;
    return P;
  }
  P.u0 = decode_unit<BN, KIND>(p, list[2 * i]);
  P.valid0 = 1;
  P.valid1 = 2 * i + 1 < n_list;
  if (P.valid1) {
    P.u1 = decode_unit<BN, KIND>(p, list[2 * i + 1]);
  } else {
    P.u1 = P.u0;
    P.u1.lt = 0;
    P.u1.cnt = 0;
  }
  P.shared = P.valid1 && P.u0.kh == P.u1.kh && P.u0.seg0 == P.u1.seg0;
  P.L = P.shared ? max(P.u0.lt, P.u1.lt) : P.u0.lt + P.u1.lt;
  P.total = P.L + P.u0.cnt + P.u1.cnt;
  P.tb = P.t0 = P.t1 = 0;
  P.chunk0 = 0;
  P.ch0 = P.ch1 = 0;
  return P;
}

// Position j of a two-way interleaving of a items of unit 0 and b items of unit 1 (alternating
// while both have items left): the unit x and its item index.
__device__ __forceinline__ void interleave(int a, int b, int j, int &x, int &idx) {
  const int m = min(a, b);
  if (j < 2 * m) {
    x = j & 1;
    idx = j >> 1;
  } else {
    x = a > b ? 0 : 1;
    idx = m + (j - 2 * m);
  }
}

// Packed stream item j: the units that use it (bit x for unit x), the tile's index in the pair's
// chunk list, and the copy rows it is loaded from.
struct PackedItem {
  int users, tile;
  long long ch;
};
__device__ __forceinline__ PackedItem packed_item(const Pair &P, int j) {
  PackedItem it;
  if (j >= P.total) {
    it.users = 0;
    it.tile = 0;
    it.ch = P.ch0;
  } else if (j < P.tb) {
    it.users = 3;
    it.tile = j;
    it.ch = P.ch0;
  } else {
    int x, idx;
    interleave(P.t0, P.t1, j - P.tb, x, idx);
    it.users = 1 << x;
    it.tile = P.tb + (x ? P.t0 : 0) + idx;
    it.ch = x ? P.ch1 : P.ch0;
  }
  return it;
}
// The chunk-list tile of unit x's n-th packed tile.
__device__ __forceinline__ int packed_unit_tile(const Pair &P, int x, int n) {
  return n < P.tb ? n : P.tb + (x ? P.t0 : 0) + (n - P.tb);
}

// Stream item j: which units use it (bit x), the unit whose indices locate its rows, whether it is
// a local tile, and the tile index (local) or the position in that unit's selected list.
struct Item {
  int users, x, local, t;
};

__device__ __forceinline__ Item item_at(const Pair &P, int j) {
  Item it;
  if (j >= P.total) {
    it.users = 0;
    it.x = 0;
    it.local = 0;
    it.t = 0;
    return it;
  }
  if (j < P.L) {
    it.local = 1;
    if (P.shared) {
      it.users = (j < P.u0.lt ? 1 : 0) | (j < P.u1.lt ? 2 : 0);
      it.x = (it.users & 1) ? 0 : 1;
      it.t = j;
    } else {
      interleave(P.u0.lt, P.u1.lt, j, it.x, it.t);
      it.users = 1 << it.x;
    }
  } else {
    it.local = 0;
    interleave(P.u0.cnt, P.u1.cnt, j - P.L, it.x, it.t);
    it.users = 1 << it.x;
  }
  return it;
}

// The units that use stream item j (bit x for unit x; 0 past the end).
template <int KIND>
__device__ __forceinline__ int users_at(const Pair &P, int j) {
  if (KIND == kKindPacked) return packed_item(P, j).users;
  if (j >= P.total) return 0;
  int x, idx;
  if (j < P.L) {
    if (P.shared) return (j < P.u0.lt ? 1 : 0) | (j < P.u1.lt ? 2 : 0);
    interleave(P.u0.lt, P.u1.lt, j, x, idx);
  } else {
    interleave(P.u0.cnt, P.u1.cnt, j - P.L, x, idx);
  }
  return 1 << x;
}

// The selected block of a unit's list position (clamped), or -1 past the list.
__device__ __forceinline__ int sel_block(const Params &p, const Unit &u, int t) {
  return t < u.cnt ? min(max(__ldg(u.sel + t), 0), p.nB - 1) : -1;
}

// This lane's four gathered key rows of permuted block c of unit u (flattened row indices,
// clamped into the KV head); lanes >= B/4 and c < 0 give zeros.
template <int BN>
__device__ __forceinline__ int4 block_rows(const Params &p, const Unit &u, int c, int lane) {
  if (c < 0 || lane >= BN / 4) return make_int4(0, 0, 0, 0);
  const int4 r4 =
      __ldg(reinterpret_cast<const int4 *>(p.perm_k + u.qh * p.N + (size_t)c * BN) + lane);
  const int row0 = (int)(u.kh * p.N), hi = p.N - 1;
  return make_int4(row0 + min(max(r4.x, 0), hi), row0 + min(max(r4.y, 0), hi),
                   row0 + min(max(r4.z, 0), hi), row0 + min(max(r4.w, 0), hi));
}

// Loads the K or V rows of stream item `it` into one ring stage (all 32 lanes of the warp call it;
// the transaction count has been set). Contiguous local tiles: one TMA tile load per 64-column
// atom; gathered rows (prepared by block_rows): tile::gather4, four rows per lane.
template <int D, int BN>
__device__ __forceinline__ void load_kv(uint32_t dst, const CUtensorMap *tm_tile,
                                        const CUtensorMap *tm_row, const Params &p,
                                        const Pair &P, const Item &it, int4 rows, uint32_t bar,
                                        int lane) {
  using L = Layout<D, BN>;
  const Unit &u = it.x ? P.u1 : P.u0;
  if (it.local) {
    if (lane == 0)
      for (int a = 0; a < D / 64; ++a)
        tma_load_tile(dst + a * L::ATOM_KV, tm_tile, a * 64,
                      (int)(u.kh * p.N) + u.seg0 + it.t * BN, bar);
  } else if (lane < BN / 4) {
    for (int a = 0; a < D / 64; ++a)
      tma_gather4(dst + a * L::ATOM_KV + lane * 4 * 128, tm_row, a * 64, rows.x, rows.y, rows.z,
                  rows.w, bar);
  }
}

// Chunks of a packed tile: 16 rows of the permuted copy each (BN/16 per tile).
constexpr int kChunkRows = 16;

// Loads one packed tile (all 32 lanes call it; the transaction count has been set): lane c < BN/16
// loads chunk c, the 16 copy rows its chunk word names (row16 = word >> 5, in units of 16 rows of
// the copy head whose first row is `ch`), with one TMA tile load of a {64, 16} box per 64-column
// atom into rows 16c..16c+15 of the stage. Chunks past a group's end name rows 0..15 of the copy
// head and are masked by the softmax.
template <int D, int BN>
__device__ __forceinline__ void load_packed(uint32_t dst, const CUtensorMap *tm_copy16,
                                            long long ch, uint32_t word, uint32_t bar, int lane) {
  using L = Layout<D, BN>;
  if (lane < BN / kChunkRows) {
    const int row = (int)(ch + (long long)(word >> 5) * kChunkRows);
    for (int a = 0; a < D / 64; ++a)
      tma_load_tile(dst + a * L::ATOM_KV + lane * kChunkRows * 128, tm_copy16, a * 64, row, bar);
  }
}

// Waits (lane 0, bounded) and broadcasts the outcome to the warp.
__device__ __forceinline__ bool warp_wait(uint32_t bar_addr, uint32_t parity, uint64_t lim,
                                          int lane) {
  bool got = true;
  if (lane == 0) got = mbar_wait(bar_addr, parity, lim);
  return __shfl_sync(0xffffffffu, got, 0);
}

// Lane 0 waits (bounded) for the last fill of each stage of a ring of `stages` slots that has
// received `filled` fills in total.
__device__ __forceinline__ void drain_ring(uint32_t full0, int stages, long long filled) {
  for (int st = 0; st < stages; ++st) {
    if (filled <= st) continue;
    const long long last = st + ((filled - 1 - st) / stages) * stages;
    mbar_wait(full0 + 8u * (uint32_t)st, (uint32_t)((last / stages) & 1), kDrainNs);
  }
}

// Eight tcgen05.mma (kind::f16) into one accumulator, issued back to back from registers: A and B
// shared-memory descriptors per K step; the first product accumulates only if `acc0` is set.
__device__ __forceinline__ void mma8_ss(uint32_t d, uint32_t idesc, const uint64_t (&a)[8],
                                        const uint64_t (&b)[8], uint32_t acc0) {
  asm volatile(
      "{\n\t.reg .pred p0, p1;\n\t"
      "setp.ne.b32 p0, %18, 0;\n\t"
      "setp.eq.b32 p1, %0, %0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %2, %10, %1, p0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %11, %1, p1;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %4, %12, %1, p1;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %5, %13, %1, p1;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %6, %14, %1, p1;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %7, %15, %1, p1;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %8, %16, %1, p1;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %9, %17, %1, p1;\n\t}\n" ::"r"(d),
      "r"(idesc), "l"(a[0]), "l"(a[1]), "l"(a[2]), "l"(a[3]), "l"(a[4]), "l"(a[5]), "l"(a[6]),
      "l"(a[7]), "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]), "l"(b[4]), "l"(b[5]), "l"(b[6]),
      "l"(b[7]), "r"(acc0)
      : "memory");
}

// As mma8_ss with A read from TMEM (eight column addresses).
__device__ __forceinline__ void mma8_ts(uint32_t d, uint32_t idesc, const uint32_t (&a)[8],
                                        const uint64_t (&b)[8], uint32_t acc0) {
  asm volatile(
      "{\n\t.reg .pred p0, p1;\n\t"
      "setp.ne.b32 p0, %18, 0;\n\t"
      "setp.eq.b32 p1, %0, %0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%2], %10, %1, p0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%3], %11, %1, p1;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%4], %12, %1, p1;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%5], %13, %1, p1;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%6], %14, %1, p1;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%7], %15, %1, p1;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%8], %16, %1, p1;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%9], %17, %1, p1;\n\t}\n" ::"r"(d),
      "r"(idesc), "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(a[4]), "r"(a[5]), "r"(a[6]),
      "r"(a[7]), "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]), "l"(b[4]), "l"(b[5]), "l"(b[6]),
      "l"(b[7]), "r"(acc0)
      : "memory");
}

// TMA tile store shared -> global (bulk async-group of the issuing thread), its commit, and the
// waits for the group's source reads / full completion.
__device__ __forceinline__ void tma_store_tile(const CUtensorMap *tm, int x, int y, uint32_t src) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
          reinterpret_cast<uint64_t>(tm)),
      "r"(x), "r"(y), "r"(src)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// 32-byte global store of eight 32-bit words (one full sector).
__device__ __forceinline__ void st_global_v8(void *dst, const uint32_t (&w)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(w[0]),
               "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
// Named barrier that also returns whether any participating thread passed `v`.
__device__ __forceinline__ bool named_bar_or(int id, int threads, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %3, 0;\n\t"
      "bar.red.or.pred p, %1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(r)
      : "r"(id), "r"(threads), "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Fills the work list for window k0 of this CTA's share (warp 0; returns the entry count, or -1
// past the end of the share). Without skipping, the share is one work item per round k of
// gridDim.x consecutive items, each contributing its units 2w and 2w+1 (adjacent units, which
// usually share local tiles): w = k·gridDim.x + blockIdx.x, and in the local pass, in odd rounds,
// w = k·gridDim.x + (gridDim.x − 1 − blockIdx.x). A round spans a few segments whose items repeat
// the lengths 1..S/B, and a plain round robin with gridDim.x = 148 and 16 blocks per segment hands
// a CTA only even or only odd block indices (units of 8 against 9 tiles on average); reversing
// every other round gives each CTA both. With skip_empty (list streams) the share is the units
// u = blockIdx.x + k·gridDim.x whose selected list is not empty, paired in list order. Packed
// streams: the share is the pairs w = blockIdx.x + k·gridDim.x that have a tile, each pair index
// at an even list position.
template <int BN, int KIND>
__device__ int build_list(const Params &p, long long k0, uint32_t *list, int lane) {
  constexpr bool PACKED = KIND == kKindPacked;
  const bool by_unit = p.skip_empty && !PACKED;
  const long long span = by_unit ? kList : kList / 2;
  const bool snake = !by_unit && !PACKED && p.mode == kLocal;
  const long long first = snake ? k0 * gridDim.x : blockIdx.x + k0 * gridDim.x;
  if (first >= (by_unit ? p.n_units : p.n_items)) return -1;
  // Whether unit u (list-stream order) has a non-empty selected list.
  auto busy = [&](long long u) -> bool {
    if (u >= p.n_units || !p.sel_cnt) return false;
    const int per_seg = p.S / BN;
    const int hi = (int)(u % p.G);
    u /= p.G;
    const int bl = (int)(u % per_seg);
    u /= per_seg;
    const int sg = (int)(u % p.nSeg);
    u /= p.nSeg;
    const int g = (int)(u % p.Hkv);
    const long long qh = (u / p.Hkv) * p.Hq + (long long)g * p.G + hi;
    return __ldg(p.sel_cnt + qh * p.nB + sg * per_seg + bl) > 0;
  };
  int n = 0;
  for (long long k = k0; k < k0 + span; k += 32) {
    const long long round = k + lane;
    const long long pos = round * gridDim.x +
                          (snake && (round & 1) ? gridDim.x - 1 - blockIdx.x : blockIdx.x);
    if (by_unit) {
      const bool keep = busy(pos);
      const unsigned m = __ballot_sync(0xffffffffu, keep);
      if (keep) list[n + __popc(m & ((1u << lane) - 1u))] = (uint32_t)pos;
      n += __popc(m);
    } else if (PACKED) {
      bool keep = false;
      if (pos < p.n_items) {
        const int4 m = __ldg(p.pair_meta + pos);
        keep = m.x + m.y + m.z > 0;
      }
      const unsigned m = __ballot_sync(0xffffffffu, keep);
      if (keep) {
        const int at = n + 2 * __popc(m & ((1u << lane) - 1u));
        list[at] = (uint32_t)pos;
        list[at + 1] = kNoUnit;
      }
      n += 2 * __popc(m);
    } else {
      const bool keep = pos < p.n_items;
      const bool two = 2 * pos + 1 < p.n_units;
      const unsigned m = __ballot_sync(0xffffffffu, keep);
      const unsigned m2 = __ballot_sync(0xffffffffu, keep && two);
      // Only the last item of all can hold a single unit, so lower lanes hold two each.
      if (keep) {
        const int at = n + 2 * __popc(m & ((1u << lane) - 1u));
        list[at] = (uint32_t)(2 * pos);
        if (two) list[at + 1] = (uint32_t)(2 * pos + 1);
      }
      n += __popc(m) + __popc(m2);
    }
  }
  return n;
}

// ------------------------------------------------------------------ the kernel

// One instantiation per Kind (see the Kind enum), so that the hot local pass carries none of the
// permuted pass's code. A permuted launch that has a decision flag runs only when the flag chose
// its form (packed streams when bit 0 is set, list streams when it is clear): the host launches
// both and one returns at once.
template <int D, int BN, int KIND>
__global__ void __launch_bounds__(kThreads, 1)
    s2o_attention_kernel(const __grid_constant__ CUtensorMap tm_q_tile,
                         const __grid_constant__ CUtensorMap tm_q_row,
                         const __grid_constant__ CUtensorMap tm_k_tile,
                         const __grid_constant__ CUtensorMap tm_k_row,
                         const __grid_constant__ CUtensorMap tm_v_tile,
                         const __grid_constant__ CUtensorMap tm_v_row,
                         const __grid_constant__ CUtensorMap tm_o_tile,
                         const __grid_constant__ CUtensorMap tm_kp16,
                         const __grid_constant__ CUtensorMap tm_vp16, const Params p) {
  using L = Layout<D, BN>;
  constexpr bool PERM = KIND == kKindList || KIND == kKindPacked || KIND == kKindOnline;
  constexpr bool PACKED = KIND == kKindPacked;
  constexpr bool MERGE = KIND == kKindMerge;
  constexpr bool ONLINE = KIND == kKindOnline;
  constexpr int CPT = BN / kChunkRows;  // chunks per packed tile
  if (p.copy_flag != nullptr && (__ldg(p.copy_flag) & p.run_mask) != p.run_value) return;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + L::OFF_Q, sK = sbase + L::OFF_K, sV = sbase + L::OFF_V,
                 sBar = sbase + L::OFF_BAR;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::OFF_BAR + kNumBars * 8);
  // kKindOnline: per query tile, set by its softmax group when the unit's list stops early.
  volatile int *stop_flag = reinterpret_cast<volatile int *>(smem + L::OFF_BAR + kStopFlagAt);
  auto bar = [&](int i) { return sBar + 8u * (uint32_t)i; };
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar(kQFull + x), 1);
      mbar_init(bar(kQEmpty + x), 1);
      mbar_init(bar(kSFull + x), 1);
      mbar_init(bar(kPFull + x), 4);  // one arrival per softmax warp
      mbar_init(bar(kOFull + x), 1);
      mbar_init(bar(kOSel + x), 1);
    }
    for (int i = 0; i < L::KST; ++i) {
      mbar_init(bar(kKFull + i), 1);
      mbar_init(bar(kKEmpty + i), 1);
    }
    for (int i = 0; i < L::VST; ++i) {
      mbar_init(bar(kVFull + i), 1);
      mbar_init(bar(kVEmpty + i), 1);
    }
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
  if (BN < kM && warp >= 3 && warp < 11) {
    // Rows BN..127 of both Q tiles are padding: zero them once (TMA writes rows 0..BN-1 only).
    const int x = (warp - 3) >> 2, row = (warp & 3) * 32 + lane;
    if (row >= BN) {
      for (int a = 0; a < D / 64; ++a) {
        uint4 *dst = reinterpret_cast<uint4 *>(smem + L::OFF_Q + x * L::Q_BYTES + a * L::ATOM_Q +
                                               row * 128);
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
  // Work comes in windows of this CTA's share: warp 0 fills the work list between two CTA-wide
  // barriers and every role then walks the window's items (a role that gave up a bounded wait
  // keeps meeting the barriers without working).
  uint32_t *list = reinterpret_cast<uint32_t *>(smem + L::OFF_LIST);
  volatile int *list_n = reinterpret_cast<volatile int *>(smem + L::OFF_LIST + kList * 4);
  auto for_each_window = [&](auto &&body) {
    for (long long k0 = 0;; k0 += p.skip_empty && !PACKED ? kList : kList / 2) {
      named_bar_sync(1, kThreads);
      if (warp == 0) {
        const int n = build_list<BN, KIND>(p, k0, list, lane);
        if (lane == 0) *list_n = n;
        __syncwarp();
      }
      named_bar_sync(1, kThreads);
      const int n_list = *list_n;
      if (n_list < 0) break;
      body(n_list);
    }
  };

  if (warp == 0 || warp == kThreads / 32 - 1) {
    // ---------------------------------------------------------------- K and V producers
    // Warp 0 loads K, the last warp V; both walk the same stream.
    const bool is_k = warp == 0;
    const int stages = is_k ? L::KST : L::VST;
    const uint32_t ring = is_k ? sK : sV;
    const int full0 = is_k ? kKFull : kVFull, empty0 = is_k ? kKEmpty : kVEmpty;
    const CUtensorMap *tm_tile = is_k ? &tm_k_tile : &tm_v_tile;
    const CUtensorMap *tm_row = is_k ? &tm_k_row : &tm_v_row;
    const CUtensorMap *tm_copy16 = is_k ? &tm_kp16 : &tm_vp16;
    long long kj = 0;  // stream items issued so far (all work items of this CTA)
    // Waits for the next ring stage and sets its transaction count; false if the wait ran out.
    auto next_stage = [&](uint32_t &dst, uint32_t &fb) -> bool {
      const int st = (int)(kj % stages);
      if (kj >= stages &&
          !warp_wait(bar(empty0 + st), (uint32_t)(((kj / stages) - 1) & 1), lim, lane))
        return false;
      if (lane == 0) mbar_expect_tx(bar(full0 + st), L::KV_BYTES);
      __syncwarp();
      dst = ring + st * L::KV_BYTES;
      fb = bar(full0 + st);
      ++kj;
      return true;
    };
    for_each_window([&](int n_list) {
    for (int wi = 0; ok && wi < (n_list + 1) / 2; ++wi) {
      const Pair P = decode_pair<BN, KIND>(p, list, n_list, wi);
      if (PACKED) {
        // Packed tiles: this lane's chunk word of the next item is loaded before the wait for
        // the current item's stage.
        auto word_of = [&](int j) -> uint32_t {
          if (j >= P.total || lane >= CPT) return 0u;
          const PackedItem t = packed_item(P, j);
          return __ldg(p.chunks + P.chunk0 + (long long)t.tile * CPT + lane);
        };
        uint32_t w_cur = word_of(0);
        for (int j = 0; ok && j < P.total; ++j) {
          const uint32_t w_next = word_of(j + 1);
          uint32_t dst, fb;
          if (!next_stage(dst, fb)) {
            ok = false;
            break;
          }
          load_packed<D, BN>(dst, tm_copy16, packed_item(P, j).ch, w_cur, fb, lane);
          w_cur = w_next;
        }
        continue;
      }
      if (!PERM) {
        // Contiguous modes: local tiles only.
        for (int j = 0; ok && j < P.total; ++j) {
          uint32_t dst, fb;
          if (!next_stage(dst, fb)) {
            ok = false;
            break;
          }
          load_kv<D, BN>(dst, tm_tile, tm_row, p, P, item_at(P, j), make_int4(0, 0, 0, 0), fb,
                         lane);
        }
        continue;
      }
      // Gathered rows are looked up ahead: the rows of item j+1 and the block of item j+2 are
      // requested before item j waits for its ring stage, so the dependent index loads are off
      // the critical path.
      auto block_of = [&](int j) -> int {
        if (j >= P.total) return -1;
        const Item t = item_at(P, j);
        return t.local ? -1 : sel_block(p, t.x ? P.u1 : P.u0, t.t);
      };
      auto rows_of = [&](int j, int c) -> int4 {
        if (j >= P.total || c < 0) return make_int4(0, 0, 0, 0);
        const Item t = item_at(P, j);
        return block_rows<BN>(p, t.x ? P.u1 : P.u0, c, lane);
      };
      int c_cur = block_of(0);
      int4 rows = rows_of(0, c_cur);
      int c_next = block_of(1);
      for (int j = 0; j < P.total; ++j) {
        const Item it = item_at(P, j);
        const int4 rows_next = rows_of(j + 1, c_next);
        c_cur = c_next;
        c_next = block_of(j + 2);
        uint32_t dst, fb;
        if (!next_stage(dst, fb)) {
          ok = false;
          break;
        }
        load_kv<D, BN>(dst, tm_tile, tm_row, p, P, it, rows, fb, lane);
        rows = rows_next;
      }
    }
    });
    // Drain: the last copy issued into each stage must have landed before the CTA exits.
    if (lane == 0) drain_ring(bar(full0), stages, kj);
    __syncwarp();
  } else if (warp == 2) {
    // ---------------------------------------------------------------- Q producer
    long long qn[2] = {0, 0};
    for_each_window([&](int n_list) {
    for (int wi = 0; ok && wi < (n_list + 1) / 2; ++wi) {
      const Pair P = decode_pair<BN, KIND>(p, list, n_list, wi);
      for (int x = 0; ok && x < 2; ++x) {
        if (!(x ? P.valid1 : P.valid0)) continue;
        if (qn[x] >= 1 &&
            !warp_wait(bar(kQEmpty + x), (uint32_t)((qn[x] - 1) & 1), lim, lane)) {
          ok = false;
          break;
        }
        if (lane == 0) mbar_expect_tx(bar(kQFull + x), BN * D * 2);
        __syncwarp();
        const Unit &u = x ? P.u1 : P.u0;
        const uint32_t dst = sQ + x * L::Q_BYTES;
        const int q_row0 = (int)(u.qh * p.N);
        if (!PERM || p.perm_q == nullptr) {
          if (lane == 0)
            for (int a = 0; a < D / 64; ++a)
              tma_load_tile(dst + a * L::ATOM_Q, &tm_q_tile, a * 64, q_row0 + u.b * BN,
                            bar(kQFull + x));
        } else if (lane < BN / 4) {
          const int4 r4 = __ldg(reinterpret_cast<const int4 *>(p.perm_q + u.qh * p.N +
                                                              (size_t)u.b * BN) + lane);
          const int hi = p.N - 1;
          const int y0 = q_row0 + min(max(r4.x, 0), hi), y1 = q_row0 + min(max(r4.y, 0), hi),
                    y2 = q_row0 + min(max(r4.z, 0), hi), y3 = q_row0 + min(max(r4.w, 0), hi);
          for (int a = 0; a < D / 64; ++a)
            tma_gather4(dst + a * L::ATOM_Q + lane * 4 * 128, &tm_q_row, a * 64, y0, y1, y2, y3,
                        bar(kQFull + x));
        }
        ++qn[x];
      }
    }
    });
    if (lane == 0)
      for (int x = 0; x < 2; ++x)
        if (qn[x] > 0) mbar_wait(bar(kQFull + x), (uint32_t)((qn[x] - 1) & 1), kDrainNs);
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    // One thread issues every tensor-core operation. Its loop is kept short (32-bit counters,
    // descriptors advanced by constant offsets): it shares a scheduler with two softmax warps
    // that issue back to back, and each of its instructions delays the next product.
    {
      constexpr uint32_t kIdescQK = idesc_bf16(kM, BN, 0, 0);
      constexpr uint32_t kIdescPV = idesc_bf16(kM, D, 0, 1);
      static_assert((L::VST & (L::VST - 1)) == 0, "V ring depth must be a power of two");
      // Descriptor start addresses are 16-byte units in bits 0-13; every operand address stays
      // below 2^18 bytes, so constant offsets are added to the descriptor directly.
      const uint64_t qdesc0 = sw128_desc(sQ, 16), kdesc0 = sw128_desc(sK, 16),
                     vdesc0 = sw128_desc(sV, L::ATOM_KV);
      // Per K step: Q descriptors of both tiles, the K offset inside a stage, P columns in TMEM.
      constexpr uint64_t kOffK[8] = {0, 2, 4, 6, L::ATOM_KV >> 4, (L::ATOM_KV >> 4) + 2,
                                     (L::ATOM_KV >> 4) + 4, (L::ATOM_KV >> 4) + 6};
      constexpr uint64_t kOffQ[8] = {0, 2, 4, 6, L::ATOM_Q >> 4, (L::ATOM_Q >> 4) + 2,
                                     (L::ATOM_Q >> 4) + 4, (L::ATOM_Q >> 4) + 6};
      uint64_t qa[2][8];
      uint32_t ptm[2][8];
#pragma unroll
      for (int x = 0; x < 2; ++x)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          qa[x][kk] = qdesc0 + (uint64_t)(x * (L::Q_BYTES >> 4)) + kOffQ[kk % (D / 16)];
          ptm[x][kk] = tmem + L::S_COL + 128u * x + 8u * (kk % (BN / 16));
        }
      uint32_t k_st = 0, k_ph = 0;  // K ring stage and phase of the next stream item
      uint32_t v_base = 0;          // stream items of this CTA's earlier work items
      uint32_t q_ph[2] = {0, 0}, p_ph[2] = {0, 0};
      for_each_window([&](int n_list) {
        // Each tile x has at most one product O_x += P_x·V still to issue (its P_x lives in
        // S_x's columns): the one of stream item pend[x]. A unit's last product is issued at tile
        // x's next step, which may belong to the next work item, so the tensor core goes on to
        // the next unit's first Q_x·Kᵀ without draining; O_x is committed right after it. The
        // window's last products are issued at its end.
        constexpr uint32_t kNone = 0xffffffffu;
        uint32_t pend[2] = {kNone, kNone};
        bool pend_last[2] = {false, false};
        uint32_t acc[2] = {0u, 0u};
        uint32_t vleft = 0;  // 2 bits per V stage: products still to issue on its tile
        // kKindOnline: units of the current work item whose list stopped early.
        bool done[2] = {false, false};
        // The V stage is released once every unit using the tile has issued its product.
        auto issue_pv = [&](auto xc) -> bool {
          constexpr int x = decltype(xc)::value;
          const uint32_t vi = pend[x];
          const uint32_t vs = vi & (L::VST - 1);
          if (!mbar_wait(bar(kVFull + vs), (vi / L::VST) & 1u, lim)) return false;
          if (!mbar_wait(bar(kPFull + x), p_ph[x], lim)) return false;
          p_ph[x] ^= 1u;
          tc_fence_after();
          const uint64_t vd = vdesc0 + vs * (L::KV_BYTES >> 4);
          uint64_t b[8];
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            b[kk] = vd + (uint64_t)((kk % (BN / 16)) * (16 * 128 / 16));
          if (BN == 128) {
            mma8_ts(tmem + L::O_COL + (uint32_t)(D * x), kIdescPV, ptm[x], b, acc[x]);
          } else {
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk)
              tc_mma_ts(tmem + L::O_COL + (uint32_t)(D * x), ptm[x][kk], b[kk], kIdescPV,
                        acc[x] | (kk > 0 ? 1u : 0u));
          }
          acc[x] = 1u;
          const uint32_t left = ((vleft >> (2 * vs)) & 3u) - 1u;
          vleft = (vleft & ~(3u << (2 * vs))) | ((left & 3u) << (2 * vs));
          if (left == 0) tc_commit(bar(kVEmpty + vs));
          bool last = pend_last[x];
          if (ONLINE && !last && stop_flag[x] != 0) {
            // The softmax group stopped the unit's list at this block (its flag was written
            // before the P arrival just waited for): this is the unit's last product, and its Q
            // tile is free.
            last = true;
            done[x] = true;
            tc_commit(bar(kQEmpty + x));
          }
          if (last) {
            tc_commit(bar(kOFull + x));
            acc[x] = 0u;
          }
          pend[x] = kNone;
          return true;
        };
        auto issue_qk = [&](auto xc, const uint64_t (&kb)[8]) {
          constexpr int x = decltype(xc)::value;
          const uint32_t d_tmem = tmem + L::S_COL + 128u * x;
          if (D == 128) {
            mma8_ss(d_tmem, kIdescQK, qa[x], kb, 0u);
          } else {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              tc_mma(d_tmem, qa[x][kk], kb[kk], kIdescQK, kk > 0 ? 1u : 0u);
          }
          tc_commit(bar(kSFull + x));
        };
      if (lane == 0) {
      for (int wi = 0; ok && wi < (n_list + 1) / 2; ++wi) {
        const Pair P = decode_pair<BN, KIND>(p, list, n_list, wi);
        auto users_seq = [&](int j) -> int { return users_at<KIND>(P, j); };
        const int n_of[2] = {P.u0.lt + P.u0.cnt, P.valid1 ? P.u1.lt + P.u1.cnt : 0};
        int qk[2] = {0, 0};
        int issued = 0;  // units that ran a product on the current stream item
        done[0] = done[1] = false;
        // One unit's step at stream item j: its pending product goes first, or now if the unit
        // skips the next item (its V tile must leave the ring); a unit's first Q_x·Kᵀ waits for
        // its Q_x tile.
        auto step = [&](auto xc, int j, int users, int nusers, const uint64_t (&kb)[8]) -> bool {
          constexpr int x = decltype(xc)::value;
          bool use = ((users >> x) & 1) && !(ONLINE && done[x]);
          if (pend[x] != kNone && (use || !((nusers >> x) & 1)) && !issue_pv(xc)) return false;
          if (ONLINE) use = use && !done[x];  // the pending product may have ended the unit
          if (use) {
            issued |= 1 << x;
            if (qk[x] == 0) {
              if (!mbar_wait(bar(kQFull + x), q_ph[x], lim)) return false;
              q_ph[x] ^= 1u;
              tc_fence_after();
            }
            issue_qk(xc, kb);
            pend[x] = v_base + (uint32_t)j;
            pend_last[x] = ++qk[x] == n_of[x];
            if (pend_last[x]) tc_commit(bar(kQEmpty + x));
          }
          return true;
        };
        int users = users_seq(0);
        for (int j = 0; j < P.total; ++j) {
          const int nusers = users_seq(j + 1);
          if (!mbar_wait(bar(kKFull + k_st), k_ph, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t kd = kdesc0 + k_st * (L::KV_BYTES >> 4);
          uint64_t kb[8];
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) kb[kk] = kd + kOffK[kk % (D / 16)];
          issued = 0;
          if (!step(std::integral_constant<int, 0>{}, j, users, nusers, kb) ||
              !step(std::integral_constant<int, 1>{}, j, users, nusers, kb)) {
            ok = false;
            break;
          }
          tc_commit(bar(kKEmpty + k_st));
          const uint32_t vs = (v_base + (uint32_t)j) & (L::VST - 1);
          const int eff = ONLINE ? issued : users;
          vleft = (vleft & ~(3u << (2 * vs))) | ((uint32_t)__popc(eff) << (2 * vs));
          if (ONLINE && eff == 0) {
            // No unit uses this item any more (its list stopped): the V tile is released once
            // it has landed.
            if (!mbar_wait(bar(kVFull + vs), ((v_base + (uint32_t)j) / L::VST) & 1u, lim)) {
              ok = false;
              break;
            }
            tc_commit(bar(kVEmpty + vs));
          }
          if (++k_st == (uint32_t)L::KST) {
            k_st = 0;
            k_ph ^= 1u;
          }
          users = nusers;
        }
        v_base += (uint32_t)P.total;
      }
      // The window's last products: every role meets the next window barrier only after its
      // units are complete.
      if (ok && pend[0] != kNone) ok = issue_pv(std::integral_constant<int, 0>{});
      if (ok && pend[1] != kNone) ok = issue_pv(std::integral_constant<int, 1>{});
      }
      __syncwarp();
      });
      // Drain: every tensor-core operation issued above completes before TMEM is freed.
      if (lane == 0) {
        tc_commit(bar(kDrain));
        mbar_wait(bar(kDrain), 0, kDrainNs);
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- softmax + epilogue
    const int x = (warp - 3) >> 2;  // query tile of this warp's group
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    const uint32_t s_addr = trow + L::S_COL + 128u * (uint32_t)x;
    const uint32_t o_addr = trow + L::O_COL + (uint32_t)(D * x);
    const unsigned full = 0xffffffffu;
    const float sl2 = p.scale_log2;
    long long sn = 0, on = 0;  // S_x tiles and work items consumed
    long long osel_n = 0;      // partial-row atoms loaded into this group's output stage (MERGE)
    for_each_window([&](int n_list) {
    for (int wi = 0; ok && wi < (n_list + 1) / 2; ++wi) {
      const Pair P = decode_pair<BN, KIND>(p, list, n_list, wi);
      if (x == 1 ? !P.valid1 : (PACKED && !P.valid0)) continue;
      const Unit u = x ? P.u1 : P.u0;
      const int seg0 = u.seg0;
      // Original position of this row's query (padding rows: the segment's last position).
      int i_orig = seg0 + p.S - 1;
      bool store_row = false;
      if (row < BN) {
        const int v = (!PERM || p.perm_q == nullptr)
                          ? u.b * BN + row
                          : __ldg(p.perm_q + u.qh * p.N + (size_t)u.b * BN + row);
        store_row = v >= seg0 && v < seg0 + p.S;
        i_orig = store_row ? v : seg0;
      }
      float m_run = -INFINITY, l_run = 0.f;
      const int n_items = u.lt + u.cnt;
      // kKindOnline: the listed blocks this unit keeps (all, unless its list stops early); the
      // flag is cleared before this unit's first P arrival.
      int kept = u.cnt;
      if (ONLINE && quad == 0 && lane == 0) stop_flag[x] = 0;
      // Keys of a selected block (for its mask) are requested before the wait for its S, the
      // block id one tile earlier.
      auto blk = [&](int n) {
        return PERM && !PACKED && n >= u.lt && n < n_items ? sel_block(p, u, n - u.lt) : -1;
      };
      int c_cur = blk(0), c_next = blk(1);
      // MERGE: the partial result of the permuted pass for this row is requested early.
      float lse_sel = -INFINITY;
      if (MERGE && store_row) lse_sel = __ldg(p.lse_in + (size_t)u.qh * p.N + i_orig);
      for (int n = 0; n < n_items; ++n) {
        // Per column group q (columns 32q..32q+31, this lane's column 32q + lane): the key's
        // original position (list streams), or the word of the chunk holding the column (packed
        // streams: chunk 2q + lane/16 of the tile).
        int keys[BN / 32];
        if (PACKED) {
          const long long cw0 = P.chunk0 + (long long)packed_unit_tile(P, x, n) * CPT + (lane >> 4);
#pragma unroll
          for (int q = 0; q < BN / 32; ++q) keys[q] = (int)__ldg(p.chunks + cw0 + 2 * q);
        } else {
#pragma unroll
          for (int q = 0; q < BN / 32; ++q)
            keys[q] = c_cur < 0 ? 0 : __ldg(p.perm_k + u.qh * p.N + (size_t)c_cur * BN + q * 32 + lane);
          c_cur = c_next;
          c_next = blk(n + 2);
        }
        // Warp-uniform outcome: the tcgen05.ld below is a warp-collective instruction.
        if (!__all_sync(full, mbar_wait(bar(kSFull + x), (uint32_t)(sn & 1), lim))) {
          ok = false;
          break;
        }
        ++sn;
        tc_fence_after();
        uint32_t s[BN];
#pragma unroll
        for (int c0 = 0; c0 < BN / 32; ++c0)
          tmem_ld32(s_addr + c0 * 32, *reinterpret_cast<uint32_t(*)[32]>(&s[c0 * 32]));
#pragma unroll
        for (int c0 = 0; c0 < BN / 32; ++c0)
          tmem_wait_ld(*reinterpret_cast<uint32_t(*)[32]>(&s[c0 * 32]));

        // Masks on original positions.
        if (!PERM || n < u.lt) {
          const int limit = i_orig - (seg0 + n * BN);  // keys col <= limit are causal
          if (__any_sync(full, limit < BN - 1)) {
#pragma unroll
            for (int c = 0; c < BN; ++c)
              if (c > limit) s[c] = __float_as_uint(-INFINITY);
          }
        } else {
          // Permuted tiles: keys before the segment (list streams), or the first v rows of each
          // 16-row chunk, v in the chunk word's low five bits (packed streams).
          uint32_t mw[BN / 32];
          bool all = true;
#pragma unroll
          for (int q = 0; q < BN / 32; ++q) {
            const bool valid = PACKED ? (int)(lane & 15) < (keys[q] & 31)
                                      : keys[q] >= 0 && keys[q] < seg0;
            mw[q] = __ballot_sync(full, valid);
            all = all && mw[q] == full;
          }
          if (!all) {
#pragma unroll
            for (int cc = 0; cc < BN; ++cc)
              if (!((mw[cc / 32] >> (cc % 32)) & 1u)) s[cc] = __float_as_uint(-INFINITY);
          }
        }
        // Row max with 8 independent partial results (no 128-long dependency chain), three inputs
        // per instruction.
        float mp[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) mp[q] = __uint_as_float(s[q]);
#pragma unroll
        for (int c = 8; c < BN; c += 16)
#pragma unroll
          for (int q = 0; q < 8; ++q)
            mp[q] = max3f(mp[q], __uint_as_float(s[c + q]), __uint_as_float(s[c + 8 + q]));
        const float mt = max3f(max3f(mp[0], mp[1], mp[2]), max3f(mp[3], mp[4], mp[5]),
                               fmaxf(mp[6], mp[7]));
        const float m_new = fmaxf(m_run, mt * sl2);
        const bool rescale = m_new > m_run + 8.0f;
        const float m_keep = rescale ? m_new : m_run;
        // A row whose columns are all masked so far has no maximum: its exponents use 0, and (in
        // the permuted pass, where that can happen) its running maximum stays −inf.
        const float m_use = m_keep == -INFINITY ? 0.f : m_keep;
        const float alpha = rescale ? ex2(m_run - m_use) : 1.f;
        // P = 2^(s·log2(e)/√d − m) as bf16 pairs, written over the first BN/2 columns of S_x.
        float sp[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        uint32_t pk[BN / 2];
#pragma unroll
        for (int c = 0; c < BN; c += 2) {
          const float p0 = ex2(fmaf(__uint_as_float(s[c]), sl2, -m_use));
          const float p1 = ex2(fmaf(__uint_as_float(s[c + 1]), sl2, -m_use));
          sp[c % 8] += p0;
          sp[(c + 1) % 8] += p1;
          pk[c / 2] = pack_bf16(p0, p1);
        }
        const float rs = ((sp[0] + sp[1]) + (sp[2] + sp[3])) + ((sp[4] + sp[5]) + (sp[6] + sp[7]));
#pragma unroll
        for (int c0 = 0; c0 < BN / 64; ++c0)
          tmem_st32(s_addr + c0 * 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[c0 * 32]));
        // O_x holds the products of earlier tiles (S_x's completion covers them): rescale it when
        // the running max moved.
        if (n > 0 && __any_sync(full, rescale)) {
#pragma unroll
          for (int c0 = 0; c0 < D / 32; ++c0) {
            uint32_t o[32];
            tmem_ld32(o_addr + c0 * 32, o);
            tmem_wait_ld(o);
#pragma unroll
            for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
            tmem_st32(o_addr + c0 * 32, o);
          }
        }
        tmem_wait_st();
        l_run = l_run * alpha + rs;
        m_run = PERM ? m_keep : m_use;
        // kKindOnline: after a listed block that is not the list's last, the block's measured
        // share of each row's running normaliser (this tile's exp-sum over the sum after it, both
        // against the same running maximum); the list stops when it is below τ for every row of
        // the block (a reduction over the group's 128 threads), and the flag tells the issuer
        // before this tile's P arrival.
        bool stop_now = false;
        if (ONLINE && n >= u.lt && n + 1 < n_items) {
          const bool keep = row < BN && store_row && rs / l_run >= p.stop_tau;
          stop_now = !named_bar_or(2 + x, 128, keep);
          if (stop_now && quad == 0 && lane == 0) stop_flag[x] = 1;
        }
        // One arrival per warp (after the warp's tensor-memory stores): arrivals on one barrier
        // are serialised, so 128 of them would delay the product by hundreds of cycles.
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kPFull + x));
        if (ONLINE && stop_now) {
          kept = n - u.lt + 1;
          break;
        }
      }
      if (!ok) break;
      // Epilogue: O/ℓ as bf16 at the query's original row.
      if (!__all_sync(full, mbar_wait(bar(kOFull + x), (uint32_t)(on & 1), lim))) {
        ok = false;
        break;
      }
      ++on;
      tc_fence_after();
      if (ONLINE && quad == 0 && lane == 0) p.stop_cnt[u.qh * p.nB + u.b] = kept;
      const float inv_l = 1.f / l_run;
      uint16_t *orow = p.o + ((size_t)u.qh * p.N + i_orig) * D;
      // MERGE: the row's final result combines this pass's O/ℓ with the permuted pass's partial
      // result o_sel (bf16, at the row's place in O) by their log2-sum-exps:
      // o = (2^lse_loc·O/ℓ + 2^lse_sel·o_sel) / (2^lse_loc + 2^lse_sel).
      float so = inv_l, ss = 0.f;
      if (MERGE && lse_sel > -INFINITY) {
        const float ll = m_run + __log2f(l_run);
        const float mm = fmaxf(ll, lse_sel);
        const float wa = ex2(ll - mm), wb = ex2(lse_sel - mm);
        const float inv = 1.f / (wa + wb);
        so = wa * inv * inv_l;
        ss = wb * inv;
      }
      if (PERM && p.sel_only) {
        // Partial result of the selected blocks: its log2-sum-exp for the merge (−inf, and no
        // row written, when no key of the row was visible).
        if (store_row)
          p.lse_out[(size_t)u.qh * p.N + i_orig] = l_run > 0.f ? m_run + __log2f(l_run) : -INFINITY;
        store_row = store_row && l_run > 0.f;
      }
      if (!PERM) {
        // Contiguous rows: each 64-column atom is staged in shared memory (128-byte swizzle) and
        // written with one TMA tile store; the group's first thread issues the stores and, before
        // its stage is overwritten, waits until the previous store has read it.
        const bool leader = quad == 0 && lane == 0;
        const uint32_t ost = sbase + L::OFF_OST + (uint32_t)x * L::ATOM_Q;
        unsigned char *ostp = smem + L::OFF_OST + x * L::ATOM_Q + row * 128;
        // MERGE: when a row of the tile has a partial result, each atom of the tile's rows of O
        // (the permuted pass's partial rows o_sel, at these original positions) is first loaded
        // into the stage by TMA, and every thread merges its row in place.
        const bool merge_tile = MERGE && named_bar_or(2 + x, 128, ss != 0.f);
#pragma unroll
        for (int a = 0; a < D / 64; ++a) {
          // This atom's 64 columns of O from TMEM (one atom at a time keeps the live set small).
          uint32_t o[64];
          tmem_ld32(o_addr + a * 64, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
          tmem_ld32(o_addr + a * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
          tmem_wait_ld(*reinterpret_cast<uint32_t(*)[32]>(&o[0]));
          tmem_wait_ld(*reinterpret_cast<uint32_t(*)[32]>(&o[32]));
          if (leader) bulk_wait_read();
          named_bar_sync(2 + x, 128);
          if (merge_tile) {
            if (leader) {
              mbar_expect_tx(bar(kOSel + x), (uint32_t)BN * 128u);  // BN rows of the atom
              tma_load_tile(ost, &tm_o_tile, a * 64, (int)(u.qh * p.N) + u.b * BN, bar(kOSel + x));
            }
            mbar_wait(bar(kOSel + x), (uint32_t)(osel_n & 1), lim);
            ++osel_n;
          }
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const int c = ch * 8;
            uint4 v;
            if (MERGE) {
              const uint4 sel = merge_tile ? *reinterpret_cast<const uint4 *>(ostp + ((ch ^ (row & 7)) * 16))
                                           : make_uint4(0, 0, 0, 0);
              auto mix = [&](int cc, uint32_t w2) {
                const float lo = __uint_as_float(w2 << 16), hi = __uint_as_float(w2 & 0xffff0000u);
                return pack_bf16(fmaf(__uint_as_float(o[cc]), so, lo * ss),
                                 fmaf(__uint_as_float(o[cc + 1]), so, hi * ss));
              };
              v.x = mix(c + 0, sel.x);
              v.y = mix(c + 2, sel.y);
              v.z = mix(c + 4, sel.z);
              v.w = mix(c + 6, sel.w);
            } else {
              v.x = pack_bf16(__uint_as_float(o[c + 0]) * inv_l, __uint_as_float(o[c + 1]) * inv_l);
              v.y = pack_bf16(__uint_as_float(o[c + 2]) * inv_l, __uint_as_float(o[c + 3]) * inv_l);
              v.z = pack_bf16(__uint_as_float(o[c + 4]) * inv_l, __uint_as_float(o[c + 5]) * inv_l);
              v.w = pack_bf16(__uint_as_float(o[c + 6]) * inv_l, __uint_as_float(o[c + 7]) * inv_l);
            }
            *reinterpret_cast<uint4 *>(ostp + ((ch ^ (row & 7)) * 16)) = v;
          }
          fence_proxy_async_smem();
          named_bar_sync(2 + x, 128);
          if (leader) {
            tma_store_tile(&tm_o_tile, a * 64, (int)(u.qh * p.N) + u.b * BN, ost);
            bulk_commit();
          }
        }
      } else {
        // The whole row of O from TMEM (one wait), then 32-byte stores (full sectors). Every
        // thread of the warp takes part in the loads (they are warp-collective); only the rows
        // this pass writes are stored (a row of the merge path's permuted pass with no visible
        // key is not).
        uint32_t o[D];
#pragma unroll
        for (int c0 = 0; c0 < D / 32; ++c0)
          tmem_ld32(o_addr + c0 * 32, *reinterpret_cast<uint32_t(*)[32]>(&o[c0 * 32]));
#pragma unroll
        for (int c0 = 0; c0 < D / 32; ++c0) tmem_wait_ld(*reinterpret_cast<uint32_t(*)[32]>(&o[c0 * 32]));
#pragma unroll
        for (int c = 0; store_row && c < D / 16; ++c) {
          uint32_t w[8];
#pragma unroll
          for (int q = 0; q < 8; ++q)
            w[q] = pack_bf16(__uint_as_float(o[c * 16 + 2 * q]) * inv_l,
                             __uint_as_float(o[c * 16 + 2 * q + 1]) * inv_l);
          if (p.o_v8) {
            st_global_v8(orow + c * 16, w);
          } else {
            reinterpret_cast<uint4 *>(orow + c * 16)[0] = make_uint4(w[0], w[1], w[2], w[3]);
            reinterpret_cast<uint4 *>(orow + c * 16)[1] = make_uint4(w[4], w[5], w[6], w[7]);
          }
        }
      }
      tc_fence_before();
    }
    });
    // The output stores of this group's stage complete before the CTA exits (and the last
    // partial-row load into it, should a wait for it have given up).
    if (quad == 0 && lane == 0) {
      bulk_wait_all();
      if (MERGE && osel_n > 0) mbar_wait(bar(kOSel + x), (uint32_t)((osel_n - 1) & 1), kDrainNs);
    }
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

// ------------------------------------------------------------------ permuted copy of K and V

// The path of a call with a workspace, decided on the device without synchronising (one CTA):
//   bit 1 (merge path): the permuted pass runs only the selected blocks and the local pass merges
//     its partial rows; otherwise the local pass runs alone and the permuted pass reruns each busy
//     query block's local tiles. Rerunning costs about S/B tiles per busy block, the merge a
//     fixed few per cent of the local pass: merge when more than 1/25 of the query blocks have a
//     selection (mode 1), always (modes 0 and 2), never (mode 3 is decided on the host).
//   bit 0 (packed streams, with bit 1): when the selected blocks outnumber twice the blocks the
//     permuted copy writes (copying a block costs about one gather of it; mode 1), always
//     (mode 2), never (mode 0).
__global__ void __launch_bounds__(1024)
    k_copy_decide(const int32_t *__restrict__ sel_cnt, long long n_units, int nB, int mode,
                  long long copy_blocks, uint32_t *__restrict__ flag) {
  __shared__ unsigned long long part[32], part_busy[32];
  unsigned long long sum = 0, busy = 0;
  for (long long i = threadIdx.x; i < n_units; i += blockDim.x) {
    const int c = min(max(__ldg(sel_cnt + i), 0), nB);
    sum += (unsigned long long)c;
    busy += c > 0 ? 1ull : 0ull;
  }
  for (int o = 16; o > 0; o >>= 1) {
    sum += __shfl_xor_sync(0xffffffffu, sum, o);
    busy += __shfl_xor_sync(0xffffffffu, busy, o);
  }
  if (threadIdx.x % 32 == 0) {
    part[threadIdx.x / 32] = sum;
    part_busy[threadIdx.x / 32] = busy;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long total = 0, total_busy = 0;
    for (int w = 0; w < (int)(blockDim.x / 32); ++w) {
      total += part[w];
      total_busy += part_busy[w];
    }
    const bool packed =
        mode == 2 || (mode == 1 && total > 2ull * (unsigned long long)copy_blocks);
    const bool merge = mode == 0 || packed ||
                       (mode == 1 && 25ull * total_busy > (unsigned long long)n_units);
    *flag = (packed ? 1u : 0u) | (merge ? 2u : 0u);
  }
}

// The (batch, query head) of copy head h: the head itself, or the first query head of KV head h
// when the copy is per KV head.
__device__ __forceinline__ long long copy_query_head(long long h, int per_kv, int Hq, int Hkv,
                                                     int G) {
  return per_kv ? (h / Hkv) * Hq + (h % Hkv) * G : h;
}

// Key order inside each block of the permuted copy (bit 0 only): one warp per (copy head, key
// block) sorts the block's B original positions ascending (ranks by (position, slot), so any
// index contents give a permutation of the block's slots) into pos_sorted, and counts for every
// segment s the block's keys before s·S into vis[h][s][c]. With the rows of a block in position
// order, the keys of block c that a query of segment s may see (original position < s·S) are its
// first vis[h][s][c] rows.
template <int B>
__global__ void __launch_bounds__(256)
    k_block_sort(const int32_t *__restrict__ perm_k, int32_t *__restrict__ pos_sorted,
                 uint8_t *__restrict__ vis, long long copy_heads, int N, int S, int nB, int nSeg,
                 int Hq, int Hkv, int G, int per_kv, const uint32_t *__restrict__ flag) {
  if ((__ldg(flag) & 1u) == 0u) return;
  constexpr int E = B / 32;
  __shared__ int sv[8][B];
  __shared__ int ss[8][B];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long gw = (long long)blockIdx.x * 8 + warp;
  if (gw >= copy_heads * nB) return;
  const long long h = gw / nB;
  const int c = (int)(gw % nB);
  const long long qh = copy_query_head(h, per_kv, Hq, Hkv, G);
  const int32_t *src = perm_k + qh * N + (long long)c * B;
  int x[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    x[e] = min(max(__ldg(src + e * 32 + lane), 0), N - 1);
    sv[warp][e * 32 + lane] = x[e];
  }
  __syncwarp();
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = e * 32 + lane;
    int rank = 0;
    for (int j = 0; j < B; ++j) {
      const int y = sv[warp][j];
      rank += (y < x[e] || (y == x[e] && j < i)) ? 1 : 0;
    }
    ss[warp][rank] = x[e];
    pos_sorted[h * N + (long long)c * B + rank] = x[e];
  }
  __syncwarp();
  for (int s = lane; s < nSeg; s += 32) {
    const int bound = s * S;
    int lo = 0, hi = B;  // first slot whose position is >= bound
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (ss[warp][mid] < bound) lo = mid + 1;
      else hi = mid;
    }
    vis[((size_t)h * nSeg + s) * nB + c] = (uint8_t)lo;
  }
}

// kp[h·N + rank] = K row pos_sorted[h·N + rank] of h's KV head, and the same for V (h a copy
// head). 16-byte pieces, grid-stride; nothing when the flag's bit 0 is clear.
template <int D>
__global__ void __launch_bounds__(256)
    k_permute_kv(const uint4 *__restrict__ k, const uint4 *__restrict__ v,
                 const int32_t *__restrict__ pos_sorted, uint4 *__restrict__ kp,
                 uint4 *__restrict__ vp, long long copy_rows, int N, int Hq, int Hkv, int G,
                 int per_kv, const uint32_t *__restrict__ flag) {
  if ((__ldg(flag) & 1u) == 0u) return;
  constexpr int PIECES = D * 2 / 16;  // 16-byte pieces per row
  const long long n = copy_rows * PIECES;
  for (long long x = (long long)blockIdx.x * blockDim.x + threadIdx.x; x < n;
       x += (long long)gridDim.x * blockDim.x) {
    const long long row = x / PIECES;
    const int piece = (int)(x % PIECES);
    const long long h = row / N;
    // KV head of copy head h.
    const long long kh = per_kv ? h : (h / Hq) * Hkv + (h % Hq) / G;
    const int j = min(max(__ldg(pos_sorted + row), 0), N - 1);
    const long long src = (kh * N + j) * PIECES + piece;
    kp[x] = __ldg(k + src);
    vp[x] = __ldg(v + src);
  }
}

// Packed streams (bit 0 only): one warp per pair of units (units 2w and 2w+1 in packed order).
// Each unit's selected list becomes a bitmap of key blocks in shared memory. When both units have
// selections and read one copy head and one segment, the blocks both selected form the pair's
// shared group and the rest each unit's own group; otherwise each unit's blocks are its own group.
// Every group, in block order, is cut into chunks of 16 rows of the permuted copy: block c gives
// ceil(n/16) chunks for its n visible keys (n = vis of the unit's copy head, segment and c), chunk
// i covering rows 16i.. of the block, of which min(16, n − 16i) are visible. The chunk word is
// (row16 << 5) | visible, row16 = c·B/16 + i the chunk's place in the copy head. Each group is
// padded with empty chunks (row16 0, visible 0) to whole tiles of BN/16 chunks; the pair's list is
// [shared group][unit 0's group][unit 1's group] from chunks + w·cap, and pair_meta[w] holds the
// three tile counts. cap = 2·nB·B/16 + 3·B/16 holds two units' blocks with their padding.
template <int BN>
__global__ void __launch_bounds__(256)
    k_pack_pairs(const int32_t *__restrict__ sel_cnt, const int32_t *__restrict__ sel_blk,
                 const uint8_t *__restrict__ vis, uint32_t *__restrict__ chunks,
                 int4 *__restrict__ pair_meta, long long cap, long long n_units, int nB, int S,
                 int nSeg, int Hq, int Hkv, int G, int per_kv, int pair_heads,
                 const uint32_t *__restrict__ flag) {
  if ((__ldg(flag) & 1u) == 0u) return;
  constexpr int CPT = BN / kChunkRows;
  constexpr int kMaxWords = 64;  // nB <= 2048
  __shared__ uint32_t sw[8][2][kMaxWords];
  const unsigned full = 0xffffffffu;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long w = (long long)blockIdx.x * 8 + warp;
  const long long n_pairs = (n_units + 1) / 2;
  if (w >= n_pairs) return;
  const int nwords = (nB + 31) / 32, per_seg = S / BN;
  long long qh[2], hc[2];
  int sg[2], cnt[2];
  for (int x = 0; x < 2; ++x) {
    long long u = 2 * w + x;
    const bool has = u < n_units;
    if (!has) u = 2 * w;
    int hi, bl, s;
    if (!pair_heads) {
      bl = (int)(u % per_seg);
      u /= per_seg;
      s = (int)(u % nSeg);
      u /= nSeg;
      hi = (int)(u % G);
      u /= G;
    } else {
      hi = (int)(u % G);
      u /= G;
      bl = (int)(u % per_seg);
      u /= per_seg;
      s = (int)(u % nSeg);
      u /= nSeg;
    }
    const int g = (int)(u % Hkv);
    const long long beta = u / Hkv;
    qh[x] = beta * Hq + (long long)g * G + hi;
    hc[x] = per_kv ? beta * Hkv + g : qh[x];
    sg[x] = s;
    const long long qb = qh[x] * nB + (long long)s * per_seg + bl;
    cnt[x] = has ? min(max(__ldg(sel_cnt + qb), 0), nB) : 0;
    for (int i = lane; i < kMaxWords; i += 32) sw[warp][x][i] = 0u;
    __syncwarp();
    const int32_t *row = sel_blk + qb * nB;
    for (int e = lane; e < cnt[x]; e += 32) {
      const int c = min(max(__ldg(row + e), 0), nB - 1);
      atomicOr(&sw[warp][x][c >> 5], 1u << (c & 31));
    }
    __syncwarp();
  }
  const bool shared = cnt[0] > 0 && cnt[1] > 0 && hc[0] == hc[1] && sg[0] == sg[1];
  uint32_t *out = chunks + w * cap;
  long long pos = 0;  // chunks written so far (warp-uniform)
  int T[3];
  for (int grp = 0; grp < 3; ++grp) {
    const long long start = pos;
    const int x = grp == 2 ? 1 : 0;
    const uint8_t *vrow = vis + ((size_t)hc[x] * nSeg + sg[x]) * nB;
    for (int w0 = 0; w0 < nwords; w0 += 32) {
      const int wd = w0 + lane;
      uint32_t m = 0u;
      if (wd < nwords) {
        const uint32_t a = sw[warp][0][wd], b = sw[warp][1][wd];
        m = grp == 0 ? (shared ? a & b : 0u) : grp == 1 ? (shared ? a & ~b : a)
                                                       : (shared ? b & ~a : b);
      }
      int mine = 0;
      for (uint32_t r = m; r; r &= r - 1) {
        const int c = 32 * wd + __ffs(r) - 1;
        mine += (__ldg(vrow + c) + kChunkRows - 1) / kChunkRows;
      }
      int incl = mine;
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(full, incl, o);
        if (lane >= o) incl += t;
      }
      long long at = pos + incl - mine;
      for (uint32_t r = m; r; r &= r - 1) {
        const int c = 32 * wd + __ffs(r) - 1;
        const int n = __ldg(vrow + c);
        for (int i = 0; i * kChunkRows < n; ++i) {
          const uint32_t row16 = (uint32_t)c * (BN / kChunkRows) + (uint32_t)i;
          out[at++] = (row16 << 5) | (uint32_t)min(kChunkRows, n - i * kChunkRows);
        }
      }
      pos += __shfl_sync(full, incl, 31);
    }
    T[grp] = (int)((pos - start + CPT - 1) / CPT);
    const long long end = start + (long long)T[grp] * CPT;
    for (long long i = pos + lane; i < end; i += 32) out[i] = 0u;
    pos = end;
  }
  if (lane == 0) pair_meta[w] = make_int4(T[0], T[1], T[2], 0);
}

// Tile counts of the packed streams of the last call (bit 0 only): acc[0] += Σ tiles loaded
// (shared + unit 0 + unit 1), acc[1] += Σ tile products (2·shared + unit 0 + unit 1).
__global__ void __launch_bounds__(256)
    k_packed_counts(const int4 *__restrict__ pair_meta, long long n_pairs,
                    const uint32_t *__restrict__ flag, unsigned long long *__restrict__ acc) {
  if ((__ldg(flag) & 1u) == 0u) return;
  unsigned long long loaded = 0, products = 0;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n_pairs;
       i += (long long)gridDim.x * blockDim.x) {
    const int4 m = __ldg(pair_meta + i);
    loaded += (unsigned long long)(m.x + m.y + m.z);
    products += (unsigned long long)(2 * m.x + m.y + m.z);
  }
  for (int o = 16; o > 0; o >>= 1) {
    loaded += __shfl_xor_sync(0xffffffffu, loaded, o);
    products += __shfl_xor_sync(0xffffffffu, products, o);
  }
  if (threadIdx.x % 32 == 0) {
    atomicAdd(acc, loaded);
    atomicAdd(acc + 1, products);
  }
}

// Work of the permuted pass without packed streams: acc[0] += Σ over busy query blocks of
// (local tiles + selected blocks) (the path without the merge reruns the local tiles),
// acc[1] += Σ selected blocks (the merge path with gathered blocks).
__global__ void __launch_bounds__(256)
    k_busy_tiles(const int32_t *__restrict__ sel_cnt, const int32_t *__restrict__ local_tiles,
                 long long n_units, int nB, int per_seg, unsigned long long *__restrict__ acc) {
  unsigned long long rerun = 0, sel = 0;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n_units;
       i += (long long)gridDim.x * blockDim.x) {
    const int c = min(max(__ldg(sel_cnt + i), 0), nB);
    if (c > 0) rerun += (unsigned long long)(c + min(max(__ldg(local_tiles + i), 1), per_seg));
    sel += (unsigned long long)c;
  }
  for (int o = 16; o > 0; o >>= 1) {
    rerun += __shfl_xor_sync(0xffffffffu, rerun, o);
    sel += __shfl_xor_sync(0xffffffffu, sel, o);
  }
  if (threadIdx.x % 32 == 0) {
    atomicAdd(acc, rerun);
    atomicAdd(acc + 1, sel);
  }
}

// Rows without a partial result from the permuted pass: lse = −inf (merge path only).
__global__ void __launch_bounds__(256)
    k_fill_neg_inf(float *__restrict__ p, long long n, const uint32_t *__restrict__ flag) {
  if (flag != nullptr && (__ldg(flag) & 2u) == 0u) return;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x)
    p[i] = -INFINITY;
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

// Streaming multiprocessors of the current device (cached per device).
int sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  if (dev >= 0 && dev < 64) cache[dev] = n;
  return n;
}

template <int D, int BN>
cudaError_t launch_t(const Dims &d, const AttnArgs &a, uint64_t limit_ns, int max_ctas,
                     cudaStream_t st) {
  using L = Layout<D, BN>;
  static_assert(L::SMEM <= 232448, "shared memory budget");
  static_assert(kNumBars * 8 + 4 <= kStopFlagAt && kStopFlagAt + 8 <= (int)L::BAR_BYTES,
                "barrier area");
  CUtensorMap tq, tqr, tk, tkr, tv, tvr, to, tkp, tvp;
  const long long q_rows = d.bhq() * d.N, kv_rows = d.bhkv() * d.N;
  if (!make_map(&tq, a.q, q_rows, D, BN) || !make_map(&tqr, a.q, q_rows, D, 1) ||
      !make_map(&tk, a.k, kv_rows, D, BN) || !make_map(&tkr, a.k, kv_rows, D, 1) ||
      !make_map(&tv, a.v, kv_rows, D, BN) || !make_map(&tvr, a.v, kv_rows, D, 1) ||
      !make_map(&to, a.o, q_rows, D, BN))
    return cudaErrorInvalidValue;
  // The permuted copy's maps, 16-row boxes (without a copy they repeat K's and V's row maps and
  // are never used).
  const bool packed = a.merge && a.copy_flag != nullptr && a.kp != nullptr && a.vp != nullptr &&
                      a.chunks != nullptr && a.pair_meta != nullptr;
  const long long copy_rows = (a.copy_per_kv ? d.bhkv() : d.bhq()) * d.N;
  if (packed) {
    if (!make_map(&tkp, a.kp, copy_rows, D, kChunkRows) ||
        !make_map(&tvp, a.vp, copy_rows, D, kChunkRows))
      return cudaErrorInvalidValue;
  } else {
    tkp = tkr;
    tvp = tvr;
  }
  cudaError_t e = cudaSuccess;
  for (auto fn : {s2o_attention_kernel<D, BN, kKindContig>, s2o_attention_kernel<D, BN, kKindList>,
                  s2o_attention_kernel<D, BN, kKindPacked>, s2o_attention_kernel<D, BN, kKindMerge>,
                  s2o_attention_kernel<D, BN, kKindOnline>})
    if ((e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)L::SMEM)) != cudaSuccess)
      return e;
  Params p;
  p.perm_q = a.perm_q;
  p.perm_k = a.perm_k;
  p.sel_cnt = a.sel_cnt;
  p.sel_blk = a.sel_blk;
  p.local_tiles = a.local_tiles;
  p.o = static_cast<uint16_t *>(a.o);
  p.o_v8 = (reinterpret_cast<uintptr_t>(a.o) & 31u) == 0 ? 1 : 0;
  p.N = d.N;
  p.nB = d.nB;
  p.Hq = d.Hq;
  p.Hkv = d.Hkv;
  p.G = d.G;
  p.n_units = d.bhq() * d.nB;
  if (p.n_units > 0x7fffffffLL) return cudaErrorInvalidValue;  // unit ids are 32-bit
  p.n_items = (p.n_units + 1) / 2;
  p.scale_log2 = (float)(1.4426950408889634 / __builtin_sqrt((double)D));
  p.limit_ns = limit_ns;
  p.div_G.init(d.G);
  p.div_nB.init(d.nB);
  p.div_Hkv.init(d.Hkv);
  p.sel_only = 0;
  p.lse_out = nullptr;
  p.lse_in = nullptr;
  p.copy_per_kv = a.copy_per_kv ? 1 : 0;
  p.chunks = a.chunks;
  p.pair_meta = a.pair_meta;
  p.chunk_cap = a.chunk_cap;
  p.pair_heads = a.copy_per_kv ? 1 : 0;
  p.stop_cnt = a.stop_cnt;
  p.stop_tau = a.stop_tau;
  auto launch = [&](int mode, int skip_empty, int kind) -> cudaError_t {
    p.mode = mode;
    p.skip_empty = skip_empty;
    p.S = mode == kDense ? d.N : d.S;
    p.nSeg = mode == kDense ? 1 : d.nSeg;
    p.div_seg.init(p.S / BN);
    p.div_nSeg.init(p.nSeg);
    const long long work =
        skip_empty && (kind == kKindList || kind == kKindOnline) ? p.n_units : p.n_items;
    const long long cap = max_ctas > 0 && max_ctas < sm_count() ? max_ctas : sm_count();
    const long long grid = work < cap ? work : cap;
    switch (kind) {
      case kKindContig:
        s2o_attention_kernel<D, BN, kKindContig><<<(unsigned)grid, kThreads, L::SMEM, st>>>(
            tq, tqr, tk, tkr, tv, tvr, to, tkp, tvp, p);
        break;
      case kKindList:
        s2o_attention_kernel<D, BN, kKindList><<<(unsigned)grid, kThreads, L::SMEM, st>>>(
            tq, tqr, tk, tkr, tv, tvr, to, tkp, tvp, p);
        break;
      case kKindPacked:
        s2o_attention_kernel<D, BN, kKindPacked><<<(unsigned)grid, kThreads, L::SMEM, st>>>(
            tq, tqr, tk, tkr, tv, tvr, to, tkp, tvp, p);
        break;
      case kKindOnline:
        s2o_attention_kernel<D, BN, kKindOnline><<<(unsigned)grid, kThreads, L::SMEM, st>>>(
            tq, tqr, tk, tkr, tv, tvr, to, tkp, tvp, p);
        break;
      default:
        s2o_attention_kernel<D, BN, kKindMerge><<<(unsigned)grid, kThreads, L::SMEM, st>>>(
            tq, tqr, tk, tkr, tv, tvr, to, tkp, tvp, p);
    }
    note_launch();
    return cudaGetLastError();
  };
  p.copy_flag = nullptr;
  p.run_mask = p.run_value = 0u;
  if (a.dense) return launch(kDense, 0, kKindContig);
  // The path without a workspace: every row first gets the dense local window of its segment,
  // computed in original order (causal triangles, masks on diagonal tiles only); then the query
  // blocks whose selected list is not empty are recomputed in full (local tiles and selected
  // blocks, permuted order) and overwrite their rows. Each row's result is the attention over its
  // key set either way.
  auto legacy = [&]() -> cudaError_t {
    cudaError_t r = launch(kLocal, 0, kKindContig);
    if (r != cudaSuccess) return r;
    return launch(kPermuted, 1, a.stop_cnt != nullptr ? kKindOnline : kKindList);
  };
  if (!a.merge || a.lse == nullptr) return legacy();
  // With a workspace every path is launched and the device-side decision word lets one run (the
  // others return at once). Merge path: the permuted pass runs only the selected blocks (gathered,
  // or packed streams) and leaves each row's partial result and its log2-sum-exp (−inf for rows
  // it does not reach); the local pass then computes the local window in original order and
  // merges the two.
  p.copy_flag = a.copy_flag;
  const long long n_rows = d.bhq() * d.N;
  const unsigned fill_grid = (unsigned)std::min<long long>((n_rows + 255) / 256, 148ll * 16);
  k_fill_neg_inf<<<fill_grid, 256, 0, st>>>(a.lse, n_rows, a.copy_flag);
  note_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  p.sel_only = 1;
  p.lse_out = a.lse;
  p.run_mask = 3u;  // merge path with gathered blocks
  p.run_value = 2u;
  if ((e = launch(kPermuted, 1, kKindList)) != cudaSuccess) return e;
  if (packed) {
    p.run_mask = p.run_value = 1u;  // packed streams
    if ((e = launch(kPermuted, 1, kKindPacked)) != cudaSuccess) return e;
  }
  p.sel_only = 0;
  p.lse_out = nullptr;
  p.lse_in = a.lse;
  p.run_mask = p.run_value = 2u;  // the merging local pass
  if ((e = launch(kLocal, 0, kKindMerge)) != cudaSuccess) return e;
  p.lse_in = nullptr;
  p.run_mask = 2u;  // the path without the merge
  p.run_value = 0u;
  return a.copy_flag != nullptr ? legacy() : cudaSuccess;
}

}  // namespace

cudaError_t launch_permuted_copy(const Dims &d, const AttnArgs &a, int mode, uint32_t *flag,
                                 cudaStream_t st) {
  if (!a.kp || !a.vp || !flag || !a.sel_cnt || !a.perm_k || !a.pos_sorted || !a.vis ||
      !a.chunks || !a.pair_meta)
    return cudaErrorInvalidValue;
  const long long copy_heads = a.copy_per_kv ? d.bhkv() : d.bhq();
  const long long copy_rows = copy_heads * d.N;
  const long long n_units = d.bhq() * d.nB;
  k_copy_decide<<<1, 1024, 0, st>>>(a.sel_cnt, n_units, d.nB, mode, copy_rows / d.B, flag);
  note_launch();
  const unsigned sort_grid = (unsigned)((copy_heads * d.nB + 7) / 8);
  if (d.B == 128)
    k_block_sort<128><<<sort_grid, 256, 0, st>>>(a.perm_k, a.pos_sorted, a.vis, copy_heads, d.N,
                                                 d.S, d.nB, d.nSeg, d.Hq, d.Hkv, d.G,
                                                 a.copy_per_kv ? 1 : 0, flag);
  else
    k_block_sort<64><<<sort_grid, 256, 0, st>>>(a.perm_k, a.pos_sorted, a.vis, copy_heads, d.N,
                                                d.S, d.nB, d.nSeg, d.Hq, d.Hkv, d.G,
                                                a.copy_per_kv ? 1 : 0, flag);
  note_launch();
  const unsigned grid = (unsigned)sm_count() * 8u;
  if (d.D == 128)
    k_permute_kv<128><<<grid, 256, 0, st>>>(
        static_cast<const uint4 *>(a.k), static_cast<const uint4 *>(a.v), a.pos_sorted,
        static_cast<uint4 *>(const_cast<void *>(a.kp)), static_cast<uint4 *>(const_cast<void *>(a.vp)),
        copy_rows, d.N, d.Hq, d.Hkv, d.G, a.copy_per_kv ? 1 : 0, flag);
  else
    k_permute_kv<64><<<grid, 256, 0, st>>>(
        static_cast<const uint4 *>(a.k), static_cast<const uint4 *>(a.v), a.pos_sorted,
        static_cast<uint4 *>(const_cast<void *>(a.kp)), static_cast<uint4 *>(const_cast<void *>(a.vp)),
        copy_rows, d.N, d.Hq, d.Hkv, d.G, a.copy_per_kv ? 1 : 0, flag);
  note_launch();
  const long long n_pairs = (n_units + 1) / 2;
  const unsigned pack_grid = (unsigned)((n_pairs + 7) / 8);
  if (d.B == 128)
    k_pack_pairs<128><<<pack_grid, 256, 0, st>>>(a.sel_cnt, a.sel_blk, a.vis, a.chunks,
                                                 a.pair_meta, a.chunk_cap, n_units, d.nB, d.S,
                                                 d.nSeg, d.Hq, d.Hkv, d.G, a.copy_per_kv ? 1 : 0,
                                                 a.copy_per_kv ? 1 : 0, flag);
  else
    k_pack_pairs<64><<<pack_grid, 256, 0, st>>>(a.sel_cnt, a.sel_blk, a.vis, a.chunks,
                                                a.pair_meta, a.chunk_cap, n_units, d.nB, d.S,
                                                d.nSeg, d.Hq, d.Hkv, d.G, a.copy_per_kv ? 1 : 0,
                                                a.copy_per_kv ? 1 : 0, flag);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_packed_counts(const Dims &d, const int4 *pair_meta, const uint32_t *flag,
                                 unsigned long long *acc, cudaStream_t st) {
  const long long n_pairs = (d.bhq() * d.nB + 1) / 2;
  const unsigned grid = (unsigned)std::min<long long>((n_pairs + 255) / 256, 148ll * 4);
  k_packed_counts<<<grid, 256, 0, st>>>(pair_meta, n_pairs, flag, acc);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_busy_tiles(const Dims &d, const int32_t *sel_cnt, const int32_t *local_tiles,
                              unsigned long long *acc, cudaStream_t st) {
  const long long n_units = d.bhq() * d.nB;
  const unsigned grid = (unsigned)std::min<long long>((n_units + 255) / 256, 148ll * 4);
  k_busy_tiles<<<grid, 256, 0, st>>>(sel_cnt, local_tiles, n_units, d.nB, d.S / d.B, acc);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_attention(const Dims &d, const AttnArgs &a, uint64_t wait_limit_ns,
                             int max_ctas, cudaStream_t st) {
  if (d.D == 128 && d.B == 128) return launch_t<128, 128>(d, a, wait_limit_ns, max_ctas, st);
  if (d.D == 128 && d.B == 64) return launch_t<128, 64>(d, a, wait_limit_ns, max_ctas, st);
  if (d.D == 64 && d.B == 128) return launch_t<64, 128>(d, a, wait_limit_ns, max_ctas, st);
  return launch_t<64, 64>(d, a, wait_limit_ns, max_ctas, st);
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
