// pa_decode_tc.cu -- decode attention with the grouped-query tile on the 5th-generation
// tensor cores (tcgen05, sm_100a).
//
// With g = Hq / Hkv query heads per kv head, every K/V byte the decode reads
// takes part in g multiply-adds for QK^T and g for PV: a skinny contraction
// that costs CUDA cores about as much time as the HBM read once g >= 4.  This
// kernel moves both products onto tcgen05.mma and keeps the read on TMA:
//
//   S^T[128 rows x N]  = K_tile[128 rows x 128 d] . Q^T[128 d x N]     (A K-major, B K-major)
//   O^T[128 d x N]     = V_tile^T[128 d x 128 rows] . P^T[128 rows x N] (A MN-major, B MN-major)
//
// with fp16/bf16 operands and fp32 accumulators in tensor memory (TMEM).
//
// Items.  An item is one partition (partition_tokens rows) of a row list of
// one kv head (or of two), read for a set of query columns (N = 16 or 32):
//   - a sequence: its tokens, for its g query heads; with several query
//     tokens per sequence (verifying speculated tokens, chunked prefill:
//     5688vip.com vLLM notes, section 2.2) for Tq x g columns, query t seeing
//     tokens below ctx - Tq + t + 1, so that every K/V tile is read once for
//     all of them;
//   - where kv heads pair up, two heads at once: a tile is then 64 tokens of
//     both heads as the 128 MMA rows (16-row groups of head 2e and of head
//     2e+1 alternate), so that one TMA box carries 4 KB (16 rows of both heads)
//     instead of 2 KB: the rate at which one SM issues boxes bounds this
//     kernel.  A row's logits against the other head's queries are computed
//     and discarded (p = 0), which the tensor cores can afford;
//   - a group of sequences whose block tables begin with the same physical
//     blocks (shared_prefix), for members x g columns: the row list is the
//     T shared tokens, read once for every member (zingnex.cn,
//     "vLLM与PagedAttention深度剖析", section 3.2 item 3: beam candidates share
//     blocks; jsqmd.com, "vLLM-v0.11.0性能实测", section 4.2: requests with the
//     same prefix share pages), then each member's own tokens, each run
//     rounded up to 16 rows and seen by that member's columns only.  A
//     sequence alone is a group of one with no shared tokens.
// Every 16-row group of an item carries its owner (a member, or every member)
// and its first token; every member its token limit and where its result
// goes: the output itself (a single partial), a split-K slot, or nowhere (no
// row of this partition is its).
//
// The softmax stays in fp32 on the CUDA cores: tcgen05.ld gives thread t (of
// 128) the logits of MMA row t, and thread t writes its row of P.  The output
// accumulates in TMEM across the tiles of an item: each column keeps a
// softmax reference m_ref that moves only when a logit exceeds it by more than
// 8 (log2 units).  Then the tile's column maxima are found (a transposed warp
// reduction plus shared memory), and thread d folds row d of O^T into
// registers, rescaled by 2^(m_old - m_new).  On other tiles nothing waits for
// the PV product: it is read once, at the end of the item.  The products are
// pipelined by tile: S^T(j+1) is issued as soon as every thread has read
// S^T(j), while tile j's softmax runs, and the softmax of tile j waits for
// O^T(j-1) only to store P(j) (or to fold O^T).  The probabilities enter the
// PV product as two terms of the input type, hi = round(p) and lo = round(p -
// hi), so they carry about 16 significant bits (a bf16 P alone, 8 bits, can
// move a short context's output by more than 2e-3); the two terms sit side by
// side as 2N columns of one PV product, so each V slice is read once for both.
//
// Warps.  One persistent CTA per SM.  A scheduler warp takes items (its first
// one by number, then from a counter in the workspace whose value carries the
// call's epoch), resolves each 16-row group through its block table and fills
// one of two item slots (descriptor, pool rows, group and member tables, and
// the query rows by one TMA box), up to two items ahead; two producer warps
// issue the tiles' tiled TMA loads, one the K half and one the V half of each
// stage, one box per lane (per tile and half: 8 groups of one head or 4 groups
// of two heads, x two 64-element halves, 128B-swizzled), into one of three
// stages whose halves are freed apart (K once S^T is computed, V once O^T
// is); a dedicated MMA warp issues every MMA and commits it to an mbarrier;
// the compute warps consume tiles in order and tell it through two more
// mbarriers when S^T(g) has been read and when P(g) has been written.  With
// an E4M3 cache, converter warps widen K into TMEM and V into shared memory
// (see Layout).  A launch over shared-prefix row lists may also take the
// per-sequence items of the own tokens no list holds (WIDE).  Without a plan, items are numbered partition 0 of
// every sequence first, then each sequence's further partitions (measured 2 %
// faster on mistral_7b_gqa than full partitions first and the shorter last
// ones after them); with one (only some sequences are units), full partitions
// first and the shorter last ones after them.
// Rows that are no token of any column are masked in P and their V rows are
// zeroed in shared memory before the PV product, so stale or NaN rows never
// reach the result.
//
// Split-K partials and the merge kernel are shared with the CUDA-core path.
//
// Every wait is bounded.  The compute warps wait per warp, and an OR-reduced
// named barrier then makes them all take the same way out when any wait
// failed (every decision before a named barrier comes from a barrier result).
// On the way out the producer waits for its TMA copies, the MMA warp commits
// once more and waits for all its MMAs, and warp 0 frees the TMEM columns.
#include <cuda.h>
#include <cuda_runtime.h>

#include <climits>
#include <type_traits>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {
namespace tc {

constexpr int kTile = 128;          // MMA rows per tile (M)
constexpr int kD = 128;             // head_dim of this path
constexpr int kGroupRows = 16;      // rows per TMA box (a block is a multiple)
constexpr int kSlots = 2;           // item slots
constexpr int kStages = 3;          // K/V stages of 64 KB (K and V halves filled and freed apart)
constexpr int kMaxGroups = 32;      // 16-row groups per item (partition_tokens <= 512)
constexpr int kMaxUnits = kSharedPrefixSeqsPerLaunch;  // sequences per launch (256)
// Where a member's result for an item goes (codes >= 0 are split-K slots).
constexpr int kSkip = -1, kDirect = -2, kZero = -3;

// Compute warpgroups split the NC query columns: warp w of the compute
// warps reads TMEM lane quarter w % 4 (MMA rows 32 (w % 4) .. +31, output rows
// likewise) and handles columns [(w / 4) NCW, (w / 4 + 1) NCW).  More warps
// per scheduler hide the latency of the per-column softmax arithmetic.
template <int NC, bool KV8>
struct Warps {
  static constexpr int kNCW = NC >= 16 ? 8 : (NC >= 8 ? 4 : NC);  // columns per warpgroup
  static constexpr int kNWG = NC / kNCW;                           // compute warpgroups
  static constexpr int kCompute = 128 * kNWG;                      // compute threads
  // + MMA, K producer, scheduler, V producer warps; with an E4M3 cache the
  // converter warps: one or two warpgroups (each row of a tile taken by one or
  // two threads: K into TMEM, V into shared memory).  Two, unless the four
  // compute warpgroups need the registers.
  static constexpr int kConvWarps = KV8 ? (kNWG == 4 ? 4 : 8) : 0;
  static constexpr int kThreads = kCompute + 128 + 32 * kConvWarps;
  static_assert(kNCW * kNWG == NC, "columns split evenly");
};

// Shared memory.  A small region at the start of the dynamic allocation
// (barriers and per-item tables), then, from the next 1024-byte boundary, the
// stages, the query slots and P, whose swizzled layouts need that alignment.
// TMEM: S^T in [0, N); O^T hi in [N, 2N), O^T lo in [2N, 3N).
// With an E4M3 cache (KV8) the stages only land the 8-bit tiles (32 KB); the
// converter warps widen each K tile into TMEM (two buffers of 64 columns,
// alternating by tile: S^T's A operand) and each V tile into a 16-bit V tile
// in shared memory (two buffers, alternating by tile).
template <int N, bool KV8>
struct Layout {
  // small region (byte offsets from the dynamic base)
  // barriers: K full[3], K empty[3], ready[2], free[2], meta[2], qk, pv, drain, s_free,
  // p_ready, conv, qconv, V full[3], V empty[3], then (KV8) per widened V buffer: widened[2],
  // free[2], and per widened K buffer: widened[2], free[2]
  static constexpr int kNumBars = 4 * kStages + 3 * kSlots + 7 + (KV8 ? 8 : 0);
  static constexpr int kBars = 0;
  static constexpr int kMisc = kBars + kNumBars * 8;        // tmem address, abort flag, accumulate flags [2]
  static constexpr int kDesc = kMisc + 16;                  // [slots][16] int
  static constexpr int kRows = kDesc + kSlots * 16 * 4;     // [slots][2][32] int: pool rows of the groups
  static constexpr int kGTok = kRows + kSlots * 64 * 4;     // [slots][32] int: first token of each group
  static constexpr int kGMeta = kGTok + kSlots * 32 * 4;    // [slots][32] int: owner + 1 | valid rows << 8
  static constexpr int kMLim = kGMeta + kSlots * 32 * 4;    // [slots][32] int: token limit of each member
  static constexpr int kMCode = kMLim + kSlots * 32 * 4;    // [slots][32] int: destination of each member
  static constexpr int kRed = kMCode + kSlots * 32 * 4;     // [4 warps][N] f32
  static constexpr int kStat = kRed + 4 * N * 4;            // m[N], then l[N], f32
  static constexpr int kQScale = kStat + 2 * N * 4;        // KV8: [slots][32] f32, query row scales
  static constexpr int kSmall = kQScale + kSlots * 32 * 4;
  // big region (byte offsets from the first 1024-byte boundary after the small one)
  static constexpr int kHalf = kTile * 128;  // a 64-element half of a 16-bit tile, or an 8-bit tile (16 KB)
  static constexpr int kStageBytes = KV8 ? 2 * kHalf : 4 * kHalf;  // K tile then V tile
  static constexpr int kStages0 = 0;
  static constexpr int kV16 = kStages0 + kStages * kStageBytes;  // KV8: widened V [2][2 halves]
  static constexpr int kQ = kV16 + (KV8 ? 4 * kHalf : 0);         // [slots][2 halves][N rows][128 B]
  static constexpr int kQBytes = 2 * N * 128;
  static constexpr int kP = kQ + kSlots * kQBytes;          // P hi, then P lo
  static constexpr int kPBytes = kTile * N * 2;             // [N/16 atoms][128 rows][32 B]
  static constexpr int kPAtom = kTile * 32;                 // bytes of one 16-column atom
  static constexpr int kBig = kP + 2 * kPBytes;
  // the allocation when the dynamic base is 1024-aligned (the kernel checks)
  static constexpr int kAlloc = (kSmall + 1023) / 1024 * 1024 + kBig;
  static_assert(kQ % 1024 == 0 && kQBytes % 1024 == 0 && kP % 256 == 0, "swizzle atoms");
  static_assert(kAlloc <= 232448, "shared memory per CTA");
};

// Item descriptor fields.
enum { kDS = 0, kDKvh, kDPart, kDBegin, kDEnd, kDTiles, kDMembers, kDVbase, kDNumFields };

// ---------------------------------------------------------------------------
// tcgen05 / descriptor helpers

// Shared-memory matrix descriptor (sm100 layout): start >> 4 in bits [0,14),
// leading-dimension byte offset >> 4 in [16,30), stride-dimension byte offset
// >> 4 in [32,46), version 1 in [46,48), swizzle mode in [61,64).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo,
                                              uint32_t swizzle) {
  return (uint64_t)((addr >> 4) & 0x3fff) | ((uint64_t)((lbo >> 4) & 0x3fff) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3fff) << 32) | (1ull << 46) | ((uint64_t)swizzle << 61);
}
constexpr uint32_t kSw128 = 2, kSw32 = 6;

// Instruction descriptor of kind::f16: fp32 accumulator, A and B of one type
// (0 = f16, 1 = bf16), per-operand major-ness (0 = K-major, 1 = MN-major),
// N >> 3 in [17,23), M >> 4 in [24,29).
__host__ __device__ constexpr uint32_t instr_desc(uint32_t ab_format, uint32_t a_mn, uint32_t b_mn,
                                                  uint32_t m, uint32_t n) {
  return (1u << 4) | (ab_format << 7) | (ab_format << 10) | (a_mn << 15) | (b_mn << 16) |
         ((n >> 3) << 17) | ((m >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
// As mma_f16, with A read from TMEM (rows in lanes, two 16-bit elements per column).
__device__ __forceinline__ void mma_f16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// NCOL (1 .. 32) consecutive fp32 columns of this thread's TMEM lane.
template <int NCOL>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, float (&v)[NCOL]) {
  uint32_t r[NCOL];
  if constexpr (NCOL == 1) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r[0]) : "r"(taddr));
  } else if constexpr (NCOL == 2) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];"
                 : "=r"(r[0]), "=r"(r[1])
                 : "r"(taddr));
  } else if constexpr (NCOL == 4) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
  } else if constexpr (NCOL == 8) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
  } else if constexpr (NCOL == 16) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
        "%12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
  } else {
    static_assert(NCOL == 32, "1, 2, 4, 8, 16 or 32 columns");
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
        "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
        "%30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
  }
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < NCOL; ++i) v[i] = __uint_as_float(r[i]);
}

// Zero NCOL (1 .. 8) consecutive fp32 columns of this thread's TMEM lane.
// Store 16 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

template <int NCOL>
__device__ __forceinline__ void tmem_zero(uint32_t taddr) {
  const uint32_t z = 0u;
  if constexpr (NCOL == 1) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(z) : "memory");
  } else if constexpr (NCOL == 2) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x2.b32 [%0], {%1, %1};" ::"r"(taddr), "r"(z) : "memory");
  } else if constexpr (NCOL == 4) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %1, %1, %1};" ::"r"(taddr), "r"(z)
                 : "memory");
  } else {
    static_assert(NCOL == 8, "1, 2, 4 or 8 columns");
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %1, %1, %1, %1, %1, %1, %1};" ::"r"(
                     taddr),
                 "r"(z)
                 : "memory");
  }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, uint32_t bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi, bool bf16) {
  if (bf16) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Column-wise reduction of a warp's 32 rows of NC values: on return lane l
// holds the maximum (or sum) of column l % NC over the warp.  Lanes first
// combine with the partners that will end up holding the same column; then
// each step of width w hands half of a lane's columns to the partner lane^w.
// NC - 1 + NC * (5 - log2 NC) shuffles instead of 5 * NC.  `v` is consumed.
template <int NC, bool MAX>
__device__ __forceinline__ float column_reduce(float (&v)[NC], int lane) {
#pragma unroll
  for (int w = 16; w >= NC; w >>= 1)
#pragma unroll
    for (int i = 0; i < NC; ++i) {
      const float o = __shfl_xor_sync(0xffffffffu, v[i], w);
      v[i] = MAX ? fmaxf(v[i], o) : v[i] + o;
    }
#pragma unroll
  for (int w = NC / 2; w >= 1; w >>= 1) {
    const bool upper = (lane & w) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const float send = upper ? v[i] : v[i + w];
      const float keep = upper ? v[i + w] : v[i];
      const float got = __shfl_xor_sync(0xffffffffu, send, w);
      v[i] = MAX ? fmaxf(keep, got) : keep + got;
    }
  }
  return v[0];
}

// Entry k >> 5 of a per-lane register array, then lane k & 31's copy of it.
template <int PPL>
__device__ __forceinline__ int lane_entry(const int (&v)[PPL], int k) {
  int mine = 0;
#pragma unroll
  for (int i = 0; i < PPL; ++i)
    if (i == (k >> 5)) mine = v[i];
  return __shfl_sync(0xffffffffu, mine, k & 31);
}

// Largest unit u with pre[u] <= r (pre non-decreasing, INT_MAX past the end).
template <int PPL>
__device__ __forceinline__ int last_at_most(const int (&pre)[PPL], int r) {
  int cnt = 0;
#pragma unroll
  for (int k = 0; k < PPL; ++k) cnt += pre[k] <= r ? 1 : 0;
  return __reduce_add_sync(0xffffffffu, cnt) - 1;
}

// Item number -> (unit, kv unit, partition).  A unit whose row list holds R
// rows has R / PT full partitions and, when PT does not divide R (or R == 0),
// one last shorter one.  Items 0 .. Hu F - 1 are the full partitions of every
// unit (F in all), the rest the last ones; the kv unit varies fastest.
// pre_f / pre_p: exclusive prefix counts of full / last partitions over the
// units, lane l holding entries l, l + 32, ...  (Per-sequence items number
// partition 0 of every sequence first and locate the rest with pre_f
// counting further partitions and pre_p zero.)  Called by all 32 lanes.
template <int PPL>
__device__ __forceinline__ void locate(int f, int Hu, int F, const int (&pre_f)[PPL],
                                       const int (&pre_p)[PPL], int& u, int& kvu, int& part) {
  if (f < Hu * F) {
    kvu = f % Hu;
    const int r = f / Hu;
    u = last_at_most(pre_f, r);
    part = r - lane_entry(pre_f, u);
  } else {
    const int g = f - Hu * F;
    kvu = g % Hu;
    u = last_at_most(pre_p, g / Hu);
    part = lane_entry(pre_f, u + 1) - lane_entry(pre_f, u);
  }
}

// Work counter tagged with the call's epoch in bits 24..63 (see pa_decode.cu):
// take_begin issues the increment, take_end (later, so that the round trip
// overlaps other work) reads its result, installing this call's epoch if the
// word still carries another one.
__device__ __forceinline__ unsigned long long take_begin(unsigned long long* ctr) {
  return atomicAdd(ctr, 1ull);
}
__device__ __forceinline__ int take_end(unsigned long long* ctr, unsigned long long old,
                                        unsigned long long epoch, unsigned int* err) {
  if ((old >> 24) == epoch) return (int)(old & 0xffffffull);
  for (int round = 0; round < (1 << 20); ++round) {
    const unsigned long long cur = atomicAdd(ctr, 0ull);
    if ((cur >> 24) == epoch) return (int)(atomicAdd(ctr, 1ull) & 0xffffffull);
    if (atomicCAS(ctr, cur, (epoch << 24) | 1ull) == cur) return 0;
  }
  report(err, kErrWaitTimeout);
  return -1;
}

// Columns an item of this launch fills at most: members x g with shared
// prefixes (32), else query tokens x heads per item x g.
__host__ __device__ inline int tc_columns(int group, int query_tokens, bool pair, bool grouped) {
  return grouped ? kTcMaxColumns : query_tokens * (pair ? 2 : 1) * group;
}

// Every unit's partition counts and their exclusive prefix over the units of
// the launch (see locate).  Called by all 32 lanes of the scheduler warp.  A
// unit's rows come from one load per sequence, all of them issued before any
// is used (indices clamped to the batch), so they are in flight together:
// without a plan every sequence is a unit (rows = its context; p0_first:
// pre_f counts the partitions after partition 0); grouped, the leaders of
// groups of two or more (rows = their list's, the plan's fourth field);
// own pass, the sequences whose own tokens are in no list (rows = ctx - T,
// the plan's third field).  -1: no unit.  With both (a list launch that also
// takes the own tokens) units 0 .. S - 1 are the lists' and S .. 2 S - 1 the
// own tokens'.
template <int PPL>
__device__ __forceinline__ void unit_prefix(const DecodeArgs& a, bool grouped, bool both, bool p0_first,
                                            int PT, int lane, int (&pre_f)[PPL], int (&pre_p)[PPL],
                                            int& carry_f, int& carry_p) {
  const int S = both ? 2 * a.num_seqs : a.num_seqs;  // units
  int rows_k[PPL];
#pragma unroll
  for (int k = 0; k < PPL; ++k) {
    const int u = min(k * 32 + lane, S - 1);
    const bool own = both && u >= a.num_seqs;
    const int sc = own ? u - a.num_seqs : u;
    rows_k[k] = grouped && !own ? __ldg(&a.plan2[sc].w)
                : a.plan        ? __ldg(&a.plan2[sc].z)
                                : __ldg(a.context_lens + sc);
  }
#pragma unroll
  for (int k = 0; k < PPL; ++k) {
    const int s = k * 32 + lane;  // this lane's unit
    int rows = rows_k[k];
    if (!a.plan) {
      if (s < S && (rows < 0 || rows > a.max_context_len) && blockIdx.x == 0) report(a.err, kErrContextLen);
      rows = max(0, min(rows, a.max_context_len));
    }
    int full = 0, last = 0;
    if (s < S && rows >= 0) {
      full = rows / PT;
      last = (rows % PT != 0 || rows == 0) ? 1 : 0;
      if (p0_first) {
        full = full + last - 1;  // further partitions after partition 0
        last = 0;
      }
    }
    pre_f[k] = full;
    pre_p[k] = last;
  }
  carry_f = 0, carry_p = 0;
#pragma unroll
  for (int k = 0; k < PPL; ++k) {
    const int s = k * 32 + lane;
    const int full = pre_f[k], last = pre_p[k];
    int inc_f = full, inc_p = last;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int tf = __shfl_up_sync(0xffffffffu, inc_f, o);
      const int tp = __shfl_up_sync(0xffffffffu, inc_p, o);
      if (lane >= o) inc_f += tf, inc_p += tp;
    }
    pre_f[k] = s <= S ? carry_f + inc_f - full : INT_MAX;
    pre_p[k] = s <= S ? carry_p + inc_p - last : INT_MAX;
    carry_f += __shfl_sync(0xffffffffu, inc_f, 31);
    carry_p += __shfl_sync(0xffffffffu, inc_p, 31);
  }
}

// Sixteen E4M3 codes (one 16-byte piece of a row, first element in the lowest
// byte) -> sixteen 16-bit values of T, two per word, first element in the low
// half.  Exact: every E4M3 value is an f16 (the hardware conversion) and a bf16.
template <typename T>
__device__ __forceinline__ void widen16(const uint4 x, uint32_t (&w)[8]) {
  const uint32_t in[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int hw = 0; hw < 2; ++hw) {
      const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(
          static_cast<__nv_fp8x2_storage_t>((in[i] >> (16 * hw)) & 0xffffu), __NV_E4M3);
      uint32_t r;
      if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        const __nv_bfloat162 b = __float22bfloat162_rn(__half22float2(*reinterpret_cast<const __half2*>(&h)));
        r = *reinterpret_cast<const uint32_t*>(&b);
      } else {
        r = *reinterpret_cast<const uint32_t*>(&h);
      }
      w[2 * i + hw] = r;
    }
}

// WIDE: a row-list launch that also takes the own-token items (2 x 256 units).
template <typename T, int NC, bool PAIR, bool KV8, bool WIDE>
__global__ void __launch_bounds__(Warps<NC, KV8>::kThreads, 1)
decode_tc_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_q) {
  constexpr int N = NC <= 16 ? 16 : 32;          // MMA columns
  // S^T, O^T hi and lo, and with an 8-bit cache two widened K tiles (A operands)
  constexpr uint32_t kACol = 3 * N;  // KV8: K buffer b at kACol + 64 b (two f16 per column)
  constexpr uint32_t kTmemCols = KV8 ? 256 : (N == 16 ? 64 : 128);
  // A tile is kTok tokens of each of the item's kHeads kv heads, as kTile MMA
  // rows (with two heads, 16-row groups of head 2e and head 2e+1 alternate)
  constexpr int kHeads = PAIR ? 2 : 1;
  constexpr int kTok = kTile / kHeads;
  constexpr int kGroupsPerTile = kTok / kGroupRows;
  using W = Warps<NC, KV8>;
  constexpr int kComputeThreads = W::kCompute, kThreads = W::kThreads, NCW = W::kNCW;
  constexpr int kComputeWarps = kComputeThreads / 32;
  constexpr int kMmaWarp = kComputeWarps, kProducerWarp = kComputeWarps + 1,
                kSchedWarp = kComputeWarps + 2, kProducerVWarp = kComputeWarps + 3,
                kConvWarp0 = kComputeWarps + 4;  // KV8: K converters, then V converters
  using L = Layout<N, KV8>;
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  // An 8-bit cache is widened to f16 (one conversion per pair) and the
  // products run in f16 whatever the query type: bf16 query rows are
  // converted to f16 at the start of each item (kQToF16).
  constexpr bool kQToF16 = KV8 && kBf16;
  using MT = typename std::conditional<KV8, __half, T>::type;  // operand type of the products
  constexpr bool kMmaBf16 = std::is_same<MT, __nv_bfloat16>::value;
  constexpr uint32_t kIdescQK = instr_desc(kMmaBf16 ? 1 : 0, 0, 0, kTile, N);
  // PV has 2N columns: P hi and P lo sit in consecutive 16-column atoms, so one
  // MMA reads each V slice once for both and writes O^T hi and O^T lo side by side
  constexpr uint32_t kIdescPV = instr_desc(kMmaBf16 ? 1 : 0, 1, 1, kTile, 2 * N);
  extern __shared__ __align__(16) unsigned char smem_raw[];

  // Until pdl_wait() below, this CTA touches only its own shared and tensor
  // memory: that part overlaps the end of the kernel before it on the stream.
  // The big region starts at the first 1024-byte boundary after the small one;
  // the allocation assumes a 1024-aligned base.  Any other base that leaves
  // too little room is reported, and the CTA does nothing.
  unsigned char* smem;
  {
    uint32_t dyn;
    asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t off = ((raw + L::kSmall + 1023u) & ~1023u) - raw;
    if (off + (uint32_t)L::kBig > dyn) {
      pdl_wait();
      if (threadIdx.x == 0) report(a.err, kErrConfig);
      return;
    }
    smem = smem_raw + off;
  }
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Hkv = a.num_kv_heads, PT = a.partition_tokens, G = a.group, Tq = a.query_tokens;
  // row lists of shared-prefix groups; else per-sequence items (with a plan:
  // the own tokens of the sequences whose own tokens are in no list)
  const bool grouped = a.plan != nullptr && !a.own_pass;
  int* desc_all = reinterpret_cast<int*>(smem_raw + L::kDesc);
  int* rows_all = reinterpret_cast<int*>(smem_raw + L::kRows);
  int* gtok_all = reinterpret_cast<int*>(smem_raw + L::kGTok);
  int* gmeta_all = reinterpret_cast<int*>(smem_raw + L::kGMeta);
  int* mlim_all = reinterpret_cast<int*>(smem_raw + L::kMLim);
  int* mcode_all = reinterpret_cast<int*>(smem_raw + L::kMCode);
  float* red = reinterpret_cast<float*>(smem_raw + L::kRed);
  float* stat = reinterpret_cast<float*>(smem_raw + L::kStat);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem_raw + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem_raw + L::kMisc + 4);
  volatile int* acc_flag = reinterpret_cast<volatile int*>(smem_raw + L::kMisc + 8);  // [2]
  const uint32_t bars = smem_addr(smem_raw + L::kBars);
  // stage st's K half and V half: landed (full), and free again (empty)
  auto full_bar = [&](int st) { return bars + st * 8; };
  auto empty_bar = [&](int st) { return bars + (kStages + st) * 8; };
  auto vfull_bar = [&](int st) { return bars + (2 * kStages + 3 * kSlots + 7 + st) * 8; };
  auto vempty_bar = [&](int st) { return bars + (3 * kStages + 3 * kSlots + 7 + st) * 8; };
  // KV8, 16-bit V buffer b: widened for its tile, and free again (O^T done)
  auto vconv_bar = [&](int b) { return bars + (4 * kStages + 3 * kSlots + 7 + b) * 8; };
  auto vfree_bar = [&](int b) { return bars + (4 * kStages + 3 * kSlots + 9 + b) * 8; };
  // KV8, TMEM K buffer b: widened for its tile, and free again (S^T done)
  auto aconv_bar = [&](int b) { return bars + (4 * kStages + 3 * kSlots + 11 + b) * 8; };
  auto afree_bar = [&](int b) { return bars + (4 * kStages + 3 * kSlots + 13 + b) * 8; };
  auto ready_bar = [&](int sl) { return bars + (2 * kStages + sl) * 8; };
  auto free_bar = [&](int sl) { return bars + (2 * kStages + kSlots + sl) * 8; };
  auto meta_bar = [&](int sl) { return bars + (2 * kStages + 2 * kSlots + sl) * 8; };
  const uint32_t qk_bar = bars + (2 * kStages + 3 * kSlots) * 8;
  const uint32_t pv_bar = qk_bar + 8;
  const uint32_t drain_bar = qk_bar + 16;
  const uint32_t s_free_bar = qk_bar + 24;   // compute warps have read S^T(g)
  const uint32_t p_ready_bar = qk_bar + 32;  // compute warps have written P(g)
  const uint32_t qconv_bar = qk_bar + 48;    // the item's query rows are f16 (kQToF16)
  const uint32_t sm_stages = smem_addr(smem + L::kStages0);
  const uint32_t sm_q = smem_addr(smem + L::kQ);
  const uint32_t sm_p = smem_addr(smem + L::kP);
  // query rows one item's TMA box fills (the rest of the N rows stay zero)
  const int q_rows = grouped ? kTcMaxColumns : Tq * kHeads * G;

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_holder)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    for (int st = 0; st < kStages; ++st) {
      mbar_init(full_bar(st), 1);
      mbar_init(vfull_bar(st), 1);
      // a half is released by the MMA warp's commit after its products, or
      // with an 8-bit cache by every compute warp once it has widened it
      mbar_init(empty_bar(st), KV8 ? W::kConvWarps : 1);
      mbar_init(vempty_bar(st), KV8 ? W::kConvWarps : 1);
    }
    if constexpr (KV8) {
      for (int b = 0; b < 2; ++b) {
        mbar_init(vconv_bar(b), W::kConvWarps);
        mbar_init(vfree_bar(b), 1);
        mbar_init(aconv_bar(b), W::kConvWarps);
        mbar_init(afree_bar(b), 1);
      }
    }
    for (int sl = 0; sl < kSlots; ++sl) {
      mbar_init(ready_bar(sl), 1);
      mbar_init(free_bar(sl), kComputeWarps);
      mbar_init(meta_bar(sl), 1);
    }
    mbar_init(qk_bar, 1);
    mbar_init(pv_bar, 1);
    mbar_init(drain_bar, 1);
    mbar_init(s_free_bar, kComputeWarps);
    mbar_init(p_ready_bar, kComputeWarps);
    mbar_init(qconv_bar, W::kNWG);
    *abort_flag = 0;
    mbar_init_fence();
  }
  // Query rows past the item's box stay zero (padded columns).
  for (int i = tid; i < kSlots * 2 * N * 8; i += kThreads) {
    const int row = (i / 8) % N;
    if (row >= q_rows)
      *reinterpret_cast<uint4*>(smem + L::kQ + (i / 8 / N) * N * 128 + row * 128 + (i % 8) * 16) =
          make_uint4(0, 0, 0, 0);
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  pdl_wait();  // the kernels before this decode (append, plan, expansion) have landed
  pdl_launch_dependents();

  if (warp == kSchedWarp) {
    // =====================================================================
    // scheduler warp: takes items, resolves them (unit, kv head, row range,
    // the pool row, owner and first token of each 16-row group, each
    // member's token limit and destination) and fills an item slot:
    // descriptor and rows (meta, for the producer), query rows (ready, for
    // the MMA and compute warps).  It runs up to two items ahead of the
    // compute warps, so none of its global round trips holds up the loads.
    // =====================================================================
    const int S = a.num_seqs;
    // partition 0 of every sequence first when every sequence is a unit (no
    // plan): the first item of every CTA is then known without the prefix
    // counts, which are computed while its tiles load; with a plan (groups, or
    // own tokens read on their own) only some sequences are units: full
    // partitions first, then the last ones, counted before the first item
    const bool p0_first = a.plan == nullptr;
    // a list launch that also takes the own tokens read on their own: units
    // S .. 2 S - 1 are those sequences' own tokens, as per-sequence items
    const bool both = WIDE && grouped && a.own_in_lists != 0;
    const int Hu = Hkv / kHeads;  // kv units of the item numbering
    constexpr int PPL = (WIDE ? 2 : 1) * kMaxUnits / 32 + 1;  // prefix[0..units] over the lanes
    int pre_f[PPL], pre_p[PPL];
    int carry_f = 0, carry_p = 0;
    if (!p0_first) unit_prefix(a, grouped, both, p0_first, PT, lane, pre_f, pre_p, carry_f, carry_p);
    // items known so far (without a plan, the partition-0 items until the
    // prefix is in)
    int total = p0_first ? S * Hu : Hu * (carry_f + carry_p);

    bool ok = true;
    int it = 0;
    int f = blockIdx.x;
    for (;; ++it) {
      const int slot = it % kSlots;
      if (it >= kSlots) {
        bool w = true;
        if (lane == 0) w = mbar_wait_or_abort(free_bar(slot), ((it / kSlots) - 1) & 1, a.err, abort_flag);
        if (!__shfl_sync(0xffffffffu, (int)w, 0)) {
          ok = false;
          break;
        }
      }
      int* desc = desc_all + slot * 16;
      if (f >= total) {
        if (lane == 0) {
          desc[kDTiles] = -1;  // end of work
          mbar_arrive(meta_bar(slot));
          mbar_arrive(ready_bar(slot));
        }
        break;
      }
      int s, kvu, part;
      if (p0_first) {
        // partition 0 of every sequence, then further partitions by sequence
        if (f < S * Hu) {
          s = f / Hu, kvu = f % Hu, part = 0;
        } else {
          locate(f - S * Hu, Hu, carry_f, pre_f, pre_p, s, kvu, part);
          part += 1;
        }
      } else {
        locate(f, Hu, carry_f, pre_f, pre_p, s, kvu, part);
      }
      bool g_item = grouped;  // this item reads a group's row list
      if (both && s >= S) {
        s -= S;
        g_item = false;
      }
      const int kvh = kvu * kHeads;  // the item's first kv head
      // query rows: one TMA box per 64-element half, [members][heads][64]
      const uint32_t rb = ready_bar(slot);
      if (lane == 0) {
        const int qrow = g_item || grouped ? a.seq_offset + s : (a.seq_offset + s) * Tq;
        mbar_expect_tx(rb, 2 * q_rows * 128);  // the phase also needs the arrival below
        tma_load_3d(sm_q + slot * L::kQBytes, &tm_q, rb, 0, kvh * G, qrow);
        tma_load_3d(sm_q + slot * L::kQBytes + N * 128, &tm_q, rb, 64, kvh * G, qrow);
      }
      // ---- members (lane m): token limit, destination of the result; the
      // row list of the item
      int members, T, n_list, vbase;  // shared rows, rows in the unit's list
      int tok_base = 0;               // token of the list's first row (own-token pass)
      int m_ctx = 0, m_off = 0, m_code = kSkip;
      const int p0 = part * PT;
      const int r0 = p0 + lane * kGroupRows;  // this lane's 16-row group of the list
      // without a plan a lane's group is the sequence's tokens r0 .. r0 + 15:
      // its table entries are read at once, with the context (entries below
      // max_context_len lie inside the table; only a group below the context
      // uses its entry)
      int spec_blk = -1, spec_blk2 = -1;
      const int32_t* stable = a.block_tables + (size_t)s * a.max_blocks_per_seq;
      if (!a.plan) {
        if (r0 < a.max_context_len) spec_blk = __ldg(stable + r0 / a.block_size);
        if (a.half_boxes && r0 + kGroupRows / 2 < a.max_context_len)
          spec_blk2 = __ldg(stable + (r0 + kGroupRows / 2) / a.block_size);
      }
      if (g_item) {
        // the group's plan and every member's record and context in one round
        // trip (lanes past the group read a neighbour, unused)
        const int sl = min(s + lane, S - 1);
        const int4 pl = __ldg(a.plan + s);
        const int4 p2 = __ldg(a.plan2 + sl);
        const int cx = __ldg(a.context_lens + sl);
        members = pl.y;
        T = pl.z;
        const int p_sh = pl.w;
        vbase = s;
        n_list = __shfl_sync(0xffffffffu, p2.w, 0);
        if (lane < members) {
          m_off = p2.x;
          m_ctx = max(0, min(cx, a.max_context_len));
          const int own = m_ctx - T;
          const int first_own = max(m_off / PT, p_sh);
          const bool mine = part < p_sh || (m_off >= 0 && own > 0 && part >= m_off / PT &&
                                            part <= (m_off + own - 1) / PT);
          if (m_ctx == 0) m_code = part == 0 ? kZero : kSkip;
          else if (!mine) m_code = kSkip;
          else if (p2.y == 1) m_code = kDirect;
          else m_code = part < p_sh ? part : p_sh + part - first_own;
        }
      } else {
        int ctx = __ldg(a.context_lens + s);
        // with a plan, the own tokens [base, ctx) after the partials of the
        // sequence's shared tokens
        int slot0 = 0, n_slots = 0;
        if (a.plan) {
          const int4 pl = __ldg(a.plan + s);
          tok_base = pl.z;
          slot0 = pl.w;
          n_slots = __ldg(a.plan2 + s).y;
        }
        ctx = max(0, min(ctx, a.max_context_len));
        members = Tq;
        T = ctx;  // every row is every query's, up to its limit
        vbase = s * Tq;
        n_list = ctx - tok_base;
        if (lane < Tq) {
          m_ctx = ctx - Tq + 1 + lane;  // causal limit of query token `lane`
          const int P_t = m_ctx > 0 ? (m_ctx + PT - 1) / PT : 0;
          if (m_ctx <= 0) m_code = part == 0 ? kZero : kSkip;
          else if (a.plan) m_code = n_slots == 1 ? kDirect : slot0 + part;
          else if (part >= P_t) m_code = kSkip;
          else if (P_t == 1) m_code = kDirect;
          else m_code = part;
        }
      }
      const int t_end = min(n_list, p0 + PT);
      const int n_rows = max(0, t_end - p0);
      const int n_tiles = (n_rows + kTok - 1) / kTok;
      const int n_groups = (n_rows + kGroupRows - 1) / kGroupRows;  // <= 32
      // ---- 16-row groups (lane i): owner, first token, valid rows, pool rows
      int g_own = -1, g_tok = 0, g_valid = 0, g_row = 0, g_row2 = 0;
      // own rows: the member whose run holds r0 (runs are in member order,
      // offsets non-decreasing; an empty run holds nothing): a binary search
      int own = 0;
      if (g_item) {
#pragma unroll
        for (int step = 16; step >= 1; step >>= 1) {
          const int cand = own + step;
          const int o = __shfl_sync(0xffffffffu, m_off, cand & 31);
          if (cand < members && o <= r0) own = cand;
        }
      }
      const int own_off = __shfl_sync(0xffffffffu, m_off, own);
      const int own_ctx = __shfl_sync(0xffffffffu, m_ctx, own);
      if (lane < n_groups) {
        int seq = s, lim;
        if (tok_base + r0 < T) {
          g_tok = tok_base + r0;
          lim = T;
        } else {
          g_own = own;
          g_tok = T + r0 - own_off;
          lim = own_ctx;
          seq = s + own;
        }
        g_valid = min(kGroupRows, lim - g_tok);
        // With 8-token blocks (half_boxes) rows 8..15 of a group have their own
        // entry; past the group's valid rows they re-read the first block (masked).
        const int32_t* table = a.block_tables + (size_t)seq * a.max_blocks_per_seq;
        auto resolve = [&](int tok, int blk) {
          if (blk < 0 || blk >= a.num_blocks) {
            report(a.err, kErrBlockId);
            return a.num_blocks * a.block_size;  // outside the map: TMA fills zeros
          }
          return blk * a.block_size + tok % a.block_size;
        };
        g_row = resolve(g_tok, a.plan ? __ldg(table + g_tok / a.block_size) : spec_blk);
        if (a.half_boxes) {
          const int t2 = g_tok + kGroupRows / 2;
          g_row2 = g_valid > kGroupRows / 2
                       ? resolve(t2, a.plan ? __ldg(table + t2 / a.block_size) : spec_blk2)
                       : g_row;
        }
      }
      {
        int* rows = rows_all + slot * 64;
        rows[lane] = g_row;
        rows[32 + lane] = g_row2;
        gtok_all[slot * 32 + lane] = g_tok;
        gmeta_all[slot * 32 + lane] = (g_own + 1) | (max(g_valid, 0) << 8);
        mlim_all[slot * 32 + lane] = lane < members ? m_ctx : -1;
        mcode_all[slot * 32 + lane] = lane < members ? m_code : kSkip;
      }
      __syncwarp();  // every lane's tables before the arrivals
      if (lane == 0) {
        desc[kDS] = s;
        desc[kDKvh] = kvh;
        desc[kDPart] = part;
        desc[kDBegin] = p0;
        desc[kDEnd] = t_end;
        desc[kDTiles] = n_tiles;
        desc[kDMembers] = members;
        desc[kDVbase] = vbase;
        mbar_arrive(meta_bar(slot));
        mbar_arrive(rb);  // with the query rows' bytes, completes the ready phase
      }
      if (p0_first && it == 0) {
        // the counts of the further partitions, while this item's tiles load
        unit_prefix(a, grouped, both, p0_first, PT, lane, pre_f, pre_p, carry_f, carry_p);
        total = Hu * carry_f + S * Hu;
      }
      // the next item: a launch with no more items than CTAs takes none
      // (every CTA had its one item); else from the work counter
      int nf = total;
      if (lane == 0 && total > (int)gridDim.x) {
        const int t = take_end(a.work_counter, take_begin(a.work_counter), a.epoch, a.err);
        nf = t < 0 ? total : (int)gridDim.x + t;
      }
      f = __shfl_sync(0xffffffffu, nf, 0);
    }
    if (!ok) *abort_flag = 1;
    // The query rows this warp loaded by TMA land before the CTA leaves
    // (bounded waits).  Items it-2 and it-1 may still be in flight, unless the
    // end-of-work mark went into item it-2's slot: that needed the slot freed,
    // so its rows had landed, and its phase parity now names a later phase.
    if (lane == 0)
      for (int k = max(0, it - (ok ? 1 : kSlots)); k < it; ++k)
        mbar_wait(ready_bar(k % kSlots), (k / kSlots) & 1, a.err);
  } else if (warp == kProducerWarp || warp == kProducerVWarp) {
    // =====================================================================
    // producer warps: one loads the K half of each tile, the other the V
    // half, by TMA from the rows the scheduler resolved.  Each half of a
    // stage is freed on its own (K once S^T is computed, V once O^T is), so
    // the K loads run up to a tile further ahead than the V loads.
    // =====================================================================
    const bool is_v = warp == kProducerVWarp;
    int issued = 0;  // tiles armed so far (stage ring position)
    bool ok = true;
    for (int it = 0; ok; ++it) {
      const int slot = it % kSlots;
      {
        bool w = true;
        if (lane == 0) w = mbar_wait_or_abort(meta_bar(slot), (it / kSlots) & 1, a.err, abort_flag);
        if (!__shfl_sync(0xffffffffu, (int)w, 0)) {
          ok = false;
          break;
        }
        __syncwarp();  // lane 0's acquire orders the other lanes' reads below
      }
      const int* desc = desc_all + slot * 16;
      const int n_tiles = desc[kDTiles];
      if (n_tiles < 0) break;  // end of work
      const int kvh = desc[kDKvh];
      const int n_groups = (desc[kDEnd] - desc[kDBegin] + kGroupRows - 1) / kGroupRows;
      const int my_row = rows_all[slot * 64 + lane];
      const int my_row2 = rows_all[slot * 64 + 32 + lane];
      const void* map = is_v ? &tm_v : &tm_k;
      for (int j = 0; j < n_tiles && ok; ++j) {
        const int st = issued % kStages;
        if (issued >= kStages &&
            !mbar_wait_or_abort(is_v ? vempty_bar(st) : empty_bar(st), ((issued / kStages) - 1) & 1, a.err,
                                abort_flag)) {
          ok = false;
          break;
        }
        const int g0 = j * kGroupsPerTile;
        const int ng = min(kGroupsPerTile, n_groups - g0);
        const uint32_t fb = is_v ? vfull_bar(st) : full_bar(st);
        // this warp's half of the stage: K at its start, V after it
        const uint32_t dst = sm_stages + st * L::kStageBytes + (is_v ? L::kStageBytes / 2 : 0);
        constexpr int kBoxBytes = kHeads * kGroupRows * 128;  // one box: a group of kHeads heads
        if (lane == 0) mbar_arrive_expect_tx(fb, ng * (KV8 ? 1 : 2) * kBoxBytes);
        __syncwarp();
        if constexpr (KV8) {
          // lane r loads group r: 128 one-byte elements x 16 rows (x 2 heads),
          // the whole head_dim in one box
          const int r = lane;
          const int row = __shfl_sync(0xffffffffu, my_row, min(g0 + r, 31));
          const int row2 = __shfl_sync(0xffffffffu, my_row2, min(g0 + r, 31));
          if (r < ng) {
            const uint32_t d = dst + r * kBoxBytes;
            if constexpr (PAIR) {
              tma_load_3d(d, map, fb, 0, row, kvh);
            } else {
              tma_load_3d(d, map, fb, 0, kvh, row);
              if (a.half_boxes) tma_load_3d(d + (kGroupRows / 2) * 128, map, fb, 0, kvh, row2);
            }
          }
        } else {
          // lane 2 r + k loads the 64-element half k of group r
          const int r = lane >> 1, k = lane & 1;
          const int row = __shfl_sync(0xffffffffu, my_row, min(g0 + r, 31));
          const int row2 = __shfl_sync(0xffffffffu, my_row2, min(g0 + r, 31));
          if (r < ng) {
            const uint32_t d = dst + k * L::kHalf + r * kBoxBytes;
            if constexpr (PAIR) {
              // maps of this kind are [rows][head] with the head innermost
              // after the dims: a box is 16 rows of head kvh, then of kvh + 1
              tma_load_3d(d, map, fb, k * 64, row, kvh);
            } else {
              tma_load_3d(d, map, fb, k * 64, kvh, row);
              if (a.half_boxes) tma_load_3d(d + (kGroupRows / 2) * 128, map, fb, k * 64, kvh, row2);
            }
          }
        }
        ++issued;
      }
    }
    if (!ok) *abort_flag = 1;
    // Every TMA copy armed by this warp lands before the CTA leaves.
    if (lane == 0)
      for (int k = max(0, issued - kStages); k < issued; ++k)
        mbar_wait(is_v ? vfull_bar(k % kStages) : full_bar(k % kStages), (k / kStages) & 1, a.err);
  } else if (warp == kMmaWarp) {
    // =====================================================================
    // MMA warp (lane 0): every tcgen05.mma of the CTA, so that issuing them
    // never holds up the compute warps.  Per tile g (numbered across items):
    //   S^T(g) = K(g) . Q^T   once stage g has landed and S^T(g-1) was read;
    //   O^T (+)= V^T . P^T(g) once the compute warps have written P(g).
    // Each of qk, pv, s_free and p_ready completes once per tile, in order,
    // so tile g waits on phase parity g & 1.
    // =====================================================================
    bool ok = true;
    int g = 0;  // tiles issued so far
    auto issue_qk = [&](int h, uint32_t q_addr) {
      tc_fence_after();
      const int st = h % kStages;
      const uint32_t kt = sm_stages + st * L::kStageBytes;
#pragma unroll
      for (int kk = 0; kk < kD / 16; ++kk) {
        const uint32_t qo = (kk / 4) * N * 128 + (kk % 4) * 32;
        if constexpr (KV8) {
          // A = the widened K tile in TMEM: row r in lane r, dims 16 kk .. 16 kk + 15
          // in columns 8 kk .. 8 kk + 7
          mma_f16_ta(tmem, tmem + kACol + 64 * (h & 1) + 8 * kk, smem_desc(q_addr + qo, 16, 1024, kSw128),
                     kIdescQK, kk > 0);
        } else {
          const uint32_t ko = (kk / 4) * L::kHalf + (kk % 4) * 32;
          mma_f16(tmem, smem_desc(kt + ko, 16, 1024, kSw128), smem_desc(q_addr + qo, 16, 1024, kSw128),
                  kIdescQK, kk > 0);
        }
      }
      mma_commit(qk_bar);
      if constexpr (!KV8) mma_commit(empty_bar(st));  // the K half is free once S^T is done
      if constexpr (KV8) mma_commit(afree_bar(h & 1));  // the TMEM K buffer too
    };
    if (lane == 0) {
      for (int it = 0; ok; ++it) {
        const int slot = it % kSlots;
        ok = mbar_wait_or_abort(ready_bar(slot), (it / kSlots) & 1, a.err, abort_flag);
        if (!ok) break;
        const int n_tiles = desc_all[slot * 16 + kDTiles];
        if (n_tiles < 0) break;  // end of work
        if constexpr (kQToF16) {
          ok = mbar_wait_or_abort(qconv_bar, it & 1, a.err, abort_flag);
          if (!ok) break;
        }
        const uint32_t q_addr = sm_q + slot * L::kQBytes;
        // S^T(h) needs its stage landed (with an 8-bit cache: widened) and
        // S^T(h-1) read by the compute warps
        auto qk_for = [&](int h) {
          bool w = KV8 ? mbar_wait_or_abort(aconv_bar(h & 1), (h >> 1) & 1, a.err, abort_flag)
                       : mbar_wait_or_abort(full_bar(h % kStages), (h / kStages) & 1, a.err, abort_flag);
          if (w && h > 0) w = mbar_wait_or_abort(s_free_bar, (h - 1) & 1, a.err, abort_flag);
          if (w) issue_qk(h, q_addr);
          return w;
        };
        if (n_tiles > 0) ok = qk_for(g);
        for (int j = 0; j < n_tiles && ok; ++j, ++g) {
          const int st = g % kStages;
          // S^T(g+1) as soon as S^T(g) has been read: it runs during tile g's
          // softmax; then, once P(g) is written, O^T(g)
          if (j + 1 < n_tiles) {
            ok = qk_for(g + 1);
            if (!ok) break;
          }
          ok = mbar_wait_or_abort(p_ready_bar, g & 1, a.err, abort_flag);
          // the V half has landed (with an 8-bit cache: has been widened)
          if (ok && !KV8) ok = mbar_wait_or_abort(vfull_bar(st), (g / kStages) & 1, a.err, abort_flag);
          if (ok && KV8) ok = mbar_wait_or_abort(vconv_bar(g & 1), (g >> 1) & 1, a.err, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t vt = KV8 ? smem_addr(smem + L::kV16) + (g & 1) * 2 * L::kHalf
                                  : sm_stages + st * L::kStageBytes + 2 * L::kHalf;
          const uint32_t acc0 = (uint32_t)acc_flag[g & 1];
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            mma_f16(tmem + N, smem_desc(vt + kk * 2048, L::kHalf, 1024, kSw128),
                    smem_desc(sm_p + kk * 512, L::kPAtom, 256, kSw32), kIdescPV,
                    acc0 | (uint32_t)(kk > 0));
          mma_commit(pv_bar);
          if constexpr (!KV8) mma_commit(vempty_bar(st));  // the V half is free once these MMAs are done
          if constexpr (KV8) mma_commit(vfree_bar(g & 1));    // the 16-bit V buffer too
        }
      }
      if (!ok) *abort_flag = 1;
      // every MMA issued here completes before TMEM is freed (bounded wait)
      mma_commit(drain_bar);
      mbar_wait(drain_bar, 0, a.err);
    }
    __syncwarp();
  } else if (KV8 && warp >= kConvWarp0) {
    // =====================================================================
    // converter warps (E4M3 cache): row t of every tile (TMEM lane t) is taken
    // by the threads of lane t % 32 in the warps of lane quarter t / 32, each
    // widening a share of its 16-byte pieces.  Per tile g: the 8-bit K row
    // widened into TMEM K buffer g & 1 once S^T(g-2) is done with it; then the
    // 8-bit V row widened into shared V buffer g & 1 once O^T(g-2) is done
    // with it.  A row that is no token of
    // its tile gets a zero V row, so a stale NaN never meets p = 0.  The 8-bit
    // tiles and the 16-bit V tiles are 128B-swizzled: 16-byte piece c of row
    // t sits at c ^ (t & 7).  The buffers let the widening run up to two
    // tiles ahead of the products.
    // =====================================================================
    const int quarter = warp & 3;
    const int t = quarter * 32 + lane;
    const uint32_t t_lane = (uint32_t)(quarter * 32) << 16;
    const int sw = t & 7;
    constexpr int kShares = W::kConvWarps >= 8 ? 2 : 1;  // threads per row
    constexpr int kPieces = 8 / kShares;            // 16-byte 8-bit pieces per thread
    const int p0 = ((warp - kConvWarp0) >> 2) * kPieces;  // this thread's first piece
    bool ok = true;
    int g = 0;  // tiles widened so far, numbered across items
    auto conv_wait = [&](uint32_t bar, uint32_t parity) {
      bool r = true;
      if (lane == 0) r = mbar_wait_or_abort(bar, parity, a.err, abort_flag);
      return __shfl_sync(0xffffffffu, (int)r, 0) != 0;
    };
    for (int it = 0; ok; ++it) {
      const int slot = it % kSlots;
      if (!conv_wait(meta_bar(slot), (it / kSlots) & 1)) {
        ok = false;
        break;
      }
      __syncwarp();  // lane 0's acquire orders the other lanes' reads below
      const int* desc = desc_all + slot * 16;
      const int n_tiles = desc[kDTiles];
      if (n_tiles < 0) break;  // end of work
      const int* gmeta = gmeta_all + slot * 32;
      for (int j = 0; j < n_tiles; ++j, ++g) {  // tile j of the item
        const int st = g % kStages;
        // ---- K: row t into TMEM K buffer g & 1
        bool wt = g < 2 || conv_wait(afree_bar(g & 1), ((g >> 1) - 1) & 1);
        if (wt) wt = conv_wait(full_bar(st), (g / kStages) & 1);
        if (!wt) {
          ok = false;
          break;
        }
        {
          const unsigned char* in = smem + L::kStages0 + st * L::kStageBytes + t * 128;
          const uint32_t dst = tmem + t_lane + kACol + 64 * (g & 1);
#pragma unroll
          for (int hq = p0 / 2; hq < (p0 + kPieces) / 2; ++hq) {  // dims 32 hq .. 32 hq + 31: 16 columns
            uint32_t wd[16];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int jc = 2 * hq + u;
              const uint4 x = *reinterpret_cast<const uint4*>(in + ((jc ^ sw) << 4));
              uint32_t w8[8];
              widen16<MT>(x, w8);
#pragma unroll
              for (int e = 0; e < 8; ++e) wd[8 * u + e] = w8[e];
            }
            tmem_st16(dst + 16 * hq, wd);
          }
          asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(empty_bar(st));      // the 8-bit K half back to its producer
          mbar_arrive(aconv_bar(g & 1));   // the MMA warp may issue S^T(g)
        }
        // ---- V: row t into shared V buffer g & 1
        wt = g < 2 || conv_wait(vfree_bar(g & 1), ((g >> 1) - 1) & 1);
        if (wt) wt = conv_wait(vfull_bar(st), (g / kStages) & 1);
        if (!wt) {
          ok = false;
          break;
        }
        {
          const int grp = j * kGroupsPerTile + (PAIR ? (t >> 5) : (t >> 4));
          const bool zero = (t & 15) >= (gmeta[grp] >> 8);
          const unsigned char* in = smem + L::kStages0 + st * L::kStageBytes + L::kHalf + t * 128;
          unsigned char* out = smem + L::kV16 + (g & 1) * 2 * L::kHalf + t * 128;
#pragma unroll
          for (int jc = p0; jc < p0 + kPieces; ++jc) {  // elements 16 jc .. 16 jc + 15 of the row
            const uint4 x = *reinterpret_cast<const uint4*>(in + ((jc ^ sw) << 4));
            uint32_t wd[8];
            widen16<MT>(x, wd);
            if (zero) {
#pragma unroll
              for (int e = 0; e < 8; ++e) wd[e] = 0u;
            }
            const int h = jc >> 2, c = 2 * (jc & 3);  // half, first 16-byte piece of it
            unsigned char* o = out + h * L::kHalf;
            *reinterpret_cast<uint4*>(o + ((c ^ sw) << 4)) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
            *reinterpret_cast<uint4*>(o + (((c + 1) ^ sw) << 4)) = make_uint4(wd[4], wd[5], wd[6], wd[7]);
          }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(vempty_bar(st));     // the 8-bit V half back to its producer
          mbar_arrive(vconv_bar(g & 1));   // the MMA warp may issue O^T(g)
        }
      }
    }
    if (!ok) *abort_flag = 1;
  } else {
    // =====================================================================
    // compute warps: thread (t, cg) = MMA row t of S^T and row d = t of O^T,
    // for the columns of warpgroup cg.  Per tile g: wait for S^T(g), read it
    // and release it (s_free) so the MMA warp can issue S^T(g+1); the softmax
    // writes P(g) after O^T(g-1), its last reader, completed; then p_ready.
    // The output stays in TMEM across tiles: each column's softmax reference
    // m_ref only moves when a logit exceeds it by more than kRescale (log2
    // units), and only then is O^T folded into registers and rescaled (and
    // the next PV overwrites instead of accumulating).  Hence p <= 2^kRescale.
    // =====================================================================
    constexpr float kRescale = 8.f;
    const int t = tid & 127;         // MMA row of S^T, output row of O^T
    const int cg = tid >> 7;         // column group
    const int c0 = cg * NCW;         // first column of this thread
    const int quarter = warp & 3;    // TMEM lane quarter of this warp
    const uint32_t t_lane = ((uint32_t)(quarter * 32) << 16);
    // MMA row t: kv head e_row of the item, 16-row group t / 16 of the tile
    // (with two heads: token group t / 32)
    const int e_row = PAIR ? (t >> 4) & 1 : 0;
    const int grp_in_tile = PAIR ? (t >> 5) : (t >> 4);
    // column c: member m_c (query token, or group member), kv head e_c of the
    // item, query head h_c of that kv head
    int m_c[NCW], e_c[NCW], h_c[NCW];
#pragma unroll
    for (int c = 0; c < NCW; ++c) {
      const int col = c0 + c;
      m_c[c] = col / (kHeads * G);
      e_c[c] = (col / G) % kHeads;
      h_c[c] = col % G;
    }
    int g = 0;  // tiles consumed, numbered across items
    bool ok = true;
    // one lane per warp waits on an mbarrier, the warp follows
    auto warp_wait = [&](uint32_t bar, uint32_t parity) {
      bool w = true;
      if (lane == 0) w = mbar_wait_or_abort(bar, parity, a.err, abort_flag);
      return __shfl_sync(0xffffffffu, (int)w, 0) != 0;
    };
    // Each warpgroup owns its columns: its rescale decisions, column
    // reductions and the agreement on a failed wait take a named barrier of
    // its own 128 threads (id 2 + cg), never one of all compute warps.
    const int wg_bar = 2 + cg;
    for (int it = 0; ok; ++it) {
      const int slot = it % kSlots;
      if (t == 0) ok = mbar_wait_or_abort(ready_bar(slot), (it / kSlots) & 1, a.err, abort_flag);
      if (named_barrier_or(wg_bar, 128, !ok || *abort_flag)) { ok = false; break; }
      const int* desc = desc_all + slot * 16;
      const int n_tiles = desc[kDTiles];
      if (n_tiles < 0) break;  // end of work
      const int kvh = desc[kDKvh], vbase = desc[kDVbase];
      const int* gtok = gtok_all + slot * 32;
      const int* gmeta = gmeta_all + slot * 32;
      // token limit of each column's member (-1: a column no member fills)
      int lim_c[NCW];
#pragma unroll
      for (int c = 0; c < NCW; ++c) lim_c[c] = mlim_all[slot * 32 + min(m_c[c], 31)];
      float* qscale = reinterpret_cast<float*>(smem_raw + L::kQScale) + slot * 32;
      if constexpr (kQToF16) {
        // this warpgroup's query rows (its columns c0 .. c0 + NCW - 1),
        // bf16 -> f16 in place, 16 threads per row (a 16-byte piece each); a
        // row whose largest magnitude would overflow f16 is scaled down by a
        // power of two, which its logits take back (f16 keeps every bf16
        // significand)
        const int rl = t >> 4, k = t & 15;
        const int r = c0 + rl;
        const bool act = rl < NCW && r < q_rows;
        unsigned char* piece = smem + L::kQ + slot * L::kQBytes + (k >> 3) * N * 128 +
                               min(r, N - 1) * 128 + (((k & 7) ^ (r & 7)) << 4);
        const uint4 v = act ? *reinterpret_cast<const uint4*>(piece) : make_uint4(0, 0, 0, 0);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        float mx = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = Elem<__nv_bfloat16>::to_f2(w[e]);
          mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        int ex = 0;
        frexpf(mx, &ex);                  // mx < 2^ex
        const int sh = max(0, ex - 15);   // mx * 2^-sh < 2^15
        const float down = ldexpf(1.f, -sh);
        if (act) {
          uint32_t o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = Elem<__nv_bfloat16>::to_f2(w[e]);
            o[e] = pack2(f.x * down, f.y * down, false);
          }
          *reinterpret_cast<uint4*>(piece) = make_uint4(o[0], o[1], o[2], o[3]);
          if (k == 0) qscale[r] = ldexpf(1.f, sh);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        named_barrier(wg_bar, 128);
        if (t == 0) mbar_arrive(qconv_bar);  // one arrival per warpgroup
      }
      // logits in log2 units; an 8-bit cache folds each kv head's K scale in
      // (and, with f16 query rows, each row's scale)
      float kfac[NCW];
#pragma unroll
      for (int c = 0; c < NCW; ++c) {
        kfac[c] = KV8 ? a.scale_log2 * __ldg(a.k_scale + min(kvh + e_c[c], Hkv - 1)) : a.scale_log2;
        if constexpr (kQToF16) kfac[c] *= c0 + c < q_rows ? qscale[c0 + c] : 1.f;
      }

      float acc[NCW], l_tok[NCW], m_ref[NCW];
#pragma unroll
      for (int c = 0; c < NCW; ++c) acc[c] = 0.f, l_tok[c] = 0.f, m_ref[c] = -INFINITY;
      bool ok_w = true;     // every wait of this warp so far succeeded

      for (int j = 0; j < n_tiles; ++j, ++g) {
        const int st = g % kStages;
        // this row's group: owner (-1: every member), first token, valid rows
        const int grp = j * kGroupsPerTile + grp_in_tile;
        const int gm = gmeta[grp];
        const int own = (gm & 0xff) - 1;
        const int tok = gtok[grp] + (t & 15);
        const bool row_ok = (t & 15) < (gm >> 8);
        bool valid[NCW];
#pragma unroll
        for (int c = 0; c < NCW; ++c)
          valid[c] = row_ok && (own < 0 || own == m_c[c]) && (!PAIR || e_c[c] == e_row) &&
                     tok < lim_c[c];
        // ---- S^T(g).  Each warp waits on its own; the OR-barrier then makes
        // every compute thread take the same way out if this or an earlier
        // wait of its warp failed.
        float sv[NCW];
        if (ok_w) ok_w = warp_wait(qk_bar, g & 1);
        if (ok_w) {
          tc_fence_after();
          tmem_ld<NCW>(tmem + t_lane + (uint32_t)c0, sv);
          tc_fence_before();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free_bar);  // S^T(g) read: the MMA warp may reuse it
        // O^T(g-1), the last reader of P and the last writer of O^T, is
        // waited for only where this tile needs it: before O^T is folded and
        // before P(g) is written
        bool pv_done = j == 0;
        bool over = false;
#pragma unroll
        for (int c = 0; c < NCW; ++c) {
          sv[c] = valid[c] ? sv[c] * kfac[c] : -INFINITY;
          over |= sv[c] > m_ref[c] + kRescale;
        }
        // one barrier for the common case (no failure, no new maximum); the
        // rare true answer is told apart by a second one
        if (named_barrier_or(wg_bar, 128, !ok_w || *abort_flag || over)) {
          if (named_barrier_or(wg_bar, 128, !ok_w || *abort_flag)) { ok = false; break; }
          // new references: this tile's column maxima where they are higher
          {
            float tmp[NCW];
#pragma unroll
            for (int c = 0; c < NCW; ++c) tmp[c] = sv[c];
            const float wmax = column_reduce<NCW, true>(tmp, lane);
            if (lane < NCW) red[quarter * N + c0 + lane] = wmax;
          }
          named_barrier(wg_bar, 128);
          if (t < NCW) {
            const int col = c0 + t;
            stat[col] = fmaxf(fmaxf(red[col], red[N + col]), fmaxf(red[2 * N + col], red[3 * N + col]));
          }
          named_barrier(wg_bar, 128);
          float alpha[NCW];
#pragma unroll
          for (int c = 0; c < NCW; ++c) {
            const float m_new = fmaxf(m_ref[c], stat[c0 + c]);
            // 0 while m_ref is -inf; 1 while the column has seen no valid row
            alpha[c] = m_new == -INFINITY ? 1.f : exp2f(m_ref[c] - m_new);
            m_ref[c] = m_new;
            l_tok[c] *= alpha[c];
          }
          if (j > 0) {
            // fold O^T (this item's tiles before g) into acc, on the new
            // reference, and zero these columns of O^T: the next products
            // accumulate onto them (they do for every warpgroup)
            if (!pv_done) ok_w = warp_wait(pv_bar, (g - 1) & 1), pv_done = true;
            tc_fence_after();
            float ov[NCW], ow[NCW];
            tmem_ld<NCW>(tmem + t_lane + (uint32_t)(N + c0), ov);
            tmem_ld<NCW>(tmem + t_lane + (uint32_t)(2 * N + c0), ow);
#pragma unroll
            for (int c = 0; c < NCW; ++c) acc[c] = (acc[c] + (ov[c] + ow[c])) * alpha[c];
            tmem_zero<NCW>(tmem + t_lane + (uint32_t)(N + c0));
            tmem_zero<NCW>(tmem + t_lane + (uint32_t)(2 * N + c0));
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
          } else {
#pragma unroll
            for (int c = 0; c < NCW; ++c) acc[c] *= alpha[c];
          }
        }
        float p[NCW];
#pragma unroll
        for (int c = 0; c < NCW; ++c) {
          p[c] = valid[c] ? exp2f(sv[c] - m_ref[c]) : 0.f;
          l_tok[c] += p[c];
        }
        // P^T rows: per 16-column atom, a 32-byte row per MMA row (MN-major,
        // 32-byte swizzle: 16-byte piece c of row t sits at c ^ bit 2 of t),
        // once for hi = round(p) and once for lo = round(p - hi).  This
        // thread writes columns [c0, c0 + NCW): NCW * 2 bytes inside one
        // 16-byte piece.
        {
          const int atom = c0 / 16, piece = (c0 % 16) / 8, within = (c0 % 8) * 2;
          unsigned char* prow = smem + L::kP + atom * L::kPAtom + t * 32 +
                                ((piece ^ ((t >> 2) & 1)) * 16) + within;
          constexpr int NW2 = (NCW + 1) / 2;  // 32-bit words (an odd single column takes half of one)
          uint32_t hi[NW2], lo[NW2];
#pragma unroll
          for (int i = 0; i < NW2; ++i) {
            const float x0 = p[2 * i], x1 = (2 * i + 1 < NCW) ? p[2 * i + 1] : 0.f;
            hi[i] = pack2(x0, x1, kMmaBf16);
            const float2 r = Elem<MT>::to_f2(hi[i]);
            lo[i] = pack2(x0 - r.x, x1 - r.y, kMmaBf16);
          }
          // P is free once O^T(g-1) is done; a failed wait is acted on at the
          // next OR-barrier (the stores below then only race with an MMA whose
          // result is discarded)
          if (!pv_done) ok_w = warp_wait(pv_bar, (g - 1) & 1), pv_done = true;
          if constexpr (NCW == 8) {
            *reinterpret_cast<uint4*>(prow) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4*>(prow + L::kPBytes) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
          } else if constexpr (NCW == 4) {
            *reinterpret_cast<uint2*>(prow) = make_uint2(hi[0], hi[1]);
            *reinterpret_cast<uint2*>(prow + L::kPBytes) = make_uint2(lo[0], lo[1]);
          } else if constexpr (NCW == 2) {
            *reinterpret_cast<uint32_t*>(prow) = hi[0];
            *reinterpret_cast<uint32_t*>(prow + L::kPBytes) = lo[0];
          } else {
            *reinterpret_cast<uint16_t*>(prow) = (uint16_t)hi[0];
            *reinterpret_cast<uint16_t*>(prow + L::kPBytes) = (uint16_t)lo[0];
          }
        }
        if constexpr (!KV8) {
          // the V half lands apart from the K half: it is waited for before a
          // row of it is zeroed (this is a warp-wide wait, taken by the warps
          // that have such a row)
          if (__any_sync(0xffffffffu, !row_ok) && ok_w) ok_w = warp_wait(vfull_bar(st), (g / kStages) & 1);
        }
        if (!KV8 && !row_ok) {
          // this row is no token: zero its V row (both 64-element halves, 16
          // pieces shared out over the column groups) so 0 * stale never
          // enters PV
          unsigned char* vrow = smem + L::kStages0 + st * L::kStageBytes + 2 * L::kHalf + t * 128;
#pragma unroll
          for (int i = cg; i < 16; i += W::kNWG)
            *reinterpret_cast<uint4*>(vrow + (i >> 3) * L::kHalf + (i & 7) * 16) = make_uint4(0, 0, 0, 0);
        }
        // O^T(g) overwrites at an item's first tile and accumulates after it
        if (tid == 0) acc_flag[g & 1] = j > 0 ? 1 : 0;
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_ready_bar);  // P(g) written: the MMA warp issues O^T(g)
      }
      if (!ok) break;

      // ---- item result: fold the last O^T, reduce the per-row sums, write
      if (t == 0 && n_tiles > 0) ok = mbar_wait_or_abort(pv_bar, (g - 1) & 1, a.err, abort_flag);
      if (named_barrier_or(wg_bar, 128, !ok || !ok_w || *abort_flag)) { ok = false; break; }
      if (n_tiles > 0) {
        tc_fence_after();
        float ov[NCW], ow[NCW];
        tmem_ld<NCW>(tmem + t_lane + (uint32_t)(N + c0), ov);
        tmem_ld<NCW>(tmem + t_lane + (uint32_t)(2 * N + c0), ow);
#pragma unroll
        for (int c = 0; c < NCW; ++c) acc[c] += ov[c] + ow[c];
        tc_fence_before();
      }
      {
        float tmp[NCW];
#pragma unroll
        for (int c = 0; c < NCW; ++c) tmp[c] = l_tok[c];
        const float wsum = column_reduce<NCW, false>(tmp, lane);
        if (lane < NCW) red[quarter * N + c0 + lane] = wsum;
      }
      named_barrier(wg_bar, 128);
      if (t < NCW) {
        const int col = c0 + t;
        stat[N + col] = (red[col] + red[N + col]) + (red[2 * N + col] + red[3 * N + col]);
      }
      named_barrier(wg_bar, 128);
      const int d = t;  // output element this thread writes, per column
      // the shared-memory reads first, then the stores: the compiler keeps a
      // read through these pointers after a global store that came before it
      int code_c[NCW];
      float sum_c[NCW];
      {
        const int members = desc[kDMembers];
#pragma unroll
        for (int c = 0; c < NCW; ++c) {
          code_c[c] = m_c[c] < members ? mcode_all[slot * 32 + m_c[c]] : kSkip;  // padded: none
          sum_c[c] = stat[N + c0 + c];
        }
      }
#pragma unroll
      for (int c = 0; c < NCW; ++c) {
        const int code = code_c[c];
        if (code == kSkip) continue;
        const size_t qh = (size_t)(vbase + m_c[c]) * a.num_q_heads + (size_t)(kvh + e_c[c]) * G + h_c[c];
        // an 8-bit cache applies its V scale here (the merge is linear in it)
        const float o = KV8 ? acc[c] * __ldg(a.v_scale + kvh + e_c[c]) : acc[c];
        if (code == kZero) {
          a.out[qh * kD + d] = 0;
        } else if (code == kDirect) {
          a.out[qh * kD + d] = Elem<T>::from_f(__fdividef(o, sum_c[c]));
        } else {
          const size_t wslot = qh * a.num_parts + code;
          a.ws_acc[wslot * kD + d] = o;
          if (d == 0) {
            a.ws_ml[2 * wslot] = m_ref[c];
            a.ws_ml[2 * wslot + 1] = sum_c[c];
          }
        }
      }
      named_barrier(wg_bar, 128);  // this warpgroup's `red` and `stat` are reused next item
      if (lane == 0) mbar_arrive(free_bar(slot));  // its query rows have been used
    }
    if (!ok) *abort_flag = 1;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// host side

int sm_count() {
  static int count[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (!count[dev]) cudaDeviceGetAttribute(&count[dev], cudaDevAttrMultiProcessorCount, dev);
  return count[dev];
}

template <typename T, int NC, bool PAIR, bool KV8, bool WIDE = false>
cudaError_t launch_typed(const DecodeArgs& a0, const CUtensorMap& tk, const CUtensorMap& tv,
                         const CUtensorMap& tq, cudaStream_t stream, int* launches) {
  using L = Layout<(NC <= 16 ? 16 : 32), KV8>;
  auto* kern = decode_tc_kernel<T, NC, PAIR, KV8, WIDE>;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int sms = sm_count();
  const bool grouped = a0.plan != nullptr && !a0.own_pass;
  // groups never cross a multiple of the shared-prefix window
  const int chunk = kSharedPrefixSeqsPerLaunch;
  const int Tq = a0.query_tokens;
  for (int s0 = 0; s0 < a0.num_seqs; s0 += chunk) {
    DecodeArgs a = a0;
    a.num_seqs = a0.num_seqs - s0 < chunk ? a0.num_seqs - s0 : chunk;
    a.seq_offset = s0;
    const size_t rows0 = (size_t)s0 * Tq * a0.num_q_heads;  // first output row of the launch
    a.out = a0.out + rows0 * kD;
    a.block_tables = a0.block_tables + (size_t)s0 * a0.max_blocks_per_seq;
    a.context_lens = a0.context_lens + s0;
    if (a0.plan) {
      a.plan = a0.plan + s0;
      a.plan2 = a0.plan2 + s0;
    }
    if (a0.ws_acc) {
      a.ws_acc = a0.ws_acc + rows0 * a0.num_parts * kD;
      a.ws_ml = a0.ws_ml + rows0 * a0.num_parts * 2;
    }
    a.epoch = a0.epoch + (unsigned long long)(s0 / chunk);
    // at least one item per (unit, kv unit) without a plan; with one, the
    // number of items is only known on the device
    const int items0 = grouped ? sms : a.num_seqs * (a.num_kv_heads / (PAIR ? 2 : 1));
    const int grid = items0 < sms ? items0 : sms;
    constexpr int kBlock = Warps<NC, KV8>::kThreads;
    cudaError_t e = launch_pdl(kern, dim3(grid), dim3(kBlock), L::kAlloc, stream, a, tk, tv, tq);
    if (e != cudaSuccess) return e;
    ++*launches;
  }
  return cudaSuccess;
}

template <typename T, bool PAIR, bool KV8>
cudaError_t launch_cols(const DecodeArgs& a, int nc, const CUtensorMap& tk, const CUtensorMap& tv,
                        const CUtensorMap& tq, cudaStream_t st, int* n) {
  switch (nc) {
    case 1:
      if constexpr (!PAIR) return launch_typed<T, 1, false, KV8>(a, tk, tv, tq, st, n);
      break;
    case 2: return launch_typed<T, 2, PAIR, KV8>(a, tk, tv, tq, st, n);
    case 4: return launch_typed<T, 4, PAIR, KV8>(a, tk, tv, tq, st, n);
    case 8: return launch_typed<T, 8, PAIR, KV8>(a, tk, tv, tq, st, n);
    case 16: return launch_typed<T, 16, PAIR, KV8>(a, tk, tv, tq, st, n);
    case 32:  // two-head items take at most 16 columns
      if constexpr (!PAIR) {
        if (a.own_in_lists) return launch_typed<T, 32, false, KV8, true>(a, tk, tv, tq, st, n);
        return launch_typed<T, 32, false, KV8>(a, tk, tv, tq, st, n);
      }
      break;
  }
  return cudaErrorInvalidValue;
}

template <typename T, bool KV8>
cudaError_t launch_kind(const DecodeArgs& a, int nc, bool pair, const CUtensorMap& tk,
                        const CUtensorMap& tv, const CUtensorMap& tq, cudaStream_t st, int* n) {
  return pair ? launch_cols<T, true, KV8>(a, nc, tk, tv, tq, st, n)
              : launch_cols<T, false, KV8>(a, nc, tk, tv, tq, st, n);
}

}  // namespace tc

TcQueryBox tc_query_box(int group, int query_tokens, bool pair, bool grouped) {
  if (grouped) return {group, kTcMaxColumns / group};
  return {(pair ? 2 : 1) * group, query_tokens};
}

cudaError_t launch_decode_tc(const DecodeArgs& a, int dtype, const CUtensorMap& tk,
                             const CUtensorMap& tv, const CUtensorMap& tq, cudaStream_t stream,
                             int* launches, bool pair, bool fp8_cache) {
  if (a.num_seqs <= 0) return cudaSuccess;
  const int cols = tc::tc_columns(a.group, a.query_tokens, pair, a.plan != nullptr && !a.own_pass);
  if (cols < 1 || cols > kTcMaxColumns) return cudaErrorInvalidValue;
  int nc = 1;
  while (nc < cols) nc *= 2;
  if (fp8_cache) {
    if (dtype == 0) return tc::launch_kind<__half, true>(a, nc, pair, tk, tv, tq, stream, launches);
    return tc::launch_kind<__nv_bfloat16, true>(a, nc, pair, tk, tv, tq, stream, launches);
  }
  if (dtype == 0) return tc::launch_kind<__half, false>(a, nc, pair, tk, tv, tq, stream, launches);
  return tc::launch_kind<__nv_bfloat16, false>(a, nc, pair, tk, tv, tq, stream, launches);
}

int decode_tc_tile_tokens() { return tc::kTile; }

}  // namespace pa
