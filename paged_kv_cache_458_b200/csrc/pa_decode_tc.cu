// pa_decode_tc.cu -- decode attention with the grouped-query tile on the 5th-generation
// tensor cores (tcgen05, sm_100a).
//
// With g = Hq / Hkv query heads per kv head, every K/V byte the decode reads
// takes part in g multiply-adds for QK^T and g for PV: a skinny contraction
// that costs CUDA cores about as much time as the HBM read once g >= 4.  This
// kernel moves both products onto tcgen05.mma and keeps the read on TMA:
//
//   S^T[128 tok x N]  = K_tile[128 tok x 128 d] . Q^T[128 d x N]     (A K-major, B K-major)
//   O^T[128 d x N]    = V_tile^T[128 d x 128 tok] . P^T[128 tok x N] (A MN-major, B MN-major)
//
// with fp16/bf16 operands and fp32 accumulators in tensor memory (TMEM).  The
// N columns are query rows:
//   - one sequence (the plain kernel): its g query heads, padded to N = 16;
//     or, where the kv heads pair up and 2g <= 16, the 2g query heads of two
//     kv heads.  Then a tile is 64 tokens of both heads as the 128 MMA rows
//     (16-row groups of head 2e and of head 2e+1 alternate), so that one TMA
//     box carries 4 KB (16 rows of both heads) instead of 2 KB: the rate at
//     which one SM issues boxes bounds this kernel.  A row's logits against
//     the other head's queries are computed and discarded (p = 0), which the
//     tensor cores can afford;
//   - a group of sequences whose block tables begin with the same physical
//     blocks (the shared-prefix kernel): members x g query rows, N = 32.  The
//     blocks every member reads are then read once for all of them, which is
//     what sharing blocks between sequences (a common prompt prefix, beam
//     candidates forked from one parent) is for (zingnex.cn,
//     "vLLM与PagedAttention深度剖析", section 3.2 item 3; jsqmd.com,
//     "vLLM-v0.11.0性能实测", section 4.2: requests with the same prefix
//     share pages).
//
// The softmax stays in fp32 on the CUDA cores: tcgen05.ld gives thread t (of
// 128) the N logits of token t, and thread t writes its row of P.  The
// output accumulates in TMEM across the tiles of an item: each column keeps a
// softmax reference m_ref that moves only when a logit exceeds it by more than
// 8 (log2 units).  Then the tile's column maxima are found (a transposed warp
// reduction, lane c ending with column c, plus shared memory), and thread d
// folds row d of O^T into registers, rescaled by 2^(m_old - m_new).  On other
// tiles nothing waits for the PV product: it is read once, at the end of the
// item.  The products are pipelined by tile: S^T(j+1) is issued as soon as
// every thread has read S^T(j), while tile j's softmax runs, and the softmax
// of tile j waits for O^T(j-1) only to store P(j) (or to fold O^T).
// The probabilities enter the PV product as two terms of the input type, hi =
// round(p) and lo = round(p - hi), so they carry about 16 significant bits (a
// bf16 P alone, 8 bits, can move a short context's output by more than 2e-3).
// The two terms sit side by side as 2N columns of one PV product, so each V
// slice is read once for both, into O^T hi and O^T lo, summed when O^T is read.
//
// Work, plain kernel: items (sequence, kv head or pair of kv heads, partition
// of partition_tokens tokens, a multiple of 128) are numbered as in the
// CUDA-core kernel (partition 0 of every (sequence, kv head) first, then the
// further partitions of longer sequences).  Shared-prefix kernel: items
// (group leader, kv head, partition of the shared tokens), numbered over the
// leaders of the launch.  One persistent CTA per SM: a scheduler warp takes
// items (its first one by number, then from a counter in the workspace whose
// value carries the call's epoch), resolves each 16-token group of an item
// through the block table and fills one of two item slots (descriptor, pool
// rows, query rows), up to two items ahead; a producer warp then only issues
// the tiles' tiled TMA loads, one box per lane (per tile: 8 groups of one
// head or 4 groups of two heads, x {K, V} x two 64-element halves,
// 128B-swizzled), into one of NST stages.  A dedicated MMA warp issues every
// MMA and commits it to an mbarrier, so issuing them never holds up the
// softmax; the compute warps
// consume tiles in order and tell it through two more mbarriers when S^T(g)
// has been read and when P(g) has been written.  Tokens at or past the end of
// the item are masked in P and their V rows are zeroed in shared memory before
// the PV product, so stale or NaN rows never reach the result.
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

constexpr int kTile = 128;          // tokens per MMA tile (M)
constexpr int kD = 128;             // head_dim of this path
constexpr int kGroupRows = 16;      // token rows per TMA box (a block is a multiple)
constexpr int kSlots = 2;           // item slots (descriptor + query rows)

// Compute warpgroups split the NC query columns: warp w of the compute
// warps reads TMEM lane quarter w % 4 (tokens 32 (w % 4) .. +31, output rows
// likewise) and handles columns [(w / 4) NCW, (w / 4 + 1) NCW).  More warps
// per scheduler hide the latency of the per-column softmax arithmetic.
template <int NC>
struct Warps {
  static constexpr int kNCW = NC >= 16 ? 8 : (NC >= 8 ? 4 : NC);  // columns per warpgroup
  static constexpr int kNWG = NC / kNCW;                           // compute warpgroups
  static constexpr int kCompute = 128 * kNWG;                      // compute threads
  static constexpr int kThreads = kCompute + 96;                   // + MMA, producer, scheduler warps
  static_assert(kNCW * kNWG == NC, "columns split evenly");
};

// Per kernel kind: N columns, sequences per launch (the scheduler warp holds
// their prefix counts in registers) and TMEM columns (S^T in [0, N); O^T in [N, 3N), its hi part
// in [N, 2N) and its lo part in [2N, 3N), rounded up to a power of two).
template <bool GROUP>
struct Cfg {
  static constexpr int kN = GROUP ? 32 : 16;
  static constexpr int kMaxSeqs = GROUP ? kSharedPrefixSeqsPerLaunch : 512;
  static constexpr uint32_t kTmemCols = GROUP ? 128 : 64;
};

template <int NST, int N>
struct Layout {
  // offsets from a 1024-byte aligned base
  static constexpr int kStageBytes = 2 * kTile * kD * 2;      // K tile then V tile (64 KB)
  static constexpr int kHalf = kTile * 128;                    // one 64-element half of a tile (16 KB)
  static constexpr int kStages = 0;
  static constexpr int kQ = kStages + NST * kStageBytes;       // [slots][2 halves][N rows][128 B]
  static constexpr int kQBytes = 2 * N * 128;
  static constexpr int kP = kQ + kSlots * kQBytes;             // P hi, then P lo
  static constexpr int kPBytes = kTile * N * 2;                // [N/16 atoms][128 tok][32 B]
  static constexpr int kPAtom = kTile * 32;                    // bytes of one 16-column atom
  static constexpr int kRed = kP + 2 * kPBytes;                // [4 warps][N] f32
  static constexpr int kStat = kRed + 4 * N * 4;               // m[N], then alpha[N] or l[N], f32
  static constexpr int kDesc = kStat + 2 * N * 4;              // [slots][8] int
  static constexpr int kRows = kDesc + kSlots * 8 * 4;         // [slots][2][32] int: pool rows of
                                                               // the item's 16-token groups
  static constexpr int kBars = kRows + kSlots * 2 * 32 * 4;
  // full[NST], empty[NST], ready[slots], free[slots], meta[slots], qk, pv, drain,
  // s_free, p_ready
  static constexpr int kNumBars = 2 * NST + 3 * kSlots + 5;
  static constexpr int kMisc = kBars + kNumBars * 8;           // tmem address, abort flag,
                                                               // accumulate flags [2]
  static constexpr int kUsed = kMisc + 16;
  static constexpr int kAlloc = kUsed + 1024;                  // room to align the base
  static_assert(kQ % 1024 == 0 && kQBytes % 1024 == 0 && kP % 256 == 0, "swizzle atoms");
  static_assert(kAlloc <= 232448, "shared memory per CTA");
};

// Item descriptor fields (kDCtx: the context of a plain item, the number of
// member sequences of a shared-prefix item).
enum { kDS = 0, kDKvh, kDPart, kDBegin, kDEnd, kDTiles, kDParts, kDCtx };

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

// Item number -> (sequence, kv head, partition); see the file comment.  The
// first n_first numbers are partition 0 of every (sequence, kv head); the
// rest are counted by prefix[] (prefix[s] = items of sequences before s, per
// kv head, non-decreasing), numbered from `part0` within a sequence.  The
// warp holds prefix[] in registers: lane l has prefix[32 k + l] in pre[k]
// (INT_MAX past prefix[S]).  Called by all 32 lanes.
template <int PPL>
__device__ __forceinline__ void locate(int f, int n_first, int Hkv, const int (&pre)[PPL], int part0,
                                       int lane, int& s, int& kvh, int& part) {
  if (f < n_first) {
    s = f / Hkv;
    kvh = f % Hkv;
    part = 0;
    return;
  }
  const int g = f - n_first;
  kvh = g % Hkv;
  const int r = g / Hkv;
  // largest s with prefix[s] <= r: the number of such entries, less one
  int cnt = 0;
#pragma unroll
  for (int k = 0; k < PPL; ++k) cnt += pre[k] <= r ? 1 : 0;
  s = __reduce_add_sync(0xffffffffu, cnt) - 1;
  int mine = 0;
#pragma unroll
  for (int k = 0; k < PPL; ++k)
    if (k == (s >> 5)) mine = pre[k];
  part = part0 + r - __shfl_sync(0xffffffffu, mine, s & 31);
}

// Work counter tagged with the call's epoch in bits 24..63 (see pa_decode.cu).
__device__ __forceinline__ int take_item(unsigned long long* ctr, unsigned long long epoch,
                                         unsigned int* err) {
  const unsigned long long old = atomicAdd(ctr, 1ull);
  if ((old >> 24) == epoch) return (int)(old & 0xffffffull);
  for (int round = 0; round < (1 << 20); ++round) {
    const unsigned long long cur = atomicAdd(ctr, 0ull);
    if ((cur >> 24) == epoch) return (int)(atomicAdd(ctr, 1ull) & 0xffffffull);
    if (atomicCAS(ctr, cur, (epoch << 24) | 1ull) == cur) return 0;
  }
  report(err, kErrWaitTimeout);
  return -1;
}

// Query columns of a kernel kind: members x g (shared-prefix), 2g (an item of
// two kv heads), g.
template <int G, bool GROUP, bool PAIR>
__host__ __device__ constexpr int columns() { return GROUP ? Cfg<GROUP>::kN : (PAIR ? 2 * G : G); }

template <typename T, int G, int NST, bool GROUP, bool PAIR>
__global__ void __launch_bounds__(Warps<columns<G, GROUP, PAIR>()>::kThreads, 1)
decode_tc_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_q) {
  using C = Cfg<GROUP>;
  constexpr int N = C::kN;
  constexpr int NC = columns<G, GROUP, PAIR>();  // columns that carry query rows
  // An item covers kHeads kv heads; a tile is kTok tokens of each, as kTile
  // MMA rows (with two heads, 16-row groups of head 2e and head 2e+1 alternate)
  constexpr int kHeads = PAIR ? 2 : 1;
  constexpr int kTok = kTile / kHeads;
  static_assert(!(GROUP && PAIR), "a shared-prefix item covers one kv head");
  using W = Warps<NC>;
  constexpr int kComputeThreads = W::kCompute, kThreads = W::kThreads, NCW = W::kNCW;
  constexpr int kComputeWarps = kComputeThreads / 32;
  constexpr int kMmaWarp = kComputeWarps, kProducerWarp = kComputeWarps + 1,
                kSchedWarp = kComputeWarps + 2;
  using L = Layout<NST, N>;
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr uint32_t kIdescQK = instr_desc(kBf16 ? 1 : 0, 0, 0, kTile, N);
  // PV has 2N columns: P hi and P lo sit in consecutive 16-column atoms, so one
  // MMA reads each V slice once for both and writes O^T hi and O^T lo side by side
  constexpr uint32_t kIdescPV = instr_desc(kBf16 ? 1 : 0, 1, 1, kTile, 2 * N);
  static_assert(GROUP || kHeads * G <= N, "query heads per tile");
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  pdl_wait();  // the kernels before this decode (append, plan) must have landed
  pdl_launch_dependents();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int S = a.num_seqs, Hkv = a.num_kv_heads, PT = a.partition_tokens;
  int* desc_all = reinterpret_cast<int*>(smem + L::kDesc);
  int* rows_all = reinterpret_cast<int*>(smem + L::kRows);
  float* red = reinterpret_cast<float*>(smem + L::kRed);
  float* stat = reinterpret_cast<float*>(smem + L::kStat);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  const uint32_t bars = smem_addr(smem + L::kBars);
  auto full_bar = [&](int st) { return bars + st * 8; };
  auto empty_bar = [&](int st) { return bars + (NST + st) * 8; };
  auto ready_bar = [&](int sl) { return bars + (2 * NST + sl) * 8; };
  auto free_bar = [&](int sl) { return bars + (2 * NST + kSlots + sl) * 8; };
  auto meta_bar = [&](int sl) { return bars + (2 * NST + 2 * kSlots + sl) * 8; };
  const uint32_t qk_bar = bars + (2 * NST + 3 * kSlots) * 8;
  const uint32_t pv_bar = qk_bar + 8;
  const uint32_t drain_bar = qk_bar + 16;
  const uint32_t s_free_bar = qk_bar + 24;   // compute warps have read S^T(g)
  const uint32_t p_ready_bar = qk_bar + 32;  // compute warps have written P(g)
  volatile int* acc_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 8);  // [2]
  const uint32_t sm_stages = smem_addr(smem + L::kStages);
  const uint32_t sm_q = smem_addr(smem + L::kQ);
  const uint32_t sm_p = smem_addr(smem + L::kP);

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_holder)),
                 "r"(C::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    for (int st = 0; st < NST; ++st) {
      mbar_init(full_bar(st), 1);
      mbar_init(empty_bar(st), 1);
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
    *abort_flag = 0;
    mbar_init_fence();
  }
  // Query rows that no item fills stay zero (padded heads); a shared-prefix
  // item fills members x g rows, so the slots start all zero.
  constexpr int kRow0 = GROUP ? 0 : kHeads * G;
  constexpr int kPad = N - kRow0;
  if constexpr (kPad > 0) {
    for (int i = tid; i < kSlots * 2 * kPad * 8; i += kThreads) {
      const int chunk = i % 8, row = kRow0 + (i / 8) % kPad, half = (i / 8 / kPad) % 2,
                slot = i / 8 / kPad / 2;
      *reinterpret_cast<uint4*>(smem + L::kQ + slot * L::kQBytes + half * N * 128 + row * 128 +
                                chunk * 16) = make_uint4(0, 0, 0, 0);
    }
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == kSchedWarp) {
    // =====================================================================
    // scheduler warp: takes items, resolves them (sequence, kv head, token
    // range, the pool row of each 16-token group) and fills an item slot:
    // descriptor and rows (meta, for the producer), query rows (ready, for
    // the MMA and compute warps).  It runs up to two items ahead of the
    // compute warps, so none of its global round trips holds up the loads.
    // =====================================================================
    // Per sequence, the items numbered through prefix[]: further partitions
    // (plain) or the shared partitions of a group leader (shared-prefix).
    constexpr int PPL = C::kMaxSeqs / 32 + 1;  // prefix[0..S] over the lanes
    int pre[PPL];
    int carry = 0;
#pragma unroll
    for (int k = 0; k < PPL; ++k) {
      const int s = k * 32 + lane;  // this lane's entry prefix[s] = carry + counts before s
      int cnt = 0;
      if (s < S) {
        if constexpr (GROUP) {
          const int4 pl = __ldg(a.plan + s);
          cnt = (pl.x == 0 && pl.y >= 2) ? pl.w : 0;
        } else {
          int ctx = __ldg(a.context_lens + s);
          if (ctx < 0 || ctx > a.max_context_len) {
            if (blockIdx.x == 0) report(a.err, kErrContextLen);
            ctx = max(0, min(ctx, a.max_context_len));
          }
          cnt = max((ctx + PT - 1) / PT - 1, 0);
        }
      }
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      pre[k] = s <= S ? carry + incl - cnt : INT_MAX;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    const int Hitem = Hkv / kHeads;  // kv-head units of the item numbering
    const int n_first = GROUP ? 0 : S * Hitem;
    const int total = n_first + Hitem * carry;

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
      int* desc = desc_all + slot * 8;
      if (f >= total) {
        if (lane == 0) {
          desc[kDTiles] = -1;  // end of work
          mbar_arrive(meta_bar(slot));
          mbar_arrive(ready_bar(slot));
        }
        break;
      }
      int s, kvh, part;
      locate(f, n_first, Hitem, pre, GROUP ? 0 : 1, lane, s, kvh, part);
      kvh *= kHeads;  // the item's first kv head
      int t_end, ctx_or_members;
      const int t_begin = part * PT;
      if constexpr (GROUP) {
        const int4 pl = __ldg(a.plan + s);
        t_end = min(pl.z, t_begin + PT);
        ctx_or_members = pl.y;
      } else {
        const int ctx = max(0, min(__ldg(a.context_lens + s), a.max_context_len));
        t_end = min(ctx, t_begin + PT);
        ctx_or_members = ctx;
      }
      const int n_tok = max(0, t_end - t_begin);
      const int n_tiles = (n_tok + kTok - 1) / kTok;
      const int n_groups = (n_tok + kGroupRows - 1) / kGroupRows;  // <= 32
      // With 8-token blocks (half_boxes) rows 8..15 of a group have their own
      // entry; past the end of the item they re-read the first block (masked).
      const int32_t* table = a.block_tables + (size_t)s * a.max_blocks_per_seq;
      auto resolve = [&](int tok) {
        const int blk = __ldg(table + tok / a.block_size);
        if (blk < 0 || blk >= a.num_blocks) {
          report(a.err, kErrBlockId);
          return a.num_blocks * a.block_size;  // outside the map: TMA fills zeros
        }
        return blk * a.block_size + tok % a.block_size;
      };
      if (lane < n_groups) {
        const int tok = t_begin + lane * kGroupRows;
        const int row = resolve(tok);
        int* rows = rows_all + slot * 64;
        rows[lane] = row;
        if (a.half_boxes) rows[32 + lane] = tok + kGroupRows / 2 < t_end ? resolve(tok + kGroupRows / 2) : row;
      }
      if constexpr (GROUP) {
        // members x g query rows, 16-byte pieces stored in the 128B-swizzled
        // K-major layout the QK descriptor reads (piece c of row r at c ^ (r & 7))
        const int rows = ctx_or_members * G;
        const uint32_t qs = sm_q + slot * L::kQBytes;
        for (int i = lane; i < rows * 16; i += 32) {
          const int r = i >> 4, cc = i & 15;
          const int m = r / G, h = r % G;
          const size_t qrow = (size_t)(a.seq_offset + s + m) * a.num_q_heads + kvh * G + h;
          const uint4 v = __ldg(reinterpret_cast<const uint4*>(a.q + qrow * kD) + cc);
          const uint32_t dst = qs + (cc >> 3) * N * 128 + r * 128 + (((cc & 7) ^ (r & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(v.x), "r"(v.y),
                       "r"(v.z), "r"(v.w)
                       : "memory");
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      }
      // shared-prefix item: bit m set when member m's result is this
      // partition alone (written directly, not as a split-K partial)
      int direct_mask = 0;
      if constexpr (GROUP) {
        bool dm = false;
        if (lane < ctx_or_members) {
          const int ctx = max(0, min(__ldg(a.context_lens + s + lane), a.max_context_len));
          dm = seq_split(a.plan, s + lane, ctx, a.own_tokens).total <= 1;
        }
        direct_mask = (int)__ballot_sync(0xffffffffu, dm);
      }
      __syncwarp();  // every lane's rows (and query rows) before the arrivals
      if (lane == 0) {
        desc[kDS] = s;
        desc[kDKvh] = kvh;
        desc[kDPart] = part;
        desc[kDBegin] = t_begin;
        desc[kDEnd] = t_end;
        desc[kDTiles] = n_tiles;
        desc[kDParts] = GROUP ? direct_mask : (ctx_or_members + PT - 1) / PT;
        desc[kDCtx] = ctx_or_members;
        mbar_arrive(meta_bar(slot));
        const uint32_t rb = ready_bar(slot);
        if constexpr (GROUP) {
          mbar_arrive(rb);
        } else {
          mbar_arrive_expect_tx(rb, 2 * kHeads * G * 128);
          const int qrow = (a.seq_offset + s) * a.num_q_heads + kvh * G;
          tma_load_2d(sm_q + slot * L::kQBytes, &tm_q, rb, 0, qrow);
          tma_load_2d(sm_q + slot * L::kQBytes + N * 128, &tm_q, rb, 64, qrow);
        }
      }
      int nf = 0;
      if (lane == 0) {
        const int t = take_item(a.work_counter, a.epoch, a.err);
        nf = t < 0 ? total : (int)gridDim.x + t;
      }
      f = __shfl_sync(0xffffffffu, nf, 0);
    }
    if (!ok) *abort_flag = 1;
    // The query rows this warp loaded by TMA land before the CTA leaves
    // (bounded waits).  Items it-2 and it-1 may still be in flight, unless the
    // end-of-work mark went into item it-2's slot: that needed the slot freed,
    // so its rows had landed, and its phase parity now names a later phase.
    if (!GROUP && lane == 0)
      for (int k = max(0, it - (ok ? 1 : kSlots)); k < it; ++k)
        mbar_wait(ready_bar(k % kSlots), (k / kSlots) & 1, a.err);
  } else if (warp == kProducerWarp) {
    // =====================================================================
    // producer warp: the K/V tiles of each item, from the rows the scheduler
    // resolved, by TMA into the stage ring
    // =====================================================================
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
      const int* desc = desc_all + slot * 8;
      const int n_tiles = desc[kDTiles];
      if (n_tiles < 0) break;  // end of work
      const int kvh = desc[kDKvh];
      const int n_groups = (desc[kDEnd] - desc[kDBegin] + kGroupRows - 1) / kGroupRows;
      const int my_row = rows_all[slot * 64 + lane];
      const int my_row2 = a.half_boxes ? rows_all[slot * 64 + 32 + lane] : 0;
      for (int j = 0; j < n_tiles && ok; ++j) {
        const int st = issued % NST;
        if (issued >= NST &&
            !mbar_wait_or_abort(empty_bar(st), ((issued / NST) - 1) & 1, a.err, abort_flag)) {
          ok = false;
          break;
        }
        const int g0 = j * (kTok / kGroupRows);
        const int ng = min(kTok / kGroupRows, n_groups - g0);
        const uint32_t fb = full_bar(st);
        const uint32_t dst = sm_stages + st * L::kStageBytes;
        constexpr int kBoxBytes = kHeads * kGroupRows * 128;  // one box: a group of kHeads heads
        if (lane == 0) mbar_arrive_expect_tx(fb, ng * 4 * kBoxBytes);
        __syncwarp();
        {
          // lane 4 r + k loads piece k (K or V, 64-element half) of group r
          const int r = lane >> 2, k = lane & 3;
          const int row = __shfl_sync(0xffffffffu, my_row, min(g0 + r, 31));
          const int row2 = __shfl_sync(0xffffffffu, my_row2, min(g0 + r, 31));
          if (r < ng) {
            const uint32_t d = dst + k * L::kHalf + r * kBoxBytes;
            const void* map = k < 2 ? &tm_k : &tm_v;
            if constexpr (PAIR) {
              // maps of this kind are [rows][head] with the head innermost
              // after the dims: a box is 16 rows of head kvh, then of kvh + 1
              tma_load_3d(d, map, fb, (k & 1) * 64, row, kvh);
            } else {
              tma_load_3d(d, map, fb, (k & 1) * 64, kvh, row);
              if (a.half_boxes) tma_load_3d(d + (kGroupRows / 2) * 128, map, fb, (k & 1) * 64, kvh, row2);
            }
          }
        }
        ++issued;
      }
    }
    if (!ok) *abort_flag = 1;
    // Every TMA copy armed by this warp lands before the CTA leaves.
    if (lane == 0)
      for (int k = max(0, issued - NST); k < issued; ++k)
        mbar_wait(full_bar(k % NST), (k / NST) & 1, a.err);
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
    auto issue_qk = [&](int st, uint32_t q_addr) {
      tc_fence_after();
      const uint32_t kt = sm_stages + st * L::kStageBytes;
#pragma unroll
      for (int kk = 0; kk < kD / 16; ++kk) {
        const uint32_t ko = (kk / 4) * L::kHalf + (kk % 4) * 32;
        const uint32_t qo = (kk / 4) * N * 128 + (kk % 4) * 32;
        mma_f16(tmem, smem_desc(kt + ko, 16, 1024, kSw128), smem_desc(q_addr + qo, 16, 1024, kSw128),
                kIdescQK, kk > 0);
      }
      mma_commit(qk_bar);
    };
    if (lane == 0) {
      for (int it = 0; ok; ++it) {
        const int slot = it % kSlots;
        ok = mbar_wait_or_abort(ready_bar(slot), (it / kSlots) & 1, a.err, abort_flag);
        if (!ok) break;
        const int n_tiles = desc_all[slot * 8 + kDTiles];
        if (n_tiles < 0) break;  // end of work
        const uint32_t q_addr = sm_q + slot * L::kQBytes;
        // S^T(h) needs its stage landed and S^T(h-1) read by the compute warps
        auto qk_for = [&](int h) {
          bool w = mbar_wait_or_abort(full_bar(h % NST), (h / NST) & 1, a.err, abort_flag);
          if (w && h > 0) w = mbar_wait_or_abort(s_free_bar, (h - 1) & 1, a.err, abort_flag);
          if (w) issue_qk(h % NST, q_addr);
          return w;
        };
        if (n_tiles > 0) ok = qk_for(g);
        for (int j = 0; j < n_tiles && ok; ++j, ++g) {
          const int st = g % NST;
          // S^T(g+1) as soon as S^T(g) has been read: it runs during tile g's
          // softmax; then, once P(g) is written, O^T(g)
          if (j + 1 < n_tiles) {
            ok = qk_for(g + 1);
            if (!ok) break;
          }
          ok = mbar_wait_or_abort(p_ready_bar, g & 1, a.err, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t vt = sm_stages + st * L::kStageBytes + 2 * L::kHalf;
          const uint32_t acc0 = (uint32_t)acc_flag[g & 1];
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            mma_f16(tmem + N, smem_desc(vt + kk * 2048, L::kHalf, 1024, kSw128),
                    smem_desc(sm_p + kk * 512, L::kPAtom, 256, kSw32), kIdescPV,
                    acc0 | (uint32_t)(kk > 0));
          mma_commit(pv_bar);
          mma_commit(empty_bar(st));  // the stage is free once these MMAs are done
        }
      }
      if (!ok) *abort_flag = 1;
      // every MMA issued here completes before TMEM is freed (bounded wait)
      mma_commit(drain_bar);
      mbar_wait(drain_bar, 0, a.err);
    }
    __syncwarp();
  } else {
    // =====================================================================
    // compute warps: thread (t, cg) = token row t of S^T and row d = t of O^T,
    // for the columns of warpgroup cg.  Per tile g: wait for S^T(g), read it
    // and release it (s_free) so the MMA warp can issue S^T(g+1); the softmax
    // writes P(g) after O^T(g-1), its last reader, completed; then p_ready.
    // The output stays in TMEM across tiles: each column's softmax reference
    // m_ref only moves when a logit exceeds it by more than kRescale (log2
    // units), and only then is O^T folded into registers and rescaled (and
    // the next PV overwrites instead of accumulating).  Hence p <= 2^kRescale.
    // =====================================================================
    constexpr float kRescale = 8.f;
    const int t = tid & 127;         // token row of S^T, output row of O^T
    const int cg = tid >> 7;         // column group
    const int c0 = cg * NCW;         // first column of this thread
    const int quarter = warp & 3;    // TMEM lane quarter of this warp
    const uint32_t t_lane = ((uint32_t)(quarter * 32) << 16);
    // MMA row t: kv head e_row of the item, token tok_row of the tile; with
    // two heads only the columns of head e_row are this row's logits
    const int e_row = PAIR ? (t >> 4) & 1 : 0;
    const int tok_row = PAIR ? ((t >> 5) << 4) + (t & 15) : t;
    bool col_ok[NCW];
#pragma unroll
    for (int c = 0; c < NCW; ++c) col_ok[c] = !PAIR || (c0 + c) / G == e_row;
    int g = 0;  // tiles consumed, numbered across items
    bool ok = true;
    // one lane per warp waits on an mbarrier, the warp follows
    auto warp_wait = [&](uint32_t bar, uint32_t parity) {
      bool w = true;
      if (lane == 0) w = mbar_wait_or_abort(bar, parity, a.err, abort_flag);
      return __shfl_sync(0xffffffffu, (int)w, 0) != 0;
    };
    for (int it = 0; ok; ++it) {
      const int slot = it % kSlots;
      if (tid == 0) ok = mbar_wait_or_abort(ready_bar(slot), (it / kSlots) & 1, a.err, abort_flag);
      if (named_barrier_or(1, kComputeThreads, !ok || *abort_flag)) { ok = false; break; }
      const int* desc = desc_all + slot * 8;
      const int n_tiles = desc[kDTiles];
      if (n_tiles < 0) break;  // end of work
      const int s = desc[kDS], kvh = desc[kDKvh], part = desc[kDPart];
      const int t_begin = desc[kDBegin], t_end = desc[kDEnd], n_parts = desc[kDParts];
      const int ctx_or_members = desc[kDCtx];
      const int cols = GROUP ? ctx_or_members * G : kHeads * G;

      float acc[NCW], l_tok[NCW], m_ref[NCW];
#pragma unroll
      for (int c = 0; c < NCW; ++c) acc[c] = 0.f, l_tok[c] = 0.f, m_ref[c] = -INFINITY;
      bool pv_acc = false;  // O^T in TMEM holds tiles not folded into acc yet
      bool ok_w = true;     // every wait of this warp so far succeeded

      for (int j = 0; j < n_tiles; ++j, ++g) {
        const int st = g % NST;
        const int n_valid = min(kTok, t_end - (t_begin + j * kTok));
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
        if (named_barrier_or(1, kComputeThreads, !ok_w || *abort_flag)) { ok = false; break; }
        // O^T(g-1), the last reader of P and the last writer of O^T, is
        // waited for only where this tile needs it: before O^T is folded and
        // before P(g) is written
        bool pv_done = j == 0;
        const bool valid = tok_row < n_valid;
        bool over = false;
#pragma unroll
        for (int c = 0; c < NCW; ++c) {
          sv[c] = valid && col_ok[c] ? sv[c] * a.scale_log2 : -INFINITY;
          over |= (c0 + c < cols) && (sv[c] > m_ref[c] + kRescale);
        }
        const bool rescale = named_barrier_or(1, kComputeThreads, over);
        if (rescale) {
          // new references: this tile's column maxima where they are higher
          {
            float tmp[NCW];
#pragma unroll
            for (int c = 0; c < NCW; ++c) tmp[c] = sv[c];
            const float wmax = column_reduce<NCW, true>(tmp, lane);
            if (lane < NCW) red[quarter * N + c0 + lane] = wmax;
          }
          named_barrier(1, kComputeThreads);
          if (tid < NC)
            stat[tid] = fmaxf(fmaxf(red[tid], red[N + tid]), fmaxf(red[2 * N + tid], red[3 * N + tid]));
          named_barrier(1, kComputeThreads);
          float alpha[NCW];
#pragma unroll
          for (int c = 0; c < NCW; ++c) {
            const float m_new = fmaxf(m_ref[c], stat[c0 + c]);
            alpha[c] = exp2f(m_ref[c] - m_new);  // 0 while m_ref is -inf
            m_ref[c] = m_new;
            l_tok[c] *= alpha[c];
          }
          if (pv_acc) {
            // fold O^T (tiles before g) into acc, on the new reference
            if (!pv_done) ok_w = warp_wait(pv_bar, (g - 1) & 1), pv_done = true;
            tc_fence_after();
            float ov[NCW], ow[NCW];
            tmem_ld<NCW>(tmem + t_lane + (uint32_t)(N + c0), ov);
            tmem_ld<NCW>(tmem + t_lane + (uint32_t)(2 * N + c0), ow);
#pragma unroll
            for (int c = 0; c < NCW; ++c) acc[c] = (acc[c] + (ov[c] + ow[c])) * alpha[c];
          } else {
#pragma unroll
            for (int c = 0; c < NCW; ++c) acc[c] *= alpha[c];
          }
          pv_acc = false;
        }
        float p[NCW];
#pragma unroll
        for (int c = 0; c < NCW; ++c) {
          p[c] = valid && col_ok[c] ? exp2f(sv[c] - m_ref[c]) : 0.f;
          l_tok[c] += p[c];
        }
        // P^T rows: per 16-column atom, a 32-byte row per token (MN-major,
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
            hi[i] = pack2(x0, x1, kBf16);
            const float2 r = Elem<T>::to_f2(hi[i]);
            lo[i] = pack2(x0 - r.x, x1 - r.y, kBf16);
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
        if (!valid) {
          // zero this token's V row (both 64-element halves, 16 pieces shared
          // out over the column groups) so 0 * stale never enters PV
          unsigned char* vrow = smem + L::kStages + st * L::kStageBytes + 2 * L::kHalf + t * 128;
#pragma unroll
          for (int i = cg; i < 16; i += W::kNWG)
            *reinterpret_cast<uint4*>(vrow + (i >> 3) * L::kHalf + (i & 7) * 16) = make_uint4(0, 0, 0, 0);
        }
        if (tid == 0) acc_flag[g & 1] = pv_acc ? 1 : 0;  // does O^T(g) accumulate?
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_ready_bar);  // P(g) written: the MMA warp issues O^T(g)
        pv_acc = true;
      }
      if (!ok) break;

      // ---- item result: fold the last O^T, reduce the per-token sums, write
      if (tid == 0 && n_tiles > 0) ok = mbar_wait_or_abort(pv_bar, (g - 1) & 1, a.err, abort_flag);
      if (named_barrier_or(1, kComputeThreads, !ok || !ok_w || *abort_flag)) { ok = false; break; }
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
      named_barrier(1, kComputeThreads);
      if (tid < NC) stat[N + tid] = (red[tid] + red[N + tid]) + (red[2 * N + tid] + red[3 * N + tid]);
      named_barrier(1, kComputeThreads);
      const int d = t;  // output element this thread writes, per column
#pragma unroll
      for (int c = 0; c < NCW; ++c) {
        const int col = c0 + c;
        if (col >= cols) break;
        const float L_c = stat[N + col];
        const int m = GROUP ? col / G : 0, h = GROUP ? col % G : col;
        const size_t qh = (size_t)(s + m) * a.num_q_heads + (size_t)kvh * G + h;
        bool zero = false, direct;
        if constexpr (GROUP) {
          direct = (n_parts >> m) & 1;  // from the producer: this partition is the member's result
        } else {
          zero = ctx_or_members == 0;
          direct = n_parts <= 1;
        }
        if (zero) {
          a.out[qh * kD + d] = 0;
        } else if (direct) {
          a.out[qh * kD + d] = Elem<T>::from_f(acc[c] / L_c);
        } else {
          const size_t wslot = qh * a.num_parts + part;
          a.ws_acc[wslot * kD + d] = acc[c];
          if (d == 0) {
            a.ws_ml[2 * wslot] = m_ref[c];
            a.ws_ml[2 * wslot + 1] = L_c;
          }
        }
      }
      named_barrier(1, kComputeThreads);  // `red` and `stat` are reused by the next item
      if (lane == 0) mbar_arrive(free_bar(slot));  // its query rows have been used
    }
    if (!ok) *abort_flag = 1;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(C::kTmemCols)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// host side

constexpr int kStagesTc = 3;

int sm_count() {
  static int count[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (!count[dev]) cudaDeviceGetAttribute(&count[dev], cudaDevAttrMultiProcessorCount, dev);
  return count[dev];
}

template <typename T, int G, bool GROUP, bool PAIR>
cudaError_t launch_typed(const DecodeArgs& a0, const CUtensorMap& tk, const CUtensorMap& tv,
                         const CUtensorMap& tq, cudaStream_t stream, int* launches) {
  using C = Cfg<GROUP>;
  using L = Layout<kStagesTc, C::kN>;
  auto* kern = decode_tc_kernel<T, G, kStagesTc, GROUP, PAIR>;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int sms = sm_count();
  constexpr int kChunk = C::kMaxSeqs;
  for (int s0 = 0; s0 < a0.num_seqs; s0 += kChunk) {
    DecodeArgs a = a0;
    a.num_seqs = a0.num_seqs - s0 < kChunk ? a0.num_seqs - s0 : kChunk;
    a.seq_offset = s0;
    a.out = a0.out + (size_t)s0 * a0.num_q_heads * kD;
    a.block_tables = a0.block_tables + (size_t)s0 * a0.max_blocks_per_seq;
    a.context_lens = a0.context_lens + s0;
    if (a0.plan) a.plan = a0.plan + s0;
    if (a0.ws_acc) {
      a.ws_acc = a0.ws_acc + (size_t)s0 * a0.num_q_heads * a0.num_parts * kD;
      a.ws_ml = a0.ws_ml + (size_t)s0 * a0.num_q_heads * a0.num_parts * 2;
    }
    a.epoch = a0.epoch + (unsigned long long)(s0 / kChunk);
    // plain: at least one item per (sequence, kv head); shared-prefix: the
    // number of items is only known on the device
    const int items0 = GROUP ? sms : a.num_seqs * (a.num_kv_heads / (PAIR ? 2 : 1));
    const int grid = items0 < sms ? items0 : sms;
    constexpr int kBlock = Warps<columns<G, GROUP, PAIR>()>::kThreads;
    cudaError_t e = launch_pdl(kern, dim3(grid), dim3(kBlock), L::kAlloc, stream, a, tk, tv, tq);
    if (e != cudaSuccess) return e;
    ++*launches;
  }
  return cudaSuccess;
}

template <typename T, bool GROUP, bool PAIR>
cudaError_t launch_group(const DecodeArgs& a, int G, const CUtensorMap& tk, const CUtensorMap& tv,
                         const CUtensorMap& tq, cudaStream_t st, int* n) {
  switch (G) {
    case 1: return launch_typed<T, 1, GROUP, PAIR>(a, tk, tv, tq, st, n);
    case 2: return launch_typed<T, 2, GROUP, PAIR>(a, tk, tv, tq, st, n);
    case 4: return launch_typed<T, 4, GROUP, PAIR>(a, tk, tv, tq, st, n);
    case 8: return launch_typed<T, 8, GROUP, PAIR>(a, tk, tv, tq, st, n);
    case 16:
      if constexpr (!PAIR) return launch_typed<T, 16, GROUP, false>(a, tk, tv, tq, st, n);
  }
  return cudaErrorInvalidValue;
}

}  // namespace tc

cudaError_t launch_decode_tc(const DecodeArgs& a, int dtype, int group, const CUtensorMap& tk,
                             const CUtensorMap& tv, const CUtensorMap& tq, cudaStream_t stream,
                             int* launches, bool pair) {
  if (a.num_seqs <= 0) return cudaSuccess;
  if (pair) {
    if (dtype == 0) return tc::launch_group<__half, false, true>(a, group, tk, tv, tq, stream, launches);
    return tc::launch_group<__nv_bfloat16, false, true>(a, group, tk, tv, tq, stream, launches);
  }
  if (dtype == 0) return tc::launch_group<__half, false, false>(a, group, tk, tv, tq, stream, launches);
  return tc::launch_group<__nv_bfloat16, false, false>(a, group, tk, tv, tq, stream, launches);
}

cudaError_t launch_decode_shared_tc(const DecodeArgs& a, int dtype, int group, const CUtensorMap& tk,
                                    const CUtensorMap& tv, cudaStream_t stream, int* launches) {
  if (a.num_seqs <= 0 || !a.plan) return cudaSuccess;
  if (dtype == 0) return tc::launch_group<__half, true, false>(a, group, tk, tv, tk, stream, launches);
  return tc::launch_group<__nv_bfloat16, true, false>(a, group, tk, tv, tk, stream, launches);
}

int decode_tc_tile_tokens() { return tc::kTile; }

}  // namespace pa
