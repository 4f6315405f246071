// pa_decode_tc.cu -- decode attention with the grouped-query tile on the 5th-generation
// tensor cores (tcgen05, sm_100a).
//
// With g = Hq / Hkv query heads per kv head, every K/V byte the decode reads
// takes part in g multiply-adds for QK^T and g for PV: a skinny contraction
// that costs CUDA cores about as much time as the HBM read once g >= 4.  This
// kernel moves both products onto tcgen05.mma and keeps the read on TMA:
//
//   S^T[128 tok x 16]  = K_tile[128 tok x 128 d] . Q^T[128 d x 16]   (A K-major, B K-major)
//   O^T[128 d x 16]    = V_tile^T[128 d x 128 tok] . P^T[128 tok x 16] (A MN-major, B MN-major)
//
// with the g heads padded to N = 16 (zero rows of Q), fp16/bf16 operands and
// fp32 accumulators in tensor memory (TMEM).  The softmax stays in fp32 on the
// CUDA cores: tcgen05.ld gives thread t (of 128) the 16 logits of token t, the
// per-head tile maximum is a warp + shared-memory reduction, and thread t writes
// its row of P.  After the PV product thread d reads row d of O^T and folds it
// into its running output (rescaled by 2^(m_old - m_new) per head).  The
// probabilities enter the PV product as two terms of the input type, hi =
// round(p) and lo = round(p - hi), so they carry about 16 significant bits (a
// bf16 P alone, 8 bits, can move a short context's output by more than 2e-3);
// the tensor cores have ample room for the second set of MMAs.
//
// Work: items (sequence, kv head, partition of partition_tokens tokens, a
// multiple of 128) are numbered as in the CUDA-core kernel (partition 0 of
// every (sequence, kv head) first, then the further partitions of longer
// sequences).  One persistent CTA per SM: a producer warp takes items (its
// first one by number, then from a counter in the workspace whose value
// carries the call's epoch), resolves each 16-token group of an item through
// the block table and issues per 128-token tile 32 tiled TMA loads (8 groups x
// {K, V} x two 64-element halves, 128B-swizzled) into one of NST stages, plus
// the item's query rows into an item slot.  Four compute warps consume tiles
// in order; thread 0 issues the MMAs and commits them to mbarriers.  Tokens at
// or past the context are masked in P and their V rows are zeroed in shared
// memory before the PV product, so stale or NaN rows never reach the result.
//
// Split-K partials and the merge kernel are shared with the CUDA-core path.
//
// Every wait is bounded; a compute-side wait is made by thread 0 and its
// outcome shared through an OR-reduced named barrier, so the four compute
// warps always agree whether to go on.  On the way out the producer waits for
// its TMA copies, thread 0 for its MMAs, and warp 0 frees the TMEM columns.
#include <cuda.h>
#include <cuda_runtime.h>

#include <type_traits>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {
namespace tc {

constexpr int kTile = 128;          // tokens per MMA tile (M)
constexpr int kN = 16;              // padded query heads (N)
constexpr int kD = 128;             // head_dim of this path
constexpr int kGroupRows = 16;      // token rows per TMA box (a block is a multiple)
constexpr int kSlots = 2;           // item slots (descriptor + query rows)
constexpr int kMaxSeqs = 512;       // sequences per launch (prefix in shared memory)
constexpr int kComputeThreads = 128;
constexpr int kThreads = kComputeThreads + 32;
constexpr uint32_t kTmemCols = 32;  // S^T in columns [0,16), O^T in [16,32)

template <int NST>
struct Layout {
  // offsets from a 1024-byte aligned base
  static constexpr int kStageBytes = 2 * kTile * kD * 2;      // K tile then V tile (64 KB)
  static constexpr int kHalf = kTile * 128;                    // one 64-element half of a tile (16 KB)
  static constexpr int kStages = 0;
  static constexpr int kQ = kStages + NST * kStageBytes;       // [slots][2 halves][16 rows][128 B]
  static constexpr int kQBytes = 2 * kN * 128;
  static constexpr int kP = kQ + kSlots * kQBytes;             // P hi, then P lo: [128 tok][16] 32-B rows
  static constexpr int kPBytes = kTile * kN * 2;
  static constexpr int kRed = kP + 2 * kPBytes;                // [4 warps][16] f32
  static constexpr int kDesc = kRed + 4 * kN * 4;              // [slots][8] int
  static constexpr int kPrefix = kDesc + kSlots * 8 * 4;       // [kMaxSeqs + 1] int
  static constexpr int kBars = (kPrefix + (kMaxSeqs + 1) * 4 + 7) / 8 * 8;
  // full[NST], empty[NST], ready[slots], free[slots], qk, pv
  static constexpr int kNumBars = 2 * NST + 2 * kSlots + 2;
  static constexpr int kMisc = kBars + kNumBars * 8;           // tmem address, abort flag
  static constexpr int kUsed = kMisc + 16;
  static constexpr int kAlloc = kUsed + 1024;                  // room to align the base
  static_assert(kQ % 1024 == 0 && kQBytes % 1024 == 0 && kP % 256 == 0, "swizzle atoms");
};

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
// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
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

// Item number -> (sequence, kv head, partition); see the file comment.
__device__ __forceinline__ void locate(int f, int n_first, int Hkv, int S, const int* prefix, int& s,
                                       int& kvh, int& part) {
  if (f < n_first) {
    s = f / Hkv;
    kvh = f % Hkv;
    part = 0;
    return;
  }
  const int g = f - n_first;
  kvh = g % Hkv;
  const int r = g / Hkv;
  int lo = 0, hi = S;  // largest s with prefix[s] <= r
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= r) lo = mid; else hi = mid;
  }
  s = lo;
  part = 1 + r - prefix[lo];
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

template <typename T, int G, int NST>
__global__ void __launch_bounds__(kThreads, 1)
decode_tc_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_q) {
  using L = Layout<NST>;
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr uint32_t kIdescQK = instr_desc(kBf16 ? 1 : 0, 0, 0, kTile, kN);
  constexpr uint32_t kIdescPV = instr_desc(kBf16 ? 1 : 0, 1, 1, kTile, kN);
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  pdl_wait();  // the append before this decode must have landed
  pdl_launch_dependents();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int S = a.num_seqs, Hkv = a.num_kv_heads, PT = a.partition_tokens;
  int* desc_all = reinterpret_cast<int*>(smem + L::kDesc);
  int* prefix = reinterpret_cast<int*>(smem + L::kPrefix);
  float* red = reinterpret_cast<float*>(smem + L::kRed);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  const uint32_t bars = smem_addr(smem + L::kBars);
  auto full_bar = [&](int st) { return bars + st * 8; };
  auto empty_bar = [&](int st) { return bars + (NST + st) * 8; };
  auto ready_bar = [&](int sl) { return bars + (2 * NST + sl) * 8; };
  auto free_bar = [&](int sl) { return bars + (2 * NST + kSlots + sl) * 8; };
  const uint32_t qk_bar = bars + (2 * NST + 2 * kSlots) * 8;
  const uint32_t pv_bar = qk_bar + 8;
  const uint32_t sm_stages = smem_addr(smem + L::kStages);
  const uint32_t sm_q = smem_addr(smem + L::kQ);
  const uint32_t sm_p = smem_addr(smem + L::kP);

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_holder)),
                 "r"(kTmemCols)
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
      mbar_init(free_bar(sl), 4);
    }
    mbar_init(qk_bar, 1);
    mbar_init(pv_bar, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  // Query rows G..15 of both slots are zero for good (the padded heads).
  if constexpr (G < kN) {
    constexpr int kPad = kN - G;
    for (int i = tid; i < kSlots * 2 * kPad * 8; i += kThreads) {
      const int chunk = i % 8, row = G + (i / 8) % kPad, half = (i / 8 / kPad) % 2,
                slot = i / 8 / kPad / 2;
      *reinterpret_cast<uint4*>(smem + L::kQ + slot * L::kQBytes + half * kN * 128 + row * 128 +
                                chunk * 16) = make_uint4(0, 0, 0, 0);
    }
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 4) {
    // =====================================================================
    // producer warp: items, table entries, TMA loads
    // =====================================================================
    int carry = 0;
    if (lane == 0) prefix[0] = 0;
    for (int base = 0; base < S; base += 32) {
      const int s = base + lane;
      int extra = 0;
      if (s < S) {
        int ctx = __ldg(a.context_lens + s);
        if (ctx < 0 || ctx > a.max_context_len) {
          if (blockIdx.x == 0) report(a.err, kErrContextLen);
          ctx = max(0, min(ctx, a.max_context_len));
        }
        extra = max((ctx + PT - 1) / PT - 1, 0);
      }
      int incl = extra;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      if (s < S) prefix[s + 1] = carry + incl;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    __syncwarp();
    const int n_first = S * Hkv;
    const int total = n_first + Hkv * carry;

    int issued = 0;  // tiles armed so far (stage ring position)
    bool ok = true;
    int f = blockIdx.x;
    for (int it = 0;; ++it) {
      const int slot = it % kSlots;
      if (it >= kSlots &&
          !mbar_wait_or_abort(free_bar(slot), ((it / kSlots) - 1) & 1, a.err, abort_flag)) {
        ok = false;
        break;
      }
      int* desc = desc_all + slot * 8;
      if (f >= total) {
        if (lane == 0) {
          desc[kDTiles] = -1;  // end of work
          mbar_arrive(ready_bar(slot));
        }
        break;
      }
      int s, kvh, part;
      locate(f, n_first, Hkv, S, prefix, s, kvh, part);
      const int ctx = max(0, min(__ldg(a.context_lens + s), a.max_context_len));
      const int t_begin = part * PT;
      const int t_end = min(ctx, t_begin + PT);
      const int n_tok = max(0, t_end - t_begin);
      const int n_tiles = (n_tok + kTile - 1) / kTile;
      const int n_groups = (n_tok + kGroupRows - 1) / kGroupRows;  // <= 32
      int my_row = 0;
      if (lane < n_groups) {
        const int tok = t_begin + lane * kGroupRows;
        const int blk = __ldg(a.block_tables + (size_t)s * a.max_blocks_per_seq + tok / a.block_size);
        if (blk < 0 || blk >= a.num_blocks) {
          report(a.err, kErrBlockId);
          my_row = a.num_blocks * a.block_size;  // outside the map: TMA fills zeros
        } else {
          my_row = blk * a.block_size + tok % a.block_size;
        }
      }
      if (lane == 0) {
        desc[kDS] = s;
        desc[kDKvh] = kvh;
        desc[kDPart] = part;
        desc[kDBegin] = t_begin;
        desc[kDEnd] = t_end;
        desc[kDTiles] = n_tiles;
        desc[kDParts] = (ctx + PT - 1) / PT;
        desc[kDCtx] = ctx;
        const uint32_t rb = ready_bar(slot);
        mbar_arrive_expect_tx(rb, 2 * G * 128);
        const int qrow = (a.seq_offset + s) * a.num_q_heads + kvh * G;
        tma_load_2d(sm_q + slot * L::kQBytes, &tm_q, rb, 0, qrow);
        tma_load_2d(sm_q + slot * L::kQBytes + kN * 128, &tm_q, rb, 64, qrow);
      }
      for (int j = 0; j < n_tiles && ok; ++j) {
        const int st = issued % NST;
        if (issued >= NST &&
            !mbar_wait_or_abort(empty_bar(st), ((issued / NST) - 1) & 1, a.err, abort_flag)) {
          ok = false;
          break;
        }
        const int g0 = j * (kTile / kGroupRows);
        const int ng = min(kTile / kGroupRows, n_groups - g0);
        const uint32_t fb = full_bar(st);
        const uint32_t dst = sm_stages + st * L::kStageBytes;
        if (lane == 0) mbar_arrive_expect_tx(fb, ng * 4 * kGroupRows * 128);
        for (int r = 0; r < ng; ++r) {
          const int row = __shfl_sync(0xffffffffu, my_row, g0 + r);
          if (lane == 0) {
            const uint32_t o = r * kGroupRows * 128;
            tma_load_3d(dst + o, &tm_k, fb, 0, kvh, row);
            tma_load_3d(dst + L::kHalf + o, &tm_k, fb, 64, kvh, row);
            tma_load_3d(dst + 2 * L::kHalf + o, &tm_v, fb, 0, kvh, row);
            tma_load_3d(dst + 3 * L::kHalf + o, &tm_v, fb, 64, kvh, row);
          }
        }
        ++issued;
      }
      if (!ok) break;
      int nf = 0;
      if (lane == 0) {
        const int t = take_item(a.work_counter, a.epoch, a.err);
        nf = t < 0 ? total : (int)gridDim.x + t;
      }
      f = __shfl_sync(0xffffffffu, nf, 0);
    }
    if (!ok) *abort_flag = 1;
    // Every TMA copy armed by this warp lands before the CTA leaves.
    if (lane == 0)
      for (int k = max(0, issued - NST); k < issued; ++k)
        mbar_wait(full_bar(k % NST), (k / NST) & 1, a.err);
  } else {
    // =====================================================================
    // compute warps (128 threads): thread t = token row t of S^T, row d = t of O^T
    // =====================================================================
    const uint32_t t_lane = ((uint32_t)(warp * 32) << 16);  // this warp's TMEM lane quarter
    int n_used = 0;       // tiles consumed (stage ring position, qk/pv phases)
    int qk_commits = 0, pv_commits = 0;  // thread 0 only
    bool ok = true;
    for (int it = 0; ok; ++it) {
      const int slot = it % kSlots;
      if (tid == 0) ok = mbar_wait_or_abort(ready_bar(slot), (it / kSlots) & 1, a.err, abort_flag);
      if (named_barrier_or(1, kComputeThreads, !ok || *abort_flag)) { ok = false; break; }
      const int* desc = desc_all + slot * 8;
      const int n_tiles = desc[kDTiles];
      if (n_tiles < 0) break;  // end of work
      const int s = desc[kDS], kvh = desc[kDKvh], part = desc[kDPart];
      const int t_begin = desc[kDBegin], t_end = desc[kDEnd], n_parts = desc[kDParts];
      const int ctx = desc[kDCtx];
      const uint32_t q_addr = sm_q + slot * L::kQBytes;

      float acc[G], l_tok[G], m_run[G];
#pragma unroll
      for (int h = 0; h < G; ++h) acc[h] = 0.f, l_tok[h] = 0.f, m_run[h] = -INFINITY;

      for (int j = 0; j < n_tiles; ++j, ++n_used) {
        const int st = n_used % NST;
        const uint32_t kt = sm_stages + st * L::kStageBytes;
        const uint32_t vt = kt + 2 * L::kHalf;
        const int n_valid = min(kTile, t_end - (t_begin + j * kTile));
        // ---- S^T = K . Q^T
        if (tid == 0) {
          ok = mbar_wait_or_abort(full_bar(st), (n_used / NST) & 1, a.err, abort_flag);
          if (ok) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk) {
              const uint32_t ko = (kk / 4) * L::kHalf + (kk % 4) * 32;
              const uint32_t qo = (kk / 4) * kN * 128 + (kk % 4) * 32;
              mma_f16(tmem, smem_desc(kt + ko, 16, 1024, kSw128),
                      smem_desc(q_addr + qo, 16, 1024, kSw128), kIdescQK, kk > 0);
            }
            mma_commit(qk_bar);
            ++qk_commits;
            ok = mbar_wait_or_abort(qk_bar, n_used & 1, a.err, abort_flag);
          }
        }
        if (named_barrier_or(1, kComputeThreads, !ok || *abort_flag)) { ok = false; break; }
        tc_fence_after();
        float sv[16];
        tmem_ld16(tmem + t_lane, sv);

        // ---- softmax over this tile (log2 domain)
        const bool valid = tid < n_valid;
        float tile_max[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          sv[h] = valid ? sv[h] * a.scale_log2 : -INFINITY;
          float mx = sv[h];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          tile_max[h] = mx;
        }
        if (lane == 0)
#pragma unroll
          for (int h = 0; h < G; ++h) red[warp * kN + h] = tile_max[h];
        named_barrier(1, kComputeThreads);
        float alpha[G], p[kN];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float mt = fmaxf(fmaxf(red[h], red[kN + h]), fmaxf(red[2 * kN + h], red[3 * kN + h]));
          const float m_new = fmaxf(m_run[h], mt);
          alpha[h] = exp2f(m_run[h] - m_new);
          m_run[h] = m_new;
          p[h] = valid ? exp2f(sv[h] - m_new) : 0.f;
        }
#pragma unroll
        for (int h = G; h < kN; ++h) p[h] = 0.f;
        // P^T rows (MN-major, 32-byte rows, 32-byte swizzle: 16-byte half c of
        // row t sits at c ^ bit 2 of t), once for hi = round(p) and once for
        // lo = round(p - hi).
        {
          float plo[kN];
          uint4 lo, hi;
          lo.x = pack2(p[0], p[1], kBf16);  lo.y = pack2(p[2], p[3], kBf16);
          lo.z = pack2(p[4], p[5], kBf16);  lo.w = pack2(p[6], p[7], kBf16);
          hi.x = pack2(p[8], p[9], kBf16);  hi.y = pack2(p[10], p[11], kBf16);
          hi.z = pack2(p[12], p[13], kBf16); hi.w = pack2(p[14], p[15], kBf16);
          {
            const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float2 r = Elem<T>::to_f2(w[i]);
              plo[2 * i] = p[2 * i] - r.x;
              plo[2 * i + 1] = p[2 * i + 1] - r.y;
            }
          }
          const int sw = (tid >> 2) & 1;
          unsigned char* prow = smem + L::kP + tid * 32;
          *reinterpret_cast<uint4*>(prow + 16 * sw) = lo;
          *reinterpret_cast<uint4*>(prow + 16 * (sw ^ 1)) = hi;
          uint4 lo2, hi2;
          lo2.x = pack2(plo[0], plo[1], kBf16);   lo2.y = pack2(plo[2], plo[3], kBf16);
          lo2.z = pack2(plo[4], plo[5], kBf16);   lo2.w = pack2(plo[6], plo[7], kBf16);
          hi2.x = pack2(plo[8], plo[9], kBf16);   hi2.y = pack2(plo[10], plo[11], kBf16);
          hi2.z = pack2(plo[12], plo[13], kBf16); hi2.w = pack2(plo[14], plo[15], kBf16);
          *reinterpret_cast<uint4*>(prow + L::kPBytes + 16 * sw) = lo2;
          *reinterpret_cast<uint4*>(prow + L::kPBytes + 16 * (sw ^ 1)) = hi2;
#pragma unroll
          for (int h = 0; h < G; ++h) l_tok[h] = l_tok[h] * alpha[h] + p[h];
        }
        if (!valid) {
          // zero this token's V row (both 64-element halves) so 0 * stale never enters PV
          unsigned char* vrow = smem + L::kStages + st * L::kStageBytes + 2 * L::kHalf + tid * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            *reinterpret_cast<uint4*>(vrow + c * 16) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4*>(vrow + L::kHalf + c * 16) = make_uint4(0, 0, 0, 0);
          }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        named_barrier(1, kComputeThreads);

        // ---- O^T = V^T . P^T
        if (tid == 0) {
          tc_fence_after();
#pragma unroll
          for (int part_p = 0; part_p < 2; ++part_p)  // P = hi + lo
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk)
              mma_f16(tmem + kN, smem_desc(vt + kk * 2048, L::kHalf, 1024, kSw128),
                      smem_desc(sm_p + part_p * L::kPBytes + kk * 512, 512, 256, kSw32), kIdescPV,
                      part_p > 0 || kk > 0);
          mma_commit(pv_bar);
          mma_commit(empty_bar(st));  // the stage is free once these MMAs are done
          ++pv_commits;
          ok = mbar_wait_or_abort(pv_bar, n_used & 1, a.err, abort_flag);
        }
        if (named_barrier_or(1, kComputeThreads, !ok || *abort_flag)) { ok = false; break; }
        tc_fence_after();
        float ov[16];
        tmem_ld16(tmem + t_lane + kN, ov);
#pragma unroll
        for (int h = 0; h < G; ++h) acc[h] = acc[h] * alpha[h] + ov[h];
        tc_fence_before();
      }
      if (!ok) break;

      // ---- item result: reduce the per-token sums, write output or partial
      float lsum[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float v = l_tok[h];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        lsum[h] = v;
      }
      named_barrier(1, kComputeThreads);  // the tile maxima in `red` have been read
      if (lane == 0)
#pragma unroll
        for (int h = 0; h < G; ++h) red[warp * kN + h] = lsum[h];
      named_barrier(1, kComputeThreads);
      const int d = tid;  // output element this thread writes, per head
      const size_t qh0 = (size_t)s * a.num_q_heads + (size_t)kvh * G;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float L_h = red[h] + red[kN + h] + red[2 * kN + h] + red[3 * kN + h];
        const size_t qh = qh0 + h;
        if (ctx == 0) {
          a.out[qh * kD + d] = 0;
        } else if (n_parts <= 1) {
          a.out[qh * kD + d] = Elem<T>::from_f(acc[h] / L_h);
        } else {
          const size_t wslot = qh * a.num_parts + part;
          a.ws_acc[wslot * kD + d] = acc[h];
          if (d == 0) {
            a.ws_ml[2 * wslot] = m_run[h];
            a.ws_ml[2 * wslot + 1] = L_h;
          }
        }
      }
      named_barrier(1, kComputeThreads);  // `red` is reused by the next item
      if (lane == 0) mbar_arrive(free_bar(slot));  // its query rows have been used
    }
    if (!ok && tid == 0) *abort_flag = 1;
    // MMAs issued by thread 0 complete before TMEM is freed (bounded waits;
    // phases complete in order, so the last commit's phase covers the rest).
    if (tid == 0) {
      if (qk_commits > 0) mbar_wait(qk_bar, (qk_commits - 1) & 1, a.err);
      if (pv_commits > 0) mbar_wait(pv_bar, (pv_commits - 1) & 1, a.err);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
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

template <typename T, int G>
cudaError_t launch_typed(const DecodeArgs& a0, const CUtensorMap& tk, const CUtensorMap& tv,
                         const CUtensorMap& tq, cudaStream_t stream, int* launches) {
  using L = Layout<kStagesTc>;
  auto* kern = decode_tc_kernel<T, G, kStagesTc>;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int sms = sm_count();
  for (int s0 = 0; s0 < a0.num_seqs; s0 += kMaxSeqs) {
    DecodeArgs a = a0;
    a.num_seqs = a0.num_seqs - s0 < kMaxSeqs ? a0.num_seqs - s0 : kMaxSeqs;
    a.seq_offset = s0;
    a.out = a0.out + (size_t)s0 * a0.num_q_heads * kD;
    a.block_tables = a0.block_tables + (size_t)s0 * a0.max_blocks_per_seq;
    a.context_lens = a0.context_lens + s0;
    if (a0.ws_acc) {
      a.ws_acc = a0.ws_acc + (size_t)s0 * a0.num_q_heads * a0.num_parts * kD;
      a.ws_ml = a0.ws_ml + (size_t)s0 * a0.num_q_heads * a0.num_parts * 2;
    }
    a.epoch = a0.epoch + (unsigned long long)(s0 / kMaxSeqs);
    const int items0 = a.num_seqs * a.num_kv_heads;
    const int grid = items0 < sms ? items0 : sms;
    cudaError_t e = launch_pdl(kern, dim3(grid), dim3(kThreads), L::kAlloc, stream, a, tk, tv, tq);
    if (e != cudaSuccess) return e;
    ++*launches;
  }
  return cudaSuccess;
}

template <typename T>
cudaError_t launch_group(const DecodeArgs& a, int G, const CUtensorMap& tk, const CUtensorMap& tv,
                         const CUtensorMap& tq, cudaStream_t st, int* n) {
  switch (G) {
    case 1: return launch_typed<T, 1>(a, tk, tv, tq, st, n);
    case 2: return launch_typed<T, 2>(a, tk, tv, tq, st, n);
    case 4: return launch_typed<T, 4>(a, tk, tv, tq, st, n);
    case 8: return launch_typed<T, 8>(a, tk, tv, tq, st, n);
    case 16: return launch_typed<T, 16>(a, tk, tv, tq, st, n);
  }
  return cudaErrorInvalidValue;
}

}  // namespace tc

cudaError_t launch_decode_tc(const DecodeArgs& a, int dtype, int group, const CUtensorMap& tk,
                             const CUtensorMap& tv, const CUtensorMap& tq, cudaStream_t stream,
                             int* launches) {
  if (a.num_seqs <= 0) return cudaSuccess;
  if (dtype == 0) return tc::launch_group<__half>(a, group, tk, tv, tq, stream, launches);
  return tc::launch_group<__nv_bfloat16>(a, group, tk, tv, tq, stream, launches);
}

int decode_tc_tile_tokens() { return tc::kTile; }

}  // namespace pa
