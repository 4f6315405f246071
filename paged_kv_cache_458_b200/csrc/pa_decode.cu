// pa_decode.cu -- single-token decode attention over a paged KV cache (sm_100a).
//
// Method: PagedAttention keeps K and V in fixed-size physical blocks reached
// through a per-sequence block table (zingnex.cn, "vLLM与PagedAttention深度剖析",
// section 3.2; 5688vip.com vLLM notes, section 2.2).  Decode reads every
// cached K/V row of the sequence once per generated token and does little
// arithmetic per byte, so this kernel is organised around the HBM read
// (5688vip.com section 2.1: decode is bandwidth-bound).
//
// Work decomposition
//   One CTA per (partition, sequence, kv head).  A partition is a run of
//   partition_tokens tokens (512 by default); the CTA holds the whole grouped
//   query (g = Hq / Hkv heads) in registers.  Inside the CTA each warp owns
//   every NW-th chunk of 16 tokens and runs its own TMA pipeline of NST
//   stages: lane 0 issues two tiled TMA loads per chunk (a 16-row box of K
//   and of V of one kv head inside one physical block) on an mbarrier, so the
//   gather through the block table costs one table read per chunk and no
//   address arithmetic per byte.  Warps never wait on each other until the
//   end, where their (max, sum, output) states are merged in shared memory.
//
// Arithmetic per chunk (fp32 throughout)
//   QK^T: lane l holds D/32 consecutive dims of every query head; per token it
//   multiplies its slice of the K row, and one transposed butterfly
//   (reduce-scatter over 32 values) leaves each lane with one complete logit.
//   Online softmax (log2 domain, scale * log2 e folded into q): running max m
//   and sum l per head; the output accumulators are rescaled by 2^(m_old-m_new).
//   PV: p is staged through shared memory and every lane accumulates its dims
//   of all heads.  Tokens past the context are masked to p = 0 and their V rows
//   are never touched, so stale slots may hold NaN.
//
// Split-K: a sequence with more than one partition stores, per (head,
//   partition), m, l and the unnormalised output row in fp32; the merge
//   kernel combines them with M = max m_p, out = sum 2^(m_p-M) acc_p /
//   sum 2^(m_p-M) l_p.  A sequence with a single partition is written directly.
#include <cuda.h>
#include <cuda_runtime.h>

#include <type_traits>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

constexpr int kChunk = 16;  // tokens per TMA box (a block is a multiple of this)

template <int D, int G, int NW, int NST, int EB = 2>  // EB: bytes per cached element
struct DecodeSmem {
  static constexpr int kRowBytes = D * EB;
  static constexpr int kStageBytes = 2 * kChunk * kRowBytes;  // K box then V box
  static constexpr int kStagesBytes = NW * NST * kStageBytes;
  static constexpr int kPBytes = NW * (kChunk * G + G) * 4;   // p[16][G] + alpha[G] per warp
  static constexpr int kBarBytes = NW * NST * 8;
  static constexpr int kMergeBytes = NW * (G * D + 2 * G) * 4;
  // the warps' final merge reuses the stage buffers (grown if they are smaller)
  static constexpr int kStageArea = kMergeBytes > kStagesBytes ? kMergeBytes : kStagesBytes;
  static constexpr int kTotal = kStageArea + kPBytes + kBarBytes;
};

__device__ __forceinline__ float warp_max_xor(float v, int lo, int hi) {
  for (int o = lo; o <= hi; o <<= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum_xor(float v, int lo, int hi) {
  for (int o = lo; o <= hi; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// One halving step of the transposed reduction: lanes with bit O set keep the
// upper half of v[0..N), the others the lower half; each adds the partner's
// copy of the half it keeps.
template <int O, int N>
__device__ __forceinline__ void rs_step(float (&v)[32], int lane) {
  const bool upper = (lane & O) != 0;
#pragma unroll
  for (int i = 0; i < N / 2; ++i) {
    const float send = upper ? v[i] : v[i + N / 2];
    const float keep = upper ? v[i + N / 2] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, O);
  }
}

// Sum N in {16, 32} per-lane partial values over the warp.
// N == 32: lane l returns the total of value l.
// N == 16: lane l returns the total of value l >> 1.
template <int N>
__device__ __forceinline__ float reduce_scatter(float (&v)[32], int lane) {
  if constexpr (N == 32) {
    rs_step<16, 32>(v, lane);
    rs_step<8, 16>(v, lane);
    rs_step<4, 8>(v, lane);
    rs_step<2, 4>(v, lane);
    rs_step<1, 2>(v, lane);
    return v[0];
  } else {
    rs_step<16, 16>(v, lane);
    rs_step<8, 8>(v, lane);
    rs_step<4, 4>(v, lane);
    rs_step<2, 2>(v, lane);
    return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
  }
}

// Load this lane's D/32 elements of a row and widen them.
template <typename T, int D>
__device__ __forceinline__ void load_row_slice(const unsigned char* row, int lane, float* out) {
  if constexpr (D == 128) {
    const uint2 u = *reinterpret_cast<const uint2*>(row + lane * 8);
    const float2 a = Elem<T>::to_f2(u.x), b = Elem<T>::to_f2(u.y);
    out[0] = a.x; out[1] = a.y; out[2] = b.x; out[3] = b.y;
  } else {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(row + lane * 4);
    const float2 a = Elem<T>::to_f2(u);
    out[0] = a.x; out[1] = a.y;
  }
}

// This lane's D/32 elements of a cached row, widened: 16-bit elements as
// load_row_slice, E4M3 codes exactly (the head's scale is applied elsewhere).
template <typename KV, typename T, int D>
__device__ __forceinline__ void load_kv_slice(const unsigned char* row, int lane, float* out) {
  if constexpr (std::is_same<KV, Fp8E4M3>::value) {
    if constexpr (D == 128) {
      const uint32_t u = *reinterpret_cast<const uint32_t*>(row + lane * 4);
      const float2 a = e4m3x2_to_f2((uint16_t)(u & 0xffffu)), b = e4m3x2_to_f2((uint16_t)(u >> 16));
      out[0] = a.x; out[1] = a.y; out[2] = b.x; out[3] = b.y;
    } else {
      const float2 a = e4m3x2_to_f2(*reinterpret_cast<const uint16_t*>(row + lane * 2));
      out[0] = a.x; out[1] = a.y;
    }
  } else {
    load_row_slice<T, D>(row, lane, out);
  }
}

// KV: T (fp16/bf16 cache) or Fp8E4M3 (one-byte codes, per-kv-head scales:
// the K scale is folded into the query, the V scale into the output).
template <typename T, typename KV, int D, int G, int NW, int NST>
__global__ void __launch_bounds__(NW * 32)
decode_partition_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v) {
  constexpr bool kFp8 = std::is_same<KV, Fp8E4M3>::value;
  using L = DecodeSmem<D, G, NW, NST, kFp8 ? 1 : 2>;
  constexpr int VEC = D / 32;
  constexpr int TPP = (G == 1) ? 16 : 32 / G;  // tokens per reduce-scatter pass
  constexpr int NPASS = kChunk / TPP;          // passes per chunk
  constexpr int LPH = (G == 1) ? 32 : 32 / G;  // lanes holding one head's logits
  extern __shared__ __align__(1024) unsigned char smem[];

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  pdl_wait();  // the append before this decode must have landed
  pdl_launch_dependents();

  int bid = blockIdx.x;
  const int kvh = bid % a.num_kv_heads;
  bid /= a.num_kv_heads;
  const int s = bid % a.num_seqs;
  const int part = bid / a.num_seqs;

  int ctx = __ldg(a.context_lens + s);
  const int ctx_cap = a.max_context_len;
  if (ctx < 0 || ctx > ctx_cap) {
    if (part == 0 && kvh == 0 && threadIdx.x == 0) report(a.err, kErrContextLen);
    ctx = max(0, min(ctx, ctx_cap));
  }
  const int q_head0 = kvh * G;
  // With a shared-prefix plan this kernel reads the own tokens [T, ctx) of
  // the sequences whose own tokens are in no group's row list (every
  // sequence in no group, T = 0), as partials after its shared ones.
  int base = 0, slot0 = 0, n_parts_seq = -1;
  if (a.plan) {
    const int4 pl = __ldg(a.plan + s);
    const int4 p2 = __ldg(a.plan2 + s);
    if (!(p2.x < 0 && (pl.y == 1 || ctx > pl.z))) return;
    base = pl.z;
    slot0 = pl.w;
    n_parts_seq = p2.y;
  }
  if (ctx == 0) {
    if (part == 0) {
      uint16_t* o = a.out + ((size_t)s * a.num_q_heads + q_head0) * D;
      for (int i = threadIdx.x; i < G * D; i += NW * 32) o[i] = 0;
    }
    return;
  }
  const int PT = a.own_tokens;
  const int t_begin = base + part * PT;
  if (t_begin >= ctx) return;
  const int t_end = min(ctx, t_begin + PT);
  if (n_parts_seq < 0) n_parts_seq = (ctx + PT - 1) / PT;
  const int n_chunks = (t_end - t_begin + kChunk - 1) / kChunk;
  const int n_mine = warp < n_chunks ? (n_chunks - warp + NW - 1) / NW : 0;

  unsigned char* stages = smem;
  float* p_all = reinterpret_cast<float*>(smem + L::kStageArea);
  float* p_sm = p_all + warp * (kChunk * G + G);  // [16][G]
  float* alpha_sm = p_sm + kChunk * G;             // [G]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kStageArea + L::kPBytes);
  const uint32_t bar0 = smem_addr(bars + warp * NST);
  const uint32_t stage0 = smem_addr(stages + warp * NST * L::kStageBytes);

  if (lane == 0) {
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
#pragma unroll
    for (int st = 0; st < NST; ++st) mbar_init(bar0 + st * 8, 1);
    mbar_init_fence();
  }
  __syncwarp();

  // Lane k resolves the physical row of this warp's k-th chunk through the
  // block table (one read per chunk, all issued up front).
  // With 8-token blocks (half_boxes) the chunk's rows 8..15 have an entry of
  // their own; past the end of the range they re-read rows of the first
  // block instead (masked), so no entry beyond the context is read.
  const int32_t* table = a.block_tables + (size_t)s * a.max_blocks_per_seq;
  auto resolve = [&](int tok) {
    const int blk = __ldg(table + tok / a.block_size);
    if (blk < 0 || blk >= a.num_blocks) {
      report(a.err, kErrBlockId);
      return a.num_blocks * a.block_size;  // outside the map: TMA fills zeros
    }
    return blk * a.block_size + tok % a.block_size;
  };
  int my_row = 0, my_row2 = 0;
  if (lane < n_mine) {
    const int tok = t_begin + (warp + lane * NW) * kChunk;
    my_row = resolve(tok);
    if (a.half_boxes) my_row2 = tok + kChunk / 2 < t_end ? resolve(tok + kChunk / 2) : my_row;
  }

  auto issue = [&](int k) {
    const int row = __shfl_sync(0xffffffffu, my_row, k);
    const int row2 = __shfl_sync(0xffffffffu, my_row2, k);
    if (lane == 0) {
      const int st = k % NST;
      const uint32_t bar = bar0 + st * 8;
      const uint32_t dst = stage0 + st * L::kStageBytes;
      mbar_arrive_expect_tx(bar, L::kStageBytes);
      if (a.half_boxes) {
        constexpr uint32_t kHalfBox = (kChunk / 2) * L::kRowBytes;
        tma_load_3d(dst, &tm_k, bar, 0, kvh, row);
        tma_load_3d(dst + kHalfBox, &tm_k, bar, 0, kvh, row2);
        tma_load_3d(dst + kChunk * L::kRowBytes, &tm_v, bar, 0, kvh, row);
        tma_load_3d(dst + kChunk * L::kRowBytes + kHalfBox, &tm_v, bar, 0, kvh, row2);
      } else {
        tma_load_3d(dst, &tm_k, bar, 0, kvh, row);
        tma_load_3d(dst + kChunk * L::kRowBytes, &tm_v, bar, 0, kvh, row);
      }
    }
  };

  // Query group in registers, pre-scaled into the log2 domain (and by the K
  // scale of an E4M3 cache).
  float qscale = a.scale_log2;
  if constexpr (kFp8) qscale *= __ldg(a.k_scale + kvh);
  float qr[G][VEC];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const unsigned char* qrow = reinterpret_cast<const unsigned char*>(
        a.q + ((size_t)s * a.num_q_heads + q_head0 + h) * D);
    load_row_slice<T, D>(qrow, lane, qr[h]);
#pragma unroll
    for (int v = 0; v < VEC; ++v) qr[h][v] *= qscale;
  }

  float acc[G][VEC];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int v = 0; v < VEC; ++v) acc[h][v] = 0.f;
  // Running max / sum of the head this lane's logits belong to.
  float m_run = -INFINITY, l_run = 0.f;
  const int my_head = (G == 1) ? 0 : lane / LPH;

  const int n_pro = min(NST, n_mine);
  for (int k = 0; k < n_pro; ++k) issue(k);

  bool ok = true;
  int k = 0;
  for (; k < n_mine; ++k) {
    const int st = k % NST;
    if (!mbar_wait(bar0 + st * 8, (k / NST) & 1, a.err)) { ok = false; break; }
    const unsigned char* Ks = stages + (warp * NST + st) * L::kStageBytes;
    const unsigned char* Vs = Ks + kChunk * L::kRowBytes;
    const int tok0 = t_begin + (warp + k * NW) * kChunk;
    const int n_valid = min(kChunk, t_end - tok0);

    // ---- logits: one complete logit per lane per pass
    float x[NPASS];
#pragma unroll
    for (int ps = 0; ps < NPASS; ++ps) {
      float part_v[32];
#pragma unroll
      for (int jj = 0; jj < TPP; ++jj) {
        float kf[VEC];
        load_kv_slice<KV, T, D>(Ks + (ps * TPP + jj) * L::kRowBytes, lane, kf);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float d = 0.f;
#pragma unroll
          for (int v = 0; v < VEC; ++v) d = fmaf(qr[h][v], kf[v], d);
          part_v[h * TPP + jj] = d;
        }
      }
      float r = reduce_scatter<(G == 1) ? 16 : 32>(part_v, lane);
      const int jj = (G == 1) ? (lane >> 1) : (lane % TPP);
      x[ps] = (ps * TPP + jj < n_valid) ? r : -INFINITY;
    }

    // ---- online softmax for this lane's head
    float mx = x[0];
#pragma unroll
    for (int ps = 1; ps < NPASS; ++ps) mx = fmaxf(mx, x[ps]);
    mx = (G == 1) ? warp_max_xor(mx, 2, 16) : warp_max_xor(mx, 1, LPH / 2);
    const float m_new = fmaxf(m_run, mx);
    const float alpha = exp2f(m_run - m_new);
    float ls = 0.f;
#pragma unroll
    for (int ps = 0; ps < NPASS; ++ps) {
      const float p = exp2f(x[ps] - m_new);
      ls += p;
      const int jj = (G == 1) ? (lane >> 1) : (lane % TPP);
      if (G > 1 || (lane & 1) == 0) p_sm[(ps * TPP + jj) * G + my_head] = p;
    }
    ls = (G == 1) ? warp_sum_xor(ls, 2, 16) : warp_sum_xor(ls, 1, LPH / 2);
    l_run = l_run * alpha + ls;
    m_run = m_new;
    if (lane % LPH == 0) alpha_sm[my_head] = alpha;
    __syncwarp();

    // ---- rescale and accumulate P V
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float al = alpha_sm[h];
#pragma unroll
      for (int v = 0; v < VEC; ++v) acc[h][v] *= al;
    }
    for (int j = 0; j < n_valid; ++j) {
      float vf[VEC];
      load_kv_slice<KV, T, D>(Vs + j * L::kRowBytes, lane, vf);
      float pj[G];
#pragma unroll
      for (int h = 0; h < G; ++h) pj[h] = p_sm[j * G + h];
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int v = 0; v < VEC; ++v) acc[h][v] = fmaf(pj[h], vf[v], acc[h][v]);
    }
    __syncwarp();
    // Stage `st` is free again: refill it with chunk k + NST.
    if (k + NST < n_mine) {
      if (lane == 0) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      issue(k + NST);
    }
  }
  if (!ok) {
    // Let every copy this warp still has in flight land before the CTA exits.
    for (int kk = k; kk < min(n_mine, k + NST); ++kk) mbar_wait(bar0 + (kk % NST) * 8, (kk / NST) & 1, a.err);
  }

  // ---- merge the warps' states
  // All stages consumed (or drained): the stage area becomes the merge area.
  const int any_failed = __syncthreads_or(!ok);
  float* mg = reinterpret_cast<float*>(smem);  // [NW][G] m, [NW][G] l, [NW][G][D] acc
  float* mg_m = mg;
  float* mg_l = mg + NW * G;
  float* mg_acc = mg + 2 * NW * G;
  if (lane % LPH == 0) {
    mg_m[warp * G + my_head] = m_run;
    mg_l[warp * G + my_head] = l_run;
  }
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int v = 0; v < VEC; ++v) mg_acc[(warp * G + h) * D + lane * VEC + v] = acc[h][v];
  __syncthreads();

  const bool direct = (n_parts_seq == 1);
  for (int i = threadIdx.x; i < G * D; i += NW * 32) {
    const int h = i / D, d = i % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, mg_m[w * G + h]);
    float num = 0.f, den = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float wt = exp2f(mg_m[w * G + h] - M);  // 0 for a warp without tokens
      num = fmaf(wt, mg_acc[(w * G + h) * D + d], num);
      den = fmaf(wt, mg_l[w * G + h], den);
    }
    if constexpr (kFp8) num *= __ldg(a.v_scale + kvh);
    if (any_failed) num = __int_as_float(0x7fc00000), den = 1.f;
    const size_t qh = (size_t)s * a.num_q_heads + q_head0 + h;
    if (direct) {
      a.out[qh * D + d] = Elem<T>::from_f(num / den);
    } else {
      const size_t slot = qh * a.num_parts + slot0 + part;
      a.ws_acc[slot * D + d] = num;
      if (d == 0) {
        a.ws_ml[2 * slot] = M;
        a.ws_ml[2 * slot + 1] = den;
      }
    }
  }
}

// Merge of the partitions of every (sequence, query head) that has more than
// one.  One warp per (sequence, query head); lane l owns dims [l*VEC, l*VEC+VEC).
// Rows are [num_seqs * query_tokens][Hq]: query t of sequence s attends to
// ctx_s - query_tokens + t + 1 tokens.  With a shared-prefix plan a sequence's
// partial count is in the plan (its partials are slots 0 .. count - 1).
template <typename T, int D>
__global__ void __launch_bounds__(128) decode_merge_kernel(const DecodeArgs a) {
  constexpr int VEC = D / 32;
  pdl_wait();  // every partition's partial is written
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int Tq = a.query_tokens;
  const int n_pairs = a.num_seqs * Tq * a.num_q_heads;
  // a fixed grid strides over the pairs: most pairs of a batch whose
  // sequences were written directly need no merge and cost one load here
  for (int pair = blockIdx.x * 4 + (threadIdx.x >> 5); pair < n_pairs; pair += gridDim.x * 4) {
  const int vs = pair / a.num_q_heads;  // virtual sequence: query vs % Tq of sequence vs / Tq
  int P;
  if (a.plan2) {
    P = __ldg(a.plan2 + vs).y;
  } else {
    int ctx = __ldg(a.context_lens + vs / Tq);
    ctx = max(0, min(ctx, a.max_context_len)) - Tq + 1 + vs % Tq;
    P = ctx > 0 ? (ctx + a.own_tokens - 1) / a.own_tokens : 0;
  }
  if (P <= 1) continue;
  const size_t base = (size_t)pair * a.num_parts;
  // (m, l) of partial p in lane p % 32: the reference M and each partial's
  // weight 2^(m_p - M) come from warp reductions, not a loop of round trips
  float M = -INFINITY;
  for (int p0 = 0; p0 < P; p0 += 32) {
    float m = p0 + lane < P ? a.ws_ml[2 * (base + p0 + lane)] : -INFINITY;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    M = fmaxf(M, m);
  }
  float num[VEC];
#pragma unroll
  for (int v = 0; v < VEC; ++v) num[v] = 0.f;
  float den = 0.f;
  for (int p0 = 0; p0 < P; p0 += 32) {
    float wt = 0.f, lw = 0.f;
    if (p0 + lane < P) {
      wt = exp2f(a.ws_ml[2 * (base + p0 + lane)] - M);
      lw = wt * a.ws_ml[2 * (base + p0 + lane) + 1];
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) lw += __shfl_xor_sync(0xffffffffu, lw, o);
    den += lw;
    // partial rows four at a time: their loads are in flight together
    const int n = min(32, P - p0);
    for (int i = 0; i < n; i += 4) {
      float r[4][VEC];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int p = min(i + u, n - 1);  // past the end: re-read the last row, weight 0
        const float* row = a.ws_acc + (base + p0 + p) * D + lane * VEC;
        if constexpr (VEC == 4) {
          const float4 x = *reinterpret_cast<const float4*>(row);
          r[u][0] = x.x; r[u][1] = x.y; r[u][2] = x.z; r[u][3] = x.w;
        } else {
          const float2 x = *reinterpret_cast<const float2*>(row);
          r[u][0] = x.x; r[u][1] = x.y;
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float w = __shfl_sync(0xffffffffu, wt, (i + u) & 31);
        const float wu = i + u < n ? w : 0.f;
#pragma unroll
        for (int v = 0; v < VEC; ++v) num[v] = fmaf(wu, r[u][v], num[v]);
      }
    }
  }
  const float inv = 1.f / den;
  uint16_t* o = a.out + (size_t)pair * D + lane * VEC;
#pragma unroll
  for (int v = 0; v < VEC; ++v) o[v] = Elem<T>::from_f(num[v] * inv);
  }
}

// Grid of the merge kernel: one warp per pair up to 8 CTAs of 4 warps per SM.
inline unsigned merge_grid(int pairs) {
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
      sms = 148;
  }
  // one warp per pair: a merge is a few dependent round trips, which a warp
  // striding over several pairs would pay one after another
  (void)sms;
  return (unsigned)((pairs + 3) / 4);
}

// ---------------------------------------------------------------------------
// host side

namespace {

// Warps per CTA and TMA stages per warp (build-time choices; 4 x 2 keeps
// three CTAs resident per SM, which measured fastest on every workload).
#ifndef PA_DECODE_WARPS
#define PA_DECODE_WARPS 4
#endif
#ifndef PA_DECODE_STAGES
#define PA_DECODE_STAGES 2
#endif
constexpr int kWarps = PA_DECODE_WARPS;
constexpr int kStages = PA_DECODE_STAGES;

template <typename T, typename KV, int D, int G>
cudaError_t launch_typed(const DecodeArgs& a, const CUtensorMap& tk, const CUtensorMap& tv,
                         int grid, cudaStream_t stream, int* launches) {
  using L = DecodeSmem<D, G, kWarps, kStages, std::is_same<KV, Fp8E4M3>::value ? 1 : 2>;
  auto* kern = decode_partition_kernel<T, KV, D, G, kWarps, kStages>;
  static bool configured = false;  // per instantiation; idempotent if raced
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kTotal);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  cudaError_t e = launch_pdl(kern, dim3(grid), dim3(kWarps * 32), L::kTotal, stream, a, tk, tv);
  if (e != cudaSuccess) return e;
  ++*launches;
  if (a.num_parts <= 1 || a.skip_merge) return cudaSuccess;
  const int pairs = a.num_seqs * a.query_tokens * a.num_q_heads;
  e = launch_pdl(decode_merge_kernel<T, D>, dim3(merge_grid(pairs)), dim3(128), 0, stream, a);
  if (e == cudaSuccess) ++*launches;
  return e;
}

template <typename T, typename KV, int D>
cudaError_t launch_group(const DecodeArgs& a, int G, const CUtensorMap& tk, const CUtensorMap& tv,
                         int grid, cudaStream_t st, int* n) {
  switch (G) {
    case 1: return launch_typed<T, KV, D, 1>(a, tk, tv, grid, st, n);
    case 2: return launch_typed<T, KV, D, 2>(a, tk, tv, grid, st, n);
    case 4: return launch_typed<T, KV, D, 4>(a, tk, tv, grid, st, n);
    case 8: return launch_typed<T, KV, D, 8>(a, tk, tv, grid, st, n);
    case 16: return launch_typed<T, KV, D, 16>(a, tk, tv, grid, st, n);
  }
  return cudaErrorInvalidValue;
}

template <typename T, typename KV>
cudaError_t launch_dims(const DecodeArgs& a, int head_dim, int group, const CUtensorMap& tk,
                        const CUtensorMap& tv, int grid, cudaStream_t stream, int* launches) {
  if (head_dim == 128) return launch_group<T, KV, 128>(a, group, tk, tv, grid, stream, launches);
  return launch_group<T, KV, 64>(a, group, tk, tv, grid, stream, launches);
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a0, int dtype, int head_dim, int group,
                          const CUtensorMap& tk, const CUtensorMap& tv, cudaStream_t stream,
                          int* launches, bool fp8_cache, bool with_merge) {
  const long long grid = (long long)a0.grid_parts * a0.num_seqs * a0.num_kv_heads;
  if (grid <= 0) return cudaSuccess;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const int g = (int)grid;
  DecodeArgs a = a0;
  if (!with_merge) a.skip_merge = 1;
  if (dtype == 0)
    return fp8_cache ? launch_dims<__half, Fp8E4M3>(a, head_dim, group, tk, tv, g, stream, launches)
                     : launch_dims<__half, __half>(a, head_dim, group, tk, tv, g, stream, launches);
  return fp8_cache
             ? launch_dims<__nv_bfloat16, Fp8E4M3>(a, head_dim, group, tk, tv, g, stream, launches)
             : launch_dims<__nv_bfloat16, __nv_bfloat16>(a, head_dim, group, tk, tv, g, stream,
                                                         launches);
}

cudaError_t launch_decode_merge(const DecodeArgs& a, int dtype, int head_dim, cudaStream_t stream,
                                int* launches) {
  if (a.num_parts <= 1 || a.num_seqs <= 0) return cudaSuccess;
  const int pairs = a.num_seqs * a.query_tokens * a.num_q_heads;
  const dim3 grid(merge_grid(pairs)), block(128);
  cudaError_t e;
  if (dtype == 0) {
    e = head_dim == 128 ? launch_pdl(decode_merge_kernel<__half, 128>, grid, block, 0, stream, a)
                        : launch_pdl(decode_merge_kernel<__half, 64>, grid, block, 0, stream, a);
  } else {
    e = head_dim == 128
            ? launch_pdl(decode_merge_kernel<__nv_bfloat16, 128>, grid, block, 0, stream, a)
            : launch_pdl(decode_merge_kernel<__nv_bfloat16, 64>, grid, block, 0, stream, a);
  }
  if (e == cudaSuccess) ++*launches;
  return e;
}

int decode_chunk_tokens() { return kChunk; }
int decode_max_partition_tokens() { return kChunk * kWarps * 32; }

}  // namespace pa
