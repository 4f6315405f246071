// pa_plan.cu -- which sequences of a decode batch share a prefix of physical
// blocks, and how much of it.
//
// Sequences forked from one parent (beam candidates) or admitted with a common
// prompt hold the same physical blocks at the start of their block tables
// (zingnex.cn, "vLLM与PagedAttention深度剖析", section 3.2 item 3: blocks are
// shared by reference count and copied only on write; jsqmd.com,
// "vLLM-v0.11.0性能实测", section 4.2: requests with the same prefix share
// pages).  The shared-prefix decode reads those blocks once per group of
// sequences instead of once per sequence.  This kernel finds the groups on the
// device, from the block tables alone:
//
//   - a run is a maximal range of consecutive sequences, inside one launch
//     chunk, with context > 0 and the same first table entry;
//   - a run is cut into groups of at most `max_members` consecutive
//     sequences (members x g query rows fit one tile of the shared kernel);
//   - the group shares its first T tokens, where T = block_size x (number of
//     leading table entries equal in every member, counted only below every
//     member's own block count), capped at the shortest member context, and
//     rounded down to 16 tokens (one TMA box);
//   - a group whose T is under `min_shared` tokens is not worth a second
//     pass: its members stay alone.
//
// plan[s] = {rank of s in its group (0 = the leader), members, T, shared
// partitions ceil(T / partition_tokens)}; a sequence alone gets {0, 1, 0, 0}.
//
// The decode then reads each group (of two or more) through one row list: the
// T shared tokens and, when the members' own tokens [T, ctx) are few (in all
// at most max(T, 64 x members) rows once each member's run is rounded up to
// 16 rows, as for beam candidates), those runs in member order after them, so
// that a 16-row box never mixes members.  Own tokens not folded into a list
// (a long private continuation of a shared prompt, and every sequence in no
// group, whose T is 0) are read by per-sequence items of their own.
// plan2[s] = {offset of s's own rows in its group's list, or -1 when they are
// read on their own; number of partials s gets (the partitions of the list
// holding its rows, then those of its own tokens; 1: its result is written
// directly, 0: empty context); rows s's own tokens are read in on their own
// (ctx - T), or -1 when they are not (in a list, or none); rows in the list
// of the group s leads, or -1 when s leads no group of two or more}.  The last
// two are what the decode's item numbering counts per sequence: one load each.
#include <cuda_runtime.h>

#include <climits>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

constexpr int kPlanThreads = 128;

// One CTA per sequence.  The tables and lengths are inputs no kernel of this
// library writes (except the query expansion of pa_decode_multi, after which
// inputs_written_before is set): the search runs before waiting for the
// kernel before this one, overlapping it, and only the plan's writes wait
// (the decode and merge of an earlier call may still be reading the plan
// until then).  The search takes two rounds of independent loads: every
// sequence's context and first table entry in the chunk (the runs are found
// in shared memory), then the table entries the group's members compare.
constexpr int kPlanMaxChunk = 256;  // sequences of a chunk (groups never cross one)
constexpr int kPlanPer = kPlanMaxChunk / kPlanThreads;

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const PlanArgs p) {
  if (p.inputs_written_before) pdl_wait();
  pdl_launch_dependents();
  __shared__ int sh_ctx[kPlanMaxChunk], sh_first[kPlanMaxChunk];
  __shared__ int sh_lo, sh_hi, sh_common;
  __shared__ int sh_rows[32];  // own rows of each member, rounded up to 16
  const int s = blockIdx.x, tid = threadIdx.x;
  const int c0 = (s / p.chunk) * p.chunk;
  const int c1 = min(p.num_seqs, c0 + p.chunk);
  const int i_s = s - c0;  // s within the chunk
  // ---- every sequence's context and first entry (-1: it cannot share: an
  // empty context, or an entry outside the pool, which the decode reports)
  {
    int c[kPlanPer], b[kPlanPer];
#pragma unroll
    for (int k = 0; k < kPlanPer; ++k) {
      const int q = min(c0 + tid + k * kPlanThreads, c1 - 1);
      c[k] = __ldg(p.context_lens + q);
      // (a batch with no table entries has only empty contexts: nothing to read)
      b[k] = p.max_blocks_per_seq > 0 ? __ldg(p.block_tables + (size_t)q * p.max_blocks_per_seq) : -1;
    }
#pragma unroll
    for (int k = 0; k < kPlanPer; ++k) {
      const int i = tid + k * kPlanThreads;
      if (c0 + i < c1) {
        const int cc = max(0, min(c[k], p.max_context_len));
        sh_ctx[i] = cc;
        sh_first[i] = (cc > 0 && b[k] >= 0 && b[k] < p.num_blocks) ? b[k] : -1;
      }
    }
    if (tid == 0) sh_lo = -1, sh_hi = c1 - c0, sh_common = INT_MAX;
  }
  __syncthreads();
  const int first = sh_first[i_s];
  int leader = s, n = 1, shared = 0;
  if (first >= 0) {
    // ---- the run: the nearest breaks below and above s
#pragma unroll
    for (int k = 0; k < kPlanPer; ++k) {
      const int i = tid + k * kPlanThreads;
      if (c0 + i < c1 && sh_first[i] != first) {
        if (i < i_s) atomicMax(&sh_lo, i);
        if (i > i_s) atomicMin(&sh_hi, i);
      }
    }
    __syncthreads();
    const int a = sh_lo + 1, b = sh_hi;  // the run [a, b) within the chunk
    const int lead = a + ((i_s - a) / p.max_members) * p.max_members;
    const int nm = min(p.max_members, b - lead);
    if (nm >= 2) {
      // ---- shortest member context and block count
      int min_ctx = INT_MAX;
      for (int m = 0; m < nm; ++m) min_ctx = min(min_ctx, sh_ctx[lead + m]);
      const int lim = (min_ctx + p.block_size - 1) / p.block_size;
      // ---- leading table entries every member has in common with the
      // leader: the first entry below lim where some member differs
      const int32_t* lead_row = p.block_tables + (size_t)(c0 + lead) * p.max_blocks_per_seq;
      const int pairs = (nm - 1) * lim;
      for (int x0 = 0; x0 < pairs; x0 += 4 * kPlanThreads) {
        int mine[4], theirs[4], jj[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int x = min(x0 + u * kPlanThreads + tid, pairs - 1);
          const int m = 1 + x / lim, j = x % lim;
          jj[u] = x0 + u * kPlanThreads + tid < pairs ? j : INT_MAX;
          mine[u] = __ldg(p.block_tables + (size_t)(c0 + lead + m) * p.max_blocks_per_seq + j);
          theirs[u] = __ldg(lead_row + j);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (jj[u] != INT_MAX && mine[u] != theirs[u]) atomicMin(&sh_common, jj[u]);
      }
      __syncthreads();
      const int common = min(sh_common, lim);
      const long long t = min((long long)common * p.block_size, (long long)min_ctx);
      const int sh = (int)(t & ~15LL);
      if (sh >= p.min_shared) leader = c0 + lead, n = nm, shared = sh;
    }
  }
  // ---- this sequence's place in its group's row list
  if (tid < n) {
    const int own = sh_ctx[leader - c0 + tid] - shared;
    sh_rows[tid] = (own + 15) / 16 * 16;
  }
  __syncthreads();
  if (tid == 0) {
    const int PT = p.partition_tokens;
    int off = shared, my_off = 0;
    for (int m = 0; m < n; ++m) {
      if (leader + m == s) my_off = off;
      off += sh_rows[m];
    }
    const bool fold = n >= 2 && off - shared <= max(shared, 64 * n);
    const int rows = fold ? off : shared;
    const int p_shared = (shared + PT - 1) / PT;
    const int own = sh_ctx[i_s] - shared;
    int n_slots = p_shared;
    if (own > 0) {
      if (fold) {
        const int first_p = max(my_off / PT, p_shared), last_p = (my_off + own - 1) / PT;
        if (last_p >= first_p) n_slots += last_p - first_p + 1;
      } else {
        n_slots += (own + p.own_partition_tokens - 1) / p.own_partition_tokens;
      }
    }
    pdl_wait();
    p.plan[s] = n >= 2 ? make_int4(s - leader, n, shared, p_shared) : make_int4(0, 1, 0, 0);
    const int own_rows = !fold && (n == 1 || own > 0) ? own : -1;
    p.plan2[s] = make_int4(fold ? my_off : -1, n_slots, own_rows, n >= 2 && s == leader ? rows : -1);
  }
}

}  // namespace

cudaError_t launch_plan(const PlanArgs& p, cudaStream_t stream, int* launches) {
  if (p.num_seqs <= 0) return cudaSuccess;
  if (p.chunk <= 0 || p.chunk > kPlanMaxChunk || p.max_members > 32) return cudaErrorInvalidValue;
  cudaError_t e = launch_pdl(plan_kernel, dim3(p.num_seqs), dim3(kPlanThreads), 0, stream, p);
  if (e == cudaSuccess) ++*launches;
  return e;
}

}  // namespace pa

// ---------------------------------------------------------------------------
// Several query tokens per sequence.  Query token t of sequence s attends to
// tokens 0 .. ctx_s - Tq + t, so it is a one-token decode of a "virtual"
// sequence v = s * Tq + t with the same block table and context
// ctx_s - Tq + t + 1: the Tq virtual sequences of s are consecutive and start
// with the same blocks, so the shared-prefix plan groups them and their
// common tokens are read once.  This kernel writes the virtual tables and
// contexts (one CTA per virtual sequence; only the entries a context uses).

namespace pa {
namespace {

__global__ void __launch_bounds__(128)
expand_queries_kernel(const int32_t* __restrict__ tables, const int32_t* __restrict__ ctx,
                      int num_query_tokens, int max_blocks_per_seq, int block_size,
                      int max_context_len, int32_t* __restrict__ tables_out,
                      int32_t* __restrict__ ctx_out, unsigned int* err) {
  pdl_wait();
  pdl_launch_dependents();
  const int v = blockIdx.x;
  const int s = v / num_query_tokens, t = v % num_query_tokens;
  int c = __ldg(ctx + s);
  if (c < 0 || c > max_context_len) {
    if (t == 0 && threadIdx.x == 0) report(err, kErrContextLen);
    c = max(0, min(c, max_context_len));
  }
  const int cv = max(0, c - num_query_tokens + t + 1);
  const int nb = (cv + block_size - 1) / block_size;
  const int32_t* src = tables + (size_t)s * max_blocks_per_seq;
  int32_t* dst = tables_out + (size_t)v * max_blocks_per_seq;
  for (int j = threadIdx.x; j < nb; j += blockDim.x) dst[j] = __ldg(src + j);
  if (threadIdx.x == 0) ctx_out[v] = cv;
}

}  // namespace

cudaError_t launch_expand_queries(const int32_t* tables, const int32_t* ctx, int num_seqs,
                                  int num_query_tokens, int max_blocks_per_seq, int block_size,
                                  int max_context_len, int32_t* tables_out, int32_t* ctx_out,
                                  unsigned int* err, cudaStream_t stream, int* launches) {
  const long long n = (long long)num_seqs * num_query_tokens;
  if (n <= 0) return cudaSuccess;
  cudaError_t e = launch_pdl(expand_queries_kernel, dim3((unsigned)n), dim3(128), 0, stream, tables,
                             ctx, num_query_tokens, max_blocks_per_seq, block_size,
                             max_context_len, tables_out, ctx_out, err);
  if (e == cudaSuccess) ++*launches;
  return e;
}

}  // namespace pa
