// pa_internal.h -- declarations shared by the libpa host code and its kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace pa {

// Arguments of the decode kernels (device pointers, host-validated sizes).
struct DecodeArgs {
  const uint16_t* q;             // [S][Hq][D]
  const int32_t* block_tables;   // [S][MBS]
  const int32_t* context_lens;   // [S]
  uint16_t* out;                 // [S][Hq][D]
  float* ws_acc;                 // [S][Hq][num_parts][D] (split-K only)
  float* ws_ml;                  // [S][Hq][num_parts][2] (split-K only)
  float scale_log2;              // scale * log2(e)
  int num_seqs, num_q_heads, num_kv_heads;
  int block_size, num_blocks, max_blocks_per_seq;
  int partition_tokens, num_parts;
  int max_context_len;           // host bound on context_lens, <= max_blocks_per_seq * block_size
  unsigned int* err;             // device error word
  unsigned long long* work_counter;  // first 8 bytes of the workspace (tensor-core path)
  unsigned long long epoch;      // tag of this call's launches (< 2^40, never 0)
  int seq_offset;                // first sequence of this launch in the whole batch
  // Shared-prefix decode (nullptr: off): per sequence {rank in its group,
  // members, shared tokens T, shared partitions}.  A sequence's own items
  // then cover [T, ctx), as partitions numbered from its shared partitions.
  const float* k_scale;          // [Hkv] with an E4M3 cache (stored value = code * scale)
  const float* v_scale;          // [Hkv]
  const int4* plan;
  // With a plan, per sequence {row offset of its own tokens in its group's
  // row list, number of partials it gets (1: written directly), partitions
  // of the group's row list, rows in that list}.
  const int4* plan2;
  int own_tokens;                // partition size of the CUDA-core kernel (with a plan: of the
                                 // own tokens it reads)
  int grid_parts;                // partitions per (sequence, kv head) of the CUDA-core grid
  int query_tokens;              // query tokens per sequence (pa_decode_multi on the
                                 // tensor-core kernels; 1 otherwise): q, out and the
                                 // split-K rows are [num_seqs * query_tokens][Hq]
  int group;                     // g = Hq / Hkv
  int own_pass;                  // with a plan: 1 = items over the own tokens [T, ctx) of the
                                 // sequences whose own tokens are in no row list
  int own_in_lists;              // with a plan and own_pass 0: the row-list launch also takes
                                 // those own-token items (after the lists' items)
  int skip_merge;                // host side: 1 = the CUDA-core launch leaves the merge to its caller
  int half_boxes;                // block_size is a multiple of 8 but not of 16: each
                                 // 16-token TMA box is loaded as two 8-token boxes, which
                                 // may come from two blocks
};

// Sequences per launch of the shared-prefix kernel; groups never cross a
// multiple of it.
constexpr int kSharedPrefixSeqsPerLaunch = 256;

// Arguments of the plan kernel (pa_plan.cu).
struct PlanArgs {
  const int32_t* block_tables;   // [S][MBS]
  const int32_t* context_lens;   // [S]
  int4* plan;                    // [S] out
  int4* plan2;                   // [S] out
  int num_seqs, max_blocks_per_seq, block_size, num_blocks, max_context_len;
  int partition_tokens;
  int own_partition_tokens;      // partition of the own tokens read on their own
  int max_members;               // members per group (32 / g)
  int min_shared;                // fewer shared tokens than this: no group
  int chunk;                     // groups stay inside [k * chunk, (k + 1) * chunk)
  int inputs_written_before;     // 1: the kernel just before wrote the tables or lengths (the
                                 // plan then reads them only after waiting for it)
};
cudaError_t launch_plan(const PlanArgs& p, cudaStream_t stream, int* launches);
// Virtual one-token sequences for Tq query tokens per sequence (pa_plan.cu).
cudaError_t launch_expand_queries(const int32_t* tables, const int32_t* ctx, int num_seqs,
                                  int num_query_tokens, int max_blocks_per_seq, int block_size,
                                  int max_context_len, int32_t* tables_out, int32_t* ctx_out,
                                  unsigned int* err, cudaStream_t stream, int* launches);


// Launch the partition kernel (+ the merge kernel when num_parts > 1 and
// with_merge).  `launches` is incremented once per kernel launched.
// fp8_cache: K/V hold E4M3 codes (a.k_scale / a.v_scale set).
cudaError_t launch_decode(const DecodeArgs& a, int dtype, int head_dim, int group,
                          const CUtensorMap& tm_k, const CUtensorMap& tm_v, cudaStream_t stream,
                          int* launches, bool fp8_cache = false, bool with_merge = true);
int decode_chunk_tokens();
int decode_max_partition_tokens();
// The split-K merge alone (after a partition kernel that wrote partials).
cudaError_t launch_decode_merge(const DecodeArgs& a, int dtype, int head_dim, cudaStream_t stream,
                                int* launches);

// The tensor-core path (head_dim 128): pool maps are 128B-swizzled, boxes of
// 64 elements x 16 (or 8) token rows of one kv head; with `pair`, items cover
// two kv heads and the pool maps are [Hkv][rows][128] by strides with boxes
// of 64 x 16 rows x 2 heads.  tm_q views q as [rows][Hq][128] (rows =
// num_seqs * query_tokens) with 128B-swizzled boxes of 64 elements x
// heads_per_box x rows_per_box; see tc_query_box().
// Without a plan, items are (sequence, kv head or pair, partition) with the
// sequence's query_tokens x heads query rows as columns; with a plan
// (a.plan, a.plan2), items are (group leader, kv head, partition of the
// group's row list) with members x g columns.
// fp8_cache: the pools hold E4M3 codes (8-bit maps with boxes of 128
// one-byte elements; a.k_scale / a.v_scale set).
cudaError_t launch_decode_tc(const DecodeArgs& a, int dtype, const CUtensorMap& tm_k,
                             const CUtensorMap& tm_v, const CUtensorMap& tm_q, cudaStream_t stream,
                             int* launches, bool pair, bool fp8_cache);
int decode_tc_tile_tokens();
// Query columns one tensor-core item holds at most.
constexpr int kTcMaxColumns = 32;
// The q box of the tensor-core kernel for a launch: {heads, rows} per box.
struct TcQueryBox {
  int heads, rows;
};
TcQueryBox tc_query_box(int group, int query_tokens, bool pair, bool grouped);

cudaError_t launch_cache_append(const void* k, const void* v, const int32_t* slot_mapping,
                                int num_tokens, void* k_cache, void* v_cache, long long num_slots,
                                int row_bytes, unsigned int* err, cudaStream_t stream,
                                int* launches);
// Append into an E4M3 cache: k, v rows of Hkv * D fp16/bf16 elements (dtype
// 0 / 1) are divided by their head's scale and rounded to E4M3 (nearest,
// ties to even, saturating at 448).
cudaError_t launch_cache_append_fp8(const void* k, const void* v, const int32_t* slot_mapping,
                                    int num_tokens, void* k_cache, void* v_cache,
                                    long long num_slots, int dtype, int num_kv_heads, int head_dim,
                                    const float* k_scale, const float* v_scale, unsigned int* err,
                                    cudaStream_t stream, int* launches);
// Copy-on-write within one pool (src == dst pools) and swap between two
// pools, either of which may be host memory the device can address.
cudaError_t launch_copy_blocks(const int32_t* pairs, int num_pairs, const void* src_k,
                               const void* src_v, int src_blocks, void* dst_k, void* dst_v,
                               int dst_blocks, long long block_bytes, unsigned int* err,
                               cudaStream_t stream, int* launches);

}  // namespace pa
