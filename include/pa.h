/*
 * pa.h -- C ABI of libpa.so: paged decode attention on B200 (sm_100a).
 *
 * The method (PagedAttention) keeps each sequence's key/value cache in
 * fixed-size physical blocks of `block_size` tokens inside one pool tensor,
 * and reaches them through a per-sequence block table that maps logical block
 * j / block_size to a physical block (zingnex.cn, "vLLM与PagedAttention深度剖析",
 * section 3.2: the block tensor, items 1-4; 5688vip.com vLLM notes, section
 * 2.2: "logical block 0 -> physical block 7").  Blocks may be shared by
 * several sequences (common prefixes, beam candidates) and are copied before
 * a shared block is written (section 3.2 item 3).  Decode is bandwidth-bound
 * (5688vip.com section 2.1), so the kernels are built around the K/V read.
 *
 * Conventions for every call:
 *  - Every pointer named "device" is a CUDA device pointer on the current
 *    device, 16-byte aligned, owned by the caller; the library allocates
 *    nothing per call and keeps no pointer after the call returns.
 *  - All device work is enqueued asynchronously on `stream` (a cudaStream_t;
 *    NULL is the legacy default stream).  No call reads device memory on the
 *    host or synchronises, except pa_last_device_error().  One call forks:
 *    a shared-prefix decode whose own tokens go to the CUDA-core kernel (see
 *    pa_decode) enqueues that pass on a second stream of the library's (one
 *    per device, created on first use), ordered after the call's earlier
 *    work on `stream` by an event, and makes `stream` wait for it before the
 *    merge: every kernel of the call is still ordered before `stream`'s next
 *    work.  Make the first such call on a device before any stream capture
 *    on it (creating a stream is not allowed inside a capture); after a
 *    context reset the stream and events are made again.
 *  - Shapes and host-side arguments are validated before anything is
 *    launched; a refusal returns PA_ERR_INVALID_ARG or PA_ERR_UNSUPPORTED and
 *    launches nothing.  A failed launch returns PA_ERR_CUDA.
 *  - Values that only the device can see (block ids, slots, context lengths,
 *    copy pairs) are range-checked by the kernels.  A bad value never faults:
 *    the access is skipped (a K/V row outside the pool reads as zeros), a bit
 *    is recorded in a per-device error word, and pa_last_device_error()
 *    returns PA_ERR_DEVICE_CHECK until it is read.
 *  - No kernel waits on anything outside its own CTA: its TMA copies, its
 *    tensor-core products and its own warps' hand-offs.  Every such wait has
 *    a wall-clock limit (2 s) after which the kernel records
 *    PA_DEVERR_WAIT_TIMEOUT, lets its copies and products land, and returns.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; declared here so this header needs no CUDA
 * headers. */
typedef struct CUstream_st *pa_stream_t;

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,  /* null pointer, negative size, misaligned pointer, bad shape */
  PA_ERR_UNSUPPORTED = 2,  /* valid but not built: head_dim, group size, block size, dtype */
  PA_ERR_CUDA = 3,         /* a CUDA runtime call or a launch failed */
  PA_ERR_OOM = 4,          /* the host block allocator has no free block */
  PA_ERR_DEVICE_CHECK = 5  /* a kernel found a bad device-side value (see pa_last_device_error) */
} pa_status;

typedef enum { PA_F16 = 0, PA_BF16 = 1 } pa_dtype;

/* Bits of the device error word returned by pa_last_device_error(). */
#define PA_DEVERR_BLOCK_ID 0x1u     /* block-table entry of a token below the context is outside [0, num_blocks) */
#define PA_DEVERR_CONTEXT_LEN 0x2u  /* context length < 0, > max_context_len or > max_blocks_per_seq * block_size */
#define PA_DEVERR_SLOT 0x4u         /* append slot >= num_blocks * block_size */
#define PA_DEVERR_PAIR 0x8u         /* copy pair names a block outside [0, num_blocks) */
#define PA_DEVERR_WAIT_TIMEOUT 0x10u
#define PA_DEVERR_CONFIG 0x20u      /* a kernel found less shared memory than it laid out; it did nothing */

/*
 * Shape of one paged KV cache and of the batch that reads it.
 *
 * Layouts (all contiguous, row-major, elements of `dtype`):
 *   q, out                  [num_seqs][num_q_heads][head_dim]
 *   k_cache, v_cache        [num_blocks][block_size][num_kv_heads][head_dim]
 *                           (the pages' [num_blocks, block_size, num_heads,
 *                           head_dim] block tensor, one for K and one for V)
 *   block_tables (int32)    [num_seqs][max_blocks_per_seq]
 *   context_lens (int32)    [num_seqs]
 *   k, v for append         [num_tokens][num_kv_heads][head_dim]
 *
 * Query head h reads kv head h / (num_q_heads / num_kv_heads): grouped-query
 * heads are contiguous.
 *
 * Built values: head_dim in {64, 128}; num_q_heads / num_kv_heads in
 * {1, 2, 4, 8, 16}; block_size a multiple of 8 (8, 16 and 256 are the measured
 * ones; with a multiple of 8 that is not one of 16, every 16-token TMA box is
 * loaded as two 8-token boxes, zingnex.cn section 5: block_size 8 for short
 * sequences); num_blocks * block_size < 2^31; partition_tokens a multiple of 16 in
 * [16, 2048], or 0 for the default: 512 for the tensor-core kernels and
 * with shared_prefix (their largest item), 1024 for the CUDA-core kernel.
 */
typedef struct {
  int32_t num_seqs;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t block_size;
  int32_t num_blocks;
  int32_t max_blocks_per_seq;
  int32_t partition_tokens;
  int32_t dtype;   /* pa_dtype */
  int32_t variant; /* pa_decode_variant (pa_decode only; 0 = automatic) */
  int32_t shared_prefix; /* pa_decode only: 1 = read blocks shared by consecutive
                            sequences once per group (see pa_decode); 0 = off */
  int32_t cache_format;  /* pa_cache_format: what k_cache / v_cache hold */
} pa_shape;

/* Element format of k_cache / v_cache.
 *  PA_CACHE_AS_DTYPE   2-byte elements of shape->dtype (pa_decode,
 *                      pa_cache_append).
 *  PA_CACHE_FP8_E4M3   1-byte OCP E4M3 codes (1 sign, 4 exponent bits with
 *                      bias 7, 3 mantissa bits, no infinity, S.1111.111 =
 *                      NaN, largest finite 448) with one fp32 scale per kv
 *                      head for K and one for V: stored value = code * scale.
 *                      Read by pa_decode_fp8, written by pa_cache_append_fp8;
 *                      q and out stay in shape->dtype.  The pages name FP8
 *                      only as a quantisation format that saves memory
 *                      (zingnex.cn sections 4.1 and 6; 5688vip.com section
 *                      2.3); this encoding is the library's reading. */
typedef enum { PA_CACHE_AS_DTYPE = 0, PA_CACHE_FP8_E4M3 = 1 } pa_cache_format;

/* How pa_decode computes QK^T and PV.  Both variants read K/V with tiled TMA
 * loads through the block table and keep the softmax in fp32.
 *  PA_DECODE_AUTO          tensor cores when head_dim == 128, the group
 *                          g = Hq / Hkv is at least 8 (at least 4 when
 *                          block_size is a multiple of 16) and
 *                          partition_tokens is a multiple of 128 up to 512;
 *                          CUDA cores otherwise.  The same rule holds for an
 *                          E4M3 cache (pa_decode_fp8).
 *  PA_DECODE_CUDA_CORES    fp32 FMA on the CUDA cores (any built shape).
 *  PA_DECODE_TENSOR_CORES  tcgen05 MMA with the g heads padded to 16: fp16/bf16
 *                          operands (the probabilities enter the PV product as
 *                          two terms of the input type, hi + lo, about 16
 *                          significant bits), fp32 accumulators in tensor
 *                          memory.  Needs head_dim 128 and partition_tokens a
 *                          multiple of 128 up to 512 (else PA_ERR_UNSUPPORTED). */
typedef enum { PA_DECODE_AUTO = 0, PA_DECODE_CUDA_CORES = 1, PA_DECODE_TENSOR_CORES = 2 } pa_decode_variant;

/* The split-K partition pa_decode() uses for `shape` (partition_tokens, or
 * its default when 0), or minus the status pa_decode() would refuse the
 * shape with.  Host only. */
int pa_decode_partition_tokens(const pa_shape *shape);

/* The kernel pa_decode() runs for `shape`: PA_DECODE_CUDA_CORES or
 * PA_DECODE_TENSOR_CORES (PA_DECODE_AUTO resolved), or
 * PA_DECODE_RESOLVED_SHARED_PREFIX with shape->shared_prefix (a plan kernel,
 * then the tensor-core kernel over every group's row list), or minus the
 * status pa_decode() would refuse the shape with.  Host only; launches
 * nothing. */
#define PA_DECODE_RESOLVED_SHARED_PREFIX 3
int pa_decode_resolved_variant(const pa_shape *shape);

/* Bytes of device workspace pa_decode() needs for `shape` when no context is
 * longer than `max_context_len` tokens: 256 bytes for the work counter the
 * tensor-core variant's persistent CTAs take items from; with shared_prefix,
 * two records of 16 bytes per sequence (each rounded up to 256) for the group
 * plan; plus, when a context spans more than one partition (always with
 * shared_prefix), per (sequence, query head, partition) the running max, the
 * softmax sum and the unnormalised output row in fp32, for ceil(max_context_len
 * / partition_tokens) partitions, two more with shared_prefix.  The
 * workspace needs no initialisation (the counter carries a per-call tag, so a
 * value left by an earlier call is recognised and replaced) and is dead after
 * the call's kernels finish.  Returns 0 for an invalid shape. */
size_t pa_decode_workspace_bytes(const pa_shape *shape, int32_t max_context_len);

/*
 * Single-token decode attention over the paged cache.
 *
 * For every sequence s and query head h, with kv head h / g and
 * ctx = context_lens[s]:
 *   x_j  = scale * <q[s][h], K_j>,  K_j = k_cache[block_tables[s][j / bs]][j % bs][h / g]
 *   out[s][h] = sum_j softmax(x)_j * V_j      (j = 0 .. ctx - 1; V_j likewise)
 * computed in fp32 and rounded to nearest-even into `dtype`.  ctx == 0 gives a
 * zero row.  Table entries at or beyond ceil(ctx / bs) and cache slots at or
 * beyond ctx are never read, so they may hold anything (including NaN).
 *
 * Contexts are cut into partitions of shape->partition_tokens tokens; each
 * (sequence, kv head, partition) is one work item (one CTA on the CUDA-core
 * variant; items taken by one persistent CTA per SM on the tensor-core
 * variant), and sequences with more than one partition are merged by a
 * second kernel (log-sum-exp rule).  shape->variant picks the arithmetic.
 *
 * Shared prefixes (shape->shared_prefix = 1; needs variant PA_DECODE_AUTO,
 * head_dim 128 and partition_tokens a multiple of 128 up to 512, else
 * PA_ERR_UNSUPPORTED).  Blocks shared between sequences (zingnex.cn,
 * "vLLM与PagedAttention深度剖析", section 3.2 item 3: beam candidates forked
 * from one parent, prompts with a common prefix) are then read once per group
 * of sequences instead of once per sequence.  A first kernel finds the groups
 * on the device from the tables alone: runs of consecutive sequences (within
 * aligned windows of 256) whose tables start with the same physical block, cut
 * into groups of at most 32 / g members; a group shares its first T tokens,
 * where T counts the leading table entries equal in all members (below each
 * member's own block count), capped at the shortest member context and
 * rounded down to a multiple of 16; groups with T < 128 are dropped (their
 * members, and every sequence in no group, are groups of one with T = 0).
 * Each group is then read as one row list: its T shared tokens, followed by
 * each member's own tokens [T, ctx) rounded up to 16 rows; the tensor-core
 * kernel reads each partition of that list once, for all members x g query
 * rows (a member's columns see the shared rows and its own), and the merge
 * kernel combines a member's partitions (log-sum-exp rule).  The result is
 * the same attention, up to fp32 rounding order; only the order in which the
 * sums are formed differs.  Own tokens not in a list (a long private
 * continuation, or a sequence in no group) are read per sequence: at group
 * sizes where the plain decode runs on the tensor cores, as further items of
 * the same launch as the lists; else on the CUDA-core kernel, on the
 * library's second stream (see the conventions above), beside the lists'
 * launch.
 *
 * q, k_cache, v_cache, block_tables, context_lens, out: device, layouts above.
 * max_context_len: host-side upper bound on every context_lens[s]; it sizes the
 *   grid.  A larger device value is clamped and reported (PA_DEVERR_CONTEXT_LEN).
 * workspace: device, at least pa_decode_workspace_bytes(shape, max_context_len)
 *   bytes, 16-byte aligned, never NULL.  It must not be shared with a decode
 *   that runs concurrently.
 * An E4M3 cache (cache_format PA_CACHE_FP8_E4M3) needs pa_decode_fp8 and its
 * scales: pa_decode refuses it with PA_ERR_INVALID_ARG.
 * CUDA graphs: the call may be captured (stream capture) once the same shape
 * has run eagerly on that device, and the graph replayed any number of
 * times.  A captured call that uses the tensor-core kernels adds a memset
 * of the workspace's work counter to the graph, which resets it before each
 * replay.  The same holds for pa_decode_fp8 and pa_decode_multi.
 */
pa_status pa_decode(const void *q, const void *k_cache, const void *v_cache,
                    const int32_t *block_tables, const int32_t *context_lens, float scale,
                    void *out, const pa_shape *shape, int32_t max_context_len,
                    void *workspace, size_t workspace_bytes, pa_stream_t stream);

/*
 * Several query tokens per sequence (the scope table's multi-token queries:
 * verifying speculated tokens, chunked prefill under continuous batching,
 * 5688vip.com section 2.2).  q, out: [num_seqs][num_query_tokens][Hq][D]
 * (shape->num_seqs real sequences).  context_lens[s] counts the sequence's
 * num_query_tokens (Tq) new tokens, whose K/V are already appended; query
 * token t attends causally to tokens 0 .. ctx_s - Tq + t.  A query whose
 * range is empty (ctx_s < Tq - t) gives a zero row.
 *
 * Where the shape allows the tensor-core kernel (head_dim 128, a 16-bit
 * cache, variant not PA_DECODE_CUDA_CORES, partition_tokens 0 (then 512) or
 * a multiple of 128 up to 512) and Tq * g <= 32, the Tq x g query rows of a
 * sequence are the columns of one item per (sequence, kv head, partition),
 * each masked at its own causal limit: every K/V tile is read once for all
 * Tq queries.  Otherwise query t of s is decoded as a one-token virtual
 * sequence with the same block table and context ctx_s - Tq + t + 1: a first
 * kernel writes the virtual tables and contexts into the workspace, and the
 * virtual sequences of one sequence, which start with the same blocks, are
 * grouped as shared prefixes when the shape allows it (variant
 * PA_DECODE_AUTO).  Tq == 1 is pa_decode.
 * workspace: pa_decode_multi_workspace_bytes(shape, Tq, max_context_len).
 */
size_t pa_decode_multi_workspace_bytes(const pa_shape *shape, int32_t num_query_tokens,
                                       int32_t max_context_len);
pa_status pa_decode_multi(const void *q, const void *k_cache, const void *v_cache,
                          const int32_t *block_tables, const int32_t *context_lens, float scale,
                          void *out, const pa_shape *shape, int32_t num_query_tokens,
                          int32_t max_context_len, void *workspace, size_t workspace_bytes,
                          pa_stream_t stream);

/*
 * pa_decode for callers that cannot allocate device memory.
 *
 * The paper has no counterpart to this call (it is not part of the method);
 * it exists for callers of this library that have no way to allocate the
 * split-K workspace pa_decode needs:
 * a plug-in running inside a host runtime that owns all device memory and
 * gives its plug-ins no allocator, or a decode loop that must not call
 * cudaMalloc (which can synchronise the whole device) once it is running.
 *
 * Same arguments and result as pa_decode, minus the workspace: the split-K
 * scratch comes from one fixed array compiled into the library.  Nothing here
 * calls cudaMalloc, cudaFree or any allocating routine.
 *  - Limit: PA_NOALLOC_SCRATCH_BYTES per device.  Every GPU that loads the
 *    library holds that much device memory for the array until the process
 *    exits.  A call whose workspace (pa_decode_workspace_bytes for the same
 *    shape and max_context_len: 256 + num_seqs * num_q_heads * partitions *
 *    (head_dim + 2) * 4 bytes, rounded) exceeds the limit returns
 *    PA_ERR_UNSUPPORTED and launches nothing; pa_decode with a caller-owned
 *    workspace has no such limit.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) and caches it; make that first call before any
 *    stream capture on that device.  It returns PA_ERR_CUDA if the lookup
 *    fails.  The cached address belongs to the device's context at that
 *    time: after cudaDeviceReset(), or anything else that destroys the
 *    primary context, it is stale, so do not call pa_decode_noalloc on that
 *    device again in the same process.
 *  - Every call on a device shares the one array and finds the previous
 *    call's contents in it; nothing in it has to start at zero, because each
 *    call writes every scratch slot it later reads.  Calls whose kernels can
 *    overlap on the GPU (different streams without ordering between them)
 *    race on the array: order them, or use pa_decode with separate workspaces.
 */
#define PA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
pa_status pa_decode_noalloc(const void *q, const void *k_cache, const void *v_cache,
                            const int32_t *block_tables, const int32_t *context_lens, float scale,
                            void *out, const pa_shape *shape, int32_t max_context_len,
                            pa_stream_t stream);

/*
 * Append one new token per entry into a 16-bit cache (cache_format
 * PA_CACHE_AS_DTYPE, else PA_ERR_INVALID_ARG; the "update KV cache" step of
 * each decode iteration, 5688vip.com section 2.1): for t < num_tokens with
 * slot = slot_mapping[t] >= 0,
 *   k_cache viewed as [num_blocks * block_size][num_kv_heads][head_dim] gets
 *   row `slot` = k[t], and likewise v_cache = v[t].
 * slot = physical_block * block_size + offset.  Negative slots are skipped
 * (padding).  Slots must be distinct.  A bit-exact copy (no conversion).
 * Uses shape->num_kv_heads, head_dim, block_size, num_blocks, dtype.
 * k, v, slot_mapping (int32 [num_tokens]), k_cache, v_cache: device.
 */
pa_status pa_cache_append(const void *k, const void *v, const int32_t *slot_mapping,
                          int32_t num_tokens, void *k_cache, void *v_cache,
                          const pa_shape *shape, pa_stream_t stream);

/*
 * Append into an E4M3 cache (shape->cache_format == PA_CACHE_FP8_E4M3, else
 * PA_ERR_INVALID_ARG): as pa_cache_append, but each element x of k[t] (fp16
 * or bf16, shape->dtype, widened exactly to fp32) of kv head h is stored as
 * the E4M3 code nearest to x / k_scale[h], the division in fp32 rounded to
 * nearest, ties to the even code, magnitudes of 448 and above saturated to
 * 448 (and v likewise with v_scale).  k_scale, v_scale: device fp32
 * [num_kv_heads], finite and > 0 (not checked).
 */
pa_status pa_cache_append_fp8(const void *k, const void *v, const int32_t *slot_mapping,
                              int32_t num_tokens, void *k_cache, void *v_cache,
                              const float *k_scale, const float *v_scale,
                              const pa_shape *shape, pa_stream_t stream);

/*
 * Decode attention over an E4M3 cache (shape->cache_format ==
 * PA_CACHE_FP8_E4M3, else PA_ERR_INVALID_ARG): pa_decode's result with
 * K_j = code * k_scale[h / g] and V_j = code * v_scale[h / g].  The variant
 * and shared_prefix work as in pa_decode.  The CUDA-core kernel widens each
 * lane's codes as it reads them; the tensor-core kernels land the 8-bit tiles
 * by TMA and widen them exactly to 16 bits in shared memory before the
 * products.  The K scale is folded into the logits and the V scale into the
 * output.  Same workspace as pa_decode.  k_scale, v_scale: device fp32
 * [num_kv_heads].
 */
pa_status pa_decode_fp8(const void *q, const void *k_cache, const void *v_cache,
                        const float *k_scale, const float *v_scale,
                        const int32_t *block_tables, const int32_t *context_lens, float scale,
                        void *out, const pa_shape *shape, int32_t max_context_len,
                        void *workspace, size_t workspace_bytes, pa_stream_t stream);

/*
 * Copy-on-write of whole blocks (zingnex.cn section 3.2 item 3): for each
 * pair i, block src_dst_pairs[2i+1] of k_cache and of v_cache becomes a
 * byte copy of block src_dst_pairs[2i] (either cache format: a block is
 * block_size * num_kv_heads * head_dim elements of 2 or 1 bytes).
 * Destinations must be distinct and no
 * destination may also be a source in the same call.
 * src_dst_pairs: device int32 [num_pairs][2].  num_pairs == 0 launches nothing.
 */
pa_status pa_copy_blocks(const int32_t *src_dst_pairs, int32_t num_pairs, void *k_cache,
                         void *v_cache, const pa_shape *shape, pa_stream_t stream);

/*
 * Swap whole blocks between two pools (zingnex.cn section 5, tuning advice:
 * CPU offload through swap space): for each pair i, block src_dst_pairs[2i+1]
 * of (dst_k, dst_v) becomes a byte copy of block src_dst_pairs[2i] of
 * (src_k, src_v).  Either pool may be host memory the device can address
 * (pinned and mapped, e.g. cudaHostAlloc'd under unified addressing), so
 * swapping a preempted sequence out to the host and back in is two calls.
 * Pageable host memory, or pinned memory the device cannot address at the
 * same pointer, is refused (PA_ERR_INVALID_ARG, checked with
 * cudaPointerGetAttributes before any launch).
 * The two pools of each tensor must not overlap (else PA_ERR_INVALID_ARG);
 * src_num_blocks / dst_num_blocks size them; an entry outside either is
 * reported (PA_DEVERR_PAIR) and skipped.  shape gives the block geometry
 * and cache format (shape->num_blocks is not used).
 * src_dst_pairs: device int32 [num_pairs][2].  num_pairs == 0 launches nothing.
 */
pa_status pa_swap_blocks(const int32_t *src_dst_pairs, int32_t num_pairs, const void *src_k,
                         const void *src_v, int32_t src_num_blocks, void *dst_k, void *dst_v,
                         int32_t dst_num_blocks, const pa_shape *shape, pa_stream_t stream);

/* Synchronises `stream`, then reads and clears this device's error word.
 * Returns PA_OK when it was zero, PA_ERR_DEVICE_CHECK otherwise (bits in
 * *bits_out if non-NULL), PA_ERR_CUDA if the synchronisation failed. */
pa_status pa_last_device_error(pa_stream_t stream, uint32_t *bits_out);

/* Static description of a status code (never NULL). */
const char *pa_status_string(pa_status status);

/* Text of the CUDA error behind the calling thread's most recent
 * PA_ERR_CUDA from pa_decode(_fp8), pa_cache_append(_fp8), pa_copy_blocks or
 * pa_last_device_error ("no CUDA error" before the first one).  The string is
 * static; the caller does not free it.  Not part of the method: a diagnostic
 * of this library. */
const char *pa_last_cuda_error(void);

/* Number of kernels this library has launched in this process. */
uint64_t pa_kernel_launches(void);

/* Build description: target architecture and library version. */
const char *pa_build_info(void);

/* ------------------------------------------------------------------------
 * Host block allocator (zingnex.cn section 3.2 items 1-4; jsqmd.com
 * "vLLM-v0.11.0性能实测" section 4.2): a free list of physical blocks, a
 * reference count per block and a block table per sequence.  It builds the
 * block tables, slot mappings and copy-on-write pairs the kernels consume.
 *
 * The free list is a stack: `order` (a permutation of 0..num_blocks-1, or
 * NULL for 0, 1, 2, ...) gives the allocation order, and a block whose count
 * drops to zero goes back on top, so it is the next one handed out.  Freeing a
 * sequence releases its blocks last-to-first.  Sequence ids are arbitrary
 * int32 values.  Not thread-safe; all memory is host memory.
 */
typedef struct pa_alloc pa_alloc;

/* Returns NULL on bad arguments (order not a permutation, sizes <= 0). */
pa_alloc *pa_alloc_create(int32_t num_blocks, int32_t block_size, const int32_t *order);
void pa_alloc_destroy(pa_alloc *a);

/* New sequence with `num_tokens` tokens (blocks allocated on demand). */
pa_status pa_alloc_add_seq(pa_alloc *a, int32_t seq, int32_t num_tokens);
/* Grow a sequence by `num_tokens` tokens without copy-on-write (prefill). */
pa_status pa_alloc_extend(pa_alloc *a, int32_t seq, int32_t num_tokens);
/* `child` (new) shares every block of `parent`; each block's count + 1. */
pa_status pa_alloc_fork(pa_alloc *a, int32_t parent, int32_t child);
/* Drop a sequence; blocks whose count reaches zero return to the free list. */
pa_status pa_alloc_free_seq(pa_alloc *a, int32_t seq);

/*
 * Reserve the slot of one new token for each of seqs[0..n-1], in order.
 * A sequence whose next token starts a block gets a fresh block.  One whose
 * last block is shared gets a fresh block and a copy pair (src, dst) is
 * appended to pairs_out (capacity n pairs); the shared block's count drops
 * by one.  slot_out[i] = block * block_size + offset.
 * All-or-nothing: PA_ERR_OOM (nothing changed) when the free list cannot
 * cover the whole batch.
 */
pa_status pa_alloc_append_slots(pa_alloc *a, const int32_t *seqs, int32_t n, int32_t *slot_out,
                                int32_t *pairs_out, int32_t *num_pairs_out);

/* Write the block tables ([n][max_blocks_per_seq], padded with -1) and
 * context lengths of seqs[0..n-1].  PA_ERR_INVALID_ARG if a table is longer
 * than max_blocks_per_seq or a sequence is unknown. */
pa_status pa_alloc_block_tables(const pa_alloc *a, const int32_t *seqs, int32_t n,
                                int32_t max_blocks_per_seq, int32_t *tables_out,
                                int32_t *lens_out);

int32_t pa_alloc_num_free(const pa_alloc *a);
/* Reference count of `block`, or -1 if out of range. */
int32_t pa_alloc_refcount(const pa_alloc *a, int32_t block);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
