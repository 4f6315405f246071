// pa_api.cu -- the C ABI of libpa.so: host-side validation, TMA descriptor
// set-up and dispatch to the kernels.  See include/pa.h for the contract.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <chrono>
#include <cmath>
#include <cstring>
#include <mutex>

#include "pa.h"
#include "pa_internal.h"

namespace {

// The per-device error word the kernels report into (see pa.h).
__device__ unsigned int g_device_error = 0;

// Device address of g_device_error on the current device, looked up once per
// device (a host-side symbol name is not a device address).
unsigned int* error_word() {
  static std::mutex mu;
  static unsigned int* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<unsigned int*>(p);
  }
  return addr[dev];
}

std::atomic<uint64_t> g_launches{0};

// What the calling thread's last PA_ERR_CUDA came from.
thread_local const char* t_last_cuda_error = "no CUDA error";

pa_status cuda_failed(cudaError_t e) {
  t_last_cuda_error = cudaGetErrorString(e);
  return PA_ERR_CUDA;
}

pa_status cuda_failed(const char* what) {
  t_last_cuda_error = what;
  return PA_ERR_CUDA;
}

void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Whether the tensor-core kernels run, with partition_tokens == 0 read as
// "their default"; defined below.
bool tensor_core_kernel(const pa_shape* s, int pt);
int box_rows(const pa_shape* s);

// partition_tokens, or its default: 512 for the tensor-core kernels (their
// largest item), 1024 for the CUDA-core kernel, where fewer partials measured
// faster than 512 (llama2_7b 6025 vs 5697 GB/s, mistral_7b_gqa 4993 vs 4889).
int effective_partition(const pa_shape* s) {
  if (s->partition_tokens != 0) return s->partition_tokens;
  return (s->shared_prefix || tensor_core_kernel(s, 512)) ? 512 : 1024;
}

// Shape checks common to every call that touches the pool.
pa_status check_pool_shape(const pa_shape* s) {
  if (!s) return PA_ERR_INVALID_ARG;
  if (s->num_kv_heads <= 0 || s->head_dim <= 0 || s->block_size <= 0 || s->num_blocks < 0)
    return PA_ERR_INVALID_ARG;
  if (s->dtype != PA_F16 && s->dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
  if (s->cache_format != PA_CACHE_AS_DTYPE && s->cache_format != PA_CACHE_FP8_E4M3)
    return PA_ERR_UNSUPPORTED;
  if (s->head_dim != 64 && s->head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (s->block_size % 8 != 0) return PA_ERR_UNSUPPORTED;
  if ((long long)s->num_blocks * s->block_size >= (1LL << 31)) return PA_ERR_UNSUPPORTED;
  return PA_OK;
}

pa_status check_decode_shape(const pa_shape* s, int32_t max_context_len) {
  pa_status st = check_pool_shape(s);
  if (st != PA_OK) return st;
  if (s->num_seqs < 0 || s->num_q_heads <= 0 || s->max_blocks_per_seq < 0 || max_context_len < 0)
    return PA_ERR_INVALID_ARG;
  if (s->num_q_heads % s->num_kv_heads != 0) return PA_ERR_INVALID_ARG;
  const int g = s->num_q_heads / s->num_kv_heads;
  if (g != 1 && g != 2 && g != 4 && g != 8 && g != 16) return PA_ERR_UNSUPPORTED;
  const int pt = effective_partition(s);
  if (pt < 16 || pt % 16 != 0 || pt > pa::decode_max_partition_tokens()) return PA_ERR_UNSUPPORTED;
  if ((long long)s->num_seqs * s->num_q_heads * s->head_dim >= (1LL << 40)) return PA_ERR_INVALID_ARG;
  if (s->variant < PA_DECODE_AUTO || s->variant > PA_DECODE_TENSOR_CORES) return PA_ERR_INVALID_ARG;
  if (s->variant == PA_DECODE_TENSOR_CORES &&
      (s->head_dim != 128 || pt % pa::decode_tc_tile_tokens() != 0 || pt > 512))
    return PA_ERR_UNSUPPORTED;
  if (s->shared_prefix != 0 && s->shared_prefix != 1) return PA_ERR_INVALID_ARG;
  if (s->shared_prefix &&
      (s->variant != PA_DECODE_AUTO || s->head_dim != 128 || pt % pa::decode_tc_tile_tokens() != 0 ||
       pt > 512))
    return PA_ERR_UNSUPPORTED;
  // work items of one launch (256 sequences; the bound takes 512) must fit the
  // 24-bit counter
  const long long parts = ((long long)max_context_len + pt - 1) / pt;
  if (512LL * s->num_kv_heads * (parts > 0 ? parts : 1) >= (1LL << 23)) return PA_ERR_UNSUPPORTED;
  return PA_OK;
}

// Whether pa_decode runs the tensor-core variant for this (valid) shape.
// Bytes of one cached element.
int cache_elem_bytes(const pa_shape* s) { return s->cache_format == PA_CACHE_FP8_E4M3 ? 1 : 2; }

bool tensor_core_kernel(const pa_shape* s, int pt) {
  if (s->variant == PA_DECODE_TENSOR_CORES) return true;
  if (s->variant == PA_DECODE_CUDA_CORES) return false;
  // measured: tensor cores win from group 8 up, and at group 4 with 16-token
  // TMA boxes (mistral_7b_gqa: 5564 vs 4977 GB/s).  With 8-token blocks the
  // tensor-core kernel issues twice as many half-size boxes, and at group 4
  // that costs more than the MMAs save (3602 vs 4890 GB/s).
  const int g = s->num_q_heads / s->num_kv_heads;
  return s->head_dim == 128 && (g >= 8 || (g >= 4 && box_rows(s) == 16)) &&
         pt % pa::decode_tc_tile_tokens() == 0 && pt <= 512;
}

bool use_tensor_cores(const pa_shape* s) { return tensor_core_kernel(s, effective_partition(s)); }

// Workspace: the work counter (8 bytes used of 256); with shared_prefix the
// two plan records, int4 [S] each (each rounded up to 256 bytes); then, for
// split-K, partial outputs [S][Hq][P][D] and (max, sum) pairs [S][Hq][P][2]
// in fp32.  P is ceil(max_context_len / partition_tokens), plus two with
// shared_prefix: a member's rows in its group's row list are its shared
// tokens and its own run, which may each end in a partial partition and
// start the next one part-way.
constexpr long long kCounterBytes = 256;

long long round256(long long x) { return (x + 255) / 256 * 256; }

// A second stream per device, and two events, for the shared-prefix decode
// whose own tokens go to the CUDA-core kernel: that kernel runs beside the
// row-list launch, which often leaves most SMs idle.  Created on first use;
// the fork and join are enqueued under a lock, so that calls from several
// host threads never wait on each other's event records.
struct SideStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t forked = nullptr, done = nullptr;
};
std::mutex g_side_lock;
SideStream g_side[64];

bool side_stream(int dev, SideStream* out) {
  if (dev < 0 || dev >= 64) return false;
  SideStream& s = g_side[dev];
  if (!s.stream) {
    SideStream n;
    if (cudaEventCreateWithFlags(&n.forked, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&n.done, cudaEventDisableTiming) != cudaSuccess ||
        cudaStreamCreateWithFlags(&n.stream, cudaStreamNonBlocking) != cudaSuccess)
      return false;
    s = n;
  }
  *out = s;
  return true;
}

int num_partitions(const pa_shape* s, int32_t max_context_len);

long long plan_bytes(const pa_shape* s) {
  return s->shared_prefix ? 2 * round256(16LL * s->num_seqs) : 0;
}

// Partitions per (sequence, query head) in the workspace (0: no split-K space).
long long workspace_parts(const pa_shape* s, int32_t max_context_len) {
  const long long P = num_partitions(s, max_context_len);
  if (s->shared_prefix) return P + 2;
  return P > 1 ? P : 0;
}

// Tags of decode launches (see the work counter in pa_decode_tc.cu): unique
// per launch, never 0, below 2^40.
// Epochs start at a per-process value so that a workspace last used by another
// library instance or process is unlikely to carry a live epoch.
std::atomic<uint64_t> g_epoch{
    1 + ((reinterpret_cast<uintptr_t>(&g_launches) ^
          (uint64_t)std::chrono::steady_clock::now().time_since_epoch().count() * 0x9E3779B97F4A7C15ull) &
         ((1ull << 39) - 1))};
uint64_t next_epochs(int n) {
  uint64_t e = g_epoch.fetch_add((uint64_t)n, std::memory_order_relaxed) & ((1ull << 40) - 1);
  if (e == 0 || e + (uint64_t)n >= (1ull << 40)) e = 1;
  return e;
}

int num_partitions(const pa_shape* s, int32_t max_context_len) {
  const int pt = effective_partition(s);
  return (max_context_len + pt - 1) / pt;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point, so the
// library does not link libcuda directly.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D map over one pool viewed as [num_blocks * block_size][Hkv][D]; a box
// is `rows` consecutive token rows of one kv head.
bool make_pool_map(CUtensorMap* map, const void* pool, const pa_shape* s, int rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const int eb = cache_elem_bytes(s);
  const cuuint64_t dims[3] = {(cuuint64_t)s->head_dim, (cuuint64_t)s->num_kv_heads,
                              (cuuint64_t)s->num_blocks * s->block_size};
  const cuuint64_t strides[2] = {(cuuint64_t)s->head_dim * eb,
                                 (cuuint64_t)s->num_kv_heads * s->head_dim * eb};
  const cuuint32_t box[3] = {(cuuint32_t)s->head_dim, 1, (cuuint32_t)rows};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, eb == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16, 3,
                  const_cast<void*>(pool), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Maps of the tensor-core variant: pools viewed as [NB * bs][Hkv][128] with
// 128B-swizzled boxes of 64 elements x 16 token rows; q viewed as
// [S * Hq][128] with 128B-swizzled boxes of 64 elements x `group` rows.
// TMA box rows over the pool: 16 (one box per 16-token group), or 8 when
// blocks hold a multiple of 8 but not of 16 tokens (two boxes per group).
// With `pair` (items of two kv heads) the pools are viewed with the head as
// the outer dimension, [Hkv][NB * bs][128] by strides, so that one box holds
// 16 rows of one head and then the same rows of the next (4 KB instead of
// 2 KB: the per-SM box rate bounds this kernel), and a q box holds 2 x group
// rows.
int box_rows(const pa_shape* s) { return s->block_size % 16 == 0 ? 16 : 8; }

bool make_tc_maps(CUtensorMap* tk, CUtensorMap* tv, CUtensorMap* tq, const void* k, const void* v,
                  const void* q, const pa_shape* s, bool pair, int query_tokens, bool grouped) {
  auto fn = encode_fn();
  if (!fn) return false;
  // a box row is 128 bytes: 64 two-byte elements, or (E4M3 cache) all 128
  // one-byte elements of a head's row
  const bool fp8 = s->cache_format == PA_CACHE_FP8_E4M3;
  const cuuint64_t eb = fp8 ? 1 : 2, inner = 128 / eb;
  const cuuint64_t rows = (cuuint64_t)s->num_blocks * s->block_size, Hkv = (cuuint64_t)s->num_kv_heads;
  const cuuint64_t dims_h[3] = {128, Hkv, rows}, dims_p[3] = {128, rows, Hkv};
  const cuuint64_t strides_h[2] = {128 * eb, Hkv * 128 * eb}, strides_p[2] = {Hkv * 128 * eb, 128 * eb};
  const cuuint32_t box_h[3] = {(cuuint32_t)inner, 1, (cuuint32_t)box_rows(s)},
                   box_p[3] = {(cuuint32_t)inner, 16, 2};
  const cuuint64_t* dims = pair ? dims_p : dims_h;
  const cuuint64_t* strides = pair ? strides_p : strides_h;
  const cuuint32_t* box = pair ? box_p : box_h;
  const cuuint32_t estr[3] = {1, 1, 1};
  for (int i = 0; i < 2; ++i) {
    CUresult r = fn(i ? tv : tk, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16,
                    3, const_cast<void*>(i ? v : k), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
  }
  // q viewed as [S * Tq][Hq][128]: one box is the query rows of an item,
  // [rows][heads][64] (rows past the batch read as zeros)
  const int g = s->num_q_heads / s->num_kv_heads;
  const pa::TcQueryBox qb = pa::tc_query_box(g, query_tokens, pair, grouped);
  const cuuint64_t qdims[3] = {128, (cuuint64_t)s->num_q_heads,
                               (cuuint64_t)s->num_seqs * (cuuint64_t)query_tokens};
  const cuuint64_t qstrides[2] = {256, (cuuint64_t)s->num_q_heads * 256};
  const cuuint32_t qbox[3] = {64, (cuuint32_t)qb.heads, (cuuint32_t)qb.rows};
  return fn(tq, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(q), qdims, qstrides, qbox, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

extern "C" {

size_t pa_decode_workspace_bytes(const pa_shape* shape, int32_t max_context_len) {
  if (check_decode_shape(shape, max_context_len) != PA_OK) return 0;
  const long long head = kCounterBytes + plan_bytes(shape);
  const long long P = workspace_parts(shape, max_context_len);
  if (P == 0) return (size_t)head;
  const long long rows = (long long)shape->num_seqs * shape->num_q_heads * P;
  const long long acc = rows * shape->head_dim * 4;
  const long long ml = rows * 2 * 4;
  return (size_t)(head + round256(acc) + ml);
}

}  // extern "C"

namespace {

// pa_decode and pa_decode_fp8 (scales set iff the cache holds E4M3 codes),
// and pa_decode_multi on the tensor-core kernels (query_tokens > 1: q and out
// are [S][Tq][Hq][D]; the caller has checked that the shape takes that path).
pa_status decode_impl(const void* q, const void* k_cache, const void* v_cache,
                      const float* k_scale, const float* v_scale, const int32_t* block_tables,
                      const int32_t* context_lens, float scale, void* out, const pa_shape* shape,
                      int32_t max_context_len, void* workspace, size_t workspace_bytes,
                      pa_stream_t stream, int query_tokens = 1, bool tables_just_written = false) {
  pa_status st = check_decode_shape(shape, max_context_len);
  if (st != PA_OK) return st;
  const bool fp8 = shape->cache_format == PA_CACHE_FP8_E4M3;
  if (fp8 != (k_scale != nullptr)) return PA_ERR_INVALID_ARG;  // the entry point must match
  if (shape->num_seqs == 0) return PA_OK;
  if (fp8 && (!v_scale || (reinterpret_cast<uintptr_t>(k_scale) & 3u) ||
              (reinterpret_cast<uintptr_t>(v_scale) & 3u)))
    return PA_ERR_INVALID_ARG;
  if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !out) return PA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
    return PA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(block_tables) & 3u) || (reinterpret_cast<uintptr_t>(context_lens) & 3u))
    return PA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;
  // the split-K rows of query_tokens queries per sequence
  pa_shape ws_shape = *shape;
  ws_shape.num_seqs = shape->num_seqs * query_tokens;
  const size_t need = pa_decode_workspace_bytes(&ws_shape, max_context_len);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return PA_ERR_INVALID_ARG;
  if (max_context_len > (long long)shape->max_blocks_per_seq * shape->block_size)
    return PA_ERR_INVALID_ARG;

  const int P_ws = (int)workspace_parts(shape, max_context_len);
  const int group = shape->num_q_heads / shape->num_kv_heads;
  pa::DecodeArgs a{};
  a.q = static_cast<const uint16_t*>(q);
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.out = static_cast<uint16_t*>(out);
  a.work_counter = static_cast<unsigned long long*>(workspace);
  char* ws = static_cast<char*>(workspace) + kCounterBytes;
  int4* plan = nullptr;
  int4* plan2 = nullptr;
  if (shape->shared_prefix) {
    plan = reinterpret_cast<int4*>(ws);
    plan2 = reinterpret_cast<int4*>(ws + plan_bytes(shape) / 2);
    ws += plan_bytes(shape);
  }
  if (P_ws > 0) {
    const long long rows = (long long)ws_shape.num_seqs * shape->num_q_heads * P_ws;
    a.ws_acc = reinterpret_cast<float*>(ws);
    a.ws_ml = reinterpret_cast<float*>(ws + round256(rows * shape->head_dim * 4));
  }
  a.scale_log2 = scale * 1.4426950408889634f;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  a.num_seqs = shape->num_seqs;
  a.num_q_heads = shape->num_q_heads;
  a.num_kv_heads = shape->num_kv_heads;
  a.block_size = shape->block_size;
  a.num_blocks = shape->num_blocks;
  a.max_blocks_per_seq = shape->max_blocks_per_seq;
  a.partition_tokens = effective_partition(shape);
  a.num_parts = P_ws > 0 ? P_ws : 1;
  a.own_tokens = a.partition_tokens;
  {
    const int gp = (max_context_len + a.own_tokens - 1) / a.own_tokens;
    a.grid_parts = gp > 0 ? gp : 1;
  }
  a.query_tokens = query_tokens;
  a.group = group;
  a.half_boxes = box_rows(shape) == 8;
  a.max_context_len = max_context_len;
  a.err = error_word();
  if (!a.err) return cuda_failed("device error word lookup failed");

  if (shape->num_blocks == 0 && max_context_len > 0) return PA_ERR_INVALID_ARG;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  int launched = 0;
  cudaError_t e;
  const bool tc_path = shape->num_blocks > 0 && (shape->shared_prefix || use_tensor_cores(shape));
  // The tensor-core kernels take items from the work counter, tagged with a
  // per-call epoch.  Inside a CUDA graph that epoch is fixed at capture, so a
  // replay would find the count its previous replay left under the same
  // epoch and skip those items.  A captured call therefore zeroes the counter
  // first: the memset becomes a node of the graph and runs before each
  // replay's kernels (a zero word carries a foreign epoch, or the right one
  // with a count of zero).  Eager calls keep relying on the epoch alone.
  if (tc_path) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(cs, &cap) != cudaSuccess) return cuda_failed("cudaStreamIsCapturing failed");
    if (cap == cudaStreamCaptureStatusActive &&
        cudaMemsetAsync(a.work_counter, 0, sizeof(unsigned long long), cs) != cudaSuccess)
      return cuda_failed("cudaMemsetAsync of the work counter failed");
  }
  if (tc_path) {
    // items of two kv heads (4 KB boxes) where the heads pair up, their query
    // columns fit 16 and blocks give 16-row boxes; shared-prefix groups keep
    // one head per item
    const bool pair = shape->num_kv_heads % 2 == 0 && !a.half_boxes && 2 * group * query_tokens <= 16;
    bool own_tc = true;
    CUtensorMap tk, tv, tq;
    if (!make_tc_maps(&tk, &tv, &tq, k_cache, v_cache, q, shape, pair, query_tokens, false))
      return cuda_failed("cuTensorMapEncodeTiled failed");
    e = cudaSuccess;
    if (shape->shared_prefix) {
      // plan the groups; then every group's row list (shared tokens, and the
      // members' own tokens where they are few) on the tensor-core kernel
      // with members x g columns; then, per sequence, the own tokens that are
      // in no list
      CUtensorMap gk, gv, gq;
      if (!make_tc_maps(&gk, &gv, &gq, k_cache, v_cache, q, shape, false, 1, true))
        return cuda_failed("cuTensorMapEncodeTiled failed");
      pa::PlanArgs pl{};
      pl.block_tables = block_tables;
      pl.context_lens = context_lens;
      pl.plan = plan;
      pl.plan2 = plan2;
      pl.num_seqs = shape->num_seqs;
      pl.max_blocks_per_seq = shape->max_blocks_per_seq;
      pl.block_size = shape->block_size;
      pl.num_blocks = shape->num_blocks;
      pl.max_context_len = max_context_len;
      pl.partition_tokens = a.partition_tokens;
      pl.max_members = pa::kTcMaxColumns / group;
      pl.min_shared = pa::decode_tc_tile_tokens();
      pl.chunk = pa::kSharedPrefixSeqsPerLaunch;
      pl.inputs_written_before = tables_just_written ? 1 : 0;
      // own tokens read on their own go to the kernel this shape would get
      // without shared prefixes: tensor cores at larger groups, else CUDA
      // cores (in their largest partitions: few partials)
      own_tc = use_tensor_cores(shape);
      pl.own_partition_tokens = own_tc ? a.partition_tokens : pa::decode_max_partition_tokens();
      a.plan = plan;
      a.plan2 = plan2;
      const int chunks = (shape->num_seqs + pa::kSharedPrefixSeqsPerLaunch - 1) /
                         pa::kSharedPrefixSeqsPerLaunch;
      a.epoch = next_epochs(chunks);
      e = pa::launch_plan(pl, cs, &launched);
      if (own_tc) {
        // own tokens for the tensor cores go into the same launch as the
        // row lists, after them: no launch of their own for what is often
        // little work
        a.own_in_lists = 1;
        if (e == cudaSuccess) e = pa::launch_decode_tc(a, shape->dtype, gk, gv, gq, cs, &launched, false, fp8);
        a.own_in_lists = 0;
      } else if (e == cudaSuccess) {
        // own tokens on the CUDA-core kernel, on a second stream forked after
        // the plan, beside the row-list launch; both join before the merge
        CUtensorMap pk, pv;
        if (!make_pool_map(&pk, k_cache, shape, box_rows(shape)) ||
            !make_pool_map(&pv, v_cache, shape, box_rows(shape)))
          return cuda_failed("cuTensorMapEncodeTiled failed");
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess) return cuda_failed("cudaGetDevice failed");
        std::lock_guard<std::mutex> lock(g_side_lock);
        SideStream side;
        if (!side_stream(dev, &side)) return cuda_failed("creating the second stream failed");
        pa::DecodeArgs own = a;
        own.own_pass = 1;
        own.own_tokens = pa::decode_max_partition_tokens();
        own.grid_parts = (max_context_len + own.own_tokens - 1) / own.own_tokens;
        if (own.grid_parts < 1) own.grid_parts = 1;
        e = cudaEventRecord(side.forked, cs);
        if (e == cudaErrorInvalidResourceHandle) {
          // a context reset since the stream and events were made: make them again
          (void)cudaGetLastError();
          g_side[dev] = SideStream{};
          if (!side_stream(dev, &side)) return cuda_failed("creating the second stream failed");
          e = cudaEventRecord(side.forked, cs);
        }
        if (e == cudaSuccess) e = cudaStreamWaitEvent(side.stream, side.forked, 0);
        const bool forked = e == cudaSuccess;
        if (e == cudaSuccess)
          e = pa::launch_decode(own, shape->dtype, shape->head_dim, group, pk, pv, side.stream, &launched, fp8,
                                false);
        if (e == cudaSuccess) e = pa::launch_decode_tc(a, shape->dtype, gk, gv, gq, cs, &launched, false, fp8);
        if (forked) {
          // join whatever went onto the second stream, even after a failed
          // launch (a stream capture must not end with it unjoined)
          cudaError_t j = cudaEventRecord(side.done, side.stream);
          if (j == cudaSuccess) j = cudaStreamWaitEvent(cs, side.done, 0);
          if (e == cudaSuccess) e = j;
        }
      }
      if (e == cudaSuccess) e = pa::launch_decode_merge(a, shape->dtype, shape->head_dim, cs, &launched);
      count_launches(launched);
      return e == cudaSuccess ? PA_OK : cuda_failed(e);
    } else {
      a.epoch = next_epochs((shape->num_seqs + pa::kSharedPrefixSeqsPerLaunch - 1) / pa::kSharedPrefixSeqsPerLaunch);
    }
    if (e == cudaSuccess)
      e = pa::launch_decode_tc(a, shape->dtype, tk, tv, tq, cs, &launched, pair, fp8);
    if (e == cudaSuccess) e = pa::launch_decode_merge(a, shape->dtype, shape->head_dim, cs, &launched);
  } else {
    if (query_tokens != 1) return PA_ERR_UNSUPPORTED;  // the caller expands the queries
    CUtensorMap tk, tv;
    if (shape->num_blocks > 0) {
      if (!make_pool_map(&tk, k_cache, shape, box_rows(shape)) ||
          !make_pool_map(&tv, v_cache, shape, box_rows(shape)))
        return cuda_failed("cuTensorMapEncodeTiled failed");
    } else {
      // An empty pool can only serve empty contexts; the kernels issue no load.
      memset(&tk, 0, sizeof tk);
      memset(&tv, 0, sizeof tv);
    }
    e = pa::launch_decode(a, shape->dtype, shape->head_dim, group, tk, tv, cs, &launched, fp8);
  }
  count_launches(launched);
  return e == cudaSuccess ? PA_OK : cuda_failed(e);
}

}  // namespace

extern "C" {

pa_status pa_decode(const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, const int32_t* context_lens, float scale,
                    void* out, const pa_shape* shape, int32_t max_context_len, void* workspace,
                    size_t workspace_bytes, pa_stream_t stream) {
  return decode_impl(q, k_cache, v_cache, nullptr, nullptr, block_tables, context_lens, scale, out,
                     shape, max_context_len, workspace, workspace_bytes, stream);
}

}  // extern "C"

namespace {

// pa_decode_multi reads each sequence's K/V once for all its Tq query tokens
// on the tensor-core kernel when the shape allows it (head_dim 128, a 16-bit
// cache, the variant not forced to CUDA cores, partition_tokens 0 or a
// multiple of 128 up to 512) and Tq x g <= 32: the Tq x g query rows are the
// columns of one item, each query masked at its own causal limit.  The shape
// it runs (tensor-core variant, 512-token partitions by default):
bool multi_direct(const pa_shape* s, int num_query_tokens) {
  const int pt = s->partition_tokens;
  return s->num_kv_heads > 0 && s->head_dim == 128 && s->variant != PA_DECODE_CUDA_CORES &&
         s->cache_format == PA_CACHE_AS_DTYPE &&
         (long long)num_query_tokens * (s->num_q_heads / s->num_kv_heads) <= pa::kTcMaxColumns &&
         (pt == 0 || (pt % pa::decode_tc_tile_tokens() == 0 && pt <= 512));
}
pa_shape multi_direct_shape(const pa_shape* s) {
  pa_shape e = *s;
  e.variant = PA_DECODE_TENSOR_CORES;
  e.shared_prefix = 0;
  if (e.partition_tokens == 0) e.partition_tokens = 512;
  return e;
}
// Otherwise it runs a one-token batch of S * Tq virtual sequences, grouped by
// shared prefix when the shape allows the shared-prefix kernel.
pa_shape multi_shape(const pa_shape* s, int num_query_tokens) {
  pa_shape e = *s;
  e.num_seqs = s->num_seqs * num_query_tokens;
  const int pt = s->partition_tokens;
  e.shared_prefix = s->head_dim == 128 && s->variant == PA_DECODE_AUTO &&
                    s->cache_format == PA_CACHE_AS_DTYPE &&
                    (pt == 0 || (pt % pa::decode_tc_tile_tokens() == 0 && pt <= 512));
  return e;
}

// Virtual block tables [S * Tq][MBS] and contexts [S * Tq], each 256-aligned.
long long multi_tables_bytes(const pa_shape* s, int num_query_tokens) {
  return round256(4LL * s->num_seqs * num_query_tokens * s->max_blocks_per_seq);
}
long long multi_head_bytes(const pa_shape* s, int num_query_tokens) {
  return multi_tables_bytes(s, num_query_tokens) + round256(4LL * s->num_seqs * num_query_tokens);
}

bool multi_args_ok(const pa_shape* s, int num_query_tokens) {
  return s && num_query_tokens >= 1 && s->num_seqs >= 0 &&
         (long long)s->num_seqs * num_query_tokens <= (1LL << 30);
}

}  // namespace

extern "C" {

size_t pa_decode_multi_workspace_bytes(const pa_shape* shape, int32_t num_query_tokens,
                                       int32_t max_context_len) {
  if (!multi_args_ok(shape, num_query_tokens)) return 0;
  if (num_query_tokens == 1) return pa_decode_workspace_bytes(shape, max_context_len);
  if (multi_direct(shape, num_query_tokens)) {
    pa_shape e = multi_direct_shape(shape);
    if (check_decode_shape(&e, max_context_len) != PA_OK) return 0;
    e.num_seqs = shape->num_seqs * num_query_tokens;  // split-K rows
    return pa_decode_workspace_bytes(&e, max_context_len);
  }
  const pa_shape e = multi_shape(shape, num_query_tokens);
  const size_t inner = pa_decode_workspace_bytes(&e, max_context_len);
  if (inner == 0) return 0;
  return (size_t)multi_head_bytes(shape, num_query_tokens) + inner;
}

pa_status pa_decode_multi(const void* q, const void* k_cache, const void* v_cache,
                          const int32_t* block_tables, const int32_t* context_lens, float scale,
                          void* out, const pa_shape* shape, int32_t num_query_tokens,
                          int32_t max_context_len, void* workspace, size_t workspace_bytes,
                          pa_stream_t stream) {
  if (!multi_args_ok(shape, num_query_tokens)) return PA_ERR_INVALID_ARG;
  if (num_query_tokens == 1)
    return pa_decode(q, k_cache, v_cache, block_tables, context_lens, scale, out, shape,
                     max_context_len, workspace, workspace_bytes, stream);
  pa_status st = check_decode_shape(shape, max_context_len);
  if (st != PA_OK) return st;
  if (shape->cache_format != PA_CACHE_AS_DTYPE) return PA_ERR_INVALID_ARG;
  if (multi_direct(shape, num_query_tokens)) {
    const pa_shape d = multi_direct_shape(shape);
    return decode_impl(q, k_cache, v_cache, nullptr, nullptr, block_tables, context_lens, scale,
                       out, &d, max_context_len, workspace, workspace_bytes, stream,
                       num_query_tokens);
  }
  const pa_shape e = multi_shape(shape, num_query_tokens);
  st = check_decode_shape(&e, max_context_len);
  if (st != PA_OK) return st;
  if (shape->num_seqs == 0) return PA_OK;
  if (!block_tables || !context_lens || (reinterpret_cast<uintptr_t>(block_tables) & 3u) ||
      (reinterpret_cast<uintptr_t>(context_lens) & 3u))
    return PA_ERR_INVALID_ARG;
  const size_t need = pa_decode_multi_workspace_bytes(shape, num_query_tokens, max_context_len);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return PA_ERR_INVALID_ARG;
  if (max_context_len > (long long)shape->max_blocks_per_seq * shape->block_size)
    return PA_ERR_INVALID_ARG;
  unsigned int* err = error_word();
  if (!err) return cuda_failed("device error word lookup failed");
  char* ws = static_cast<char*>(workspace);
  int32_t* tables_v = reinterpret_cast<int32_t*>(ws);
  int32_t* ctx_v = reinterpret_cast<int32_t*>(ws + multi_tables_bytes(shape, num_query_tokens));
  const long long head = multi_head_bytes(shape, num_query_tokens);
  int launched = 0;
  cudaError_t ce = pa::launch_expand_queries(block_tables, context_lens, shape->num_seqs,
                                             num_query_tokens, shape->max_blocks_per_seq,
                                             shape->block_size, max_context_len, tables_v, ctx_v,
                                             err, reinterpret_cast<cudaStream_t>(stream), &launched);
  count_launches(launched);
  if (ce != cudaSuccess) return cuda_failed(ce);
  return decode_impl(q, k_cache, v_cache, nullptr, nullptr, tables_v, ctx_v, scale, out, &e,
                     max_context_len, ws + head, workspace_bytes - (size_t)head, stream, 1, true);
}

pa_status pa_decode_fp8(const void* q, const void* k_cache, const void* v_cache,
                        const float* k_scale, const float* v_scale, const int32_t* block_tables,
                        const int32_t* context_lens, float scale, void* out, const pa_shape* shape,
                        int32_t max_context_len, void* workspace, size_t workspace_bytes,
                        pa_stream_t stream) {
  if (!k_scale) return PA_ERR_INVALID_ARG;
  return decode_impl(q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, scale, out,
                     shape, max_context_len, workspace, workspace_bytes, stream);
}

pa_status pa_cache_append(const void* k, const void* v, const int32_t* slot_mapping,
                          int32_t num_tokens, void* k_cache, void* v_cache, const pa_shape* shape,
                          pa_stream_t stream) {
  pa_status st = check_pool_shape(shape);
  if (st != PA_OK) return st;
  if (num_tokens < 0) return PA_ERR_INVALID_ARG;
  if (num_tokens == 0) return PA_OK;
  if (shape->cache_format != PA_CACHE_AS_DTYPE) return PA_ERR_INVALID_ARG;  // pa_cache_append_fp8
  if (!k || !v || !slot_mapping || !k_cache || !v_cache) return PA_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache) ||
      (reinterpret_cast<uintptr_t>(slot_mapping) & 3u))
    return PA_ERR_INVALID_ARG;
  const int row_bytes = shape->num_kv_heads * shape->head_dim * 2;
  unsigned int* err = error_word();
  if (!err) return cuda_failed("device error word lookup failed");
  int launched = 0;
  cudaError_t e = pa::launch_cache_append(k, v, slot_mapping, num_tokens, k_cache, v_cache,
                                          (long long)shape->num_blocks * shape->block_size,
                                          row_bytes, err, reinterpret_cast<cudaStream_t>(stream),
                                          &launched);
  count_launches(launched);
  return e == cudaSuccess ? PA_OK : cuda_failed(e);
}

pa_status pa_cache_append_fp8(const void* k, const void* v, const int32_t* slot_mapping,
                              int32_t num_tokens, void* k_cache, void* v_cache,
                              const float* k_scale, const float* v_scale, const pa_shape* shape,
                              pa_stream_t stream) {
  pa_status st = check_pool_shape(shape);
  if (st != PA_OK) return st;
  if (shape->cache_format != PA_CACHE_FP8_E4M3) return PA_ERR_INVALID_ARG;
  if (num_tokens < 0) return PA_ERR_INVALID_ARG;
  if (num_tokens == 0) return PA_OK;
  if (!k || !v || !slot_mapping || !k_cache || !v_cache || !k_scale || !v_scale)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache) ||
      (reinterpret_cast<uintptr_t>(slot_mapping) & 3u) ||
      (reinterpret_cast<uintptr_t>(k_scale) & 3u) || (reinterpret_cast<uintptr_t>(v_scale) & 3u))
    return PA_ERR_INVALID_ARG;
  unsigned int* err = error_word();
  if (!err) return cuda_failed("device error word lookup failed");
  int launched = 0;
  cudaError_t e = pa::launch_cache_append_fp8(
      k, v, slot_mapping, num_tokens, k_cache, v_cache,
      (long long)shape->num_blocks * shape->block_size, shape->dtype, shape->num_kv_heads,
      shape->head_dim, k_scale, v_scale, err, reinterpret_cast<cudaStream_t>(stream), &launched);
  count_launches(launched);
  return e == cudaSuccess ? PA_OK : cuda_failed(e);
}

pa_status pa_copy_blocks(const int32_t* src_dst_pairs, int32_t num_pairs, void* k_cache,
                         void* v_cache, const pa_shape* shape, pa_stream_t stream) {
  pa_status st = check_pool_shape(shape);
  if (st != PA_OK) return st;
  if (num_pairs < 0) return PA_ERR_INVALID_ARG;
  if (num_pairs == 0) return PA_OK;
  if (num_pairs > 65535) return PA_ERR_UNSUPPORTED;
  if (!src_dst_pairs || !k_cache || !v_cache) return PA_ERR_INVALID_ARG;
  if (!aligned16(k_cache) || !aligned16(v_cache) || (reinterpret_cast<uintptr_t>(src_dst_pairs) & 3u))
    return PA_ERR_INVALID_ARG;
  const long long block_bytes = (long long)shape->block_size * shape->num_kv_heads *
                                shape->head_dim * cache_elem_bytes(shape);
  unsigned int* err = error_word();
  if (!err) return cuda_failed("device error word lookup failed");
  int launched = 0;
  cudaError_t e = pa::launch_copy_blocks(src_dst_pairs, num_pairs, k_cache, v_cache,
                                         shape->num_blocks, k_cache, v_cache, shape->num_blocks,
                                         block_bytes, err, reinterpret_cast<cudaStream_t>(stream),
                                         &launched);
  count_launches(launched);
  return e == cudaSuccess ? PA_OK : cuda_failed(e);
}

pa_status pa_swap_blocks(const int32_t* src_dst_pairs, int32_t num_pairs, const void* src_k,
                         const void* src_v, int32_t src_num_blocks, void* dst_k, void* dst_v,
                         int32_t dst_num_blocks, const pa_shape* shape, pa_stream_t stream) {
  pa_status st = check_pool_shape(shape);
  if (st != PA_OK) return st;
  if (num_pairs < 0 || src_num_blocks < 0 || dst_num_blocks < 0) return PA_ERR_INVALID_ARG;
  if (num_pairs == 0) return PA_OK;
  if (num_pairs > 65535) return PA_ERR_UNSUPPORTED;
  if (!src_dst_pairs || !src_k || !src_v || !dst_k || !dst_v) return PA_ERR_INVALID_ARG;
  if (!aligned16(src_k) || !aligned16(src_v) || !aligned16(dst_k) || !aligned16(dst_v) ||
      (reinterpret_cast<uintptr_t>(src_dst_pairs) & 3u))
    return PA_ERR_INVALID_ARG;
  // the pools must not overlap: a swap moves blocks between two pools
  const long long block_bytes = (long long)shape->block_size * shape->num_kv_heads *
                                shape->head_dim * cache_elem_bytes(shape);
  auto disjoint = [&](const void* a, long long na, const void* b, long long nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x + (uintptr_t)(na * block_bytes) <= y || y + (uintptr_t)(nb * block_bytes) <= x;
  };
  if (!disjoint(src_k, src_num_blocks, dst_k, dst_num_blocks) ||
      !disjoint(src_v, src_num_blocks, dst_v, dst_num_blocks))
    return PA_ERR_INVALID_ARG;
  // every pool must be memory the device can address at the same pointer:
  // device memory, managed memory, or pinned host memory mapped under
  // unified addressing (never pageable host memory)
  for (const void* p : {src_k, src_v, static_cast<const void*>(dst_k), static_cast<const void*>(dst_v)}) {
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
      cudaGetLastError();
      return PA_ERR_INVALID_ARG;
    }
    if (attr.type == cudaMemoryTypeUnregistered) return PA_ERR_INVALID_ARG;
    if (attr.type == cudaMemoryTypeHost && attr.devicePointer != p) return PA_ERR_INVALID_ARG;
  }
  unsigned int* err = error_word();
  if (!err) return cuda_failed("device error word lookup failed");
  int launched = 0;
  cudaError_t e = pa::launch_copy_blocks(src_dst_pairs, num_pairs, src_k, src_v, src_num_blocks,
                                         dst_k, dst_v, dst_num_blocks, block_bytes, err,
                                         reinterpret_cast<cudaStream_t>(stream), &launched);
  count_launches(launched);
  return e == cudaSuccess ? PA_OK : cuda_failed(e);
}

int pa_decode_partition_tokens(const pa_shape* shape) {
  const pa_status st = check_decode_shape(shape, 0);
  if (st != PA_OK) return -(int)st;
  return effective_partition(shape);
}

int pa_decode_resolved_variant(const pa_shape* shape) {
  const pa_status st = check_decode_shape(shape, 0);
  if (st != PA_OK) return -(int)st;
  if (shape->shared_prefix) return PA_DECODE_RESOLVED_SHARED_PREFIX;
  return use_tensor_cores(shape) ? PA_DECODE_TENSOR_CORES : PA_DECODE_CUDA_CORES;
}

pa_status pa_last_device_error(pa_stream_t stream, uint32_t* bits_out) {
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_failed(e);
  unsigned int bits = 0;
  const unsigned int zero = 0;
  if ((e = cudaMemcpyFromSymbol(&bits, g_device_error, sizeof bits)) != cudaSuccess) return cuda_failed(e);
  if (bits && (e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero)) != cudaSuccess)
    return cuda_failed(e);
  if (bits_out) *bits_out = bits;
  return bits ? PA_ERR_DEVICE_CHECK : PA_OK;
}

const char* pa_status_string(pa_status s) {
  switch (s) {
    case PA_OK: return "ok";
    case PA_ERR_INVALID_ARG: return "invalid argument";
    case PA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case PA_ERR_CUDA: return "CUDA error";
    case PA_ERR_OOM: return "out of blocks";
    case PA_ERR_DEVICE_CHECK: return "device-side check failed";
  }
  return "unknown status";
}

const char* pa_last_cuda_error(void) { return t_last_cuda_error; }

uint64_t pa_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

#define PA_STR2(x) #x
#define PA_STR(x) PA_STR2(x)
const char* pa_build_info(void) { return "libpa 0.1 for sm_100a, CUDA runtime " PA_STR(CUDART_VERSION); }

}  // extern "C"
