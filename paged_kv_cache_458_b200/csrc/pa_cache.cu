// pa_cache.cu -- the two cache-maintenance kernels of the paged KV cache.
//
// append: the "update KV cache" step of each decode iteration (5688vip.com
//   vLLM notes, section 2.1) writes the new token's K and V rows into the slot
//   the block table reserved for it (zingnex.cn, "vLLM与PagedAttention深度剖析",
//   section 3.2 item 1: a block is taken only when a token crosses into it).
// copy:   copy-on-write of a shared block before one of its sharers writes
//   into it (same page, section 3.2 item 3).
//
// Both are byte copies in 16-byte vectors; pools are [NB][bs][Hkv][D], so one
// token's K row over all kv heads is one contiguous run of Hkv * D elements
// and one block is a contiguous run of bs * Hkv * D elements.
#include <cuda_runtime.h>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

// One CTA per token: copies row_bytes of K and of V.
__global__ void __launch_bounds__(256)
cache_append_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                    const int32_t* __restrict__ slot_mapping, uint4* __restrict__ k_cache,
                    uint4* __restrict__ v_cache, long long num_slots, int row_vecs,
                    unsigned int* err) {
  pdl_wait();  // a copy-on-write of this slot's block must land first
  pdl_launch_dependents();
  const int t = blockIdx.x;
  const long long slot = __ldg(slot_mapping + t);
  if (slot < 0) return;
  if (slot >= num_slots) {
    if (threadIdx.x == 0) report(err, kErrSlot);
    return;
  }
  const uint4* ks = k + (size_t)t * row_vecs;
  const uint4* vs = v + (size_t)t * row_vecs;
  uint4* kd = k_cache + slot * row_vecs;
  uint4* vd = v_cache + slot * row_vecs;
  for (int i = threadIdx.x; i < row_vecs; i += blockDim.x) {
    kd[i] = __ldg(ks + i);
    vd[i] = __ldg(vs + i);
  }
}

// Append into an E4M3 cache.  One CTA per token; each thread converts 8
// consecutive elements (16 bytes in, 8 bytes out) per step: x / scale[head]
// in fp32 (IEEE division, round to nearest), then the nearest E4M3 code,
// ties to even, saturating at 448.
template <typename T>
__global__ void __launch_bounds__(256)
cache_append_fp8_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                        const int32_t* __restrict__ slot_mapping, uint2* __restrict__ k_cache,
                        uint2* __restrict__ v_cache, long long num_slots, int head_dim,
                        int row_vecs, const float* __restrict__ k_scale,
                        const float* __restrict__ v_scale, unsigned int* err) {
  pdl_wait();  // a copy-on-write of this slot's block must land first
  pdl_launch_dependents();
  const int t = blockIdx.x;
  const long long slot = __ldg(slot_mapping + t);
  if (slot < 0) return;
  if (slot >= num_slots) {
    if (threadIdx.x == 0) report(err, kErrSlot);
    return;
  }
  for (int i = threadIdx.x; i < row_vecs; i += blockDim.x) {
    const int h = (i * 8) / head_dim;  // 8 elements never straddle two heads
    const float ks = __ldg(k_scale + h), vs = __ldg(v_scale + h);
    const uint4 xk = __ldg(k + (size_t)t * row_vecs + i), xv = __ldg(v + (size_t)t * row_vecs + i);
    uint2 ok, ov;
    uint32_t* pk = &ok.x;
    uint32_t* pv = &ov.x;
    const uint32_t wk[4] = {xk.x, xk.y, xk.z, xk.w}, wv[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
    for (int w = 0; w < 4; w += 2) {
      const float2 k0 = Elem<T>::to_f2(wk[w]), k1 = Elem<T>::to_f2(wk[w + 1]);
      const float2 v0 = Elem<T>::to_f2(wv[w]), v1 = Elem<T>::to_f2(wv[w + 1]);
      const uint32_t ck = (uint32_t)__nv_cvt_float2_to_fp8x2(
                              make_float2(__fdiv_rn(k0.x, ks), __fdiv_rn(k0.y, ks)), __NV_SATFINITE,
                              __NV_E4M3) |
                          ((uint32_t)__nv_cvt_float2_to_fp8x2(
                               make_float2(__fdiv_rn(k1.x, ks), __fdiv_rn(k1.y, ks)), __NV_SATFINITE,
                               __NV_E4M3)
                           << 16);
      const uint32_t cv = (uint32_t)__nv_cvt_float2_to_fp8x2(
                              make_float2(__fdiv_rn(v0.x, vs), __fdiv_rn(v0.y, vs)), __NV_SATFINITE,
                              __NV_E4M3) |
                          ((uint32_t)__nv_cvt_float2_to_fp8x2(
                               make_float2(__fdiv_rn(v1.x, vs), __fdiv_rn(v1.y, vs)), __NV_SATFINITE,
                               __NV_E4M3)
                           << 16);
      pk[w / 2] = ck;
      pv[w / 2] = cv;
    }
    k_cache[slot * row_vecs + i] = ok;
    v_cache[slot * row_vecs + i] = ov;
  }
}

// grid.x = pieces of a block, grid.y = pair.  Each CTA copies kPiece vectors
// of block src of the source K pool and of the V pool into block dst of the
// destination pools.  Copy-on-write passes the same pool as source and
// destination; swap passes a device pool and a host pool the device can
// address (pinned and mapped), in either order.
constexpr int kCopyThreads = 256;
constexpr int kCopyUnroll = 4;
constexpr int kPiece = kCopyThreads * kCopyUnroll;

__global__ void __launch_bounds__(kCopyThreads)
copy_blocks_kernel(const int32_t* __restrict__ pairs, const uint4* src_k, const uint4* src_v,
                   int src_blocks, uint4* dst_k, uint4* dst_v, int dst_blocks, long long block_vecs,
                   unsigned int* err) {
  pdl_wait();
  pdl_launch_dependents();
  const int i = blockIdx.y;
  const int src = __ldg(pairs + 2 * i), dst = __ldg(pairs + 2 * i + 1);
  if (src < 0 || src >= src_blocks || dst < 0 || dst >= dst_blocks) {
    if (blockIdx.x == 0 && threadIdx.x == 0) report(err, kErrPair);
    return;
  }
  const long long base = (long long)blockIdx.x * kPiece;
  const uint4* ks = src_k + src * block_vecs;
  const uint4* vs = src_v + src * block_vecs;
  uint4* kd = dst_k + dst * block_vecs;
  uint4* vd = dst_v + dst * block_vecs;
  uint4 rk[kCopyUnroll], rv[kCopyUnroll];
#pragma unroll
  for (int u = 0; u < kCopyUnroll; ++u) {
    const long long e = base + u * kCopyThreads + threadIdx.x;
    if (e < block_vecs) { rk[u] = ks[e]; rv[u] = vs[e]; }
  }
#pragma unroll
  for (int u = 0; u < kCopyUnroll; ++u) {
    const long long e = base + u * kCopyThreads + threadIdx.x;
    if (e < block_vecs) { kd[e] = rk[u]; vd[e] = rv[u]; }
  }
}

cudaError_t launch_cache_append(const void* k, const void* v, const int32_t* slot_mapping,
                                int num_tokens, void* k_cache, void* v_cache, long long num_slots,
                                int row_bytes, unsigned int* err, cudaStream_t stream,
                                int* launches) {
  if (num_tokens == 0) return cudaSuccess;
  const int row_vecs = row_bytes / 16;
  const int threads = row_vecs >= 256 ? 256 : ((row_vecs + 31) / 32) * 32;
  cudaError_t e = launch_pdl(cache_append_kernel, dim3(num_tokens), dim3(threads), 0, stream,
                             static_cast<const uint4*>(k), static_cast<const uint4*>(v),
                             slot_mapping, static_cast<uint4*>(k_cache),
                             static_cast<uint4*>(v_cache), num_slots, row_vecs, err);
  if (e == cudaSuccess) ++*launches;
  return e;
}

cudaError_t launch_cache_append_fp8(const void* k, const void* v, const int32_t* slot_mapping,
                                    int num_tokens, void* k_cache, void* v_cache,
                                    long long num_slots, int dtype, int num_kv_heads, int head_dim,
                                    const float* k_scale, const float* v_scale, unsigned int* err,
                                    cudaStream_t stream, int* launches) {
  if (num_tokens == 0) return cudaSuccess;
  const int row_vecs = num_kv_heads * head_dim / 8;  // 8 elements per step
  const int threads = row_vecs >= 256 ? 256 : ((row_vecs + 31) / 32) * 32;
  auto* kern = dtype == 0 ? cache_append_fp8_kernel<__half> : cache_append_fp8_kernel<__nv_bfloat16>;
  cudaError_t e = launch_pdl(kern, dim3(num_tokens), dim3(threads), 0, stream,
                             static_cast<const uint4*>(k), static_cast<const uint4*>(v), slot_mapping,
                             static_cast<uint2*>(k_cache), static_cast<uint2*>(v_cache), num_slots,
                             head_dim, row_vecs, k_scale, v_scale, err);
  if (e == cudaSuccess) ++*launches;
  return e;
}

cudaError_t launch_copy_blocks(const int32_t* pairs, int num_pairs, const void* src_k,
                               const void* src_v, int src_blocks, void* dst_k, void* dst_v,
                               int dst_blocks, long long block_bytes, unsigned int* err,
                               cudaStream_t stream, int* launches) {
  if (num_pairs == 0) return cudaSuccess;
  const long long block_vecs = block_bytes / 16;
  const long long pieces = (block_vecs + kPiece - 1) / kPiece;
  if (num_pairs > 65535 || pieces > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  dim3 grid((unsigned)pieces, (unsigned)num_pairs);
  cudaError_t e = launch_pdl(copy_blocks_kernel, grid, dim3(kCopyThreads), 0, stream, pairs,
                             static_cast<const uint4*>(src_k), static_cast<const uint4*>(src_v),
                             src_blocks, static_cast<uint4*>(dst_k), static_cast<uint4*>(dst_v),
                             dst_blocks, block_vecs, err);
  if (e == cudaSuccess) ++*launches;
  return e;
}

}  // namespace pa
