// pa_noalloc.cu -- pa_decode for callers that cannot allocate device memory.
//
// pa_decode() needs a split-K workspace whenever a context spans more than
// one partition, and leaves it to the caller to allocate.  Some callers have
// no way to do that: code running as a plug-in inside a host runtime that owns
// every byte of device memory and hands its plug-ins no allocator, or a
// latency-critical decode loop that must never call cudaMalloc (which can
// synchronise the whole device) once it is running.  pa_decode_noalloc()
// serves them from a fixed scratch array compiled into this library instead.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds PA_NOALLOC_SCRATCH_BYTES of it until the process exits.  In
// host code its name is only a stand-in for the symbol, never a device
// address: the address is looked up once per device with
// cudaGetSymbolAddress(), with that device current, and handed to the
// kernels as their workspace pointer.
#include <cuda_runtime.h>

#include <mutex>

#include "pa.h"

namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[PA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

// Device address of g_decode_scratch on the current device (nullptr if the
// lookup failed).  Looked up on the first call per device, then cached.
unsigned char* scratch_on_current_device() {
  static std::mutex mu;
  static unsigned char* addr[kMaxDevices] = {};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    unsigned char* p = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_decode_scratch) != cudaSuccess)
      return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace

extern "C" pa_status pa_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                       const int32_t* block_tables, const int32_t* context_lens,
                                       float scale, void* out, const pa_shape* shape,
                                       int32_t max_context_len, pa_stream_t stream) {
  if (!shape) return PA_ERR_INVALID_ARG;
  const size_t need = pa_decode_workspace_bytes(shape, max_context_len);
  if (need > (size_t)PA_NOALLOC_SCRATCH_BYTES) return PA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (need > 0) {
    scratch = scratch_on_current_device();
    if (!scratch) return PA_ERR_CUDA;
  }
  // The split-K workspace needs no initial contents: every slot the merge
  // reads is written by the same call's partition kernel.
  return pa_decode(q, k_cache, v_cache, block_tables, context_lens, scale, out, shape,
                   max_context_len, scratch, need > 0 ? (size_t)PA_NOALLOC_SCRATCH_BYTES : 0,
                   stream);
}
