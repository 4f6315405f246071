// pa_common.cuh -- device-side helpers shared by the libpa kernels (sm_100a).
//
// * element traits for fp16 / bf16 storage with fp32 arithmetic;
// * the device error word the kernels report bad indices and expired waits in
//   (no kernel ever traps: a failed check records a bit and skips the access);
// * thin inline-PTX wrappers for mbarrier and the tiled TMA load
//   (cp.async.bulk.tensor), all waits bounded by a wall-clock limit.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace pa {

// Bits of the device error word.
enum DeviceErrorBits : unsigned int {
  kErrBlockId = 1u << 0,      // a block-table entry below the context is outside the pool
  kErrContextLen = 1u << 1,   // a context length is negative or above the host's bound
  kErrSlot = 1u << 2,         // an append slot is outside the pool
  kErrPair = 1u << 3,         // a copy pair names a block outside the pool
  kErrWaitTimeout = 1u << 4,  // an mbarrier wait ran past its time limit
  kErrConfig = 1u << 5,       // a kernel could not lay out its shared memory (did nothing)
};

// Kernels receive the address of the per-device error word (read and
// cleared by pa_last_device_error()) and OR bits into it.
__device__ __forceinline__ void report(unsigned int* err, unsigned int bits) { atomicOr(err, bits); }

// ---------------------------------------------------------------------------
// element traits

template <typename T> struct Elem;

template <> struct Elem<__half> {
  // two packed elements -> two floats
  static __device__ __forceinline__ float2 to_f2(uint32_t u) {
    __half2 h = *reinterpret_cast<__half2*>(&u);
    return __half22float2(h);
  }
  static __device__ __forceinline__ uint16_t from_f(float x) {
    __half h = __float2half_rn(x);
    return *reinterpret_cast<uint16_t*>(&h);
  }
};

template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float2 to_f2(uint32_t u) {
    // bf16 is the top half of an fp32: widening is a shift / mask
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
  }
  static __device__ __forceinline__ uint16_t from_f(float x) {
    __nv_bfloat16 b = __float2bfloat16_rn(x);
    return *reinterpret_cast<uint16_t*>(&b);
  }
};

// 8-bit E4M3 cache codes (one byte per element) and their widening.
struct Fp8E4M3 {};

// Two E4M3 codes (low byte first) -> two floats, exact (via the hardware
// E4M3 -> f16 conversion, which every E4M3 value survives unchanged).
__device__ __forceinline__ float2 e4m3x2_to_f2(uint16_t u) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(u), __NV_E4M3);
  return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

// ---------------------------------------------------------------------------
// time and shared-memory addressing

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Make barrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

// Raise the transaction count of the current phase without arriving: the
// phase then completes once its arrivals are in and those bytes have landed.
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t phase) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(phase)
      : "memory");
  return ok != 0;
}

// Non-blocking probe: has phase `phase` completed?  (test_wait never suspends.)
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t phase) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(phase)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Wall-clock limit of any single wait.  A TMA load of a few KB completes in
// microseconds; two seconds means the copy will never land.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Wait for the barrier's phase `phase` to complete.  Returns false (after
// recording kErrWaitTimeout) if it has not completed within kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t phase, unsigned int* err) {
  if (mbar_try_wait(bar, phase)) return true;
  const uint64_t t0 = globaltimer_ns();
  uint32_t spins = 0;
  while (!mbar_try_wait(bar, phase)) {
    if ((++spins & 255u) == 0 && globaltimer_ns() - t0 > kWaitLimitNs) {
      report(err, kErrWaitTimeout);
      return false;
    }
  }
  return true;
}

// As mbar_wait, but also gives up (returning false) once *abort has been set
// by another warp of the CTA; a timeout sets *abort itself.
__device__ __forceinline__ bool mbar_wait_or_abort(uint32_t bar, uint32_t phase, unsigned int* err,
                                                   volatile int* abort) {
  if (mbar_try_wait(bar, phase)) return true;
  const uint64_t t0 = globaltimer_ns();
  uint32_t spins = 0;
  while (!mbar_try_wait(bar, phase)) {
    if ((++spins & 63u) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        report(err, kErrWaitTimeout);
        *abort = 1;
        return false;
      }
    }
  }
  return true;
}

// Named barrier `id` (> 0) over `threads` threads (a multiple of 32).
__device__ __forceinline__ void named_barrier(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Named barrier that also ORs `flag` over its threads: every participant gets
// the same answer, whatever other warps write to shared memory meanwhile.
__device__ __forceinline__ bool named_barrier_or(int id, int threads, bool flag) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred pin, pout;\n\t"
      "setp.ne.u32 pin, %1, 0;\n\t"
      "barrier.red.or.pred pout, %2, %3, pin;\n\t"
      "selp.u32 %0, 1, 0, pout;\n\t}"
      : "=r"(out)
      : "r"((uint32_t)flag), "r"(id), "r"(threads)
      : "memory");
  return out != 0;
}

// ---------------------------------------------------------------------------
// TMA: tiled 3-D load global -> shared, completion counted on an mbarrier.
// The tensor map lives in kernel parameter space (__grid_constant__).

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* tmap, uint32_t bar, int c0,
                                            int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// ---------------------------------------------------------------------------
// programmatic dependent launch.  Every kernel of this library is launched
// with programmatic stream serialisation: it may start while the kernel
// before it on the stream is still running, so it first waits (pdl_wait)
// for that kernel to finish and its writes to be visible, before touching
// global memory, and then lets the kernel after it start early
// (pdl_launch_dependents).  A kernel before it that does not trigger (one
// not from this library) simply finishes first, as without the attribute.

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Host: launch `kern` with programmatic stream serialisation.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

}  // namespace pa
