// Shared device helpers of libflashsvd (sm_100a only).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/flashsvd.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libflashsvd is built for sm_100a only"
#endif

namespace fsvd {

typedef __nv_bfloat16 bf16;

// ------------------------------------------------------------ host side --

// Host-side count of kernel launches (eager) and replayed kernel nodes.
extern std::atomic<int64_t> g_launches;
// Last CUDA error seen by an entry point.
extern int g_last_cuda_error;

inline int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return FLASHSVD_OK;
  g_last_cuda_error = (int)e;
  return FLASHSVD_ERR_CUDA;
}

#define FSVD_TRY(expr)                     \
  do {                                     \
    int _st = (expr);                      \
    if (_st != FLASHSVD_OK) return _st;    \
  } while (0)

#define FSVD_CUDA(expr) FSVD_TRY(::fsvd::cuda_status(expr))

// Name and algorithmic work of one launch (for the optional profiler).
struct LaunchTag {
  const char* name;
  double bytes;   // bytes the operation must move to or from HBM
  double flops;
};

// Profiler hooks (prof.cu): when enabled, eager launches are bracketed by
// CUDA events on their stream; launches being captured are not.
bool prof_active(cudaStream_t s);
void prof_begin(cudaStream_t s);
void prof_end(const LaunchTag& tag, cudaStream_t s);

// Launch `kernel` with programmatic dependent launch enabled, so that its
// prologue (weight loads) can overlap the tail of the previous kernel on the
// stream; the kernel orders itself after that kernel with
// griddepcontrol.wait before it touches anything the previous kernel wrote.
template <typename... KArgs, typename... Args>
inline int launch_pdl(const LaunchTag& tag, void (*kernel)(KArgs...), dim3 grid,
                      dim3 block, size_t smem, cudaStream_t stream, Args&&... args) {
  const bool prof = prof_active(stream);
  if (prof) prof_begin(stream);
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
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e != cudaSuccess) return cuda_status(e);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (prof) prof_end(tag, stream);
  return FLASHSVD_OK;
}

// Raise `kernel`'s dynamic shared-memory limit to `bytes` on the current
// device.  cudaFuncSetAttribute applies to the device that is current when it
// runs, so the flag is kept per device (a call site keeps one `SmemAttrOnce`
// per kernel instantiation).  Two threads racing here both set the same
// value, which is harmless.
struct SmemAttrOnce {
  std::atomic<bool> done[64];
};

template <typename Kern>
inline int set_smem_once(SmemAttrOnce& once, Kern kernel, int bytes) {
  int dev = 0;
  FSVD_CUDA(cudaGetDevice(&dev));
  const bool tracked = dev >= 0 && dev < 64;
  if (tracked && once.done[dev].load(std::memory_order_acquire)) return FLASHSVD_OK;
  FSVD_CUDA(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  if (tracked) once.done[dev].store(true, std::memory_order_release);
  return FLASHSVD_OK;
}

// The same launch as launch_pdl, as a cooperative launch: every CTA of the
// grid is resident at once (the launch fails otherwise), which kernels whose
// CTAs wait on one another (grid barriers) rely on.
template <typename... KArgs, typename... Args>
inline int launch_pdl_coop(const LaunchTag& tag, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                           cudaStream_t stream, Args&&... args) {
  const bool prof = prof_active(stream);
  if (prof) prof_begin(stream);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeCooperative;
  attr[1].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e != cudaSuccess) return cuda_status(e);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (prof) prof_end(tag, stream);
  return FLASHSVD_OK;
}

// The same launch as launch_pdl with the grid in clusters of `cluster_x`
// CTAs along x (CTA pairs of the 2-SM tensor-core kernels).
template <typename... KArgs, typename... Args>
inline int launch_pdl_cluster(const LaunchTag& tag, int cluster_x, void (*kernel)(KArgs...), dim3 grid,
                              dim3 block, size_t smem, cudaStream_t stream, Args&&... args) {
  const bool prof = prof_active(stream);
  if (prof) prof_begin(stream);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster_x;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e != cudaSuccess) return cuda_status(e);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (prof) prof_end(tag, stream);
  return FLASHSVD_OK;
}

inline int ceil_div(int a, int b) { return (a + b - 1) / b; }
inline int round_up(int a, int b) { return ceil_div(a, b) * b; }
inline bool aligned16(const void* p) { return (((uintptr_t)p) & 15u) == 0; }

// ---------------------------------------------------------- device side --

__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// 16-byte streaming load of read-once data (weights): no L1 allocation.
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// bf16x2 packed in a 32-bit word -> two floats (exact).
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float bf2f(bf16 v) { return __bfloat162float(v); }
__device__ __forceinline__ bf16 f2bf(float v) { return __float2bfloat16_rn(v); }

__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
  __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&t);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Device status word codes (written by kernels whose bounded waits expire).
// DEV_STATUS_SCHEDULE: a kernel met a work split beyond its fixed limits
// (e.g. very unequal sequence lengths) and skipped that work.
enum : int { DEV_STATUS_OK = 0, DEV_STATUS_TIMEOUT = 1, DEV_STATUS_SCHEDULE = 2 };

}  // namespace fsvd
