// Kernel launch helper: cudaLaunchKernelEx with optional programmatic stream
// serialisation (PDL), and a once-per-kernel opt-in to large dynamic shared memory.
#pragma once
#include <cuda_runtime.h>
#include <atomic>
#include "ms_kernels.h"

namespace ms {

// Kernels launched by this process through launch_k (all threads).
std::atomic<unsigned long long>& launch_counter();

template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(const Launch& L, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                            Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = L.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = L.pdl ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  if (e == cudaSuccess) launch_counter().fetch_add(1, std::memory_order_relaxed);
  return e;
}

// Largest dynamic shared memory a CTA may use on sm_100 (227 KiB).
constexpr size_t kMaxDynSmem = 227 * 1024;

// Raise the kernel's dynamic shared memory limit when it needs more than 48 KiB.  Done once
// per device before any launch (never during stream capture).
// `bytes` is capped at the device's opt-in limit minus the kernel's static shared memory.
template <typename... KArgs>
inline cudaError_t allow_smem(void (*kernel)(KArgs...), size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  int dev = 0, optin = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  cudaFuncAttributes fa;
  if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, reinterpret_cast<const void*>(kernel));
  if (e != cudaSuccess) return e;
  const size_t most = (size_t)optin > fa.sharedSizeBytes ? (size_t)optin - fa.sharedSizeBytes : 0;
  if (bytes > most) bytes = most;
  return cudaFuncSetAttribute(reinterpret_cast<const void*>(kernel),
                              cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
}

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

}  // namespace ms
