// Device helpers shared by the kernels: status word, bulk copies into shared memory
// tracked by an mbarrier (bounded waits), programmatic dependent launch, reductions.
#pragma once
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <stdint.h>
#include "ms_kernels.h"

namespace ms {

constexpr unsigned kErrToken = kErrTokenBit;
constexpr unsigned kErrTimeout = kErrTimeoutBit;
constexpr unsigned kErrShape = kErrShapeBit;

// Iteration limit for every spin on an mbarrier: far above any legitimate wait
// (a few microseconds), far below a hang (seconds at most).
constexpr long long kSpinLimit = 1ll << 22;

__device__ __forceinline__ void flag_error(unsigned* status, unsigned bit) {
  if (status) atomicOr(status, bit);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- programmatic dependent launch ---------------------------------------------------
// Everything a kernel reads from its immediate predecessor must come after pdl_wait();
// data written two or more launches earlier may be read before it.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- mbarrier + bulk copy (global -> shared) ------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
// Bulk copy of `bytes` (multiple of 16, both addresses 16-byte aligned) into this CTA's
// shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}" : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for phase `parity` of `bar`.  Returns false (and flags kErrTimeout) if the
// limit ran out; the caller then skips its work and returns.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned* status) {
  for (long long i = 0; i < kSpinLimit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  flag_error(status, kErrTimeout);
  return false;
}

// Issue a (possibly large) contiguous copy as pieces of at most 64 KiB on one barrier.
// The caller has already posted the total with mbar_expect_tx.
__device__ __forceinline__ void bulk_g2s_pieces(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  const uint32_t piece = 65536;
  char* d = static_cast<char*>(dst);
  const char* s = static_cast<const char*>(src);
  for (uint32_t off = 0; off < bytes; off += piece) {
    uint32_t n = bytes - off < piece ? bytes - off : piece;
    bulk_g2s(d + off, s + off, n, bar);
  }
}

// ---- reductions ---------------------------------------------------------------------
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

// Sum over the whole block (blockDim.x a multiple of 32, at most 1024).  `red` holds 32
// floats of shared memory.  Every thread gets the result.
__device__ __forceinline__ float block_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = lane < nw ? red[lane] : 0.f;
  return warp_sum(t);
}

// Greedy choice order: larger value first, lower index on ties.
__device__ __forceinline__ bool argmax_better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}
// (value, index) argmax over a warp; every lane gets the result.
__device__ __forceinline__ void warp_argmax(float& v, int& i) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float v2 = __shfl_xor_sync(0xffffffffu, v, o);
    const int i2 = __shfl_xor_sync(0xffffffffu, i, o);
    if (argmax_better(v2, i2, v, i)) {
      v = v2;
      i = i2;
    }
  }
}

// fp32 INT4 nibble -> exact float of q = u - 8 (u in [0, 15]): 2^23 + u has u in its low
// mantissa bits, subtracting 2^23 + 8 is exact.
__device__ __forceinline__ float nib_to_q(uint32_t u4) {
  return __int_as_float(0x4B000000u | u4) - 8388616.0f;
}

// ---- KV cache elements: fp32 (KV = 0) or IEEE half (KV = 1, round to nearest even) ---------
// Four consecutive elements e .. e + 3 of a cache row as floats (16-byte / 8-byte loads,
// through L2: the rows may have been written by another CTA of the same kernel).
template <int KV>
__device__ __forceinline__ float4 kv_load4(const void* base, size_t e) {
  if (KV == 0) return __ldcg(reinterpret_cast<const float4*>(static_cast<const float*>(base) + e));
  const uint2 u = __ldcg(reinterpret_cast<const uint2*>(static_cast<const __half*>(base) + e));
  const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
  const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
template <int KV>
__device__ __forceinline__ void kv_store(void* base, size_t e, float v) {
  if (KV == 0) static_cast<float*>(base)[e] = v;
  else static_cast<__half*>(base)[e] = __float2half_rn(v);
}

__device__ __forceinline__ float gelu_erf(float u) {
  return 0.5f * u * (1.0f + erff(u * 0.70710678118654752f));
}

}  // namespace ms
