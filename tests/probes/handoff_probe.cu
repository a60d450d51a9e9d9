// Latency of one stamped hand-off between CTAs, measured in isolation: the building block of
// the persistent decode kernel's phase boundaries, where a producer CTA publishes 64-bit
// {value, epoch} words with relaxed GPU-scope stores and every consumer CTA loads the words it
// needs with relaxed GPU-scope loads until all carry the expected epoch.
//
// mode 0 (ping-pong): CTA 0 and CTA p pass one word back and forth `rounds` times, for every
// partner p in turn; out[p] = ns per round trip (two one-way hand-offs), measured by CTA 0 with
// %globaltimer; out[0] = -1.  The SM of every CTA goes to sm[] (placement is the scheduler's).
// mode 1 (all-to-all): every CTA publishes `width` words per round and then waits for the words
// of all CTAs (the shape of a phase boundary: a d-long vector written in slices and read whole
// by every CTA); out[c] = ns per round seen by CTA c.  mode 2: the same reads of words published
// before the timed rounds, i.e. the consumer's load alone.
// Every wait is bounded; a wait that runs out sets *fail and its CTA leaves.  The launch is
// cooperative, so every CTA is resident before any waits.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr long long kLimit = 1ll << 24;

__device__ __forceinline__ void st_word(uint64_t* p, uint32_t v, uint32_t ep) {
  const uint64_t w = ((uint64_t)ep << 32) | (uint64_t)v;
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}
__device__ __forceinline__ uint64_t ld_word(const uint64_t* p) {
  uint64_t w;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(w) : "l"(p) : "memory");
  return w;
}
__device__ __forceinline__ uint64_t gtime() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ bool wait_word(const uint64_t* p, uint32_t ep, int* fail) {
  for (long long i = 0; i < kLimit; ++i)
    if ((uint32_t)(ld_word(p) >> 32) >= ep) return true;   // a CTA may already be a round ahead
  atomicExch(fail, 1);
  return false;
}

__global__ void probe_kernel(int mode, int rounds, int width, uint64_t* words, double* out, int* sm, int* fail) {
  const int c = blockIdx.x, G = gridDim.x, tid = threadIdx.x;
  if (tid == 0) {
    int s;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(s));
    sm[c] = s;
  }
  if (mode == 0) {
    if (tid != 0) return;
    // partner p uses words[2p] (CTA 0 -> p) and words[2p + 1] (p -> CTA 0)
    if (c == 0) {
      out[0] = -1.0;
      for (int p = 1; p < G; ++p) {
        const uint64_t t0 = gtime();
        bool ok = true;
        for (int r = 1; r <= rounds && ok; ++r) {
          st_word(words + 2 * p, 0u, (uint32_t)r);
          ok = wait_word(words + 2 * p + 1, (uint32_t)r, fail);
        }
        out[p] = ok ? (double)(gtime() - t0) / rounds : -1.0;
        if (!ok) return;
      }
    } else {
      for (int r = 1; r <= rounds; ++r) {
        if (!wait_word(words + 2 * c, (uint32_t)r, fail)) return;
        st_word(words + 2 * c + 1, 0u, (uint32_t)r);
      }
    }
    return;
  }
  // mode 1: slices of `width` words per CTA, every CTA reads all G * width of them; mode 2: the
  // same reads of words that are all published before the timed rounds (the load alone).
  // A thread loads its words 8 at a time, all 8 in flight, then re-reads only the stale ones.
  __shared__ int bad;
  if (tid == 0) bad = 0;
  __syncthreads();
  const int total = G * width;
  if (mode == 2) {
    for (int i = tid; i < width; i += blockDim.x) st_word(words + (size_t)c * width + i, (uint32_t)c, 1u);
  }
  uint64_t t0 = 0;
  for (int r = 1; r <= rounds; ++r) {
    if (r == 2) t0 = gtime();   // the first pass lines the CTAs up
    const uint32_t ep = mode == 2 ? 1u : (uint32_t)r;
    if (mode == 1)
      for (int i = tid; i < width; i += blockDim.x) st_word(words + (size_t)c * width + i, (uint32_t)c, ep);
    for (int i0 = tid; i0 < total; i0 += 8 * blockDim.x) {
      uint64_t w[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int i = i0 + j * blockDim.x;
        w[j] = i < total ? ld_word(words + i) : ((uint64_t)ep << 32);
      }
      for (long long it = 0;; ++it) {
        bool stale = false;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int i = i0 + j * blockDim.x;
          if ((uint32_t)(w[j] >> 32) < ep) {
            stale = true;
            w[j] = ld_word(words + i);
          }
        }
        if (!stale) break;
        if (it == kLimit) {
          atomicExch(fail, 1);
          bad = 1;
          break;
        }
      }
    }
    __syncthreads();
    if (bad) return;
  }
  if (tid == 0 && rounds > 1) out[c] = (double)(gtime() - t0) / (rounds - 1);
}

}  // namespace

// Returns 0 on success, 1 if a wait ran out, 2 on a CUDA error.  out[ctas], sm[ctas].
extern "C" int handoff_probe(int mode, int ctas, int rounds, int width, double* out, int* sm) {
  if (ctas < 2 || rounds < 2 || mode < 0 || mode > 2 || (mode > 0 && width < 1)) return 2;
  uint64_t* words = nullptr;
  double* d_out = nullptr;
  int *d_sm = nullptr, *d_fail = nullptr;
  const size_t nwords = mode == 0 ? (size_t)2 * ctas : (size_t)ctas * width;
  int rc = 2;
  if (cudaMalloc(&words, nwords * 8) == cudaSuccess && cudaMalloc(&d_out, ctas * sizeof(double)) == cudaSuccess &&
      cudaMalloc(&d_sm, ctas * sizeof(int)) == cudaSuccess && cudaMalloc(&d_fail, sizeof(int)) == cudaSuccess &&
      cudaMemset(words, 0, nwords * 8) == cudaSuccess && cudaMemset(d_fail, 0, sizeof(int)) == cudaSuccess &&
      cudaMemset(d_out, 0, ctas * sizeof(double)) == cudaSuccess) {
    void* args[] = {&mode, &rounds, &width, &words, &d_out, &d_sm, &d_fail};
    const dim3 block(mode == 0 ? 32 : 256);   // mode 0 uses thread 0 of each CTA
    if (cudaLaunchCooperativeKernel(reinterpret_cast<void*>(probe_kernel), dim3(ctas), block, args, 0, 0) ==
            cudaSuccess &&
        cudaDeviceSynchronize() == cudaSuccess) {
      int fail = 0;
      if (cudaMemcpy(out, d_out, ctas * sizeof(double), cudaMemcpyDeviceToHost) == cudaSuccess &&
          cudaMemcpy(sm, d_sm, ctas * sizeof(int), cudaMemcpyDeviceToHost) == cudaSuccess &&
          cudaMemcpy(&fail, d_fail, sizeof(int), cudaMemcpyDeviceToHost) == cudaSuccess)
        rc = fail ? 1 : 0;
    }
  }
  cudaFree(words);
  cudaFree(d_out);
  cudaFree(d_sm);
  cudaFree(d_fail);
  return rc;
}
