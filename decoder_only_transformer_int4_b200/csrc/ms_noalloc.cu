// LM head + argmax for callers that cannot allocate device memory.
//
// ms_op_lm_head_argmax keeps its per-CTA partial results in a buffer it cudaMallocs on
// first use.  This variant keeps them in a fixed array compiled into the library instead,
// so the call itself allocates nothing.  The array exists once per device that loads the
// library and stays until the process exits.
#include <cuda_runtime.h>

#include <mutex>
#include <vector>

#include "../../include/ms.h"
#include "ms_kernels.h"

namespace {

constexpr int kStaticMaxCtas = 256;   // per-CTA result slots (the LM head uses one CTA per ~V/148 rows)
constexpr int kStaticMaxRows = 64;    // M, as for ms_op_lm_head_argmax
constexpr size_t kValBytes = sizeof(float) * kStaticMaxCtas * 64;
constexpr size_t kIdxBytes = sizeof(int) * kStaticMaxCtas * 64;
constexpr size_t kScratchBytes = kValBytes + kIdxBytes + 256;  // + the ticket counter

}  // namespace

// The scratch itself: per-CTA (value, index) pairs, then the last-CTA ticket counter.
static __device__ __align__(256) unsigned char g_lm_head_scratch[kScratchBytes];

namespace {

std::mutex g_mu;
std::vector<unsigned char*> g_addr;  // device address of g_lm_head_scratch, per device
std::vector<char> g_attrs;           // kernel attributes set, per device

// The host-side name g_lm_head_scratch is not a device address: resolve it once per
// device, with that device current.
cudaError_t scratch_of_current_device(unsigned char** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(g_mu);
  if ((int)g_addr.size() <= dev) {
    g_addr.resize(dev + 1, nullptr);
    g_attrs.resize(dev + 1, 0);
  }
  if (!g_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_lm_head_scratch);
    if (e != cudaSuccess) return e;
    g_addr[dev] = static_cast<unsigned char*>(p);
  }
  if (!g_attrs[dev]) {
    e = ms::init_attrs_gemv();
    if (e != cudaSuccess) return e;
    g_attrs[dev] = 1;
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

ms_status bad(ms_status s, const char* m) {
  ms::set_last_error(m);
  return s;
}

}  // namespace

extern "C" ms_status ms_op_lm_head_argmax_static(const float* x, int ldx, int M, int d, const float* gamma,
                                                 const float* beta, float eps, const float* W, int V, float* logits,
                                                 int32_t* argmax, void* stream) {
  if (!x || !W) return bad(MS_ERR_INVALID_ARG, "ms_op_lm_head_argmax_static: null pointer");
  if ((gamma == nullptr) != (beta == nullptr))
    return bad(MS_ERR_INVALID_ARG, "ms_op_lm_head_argmax_static: gamma and beta go together");
  if (M < 1 || M > kStaticMaxRows)
    return bad(MS_ERR_SHAPE, "ms_op_lm_head_argmax_static: M must be in [1, 64]");
  if (V < 1 || d < 128 || d % 128 != 0 || ldx < d || ldx % 4 != 0)
    return bad(MS_ERR_SHAPE, "ms_op_lm_head_argmax_static: bad sizes (d a multiple of 128, ldx >= d)");
  if (ms::lm_head_grid(V) > kStaticMaxCtas)
    return bad(MS_ERR_SHAPE, "ms_op_lm_head_argmax_static: V needs more CTAs than the fixed scratch holds (256)");
  unsigned char* base = nullptr;
  cudaError_t e = scratch_of_current_device(&base);
  if (e != cudaSuccess) return bad(MS_ERR_CUDA, cudaGetErrorString(e));
  ms::LmHeadWork w{reinterpret_cast<float*>(base), reinterpret_cast<int*>(base + kValBytes),
                   reinterpret_cast<unsigned*>(base + kValBytes + kIdxBytes)};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the ticket counter must start at zero (an interrupted earlier call may have left it set)
  e = cudaMemsetAsync(w.counter, 0, sizeof(unsigned), st);
  if (e != cudaSuccess) return bad(MS_ERR_CUDA, cudaGetErrorString(e));
  ms::Launch L{st, false, nullptr};
  e = ms::launch_lm_head(L, x, ldx, M, d, gamma, beta, eps, W, V, logits, argmax, nullptr, M, 0, nullptr, 0, w);
  if (e != cudaSuccess) return bad(MS_ERR_CUDA, cudaGetErrorString(e));
  return MS_OK;
}
