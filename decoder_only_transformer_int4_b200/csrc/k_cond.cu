// Conditioner front-end kernels (MuScriptor small — ONNX conversion, the conditioner graph
// muscriptor-small-cond.onnx: audio [B, N] at 16 kHz -> prefix [B, frames + 1 + K, d];
// MuScriptor model card, Model description: STFT with n_fft 2048 and hop 160, 512 mel bands,
// log, projection to d_model, then the dataset and instrument embedding rows).
//
// log_mel_kernel: one CTA per (frame, stream).  The frame is the reflection-padded, centred
// slice of the signal times the stored window; its real DFT is taken as a complex DFT of half
// the length (even samples in the real part, odd ones in the imaginary part; radix-2,
// decimation in time, in shared memory) followed by the split into the even and odd halves'
// spectra.  All of it in double precision: the magnitudes feed a logarithm, which turns an
// fp32 FFT's absolute error into a large relative error in low-energy bands.  Each mel band is
// the weighted sum of its own range of bins (the filterbank rows are stored compressed to
// their non-zero range), floored at 1e-6 and logged.  The result leaves as fp32 rows and / or
// as the fp16 hi / lo planes the tcgen05 GEMM takes for the projection.
//
// cond_assemble_kernel: scales the projected rows back (the projection weights are stored
// times 2^s so that their fp16 lo halves stay normal), adds the bias, and writes the dataset
// and instrument embedding rows after the frames.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ms_kernels.h"
#include "ms_launch.cuh"

namespace ms {

namespace {

__global__ void __launch_bounds__(256) log_mel_kernel(const float* __restrict__ audio, int n_samples, CondDev c,
                                                      int frames, float* __restrict__ out, __half* __restrict__ xh,
                                                      __half* __restrict__ xl) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int half = c.n_fft >> 1;
  double2* z = reinterpret_cast<double2*>(smem_raw);            // [half]
  double* mag = reinterpret_cast<double*>(z + half);            // [half + 1]
  const int t = blockIdx.x, b = blockIdx.y;
  const float* x = audio + (size_t)b * n_samples;
  const int lg = 31 - __clz(half);
  // frame samples 2n and 2n+1, windowed, into the bit-reversed slot of n
  for (int n = threadIdx.x; n < half; n += blockDim.x) {
    double f[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int m = 2 * n + e;
      int j = t * c.hop + m - half;                               // index into the unpadded signal
      if (j < 0) j = -j;                                          // reflection without the edge sample
      if (j >= n_samples) j = 2 * (n_samples - 1) - j;
      f[e] = (double)__ldg(c.window + m) * (double)__ldg(x + j);
    }
    const int r = lg ? (int)(__brev((unsigned)n) >> (32 - lg)) : 0;
    z[r] = make_double2(f[0], f[1]);
  }
  __syncthreads();
  // radix-2 stages of the half-length complex DFT; the twiddles of the full length serve it
  // at every second index
  for (int h = 1; h < half; h <<= 1) {
    const int step = c.n_fft / (2 * h);
    for (int i = threadIdx.x; i < (half >> 1); i += blockDim.x) {
      const int j = i & (h - 1);
      const int p = ((i - j) << 1) + j, q = p + h;
      const double2 w = __ldg(c.twiddle + j * step);
      const double2 u = z[p], v = z[q];
      const double vr = v.x * w.x - v.y * w.y, vi = v.x * w.y + v.y * w.x;
      z[p] = make_double2(u.x + vr, u.y + vi);
      z[q] = make_double2(u.x - vr, u.y - vi);
    }
    __syncthreads();
  }
  // X[k] = E[k] + e^{-2 pi i k / n_fft} O[k], E and O the spectra of the even and odd samples
  for (int k = threadIdx.x; k <= half; k += blockDim.x) {
    if (k == 0 || k == half) {
      const double2 z0 = z[0];
      mag[k] = fabs(k == 0 ? z0.x + z0.y : z0.x - z0.y);
    } else {
      const double2 a = z[k], cz = z[half - k];
      const double er = 0.5 * (a.x + cz.x), ei = 0.5 * (a.y - cz.y);     // (a + conj(cz)) / 2
      const double orr = 0.5 * (a.y + cz.y), oi = -0.5 * (a.x - cz.x);  // (a - conj(cz)) / 2i
      const double2 w = __ldg(c.twiddle + k);
      const double xr = er + (orr * w.x - oi * w.y), xi = ei + (orr * w.y + oi * w.x);
      mag[k] = sqrt(xr * xr + xi * xi);
    }
  }
  __syncthreads();
  const size_t row = (size_t)b * frames + t;
  for (int m = threadIdx.x; m < c.kp; m += blockDim.x) {
    float v = 0.f;
    if (m < c.n_mels) {
      const int lo = __ldg(c.band_lo + m), o0 = __ldg(c.band_off + m), o1 = __ldg(c.band_off + m + 1);
      double s = 0.0;
      for (int i = o0; i < o1; ++i) s += (double)__ldg(c.band_w + i) * mag[lo + i - o0];
      v = (float)log(fmax(s, 1e-6));
      if (out) out[row * c.n_mels + m] = v;
    }
    if (xh) {
      const __half hi = __float2half_rn(v);
      xh[row * c.kp + m] = hi;
      xl[row * c.kp + m] = __float2half_rn(v - __half2float(hi));
    }
  }
}

// One CTA per output row (frame rows, then the dataset row, then the instrument rows).
__global__ void __launch_bounds__(256) cond_assemble_kernel(const float* __restrict__ y, float yscale,
                                                            const float* __restrict__ bias,
                                                            const float* __restrict__ ds_emb, int n_ds,
                                                            const float* __restrict__ inst_emb, int n_inst,
                                                            const int32_t* __restrict__ dataset,
                                                            const int32_t* __restrict__ instruments, int K, int frames,
                                                            int d, float* __restrict__ prefix, unsigned* status) {
  const int r = blockIdx.x, b = blockIdx.y;
  const int rows = frames + 1 + K;
  float4* dst = reinterpret_cast<float4*>(prefix + ((size_t)b * rows + r) * d);
  const int d4 = d >> 2;
  if (r < frames) {
    const float4* src = reinterpret_cast<const float4*>(y + ((size_t)b * frames + r) * d);
    const float4* bb = reinterpret_cast<const float4*>(bias);
    for (int i = threadIdx.x; i < d4; i += blockDim.x) {
      const float4 v = __ldg(src + i), w = __ldg(bb + i);
      dst[i] = make_float4(v.x * yscale + w.x, v.y * yscale + w.y, v.z * yscale + w.z, v.w * yscale + w.w);
    }
    return;
  }
  int id, n;
  const float* table;
  if (r == frames) {
    id = __ldg(dataset + b), n = n_ds, table = ds_emb;
  } else {
    id = __ldg(instruments + (size_t)b * K + (r - frames - 1)), n = n_inst, table = inst_emb;
  }
  if (id < 0 || id >= n) {
    if (threadIdx.x == 0 && status) atomicOr(status, kErrTokenBit);
    id = id < 0 ? 0 : n - 1;
  }
  const float4* src = reinterpret_cast<const float4*>(table + (size_t)id * d);
  for (int i = threadIdx.x; i < d4; i += blockDim.x) dst[i] = __ldg(src + i);
}

}  // namespace

size_t log_mel_smem_bytes(int n_fft) {
  return (size_t)(n_fft / 2) * sizeof(double2) + (size_t)(n_fft / 2 + 1) * sizeof(double);
}

cudaError_t init_attrs_cond() { return allow_smem(log_mel_kernel, log_mel_smem_bytes(kCondMaxFft)); }

cudaError_t launch_log_mel(const Launch& L, const float* audio, int n_samples, int B, const CondDev& c, int frames,
                           float* out, __half* xh, __half* xl) {
  if (B <= 0) return cudaSuccess;
  return launch_k(L, log_mel_kernel, dim3(frames, B), dim3(256), log_mel_smem_bytes(c.n_fft), audio, n_samples, c,
                  frames, out, xh, xl);
}

cudaError_t launch_cond_assemble(const Launch& L, const float* y, float yscale, const float* bias,
                                 const float* ds_emb, int n_ds, const float* inst_emb, int n_inst,
                                 const int32_t* dataset, const int32_t* instruments, int K, int frames, int d, int B,
                                 float* prefix) {
  if (B <= 0) return cudaSuccess;
  return launch_k(L, cond_assemble_kernel, dim3(frames + 1 + K, B), dim3(256), 0, y, yscale, bias, ds_emb, n_ds,
                  inst_emb, n_inst, dataset, instruments, K, frames, d, prefix, L.status);
}

}  // namespace ms
