// Conditioner front-end kernels (MuScriptor small — ONNX conversion, the conditioner graph
// muscriptor-small-cond.onnx: audio [B, N] at 16 kHz -> prefix [B, frames + 1 + K, d];
// MuScriptor model card, Model description: STFT with n_fft 2048 and hop 160, 512 mel bands,
// log, projection to d_model, then the dataset and instrument embedding rows).
//
// log_mel_kernel: one CTA per (frame, stream).  The frame is the reflection-padded, centred
// slice of the signal times the stored window; its real DFT is taken as a complex DFT of half
// the length (even samples in the real part, odd ones in the imaginary part; radix-4
// decimation-in-frequency stages in shared memory, the first taken on the values as they are
// read, outputs left in digit-reversed order) followed by the split into the even and odd
// halves' spectra.  All of it in double precision: the magnitudes feed a logarithm, which turns an
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

// Position, after the decimation-in-frequency stages below, of frequency k of the half-length
// transform: the stages take radix 4 from the full length down (radix 2 last when log2(half) is
// odd), and each stage's output digit selects a quarter (half) of the current span.
__device__ __forceinline__ int dif_pos(int k, int half) {
  int p = 0, span = half;
  while (span > 1) {
    const int r = span >= 4 ? 4 : 2;
    span /= r;
    p += (k % r) * span;
    k /= r;
  }
  return p;
}

// Shared-memory slot of complex element p: one 16-byte pad after every 8 elements, so that the
// strided and digit-reversed accesses of the stages and the split spread over the banks.
__device__ __forceinline__ int zi(int p) { return p + (p >> 3); }

__device__ __forceinline__ double2 cmul(double2 a, double2 w) {
  return make_double2(a.x * w.x - a.y * w.y, a.x * w.y + a.y * w.x);
}

// One radix-4 decimation-in-frequency butterfly on a0..a3 = x[t1 + q * L/4] of a span of length
// L: the 4-point DFT over q, output digit m times W_L^{t1 m} (the twiddle table holds
// W_{n_fft}^i, so W_L^j = table[j * n_fft / L]).
__device__ __forceinline__ void dif4(double2& a0, double2& a1, double2& a2, double2& a3, int t1, int tstep,
                                     const double2* __restrict__ tw) {
  const double2 s02 = make_double2(a0.x + a2.x, a0.y + a2.y), d02 = make_double2(a0.x - a2.x, a0.y - a2.y);
  const double2 s13 = make_double2(a1.x + a3.x, a1.y + a3.y), d13 = make_double2(a1.x - a3.x, a1.y - a3.y);
  a0 = make_double2(s02.x + s13.x, s02.y + s13.y);
  const double2 c2 = make_double2(s02.x - s13.x, s02.y - s13.y);
  const double2 c1 = make_double2(d02.x + d13.y, d02.y - d13.x);   // d02 - i d13
  const double2 c3 = make_double2(d02.x - d13.y, d02.y + d13.x);   // d02 + i d13
  if (t1 == 0) {
    a1 = c1, a2 = c2, a3 = c3;
  } else {
    a1 = cmul(c1, __ldg(tw + t1 * tstep));
    a2 = cmul(c2, __ldg(tw + 2 * t1 * tstep));
    a3 = cmul(c3, __ldg(tw + 3 * t1 * tstep));
  }
}

__global__ void __launch_bounds__(256) log_mel_kernel(const float* __restrict__ audio, int n_samples, CondDev c,
                                                      int frames, float* __restrict__ out, __half* __restrict__ xh,
                                                      __half* __restrict__ xl) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int half = c.n_fft >> 1, q4 = half >> 2;
  double2* z = reinterpret_cast<double2*>(smem_raw);            // [half + half / 8], element p at zi(p)
  double* mag = reinterpret_cast<double*>(z + half + half / 8); // [half + 1]
  const int t = blockIdx.x, b = blockIdx.y;
  const float* x = audio + (size_t)b * n_samples;
  // z[n] = (f[2n], f[2n+1]), f = window x the frame; the first radix-4 stage (span = half) is
  // taken on the values as they arrive
  auto frame_pair = [&](int n) {
    double f[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int m = 2 * n + e;
      int j = t * c.hop + m - half;                               // index into the unpadded signal
      if (j < 0) j = -j;                                          // reflection without the edge sample
      if (j >= n_samples) j = 2 * (n_samples - 1) - j;
      f[e] = __ldg(c.window + m) * (double)__ldg(x + j);
    }
    return make_double2(f[0], f[1]);
  };
  int span = half;
  if (half >= 4) {
    for (int t1 = threadIdx.x; t1 < q4; t1 += blockDim.x) {
      double2 a0 = frame_pair(t1), a1 = frame_pair(t1 + q4), a2 = frame_pair(t1 + 2 * q4), a3 = frame_pair(t1 + 3 * q4);
      dif4(a0, a1, a2, a3, t1, c.n_fft / half, c.twiddle);
      z[zi(t1)] = a0, z[zi(t1 + q4)] = a1, z[zi(t1 + 2 * q4)] = a2, z[zi(t1 + 3 * q4)] = a3;
    }
    span = q4;
  } else {
    for (int n = threadIdx.x; n < half; n += blockDim.x) z[zi(n)] = frame_pair(n);
  }
  __syncthreads();
  for (; span >= 4; span >>= 2) {
    const int L4 = span >> 2, tstep = c.n_fft / span;
    for (int i = threadIdx.x; i < q4; i += blockDim.x) {
      const int t1 = i % L4, base = (i / L4) * span + t1;
      double2 a0 = z[zi(base)], a1 = z[zi(base + L4)], a2 = z[zi(base + 2 * L4)], a3 = z[zi(base + 3 * L4)];
      dif4(a0, a1, a2, a3, t1, tstep, c.twiddle);
      z[zi(base)] = a0, z[zi(base + L4)] = a1, z[zi(base + 2 * L4)] = a2, z[zi(base + 3 * L4)] = a3;
    }
    __syncthreads();
  }
  if (span == 2) {                                              // a last radix-2 stage
    for (int i = threadIdx.x; i < (half >> 1); i += blockDim.x) {
      const double2 a0 = z[zi(2 * i)], a1 = z[zi(2 * i + 1)];
      z[zi(2 * i)] = make_double2(a0.x + a1.x, a0.y + a1.y);
      z[zi(2 * i + 1)] = make_double2(a0.x - a1.x, a0.y - a1.y);
    }
    __syncthreads();
  }
  // X[k] = E[k] + e^{-2 pi i k / n_fft} O[k], E and O the spectra of the even and odd samples
  for (int k = threadIdx.x; k <= half; k += blockDim.x) {
    if (k == 0 || k == half) {
      const double2 z0 = z[zi(0)];
      mag[k] = fabs(k == 0 ? z0.x + z0.y : z0.x - z0.y);
    } else {
      const double2 a = z[zi(dif_pos(k, half))], cz = z[zi(dif_pos(half - k, half))];
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
  return (size_t)(n_fft / 2 + n_fft / 16) * sizeof(double2) + (size_t)(n_fft / 2 + 1) * sizeof(double);
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
