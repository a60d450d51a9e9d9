// General-M dequant-GEMM on CUDA cores (fp32 FMA): the reference-precision path for
// prefill and batched decode.  y[m][n] (+)= sum_k x[m][k] W[n][k], with the weight
// tile dequantised into shared memory as the fp32 product q * s ("MuScriptor Medium —
// optimized W4A32 ONNX Runtime", Model variant: MatMulNBits with INT4 g32 weights).
#include "ms_device.cuh"
#include "ms_launch.cuh"

namespace ms {

namespace {
constexpr int BM = 64, BN = 64, BK = 32;

struct GemmArgs {
  const uint8_t* wq;
  const float* ws;
  const uint16_t* wh;
  int N, K;
  int ldq, lds;
  const float* x;
  int ldx, M;
  float* y;
  int ldy;
};
}  // namespace

// 256 threads; thread (tm, tn) owns the 4x4 outputs rows m0 + 4 tm .. +3, cols n0 + 4 tn .. +3.
// BK = 32 is exactly one quantisation group, so each weight row of the tile has one scale.
template <int FMT, int EPI>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GemmArgs a) {
  __shared__ __align__(16) float As[BK][BM + 4];
  __shared__ __align__(16) float Bs[BK][BN + 4];
  const int tid = threadIdx.x, tm = tid >> 4, tn = tid & 15;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const int K = a.K;
  pdl_wait();
  pdl_trigger();
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < K; k0 += BK) {
#pragma unroll
    for (int it = 0; it < 2; ++it) {
      const int idx = tid + it * 256;
      const int r = idx >> 3, kq = idx & 7;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (m0 + r < a.M) v = *reinterpret_cast<const float4*>(a.x + (size_t)(m0 + r) * a.ldx + k0 + 4 * kq);
      As[4 * kq + 0][r] = v.x;
      As[4 * kq + 1][r] = v.y;
      As[4 * kq + 2][r] = v.z;
      As[4 * kq + 3][r] = v.w;
    }
    {
      const int r = tid >> 2, wd = tid & 3;
      const int n = n0 + r;
      if (FMT == kInt4) {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(a.wq + (size_t)n * a.ldq + k0 / 2 + wd * 4);
        const float s = a.ws[(size_t)n * a.lds + k0 / 32];
#pragma unroll
        for (int e = 0; e < 8; ++e) Bs[wd * 8 + e][r] = nib_to_q((w >> (4 * e)) & 15u) * s;
      } else {
        const uint4 hv = *reinterpret_cast<const uint4*>(a.wh + (size_t)n * K + k0 + wd * 8);
        const __half2* h2 = reinterpret_cast<const __half2*>(&hv);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __half22float2(h2[e]);
          Bs[wd * 8 + 2 * e][r] = f.x;
          Bs[wd * 8 + 2 * e + 1][r] = f.y;
        }
      }
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      const float4 av = *reinterpret_cast<const float4*>(&As[kk][tm * 4]);
      const float4 bv = *reinterpret_cast<const float4*>(&Bs[kk][tn * 4]);
      const float ar[4] = {av.x, av.y, av.z, av.w};
      const float br[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(ar[i], br[j], acc[i][j]);
    }
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + tm * 4 + i;
    if (m >= a.M) continue;
    float4* yp = reinterpret_cast<float4*>(a.y + (size_t)m * a.ldy + n0 + tn * 4);
    float4 v = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
    if (EPI == kAdd) {
      const float4 o = *yp;
      v.x += o.x;
      v.y += o.y;
      v.z += o.z;
      v.w += o.w;
    } else if (EPI == kGelu) {
      v.x = gelu_erf(v.x);
      v.y = gelu_erf(v.y);
      v.z = gelu_erf(v.z);
      v.w = gelu_erf(v.w);
    }
    *yp = v;
  }
}

cudaError_t launch_gemm(const Launch& L, const WView& w, const float* x, int ldx, int M, float* y, int ldy,
                        int epi) {
  if (M <= 0) return cudaSuccess;
  if (w.N % BN != 0 || w.K % BK != 0 || ldx % 4 != 0 || ldy % 4 != 0) return cudaErrorInvalidValue;
  GemmArgs a;
  a.wq = w.q;
  a.ws = w.s;
  a.wh = w.h;
  a.N = w.N;
  a.K = w.K;
  a.ldq = w.ldq;
  a.lds = w.lds;
  a.x = x;
  a.ldx = ldx;
  a.M = M;
  a.y = y;
  a.ldy = ldy;
  const dim3 grid(w.N / BN, (M + BM - 1) / BM);
  if (w.fmt == kInt4) {
    if (epi == kAdd) return launch_k(L, gemm_simt_kernel<kInt4, kAdd>, grid, dim3(256), 0, a);
    if (epi == kGelu) return launch_k(L, gemm_simt_kernel<kInt4, kGelu>, grid, dim3(256), 0, a);
    return launch_k(L, gemm_simt_kernel<kInt4, kStore>, grid, dim3(256), 0, a);
  }
  if (epi == kAdd) return launch_k(L, gemm_simt_kernel<kFp16, kAdd>, grid, dim3(256), 0, a);
  if (epi == kGelu) return launch_k(L, gemm_simt_kernel<kFp16, kGelu>, grid, dim3(256), 0, a);
  return launch_k(L, gemm_simt_kernel<kFp16, kStore>, grid, dim3(256), 0, a);
}

}  // namespace ms
