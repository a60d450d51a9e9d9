// W4A8: the backbone MatMuls with their activations quantised to INT8 at run time and the
// products accumulated in INT32 ("MuScriptor Medium — optimized W4A32 ONNX Runtime", Model
// variant: MatMulNBits with accuracy_level=4).  The page does not say how the activations are
// quantised; the reading used is the weight quantiser's rule at 127 levels a side on blocks of
// 32 consecutive K elements of a row (one block per weight group):
//   scale = absmax / 127, q = clamp(rint(x / scale), -127, 127), fp32 IEEE divisions, ties to
//   even; an all-zero block has scale 0 and q 0;
//   y[m][n] = sum over blocks b of (sa[m][b] * sw[n][b]) * (sum_{k in b} qa[m][k] * qw[n][k]),
// the inner sums exact in INT32 (at most 32 * 127 * 7 in magnitude), the blocks summed in fp32.
//
// Kernels: the quantiser (codes bit-exact with the definition above given the same fp32
// input), a dp4a GEMV for 1 to 8 rows (decode: HBM-bound on the INT4 weights, like the fp32
// GEMV), and a dp4a tiled GEMM for more rows (prefill, batched decode).
#include "ms_device.cuh"
#include "ms_launch.cuh"

namespace ms {

// ---- activation quantiser ------------------------------------------------------------------
// One warp per 32-element block: lane l takes element l.
__global__ void __launch_bounds__(256) quantize_act_int8_kernel(const float* __restrict__ x, int ldx, int M, int K,
                                                                int8_t* __restrict__ q, int ldq, float* __restrict__ s,
                                                                int lds) {
  pdl_wait();
  pdl_trigger();
  const int KB = K >> 5;
  const long long blk = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (blk >= (long long)M * KB) return;
  const int lane = threadIdx.x & 31;
  const int m = (int)(blk / KB), b = (int)(blk - (long long)m * KB);
  const float v = x[(size_t)m * ldx + b * 32 + lane];
  const float am = warp_max(fabsf(v));
  const float sc = __fdiv_rn(am, 127.0f);
  int qi = 0;
  if (sc != 0.f) qi = (int)fminf(fmaxf(rintf(__fdiv_rn(v, sc)), -127.f), 127.f);
  q[(size_t)m * ldq + b * 32 + lane] = (int8_t)qi;
  if (lane == 0) s[(size_t)m * lds + b] = sc;
}

cudaError_t launch_quantize_act_int8(const Launch& L, const float* x, int ldx, int M, int K, int8_t* q, int ldq,
                                     float* s, int lds) {
  if (M <= 0) return cudaSuccess;
  if (K % 32 != 0) return cudaErrorInvalidValue;
  const long long blocks = (long long)M * (K / 32);
  return launch_k(L, quantize_act_int8_kernel, dim3((unsigned)((blocks + 7) / 8)), dim3(256), 0, x, ldx, M, K, q, ldq,
                  s, lds);
}

namespace {

// Eight INT4 codes (four bytes, element 2j in the low nibble of byte j) -> two words of four
// signed bytes in element order: elements 0..3 and 4..7.
__device__ __forceinline__ void nib8_to_s8(uint32_t w, uint32_t& e0123, uint32_t& e4567) {
  const uint32_t lo = w & 0x0F0F0F0Fu;          // elements 0, 2, 4, 6
  const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;   // elements 1, 3, 5, 7
  e0123 = __vsub4(__byte_perm(lo, hi, 0x5140), 0x08080808u);
  e4567 = __vsub4(__byte_perm(lo, hi, 0x7362), 0x08080808u);
}

__device__ __forceinline__ float epi_apply(int epi, float v, const float* yp) {
  if (epi == kAdd) return v + *yp;
  if (epi == kGelu) return gelu_erf(v);
  return v;
}

}  // namespace

// ---- GEMV: M <= 8 rows ---------------------------------------------------------------------
// Each warp takes weight rows n = warp_global, + total warps, ...; lane l takes the blocks
// b = l, l + 32, ... of the row (16 code bytes and one scale each), the M rows' codes of its
// blocks come from shared memory; the per-row sums are reduced over the warp.
template <int M>
__global__ void __launch_bounds__(256) gemv_w4a8_kernel(WView w, const int8_t* __restrict__ qa, int ldqa,
                                                        const float* __restrict__ sa, int ldsa, float* __restrict__ y,
                                                        int ldy, int epi) {
  extern __shared__ __align__(16) unsigned char sm8[];
  const int K = w.K, KB = K >> 5;
  int8_t* qs = reinterpret_cast<int8_t*>(sm8);                         // [M][K]
  float* ss = reinterpret_cast<float*>(sm8 + (size_t)M * K);           // [M][KB]
  pdl_wait();
  pdl_trigger();
  for (int i = threadIdx.x; i < M * K / 16; i += blockDim.x) {
    const int m = i / (K / 16), c = i - m * (K / 16);
    reinterpret_cast<uint4*>(qs)[i] = *reinterpret_cast<const uint4*>(qa + (size_t)m * ldqa + c * 16);
  }
  for (int i = threadIdx.x; i < M * KB; i += blockDim.x) {
    const int m = i / KB, b = i - m * KB;
    ss[i] = sa[(size_t)m * ldsa + b];
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int nw = gridDim.x * (blockDim.x >> 5);
  for (int n = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); n < w.N; n += nw) {
    float acc[M];
#pragma unroll
    for (int m = 0; m < M; ++m) acc[m] = 0.f;
    const uint8_t* row = w.q + (size_t)n * w.ldq;
    const float* srow = w.s + (size_t)n * w.lds;
    for (int b = lane; b < KB; b += 32) {
      const uint4 c = __ldg(reinterpret_cast<const uint4*>(row + b * 16));
      const float swb = __ldg(srow + b);
      uint32_t wv[8];
      nib8_to_s8(c.x, wv[0], wv[1]);
      nib8_to_s8(c.y, wv[2], wv[3]);
      nib8_to_s8(c.z, wv[4], wv[5]);
      nib8_to_s8(c.w, wv[6], wv[7]);
#pragma unroll
      for (int m = 0; m < M; ++m) {
        const uint4 a0 = reinterpret_cast<const uint4*>(qs + (size_t)m * K + b * 32)[0];
        const uint4 a1 = reinterpret_cast<const uint4*>(qs + (size_t)m * K + b * 32)[1];
        int isum = 0;
        isum = __dp4a((int)wv[0], (int)a0.x, isum);
        isum = __dp4a((int)wv[1], (int)a0.y, isum);
        isum = __dp4a((int)wv[2], (int)a0.z, isum);
        isum = __dp4a((int)wv[3], (int)a0.w, isum);
        isum = __dp4a((int)wv[4], (int)a1.x, isum);
        isum = __dp4a((int)wv[5], (int)a1.y, isum);
        isum = __dp4a((int)wv[6], (int)a1.z, isum);
        isum = __dp4a((int)wv[7], (int)a1.w, isum);
        acc[m] = fmaf((float)isum, swb * ss[m * KB + b], acc[m]);
      }
    }
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const float v = warp_sum(acc[m]);
      if (lane == 0) {
        float* yp = y + (size_t)m * ldy + n;
        *yp = epi_apply(epi, v, yp);
      }
    }
  }
}

// ---- GEMM: any M (tiles of 64 activation rows x 64 weight rows) ------------------------------
// 256 threads; thread (tm, tn) computes rows m = 4 tm .. 4 tm + 3 and weight rows n = 4 tn ..
// 4 tn + 3.  Per 128-wide K chunk the CTA stages the weight codes (as signed bytes in element
// order) and the activation codes in shared memory, rows padded to 33 words (no bank
// conflicts), and the block scales; each 32-element block's INT32 sums are scaled and added
// in fp32.
namespace {
constexpr int kQm = 64, kQn = 64, kQk = 128, kQw = kQk / 4 + 1;   // padded words per row
}

__global__ void __launch_bounds__(256) gemm_w4a8_kernel(WView w, const int8_t* __restrict__ qa, int ldqa,
                                                        const float* __restrict__ sa, int ldsa, int M,
                                                        float* __restrict__ y, int ldy, int epi) {
  __shared__ uint32_t wsm[kQn][kQw];
  __shared__ uint32_t asm_[kQm][kQw];
  __shared__ float sws[kQn][4], sas[kQm][4];
  pdl_wait();
  pdl_trigger();
  const int tid = threadIdx.x, tn = tid & 15, tm = tid >> 4;
  const int n0 = blockIdx.x * kQn, m0 = blockIdx.y * kQm;
  const int K = w.K, KB = K >> 5;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int k0 = 0; k0 < K; k0 += kQk) {
    __syncthreads();
    // weights: 64 rows x 64 code bytes (128 elements): thread t takes 16 bytes of one row
    for (int i = tid; i < kQn * 4; i += 256) {
      const int r = i >> 2, c = i & 3, n = n0 + r;
      uint4 cb = make_uint4(0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u);
      if (n < w.N) cb = __ldg(reinterpret_cast<const uint4*>(w.q + (size_t)n * w.ldq + k0 / 2 + c * 16));
      uint32_t* d = &wsm[r][c * 8];
      nib8_to_s8(cb.x, d[0], d[1]);
      nib8_to_s8(cb.y, d[2], d[3]);
      nib8_to_s8(cb.z, d[4], d[5]);
      nib8_to_s8(cb.w, d[6], d[7]);
    }
    for (int i = tid; i < kQn * 4; i += 256) {
      const int r = i >> 2, g = i & 3, n = n0 + r;
      sws[r][g] = n < w.N ? __ldg(w.s + (size_t)n * w.lds + k0 / 32 + g) : 0.f;
    }
    // activations: 64 rows x 128 code bytes
    for (int i = tid; i < kQm * 8; i += 256) {
      const int r = i >> 3, c = i & 7, m = m0 + r;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (m < M) v = __ldg(reinterpret_cast<const uint4*>(qa + (size_t)m * ldqa + k0 + c * 16));
      uint32_t* d = &asm_[r][c * 4];
      d[0] = v.x;
      d[1] = v.y;
      d[2] = v.z;
      d[3] = v.w;
    }
    for (int i = tid; i < kQm * 4; i += 256) {
      const int r = i >> 2, g = i & 3, m = m0 + r;
      sas[r][g] = m < M ? sa[(size_t)m * ldsa + k0 / 32 + g] : 0.f;
    }
    __syncthreads();
    const int ng = min(4, KB - (k0 >> 5));
    for (int g = 0; g < ng; ++g) {
      int isum[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) isum[i][j] = 0;
#pragma unroll
      for (int wd = 0; wd < 8; ++wd) {
        uint32_t av[4], wv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) av[i] = asm_[tm * 4 + i][g * 8 + wd];
#pragma unroll
        for (int j = 0; j < 4; ++j) wv[j] = wsm[tn * 4 + j][g * 8 + wd];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) isum[i][j] = __dp4a((int)av[i], (int)wv[j], isum[i][j]);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf((float)isum[i][j], sas[tm * 4 + i][g] * sws[tn * 4 + j][g], acc[i][j]);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + tm * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tn * 4 + j;
      if (n < w.N) {
        float* yp = y + (size_t)m * ldy + n;
        *yp = epi_apply(epi, acc[i][j], yp);
      }
    }
  }
}

cudaError_t init_attrs_w4a8() {
  cudaError_t e = allow_smem(gemv_w4a8_kernel<1>, kMaxDynSmem);
  if (e == cudaSuccess) e = allow_smem(gemv_w4a8_kernel<2>, kMaxDynSmem);
  if (e == cudaSuccess) e = allow_smem(gemv_w4a8_kernel<4>, kMaxDynSmem);
  if (e == cudaSuccess) e = allow_smem(gemv_w4a8_kernel<8>, kMaxDynSmem);
  return e;
}

cudaError_t launch_matmul_w4a8(const Launch& L, const WView& w, const int8_t* qa, int ldqa, const float* sa, int ldsa,
                               int M, float* y, int ldy, int epi, int sms) {
  if (M <= 0) return cudaSuccess;
  if (w.fmt != kInt4 || w.K % 128 != 0 || ldqa % 16 != 0) return cudaErrorInvalidValue;
  if (M == 1 || M == 2 || M == 4 || M == 8) {
    const size_t smem = (size_t)M * w.K + (size_t)M * (w.K / 32) * sizeof(float);
    if (smem <= kMaxDynSmem) {
      int grid = (w.N + 7) / 8;
      if (grid > 2 * sms) grid = 2 * sms;
      switch (M) {
        case 1: return launch_k(L, gemv_w4a8_kernel<1>, dim3(grid), dim3(256), smem, w, qa, ldqa, sa, ldsa, y, ldy, epi);
        case 2: return launch_k(L, gemv_w4a8_kernel<2>, dim3(grid), dim3(256), smem, w, qa, ldqa, sa, ldsa, y, ldy, epi);
        case 4: return launch_k(L, gemv_w4a8_kernel<4>, dim3(grid), dim3(256), smem, w, qa, ldqa, sa, ldsa, y, ldy, epi);
        default: return launch_k(L, gemv_w4a8_kernel<8>, dim3(grid), dim3(256), smem, w, qa, ldqa, sa, ldsa, y, ldy, epi);
      }
    }
  }
  const dim3 grid((w.N + kQn - 1) / kQn, (M + kQm - 1) / kQm);
  return launch_k(L, gemm_w4a8_kernel, grid, dim3(256), 0, w, qa, ldqa, sa, ldsa, M, y, ldy, epi);
}

}  // namespace ms
