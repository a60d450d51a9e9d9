// Decode-path kernels: the W4 (and fp16-weight) dequant-GEMV for M <= 8 rows and the
// fused LM head + argmax.
//
// Both stream their whole weight slice into shared memory with bulk copies issued
// before the programmatic-dependent-launch wait, so the weight bytes (which do not
// depend on the previous kernel) are in flight while that kernel finishes.
#include <float.h>
#include <limits.h>
#include "ms_device.cuh"
#include "ms_launch.cuh"

namespace ms {

namespace {
constexpr int kGemvThreads = 256;
constexpr int kGemvWarps = kGemvThreads / 32;
constexpr int kTargetCtas = 148;       // one CTA per SM of a B200
constexpr size_t kSmemBudget = 200 * 1024;

struct GemvArgs {
  const uint8_t* wq;
  const float* ws;
  const uint16_t* wh;
  int N, K, rpc;
  int ldq, lds;       // INT4 row strides (bytes, floats)
  int inter;          // 1: scales follow each row's nibbles (one copy per slice)
  const float* x;
  int ldx;
  const float* ln_g;
  const float* ln_b;
  float eps;
  float* y;
  int ldy;
  unsigned* status;
};

// Shared memory: the slice's rows (INT4: nibbles + scales), then M activation rows.
size_t gemv_smem(int fmt, int K, int rpc, int M) {
  size_t s = 16;
  if (fmt == kInt4)
    s += align16((size_t)rpc * (K / 2)) + align16((size_t)rpc * (K / 8));
  else
    s += align16((size_t)rpc * K * 2);
  s += (size_t)M * K * 4 + 64 * 4;
  return s;
}

int gemv_rpc(int N) { return (N + kTargetCtas - 1) / kTargetCtas; }
}  // namespace

// y[m][n] (+)= sum_k xn[m][k] W[n][k], W[n][k] = q[n][k] * s[n][k/32] (INT4, "MuScriptor
// Medium — optimized W4A32 ONNX Runtime", Model variant) or the fp16 value.  xn is x or,
// with LN, the LayerNorm of x (the pre-LN of the block, fused here so the normalised row
// never goes through global memory).
//
// Layout: CTA c owns rows [c*rpc, c*rpc + rpc); warp w takes rows w, w+8, ...; lane l
// takes the 4-byte word l + 32 j of a row (8 nibbles, elements 8c..8c+7) so a warp's
// loads are contiguous.  Activations sit in shared memory de-interleaved (elements
// 8c..8c+3 and 8c+4..8c+7 in two float4 arrays) so those reads are conflict-free too.
// Per word: 8 exact int->float conversions, 8 FMAs against x, one FMA with the group
// scale.  A warp shuffle tree reduces each row.
template <int M, int FMT, bool LN, int EPI>
__global__ void __launch_bounds__(kGemvThreads) gemv_kernel(GemvArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int K = a.K;
  const int n0 = blockIdx.x * a.rpc;
  const int rows = min(a.rpc, a.N - n0);
  // Shared layout.  Interleaved INT4: rows of ldq bytes (nibbles then scales) back to
  // back.  Separate INT4: all rows' nibbles, then all rows' scales.  FP16: rows of 2K bytes.
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem);
  unsigned char* wsm = smem + 16;
  const size_t wregion = FMT == kInt4 ? align16((size_t)a.rpc * (K / 2)) + align16((size_t)a.rpc * (K / 8))
                                      : align16((size_t)a.rpc * K * 2);
  float* xsm = reinterpret_cast<float*>(wsm + wregion);
  float* red = xsm + (size_t)M * K;
  const size_t wstride = FMT == kInt4 ? (a.inter ? (size_t)a.ldq : (size_t)K / 2) : (size_t)K * 2;
  const float* ssm_sep = reinterpret_cast<const float*>(wsm + align16((size_t)a.rpc * (K / 2)));

  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (tid == 0) {
    if (FMT == kFp16) {
      const uint32_t wb = (uint32_t)((size_t)rows * K * 2);
      mbar_expect_tx(bar, wb);
      bulk_g2s_pieces(wsm, reinterpret_cast<const unsigned char*>(a.wh) + (size_t)n0 * K * 2, wb, bar);
    } else if (a.inter) {
      const uint32_t wb = (uint32_t)((size_t)rows * a.ldq);
      mbar_expect_tx(bar, wb);
      bulk_g2s_pieces(wsm, a.wq + (size_t)n0 * a.ldq, wb, bar);
    } else {
      const uint32_t wb = (uint32_t)((size_t)rows * (K / 2));
      const uint32_t sb = (uint32_t)((size_t)rows * (K / 8));
      mbar_expect_tx(bar, wb + sb);
      bulk_g2s_pieces(wsm, a.wq + (size_t)n0 * (K / 2), wb, bar);
      bulk_g2s_pieces(const_cast<float*>(ssm_sep), a.ws + (size_t)n0 * (K / 32), sb, bar);
    }
  }

  pdl_wait();
  pdl_trigger();

  const int KW = K / 8;
  float4* xs4 = reinterpret_cast<float4*>(xsm);
#pragma unroll
  for (int m = 0; m < M; ++m) {
    const float4* src = reinterpret_cast<const float4*>(a.x + (size_t)m * a.ldx);
    float4* dst = xs4 + (size_t)m * 2 * KW;
    if (LN) {
      float s = 0.f;
      for (int f = tid; f < K / 4; f += kGemvThreads) {
        const float4 v = src[f];
        s += (v.x + v.y) + (v.z + v.w);
        dst[(f & 1) * KW + (f >> 1)] = v;
      }
      const float mean = block_sum(s, red) / K;
      float q = 0.f;
      for (int f = tid; f < K / 4; f += kGemvThreads) {
        const float4 v = dst[(f & 1) * KW + (f >> 1)];
        const float p0 = v.x - mean, p1 = v.y - mean, p2 = v.z - mean, p3 = v.w - mean;
        q += (p0 * p0 + p1 * p1) + (p2 * p2 + p3 * p3);
      }
      const float var = block_sum(q, red) / K;
      const float rstd = 1.0f / sqrtf(var + a.eps);
      const float4* g4 = reinterpret_cast<const float4*>(a.ln_g);
      const float4* b4 = reinterpret_cast<const float4*>(a.ln_b);
      for (int f = tid; f < K / 4; f += kGemvThreads) {
        float4 v = dst[(f & 1) * KW + (f >> 1)];
        const float4 gg = g4[f], bb = b4[f];
        v.x = (v.x - mean) * rstd * gg.x + bb.x;
        v.y = (v.y - mean) * rstd * gg.y + bb.y;
        v.z = (v.z - mean) * rstd * gg.z + bb.z;
        v.w = (v.w - mean) * rstd * gg.w + bb.w;
        dst[(f & 1) * KW + (f >> 1)] = v;
      }
    } else {
      for (int f = tid; f < K / 4; f += kGemvThreads) dst[(f & 1) * KW + (f >> 1)] = src[f];
    }
  }
  __syncthreads();
  if (rows <= 0) return;
  if (!mbar_wait(bar, 0, a.status)) return;

  const int JW = KW / 32;
  for (int r = warp; r < rows; r += kGemvWarps) {
    float acc[M];
#pragma unroll
    for (int m = 0; m < M; ++m) acc[m] = 0.f;
    if (FMT == kInt4) {
      const uint32_t* wr = reinterpret_cast<const uint32_t*>(wsm + (size_t)r * wstride);
      const float* sr = a.inter ? reinterpret_cast<const float*>(wsm + (size_t)r * wstride + K / 2)
                                : ssm_sep + (size_t)r * (K / 32);
#pragma unroll 2
      for (int j = 0; j < JW; ++j) {
        const int c = lane + 32 * j;
        const uint32_t wd = wr[c];
        const float sc = sr[c >> 2];
        float q[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) q[e] = nib_to_q((wd >> (4 * e)) & 15u);
#pragma unroll
        for (int m = 0; m < M; ++m) {
          const float4 xa = xs4[(size_t)m * 2 * KW + c];
          const float4 xb = xs4[(size_t)m * 2 * KW + KW + c];
          float p = q[0] * xa.x;
          p = fmaf(q[1], xa.y, p);
          p = fmaf(q[2], xa.z, p);
          p = fmaf(q[3], xa.w, p);
          p = fmaf(q[4], xb.x, p);
          p = fmaf(q[5], xb.y, p);
          p = fmaf(q[6], xb.z, p);
          p = fmaf(q[7], xb.w, p);
          acc[m] = fmaf(sc, p, acc[m]);
        }
      }
    } else {
      const uint4* wr = reinterpret_cast<const uint4*>(wsm + (size_t)r * wstride);
#pragma unroll 2
      for (int j = 0; j < JW; ++j) {
        const int c = lane + 32 * j;
        const uint4 hv = wr[c];
        const __half2* h2 = reinterpret_cast<const __half2*>(&hv);
        float q[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f2 = __half22float2(h2[e]);
          q[2 * e] = f2.x;
          q[2 * e + 1] = f2.y;
        }
#pragma unroll
        for (int m = 0; m < M; ++m) {
          const float4 xa = xs4[(size_t)m * 2 * KW + c];
          const float4 xb = xs4[(size_t)m * 2 * KW + KW + c];
          float p = acc[m];
          p = fmaf(q[0], xa.x, p);
          p = fmaf(q[1], xa.y, p);
          p = fmaf(q[2], xa.z, p);
          p = fmaf(q[3], xa.w, p);
          p = fmaf(q[4], xb.x, p);
          p = fmaf(q[5], xb.y, p);
          p = fmaf(q[6], xb.z, p);
          p = fmaf(q[7], xb.w, p);
          acc[m] = p;
        }
      }
    }
#pragma unroll
    for (int m = 0; m < M; ++m) acc[m] = warp_sum(acc[m]);
    if (lane < M) {
      float v = acc[0];
#pragma unroll
      for (int m = 1; m < M; ++m)
        if (lane == m) v = acc[m];
      float* yp = a.y + (size_t)lane * a.ldy + (n0 + r);
      if (EPI == kAdd)
        *yp += v;
      else if (EPI == kGelu)
        *yp = gelu_erf(v);
      else
        *yp = v;
    }
  }
}

bool gemv_fits(const WView& w, int M) {
  if (M < 1 || M > 8) return false;
  if (w.K % 256 != 0) return false;
  return gemv_smem(w.fmt, w.K, gemv_rpc(w.N), M) <= kSmemBudget;
}

template <int M, int FMT, bool LN, int EPI>
static cudaError_t gemv_go(const Launch& L, const GemvArgs& a, int grid, size_t smem) {
  return launch_k(L, gemv_kernel<M, FMT, LN, EPI>, dim3(grid), dim3(kGemvThreads), smem, a);
}

template <int M, int FMT>
static cudaError_t gemv_attrs_mf() {
  cudaError_t e = cudaSuccess;
  if (e == cudaSuccess) e = allow_smem(gemv_kernel<M, FMT, false, kStore>, kMaxDynSmem);
  if (e == cudaSuccess) e = allow_smem(gemv_kernel<M, FMT, false, kAdd>, kMaxDynSmem);
  if (e == cudaSuccess) e = allow_smem(gemv_kernel<M, FMT, false, kGelu>, kMaxDynSmem);
  if (e == cudaSuccess) e = allow_smem(gemv_kernel<M, FMT, true, kStore>, kMaxDynSmem);
  if (e == cudaSuccess) e = allow_smem(gemv_kernel<M, FMT, true, kAdd>, kMaxDynSmem);
  if (e == cudaSuccess) e = allow_smem(gemv_kernel<M, FMT, true, kGelu>, kMaxDynSmem);
  return e;
}

template <int M, int FMT>
static cudaError_t gemv_dispatch_epi(const Launch& L, const GemvArgs& a, int grid, size_t smem, bool ln, int epi) {
  if (ln) {
    if (epi == kGelu) return gemv_go<M, FMT, true, kGelu>(L, a, grid, smem);
    if (epi == kAdd) return gemv_go<M, FMT, true, kAdd>(L, a, grid, smem);
    return gemv_go<M, FMT, true, kStore>(L, a, grid, smem);
  }
  if (epi == kGelu) return gemv_go<M, FMT, false, kGelu>(L, a, grid, smem);
  if (epi == kAdd) return gemv_go<M, FMT, false, kAdd>(L, a, grid, smem);
  return gemv_go<M, FMT, false, kStore>(L, a, grid, smem);
}

template <int M>
static cudaError_t gemv_dispatch_fmt(const Launch& L, const GemvArgs& a, int fmt, int grid, size_t smem, bool ln,
                                     int epi) {
  if (fmt == kInt4) return gemv_dispatch_epi<M, kInt4>(L, a, grid, smem, ln, epi);
  return gemv_dispatch_epi<M, kFp16>(L, a, grid, smem, ln, epi);
}

cudaError_t launch_gemv(const Launch& L, const WView& w, const float* x, int ldx, int M, const float* ln_g,
                        const float* ln_b, float eps, float* y, int ldy, int epi) {
  if (!gemv_fits(w, M)) return cudaErrorInvalidValue;
  GemvArgs a;
  a.wq = w.q;
  a.ws = w.s;
  a.wh = w.h;
  a.N = w.N;
  a.K = w.K;
  a.rpc = gemv_rpc(w.N);
  a.ldq = w.ldq;
  a.lds = w.lds;
  a.inter = w.interleaved() ? 1 : 0;
  a.x = x;
  a.ldx = ldx;
  a.ln_g = ln_g;
  a.ln_b = ln_b;
  a.eps = eps;
  a.y = y;
  a.ldy = ldy;
  a.status = L.status;
  const int grid = (w.N + a.rpc - 1) / a.rpc;
  const int Mp = M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : 8;
  const size_t smem = gemv_smem(w.fmt, w.K, a.rpc, Mp);
  const bool ln = ln_g != nullptr;
  if (Mp != M) return cudaErrorInvalidValue;  // callers pass M in {1, 2, 4, 8}
  switch (M) {
    case 1: return gemv_dispatch_fmt<1>(L, a, w.fmt, grid, smem, ln, epi);
    case 2: return gemv_dispatch_fmt<2>(L, a, w.fmt, grid, smem, ln, epi);
    case 4: return gemv_dispatch_fmt<4>(L, a, w.fmt, grid, smem, ln, epi);
    default: return gemv_dispatch_fmt<8>(L, a, w.fmt, grid, smem, ln, epi);
  }
}

// ---------------------------------------------------------------------------------
// LM head + greedy argmax.  logits[m][v] = LN_f(x_m) . W[v] with W fp32 [V][d] ("MuScriptor
// Medium — optimized W4A32 ONNX Runtime", Model variant: LM head FP32, not quantized;
// "MuScriptor small — ONNX conversion", muscriptor-small-lm.onnx: logits of the last
// position only), argmax = lowest index of the largest logit ("MuScriptor — small
// (≈100M)", Model description: greedy decoding).  Each CTA reduces its rows to one
// (value, index) per m; the last CTA to finish (atomic ticket, no waiting) reduces the
// per-CTA results, writes argmax and the token history, and advances the cache length.
// ---------------------------------------------------------------------------------
namespace {
constexpr int kLmThreads = 256;
constexpr int kLmWarps = kLmThreads / 32;
constexpr int kLmMaxChunk = 8;

struct LmArgs {
  const float* x;
  int ldx, M, m_base, d;
  const float* ln_g;
  const float* ln_b;
  float eps;
  const float* W;
  int V, rpc;
  float* logits;
  int32_t* argmax;
  int32_t* hist;
  int hist_B, hist_off;
  int* dlen;
  int len_add;
  float* part_val;
  int* part_idx;
  unsigned* counter;
  unsigned* status;
  float guidance;   // 0: argmax per row; else rows (2p, 2p+1) = (conditional, unconditional) pairs
};

int lm_rpc(int V) { return (V + kTargetCtas - 1) / kTargetCtas; }
}  // namespace

int lm_head_grid(int V) {
  const int rpc = lm_rpc(V);
  return (V + rpc - 1) / rpc;
}

__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

template <int M>
__global__ void __launch_bounds__(kLmThreads) lm_head_kernel(LmArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int d = a.d;
  const int v0 = blockIdx.x * a.rpc;
  const int rows = min(a.rpc, a.V - v0);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem);
  float* wsm = reinterpret_cast<float*>(smem + 16);
  float* hsm = wsm + (size_t)a.rpc * d;
  float* red = hsm + (size_t)M * d;
  float* bval = red + 64;                 // [warps][M]
  int* bidx = reinterpret_cast<int*>(bval + kLmWarps * M);
  __shared__ unsigned last;

  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (tid == 0 && rows > 0) {
    const uint32_t bytes = (uint32_t)((size_t)rows * d * 4);
    mbar_expect_tx(bar, bytes);
    bulk_g2s_pieces(wsm, a.W + (size_t)v0 * d, bytes, bar);
  }
  pdl_wait();
  pdl_trigger();

  for (int m = 0; m < M; ++m) {
    const float4* src = reinterpret_cast<const float4*>(a.x + (size_t)(a.m_base + m) * a.ldx);
    float4* dst = reinterpret_cast<float4*>(hsm + (size_t)m * d);
    if (a.ln_g) {
      float s = 0.f;
      for (int f = tid; f < d / 4; f += kLmThreads) {
        const float4 v = src[f];
        s += (v.x + v.y) + (v.z + v.w);
        dst[f] = v;
      }
      const float mean = block_sum(s, red) / d;
      float q = 0.f;
      for (int f = tid; f < d / 4; f += kLmThreads) {
        const float4 v = dst[f];
        const float p0 = v.x - mean, p1 = v.y - mean, p2 = v.z - mean, p3 = v.w - mean;
        q += (p0 * p0 + p1 * p1) + (p2 * p2 + p3 * p3);
      }
      const float var = block_sum(q, red) / d;
      const float rstd = 1.0f / sqrtf(var + a.eps);
      const float4* g4 = reinterpret_cast<const float4*>(a.ln_g);
      const float4* b4 = reinterpret_cast<const float4*>(a.ln_b);
      for (int f = tid; f < d / 4; f += kLmThreads) {
        float4 v = dst[f];
        const float4 gg = g4[f], bb = b4[f];
        v.x = (v.x - mean) * rstd * gg.x + bb.x;
        v.y = (v.y - mean) * rstd * gg.y + bb.y;
        v.z = (v.z - mean) * rstd * gg.z + bb.z;
        v.w = (v.w - mean) * rstd * gg.w + bb.w;
        dst[f] = v;
      }
    } else {
      for (int f = tid; f < d / 4; f += kLmThreads) dst[f] = src[f];
    }
  }
  __syncthreads();

  float best[M];
  int bi[M];
#pragma unroll
  for (int m = 0; m < M; ++m) {
    best[m] = -FLT_MAX;
    bi[m] = INT_MAX;
  }
  bool ok = true;
  if (rows > 0) ok = mbar_wait(bar, 0, a.status);
  if (ok) {
    const float4* w4 = reinterpret_cast<const float4*>(wsm);
    const float4* h4 = reinterpret_cast<const float4*>(hsm);
    const int F = d / 4;
    for (int r = warp; r < rows; r += kLmWarps) {
      float acc[M];
#pragma unroll
      for (int m = 0; m < M; ++m) acc[m] = 0.f;
      for (int f = lane; f < F; f += 32) {
        const float4 w = w4[(size_t)r * F + f];
#pragma unroll
        for (int m = 0; m < M; ++m) {
          const float4 h = h4[(size_t)m * F + f];
          acc[m] = fmaf(w.x, h.x, acc[m]);
          acc[m] = fmaf(w.y, h.y, acc[m]);
          acc[m] = fmaf(w.z, h.z, acc[m]);
          acc[m] = fmaf(w.w, h.w, acc[m]);
        }
      }
      const int v = v0 + r;
      float sv[M];
#pragma unroll
      for (int m = 0; m < M; ++m) {
        sv[m] = warp_sum(acc[m]);
        if (lane == 0 && a.logits) a.logits[(size_t)(a.m_base + m) * a.V + v] = sv[m];
      }
#pragma unroll
      for (int m = 0; m < M; ++m) {
        // classifier-free guidance: both rows of a pair choose by u + scale (k - u)
        float g = sv[m];
        if (M >= 2 && a.guidance != 0.f) {
          const int c = m & ~1;
          g = sv[c + 1] + a.guidance * (sv[c] - sv[c + 1]);
        }
        if (better(g, v, best[m], bi[m])) {
          best[m] = g;
          bi[m] = v;
        }
      }
    }
  }
  if (lane == 0) {
#pragma unroll
    for (int m = 0; m < M; ++m) {
      bval[warp * M + m] = best[m];
      bidx[warp * M + m] = bi[m];
    }
  }
  // a CTA whose weight rows never arrived marks its result with index -1, so the failure
  // reaches the argmax even when the caller passed no status word
  const int cta_failed = __syncthreads_or(!ok);
  if (tid < M) {
    float bv = -FLT_MAX;
    int bx = INT_MAX;
    for (int w = 0; w < kLmWarps; ++w)
      if (better(bval[w * M + tid], bidx[w * M + tid], bv, bx)) {
        bv = bval[w * M + tid];
        bx = bidx[w * M + tid];
      }
    a.part_val[(size_t)blockIdx.x * 64 + a.m_base + tid] = bv;
    a.part_idx[(size_t)blockIdx.x * 64 + a.m_base + tid] = cta_failed ? -1 : bx;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) last = (atomicAdd(a.counter, 1u) == gridDim.x - 1) ? 1u : 0u;
  __syncthreads();
  if (!last) return;
  __threadfence();
  const int len = a.dlen ? *reinterpret_cast<volatile int*>(a.dlen) : 0;
  // every thread takes a share of the per-CTA results, then a block argmax
  bool any_failed = false;
  for (int m = 0; m < M; ++m) {
    const int mg = a.m_base + m;
    float bv = -FLT_MAX;
    int bx = INT_MAX;
    for (int c = tid; c < (int)gridDim.x; c += kLmThreads) {
      const float v = __ldcg(a.part_val + (size_t)c * 64 + mg);
      const int i = __ldcg(a.part_idx + (size_t)c * 64 + mg);
      if (i < 0) any_failed = true;
      else if (argmax_better(v, i, bv, bx)) {
        bv = v;
        bx = i;
      }
    }
    warp_argmax(bv, bx);
    if (lane == 0) {
      bval[warp * M + m] = bv;
      bidx[warp * M + m] = bx;
    }
  }
  const int failed = __syncthreads_or(any_failed);
  if (tid < M) {
    const int mg = a.m_base + tid;
    float bv = -FLT_MAX;
    int bx = INT_MAX;
    for (int w = 0; w < kLmWarps; ++w)
      if (argmax_better(bval[w * M + tid], bidx[w * M + tid], bv, bx)) {
        bv = bval[w * M + tid];
        bx = bidx[w * M + tid];
      }
    if (bx == INT_MAX) bx = 0;
    if (failed) bx = -1;   // some CTA's weight rows never arrived: no valid choice
    if (a.argmax) a.argmax[mg] = bx;
    if (a.hist) a.hist[(size_t)(len + a.hist_off) * a.hist_B + mg] = bx;
  }
  __syncthreads();
  if (tid == 0) {
    *a.counter = 0u;
    if (a.len_add) *a.dlen = len + a.len_add;
  }
}

cudaError_t launch_lm_head(const Launch& L, const float* x, int ldx, int M, int d, const float* ln_g,
                           const float* ln_b, float eps, const float* W, int V, float* logits, int32_t* argmax,
                           int32_t* hist, int hist_B, int hist_off, int* dlen, int len_add, const LmHeadWork& w,
                           float guidance) {
  if (M < 1 || M > 64 || d % 128 != 0) return cudaErrorInvalidValue;
  if (guidance != 0.f && M % 2 != 0) return cudaErrorInvalidValue;
  LmArgs a;
  a.x = x;
  a.ldx = ldx;
  a.d = d;
  a.ln_g = ln_g;
  a.ln_b = ln_b;
  a.eps = eps;
  a.W = W;
  a.V = V;
  a.rpc = lm_rpc(V);
  a.logits = logits;
  a.argmax = argmax;
  a.hist = hist;
  a.hist_B = hist_B;
  a.hist_off = hist_off;
  a.dlen = dlen;
  a.part_val = w.part_val;
  a.part_idx = w.part_idx;
  a.counter = w.counter;
  a.status = L.status;
  a.guidance = guidance;
  const int grid = (V + a.rpc - 1) / a.rpc;
  cudaError_t e = cudaSuccess;
  // chunks of 8, 4, 2 (then 1) rows: the rows of a guidance pair stay in one launch
  for (int mb = 0, mc = 0; mb < M && e == cudaSuccess; mb += mc) {
    const int rest = M - mb;
    mc = rest >= kLmMaxChunk ? kLmMaxChunk : rest >= 4 ? 4 : rest >= 2 ? 2 : 1;
    const int mp = mc;
    a.m_base = mb;
    a.M = mc;
    a.len_add = (mb + mc >= M) ? len_add : 0;
    const size_t smem = 16 + (size_t)a.rpc * d * 4 + (size_t)mp * d * 4 + 64 * 4 + kLmWarps * mp * 8;
    Launch Lc = L;
    if (mb > 0) Lc.pdl = true;
    // A chunk of mc rows runs the mp-row kernel on rows mb .. mb + mp - 1; rows past M
    // would read past x, so only exact sizes use the padded kernel.
    switch (mp == mc ? mp : 1) {
      case 8: {
        e = launch_k(Lc, lm_head_kernel<8>, dim3(grid), dim3(kLmThreads), smem, a);
        break;
      }
      case 4: {
        e = launch_k(Lc, lm_head_kernel<4>, dim3(grid), dim3(kLmThreads), smem, a);
        break;
      }
      case 2: {
        e = launch_k(Lc, lm_head_kernel<2>, dim3(grid), dim3(kLmThreads), smem, a);
        break;
      }
      default: {
        // odd chunk sizes: one row per launch
        auto k = lm_head_kernel<1>;
        const size_t s1 = 16 + (size_t)a.rpc * d * 4 + (size_t)d * 4 + 64 * 4 + kLmWarps * 8;
        for (int j = 0; j < mc && e == cudaSuccess; ++j) {
          LmArgs b = a;
          b.m_base = mb + j;
          b.M = 1;
          b.len_add = (mb + j == M - 1) ? len_add : 0;
          Launch Lj = L;
          if (mb + j > 0) Lj.pdl = true;
          e = launch_k(Lj, k, dim3(grid), dim3(kLmThreads), s1, b);
        }
        break;
      }
    }
  }
  return e;
}

cudaError_t init_attrs_gemv() {
  cudaError_t e = cudaSuccess;
  if (e == cudaSuccess) e = gemv_attrs_mf<1, kInt4>();
  if (e == cudaSuccess) e = gemv_attrs_mf<2, kInt4>();
  if (e == cudaSuccess) e = gemv_attrs_mf<4, kInt4>();
  if (e == cudaSuccess) e = gemv_attrs_mf<8, kInt4>();
  if (e == cudaSuccess) e = gemv_attrs_mf<1, kFp16>();
  if (e == cudaSuccess) e = gemv_attrs_mf<2, kFp16>();
  if (e == cudaSuccess) e = gemv_attrs_mf<4, kFp16>();
  if (e == cudaSuccess) e = gemv_attrs_mf<8, kFp16>();
  if (e == cudaSuccess) e = allow_smem(lm_head_kernel<1>, kMaxDynSmem);
  if (e == cudaSuccess) e = allow_smem(lm_head_kernel<2>, kMaxDynSmem);
  if (e == cudaSuccess) e = allow_smem(lm_head_kernel<4>, kMaxDynSmem);
  if (e == cudaSuccess) e = allow_smem(lm_head_kernel<8>, kMaxDynSmem);
  return e;
}

}  // namespace ms
