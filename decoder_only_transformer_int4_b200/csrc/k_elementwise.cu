// Elementwise kernels of the decoder step: RTN INT4 quantiser, token embedding with
// the conditioner prefix, SkipLayerNorm, RoPE with the in-place KV-cache append.
#include "ms_device.cuh"
#include "ms_launch.cuh"

namespace ms {

// ---------------------------------------------------------------------------------
// Symmetric RTN INT4, group 32 along K ("MuScriptor Medium — optimized W4A32 ONNX
// Runtime", Model variant).  One thread per group: scale = absmax / 7 and
// q = clamp(rint(w / scale), -7, 7), both divisions IEEE fp32 (__fdiv_rn), rint ties to
// even; nibble u = q + 8 with element 2j in the low nibble of byte j.
// ---------------------------------------------------------------------------------
__global__ void quantize_int4_kernel(const float* __restrict__ w, long long groups,
                                     uint8_t* __restrict__ packed, float* __restrict__ scales) {
  const long long gi = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (gi >= groups) return;
  const float4* src = reinterpret_cast<const float4*>(w + gi * 32);
  float v[32];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 t = src[i];
    v[4 * i] = t.x;
    v[4 * i + 1] = t.y;
    v[4 * i + 2] = t.z;
    v[4 * i + 3] = t.w;
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const float s = __fdiv_rn(amax, 7.0f);
  uint32_t words[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    int q = 0;
    if (s != 0.f) {
      float r = rintf(__fdiv_rn(v[i], s));
      r = fminf(fmaxf(r, -7.f), 7.f);
      q = static_cast<int>(r);
    }
    words[i >> 3] |= static_cast<uint32_t>(q + 8) << (4 * (i & 7));
  }
  reinterpret_cast<uint4*>(packed)[gi] = make_uint4(words[0], words[1], words[2], words[3]);
  scales[gi] = s;
}

cudaError_t launch_quantize_int4(const float* w, int N, int K, uint8_t* packed, float* scales, cudaStream_t s) {
  const long long groups = (long long)N * (K / 32);
  if (groups == 0) return cudaSuccess;
  const int block = 256;
  const long long grid = (groups + block - 1) / block;
  quantize_int4_kernel<<<(unsigned)grid, block, 0, s>>>(w, groups, packed, scales);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------------
// Embedding.  Prefill rows of stream b: P prefix rows (the conditioner output is used as
// a prefix condition, "MuScriptor — small (≈100M)", Model description), then E[token]
// for each of S tokens ("MuScriptor small — ONNX conversion", muscriptor-small-lm.onnx).
// Token ids outside [0, V) are clamped and flagged in the status word.
// ---------------------------------------------------------------------------------
__global__ void embed_prefill_kernel(const int64_t* __restrict__ tokens, int S, const float* __restrict__ prefix,
                                     int P, const float* __restrict__ E, int V, int d, float* __restrict__ x,
                                     unsigned* status) {
  pdl_wait();
  pdl_trigger();
  const int r = blockIdx.x, b = blockIdx.y, n = P + S;
  const float4* src;
  if (r < P) {
    src = reinterpret_cast<const float4*>(prefix + ((size_t)b * P + r) * d);
  } else {
    long long t = tokens[(size_t)b * S + (r - P)];
    if (t < 0 || t >= V) {
      if (threadIdx.x == 0) flag_error(status, kErrToken);
      t = t < 0 ? 0 : V - 1;
    }
    src = reinterpret_cast<const float4*>(E + (size_t)t * d);
  }
  float4* dst = reinterpret_cast<float4*>(x + ((size_t)b * n + r) * d);
  for (int i = threadIdx.x; i < d / 4; i += blockDim.x) dst[i] = src[i];
}

cudaError_t launch_embed_prefill(const Launch& L, const int64_t* tokens, int S, const float* prefix, int P,
                                 const float* tok_emb, int V, int d, int B, float* x) {
  return launch_k(L, embed_prefill_kernel, dim3(P + S, B), dim3(128), 0, tokens, S, prefix, P, tok_emb, V, d, x,
                  L.status);
}

__global__ void embed_decode_kernel(const int32_t* __restrict__ tokens, const int32_t* __restrict__ hist,
                                    const int* __restrict__ dlen, const float* __restrict__ E, int V, int d, int B,
                                    float* __restrict__ x, unsigned* status) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.x;
  int t;
  if (tokens) {
    t = tokens[b];
  } else {
    const int len = *dlen;
    t = len > 0 ? hist[(size_t)(len - 1) * B + b] : 0;
  }
  if (t < 0 || t >= V) {
    if (threadIdx.x == 0) flag_error(status, kErrToken);
    t = t < 0 ? 0 : V - 1;
  }
  const float4* src = reinterpret_cast<const float4*>(E + (size_t)t * d);
  float4* dst = reinterpret_cast<float4*>(x + (size_t)b * d);
  for (int i = threadIdx.x; i < d / 4; i += blockDim.x) dst[i] = src[i];
}

cudaError_t launch_embed_decode(const Launch& L, const int32_t* tokens, const int32_t* hist, const int* dlen,
                                const float* tok_emb, int V, int d, int B, float* x) {
  return launch_k(L, embed_decode_kernel, dim3(B), dim3(128), 0, tokens, hist, dlen, tok_emb, V, d, B, x, L.status);
}

// ---------------------------------------------------------------------------------
// SkipLayerNormalization ("MuScriptor Medium — optimized W4A32 ONNX Runtime", Model
// variant): s = x + y written back to x, h = (s - mean) / sqrt(var + eps) * gamma + beta,
// biased variance, two passes over registers.  One warp per row; d a multiple of 128.
// ---------------------------------------------------------------------------------
template <int NVMAX>
__global__ void __launch_bounds__(256) skipln_kernel(float* __restrict__ x, const float* __restrict__ y,
                                                     const float* __restrict__ g, const float* __restrict__ bta,
                                                     float eps, int R, int d, float* __restrict__ h,
                                                     __half* __restrict__ hh, __half* __restrict__ hl, int ldh,
                                                     unsigned* status) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= R) return;
  const int nv = d / 128;
  float4* xr = reinterpret_cast<float4*>(x + (size_t)row * d);
  const float4* yr = y ? reinterpret_cast<const float4*>(y + (size_t)row * d) : nullptr;
  float4 v[NVMAX];
  float sum = 0.f;
#pragma unroll
  for (int j = 0; j < NVMAX; ++j) {
    if (j < nv) {
      float4 t = xr[lane + 32 * j];
      if (yr) {
        const float4 u = yr[lane + 32 * j];
        t.x += u.x;
        t.y += u.y;
        t.z += u.z;
        t.w += u.w;
        xr[lane + 32 * j] = t;
      }
      v[j] = t;
      sum += (t.x + t.y) + (t.z + t.w);
    }
  }
  const float mean = warp_sum(sum) / d;
  float sq = 0.f;
#pragma unroll
  for (int j = 0; j < NVMAX; ++j) {
    if (j < nv) {
      const float a = v[j].x - mean, b = v[j].y - mean, c = v[j].z - mean, e = v[j].w - mean;
      sq += (a * a + b * b) + (c * c + e * e);
    }
  }
  const float var = warp_sum(sq) / d;
  const float rstd = 1.0f / sqrtf(var + eps);
  const float4* g4 = reinterpret_cast<const float4*>(g);
  const float4* b4 = reinterpret_cast<const float4*>(bta);
  float4* hr = h ? reinterpret_cast<float4*>(h + (size_t)row * d) : nullptr;
  bool big = false;
#pragma unroll
  for (int j = 0; j < NVMAX; ++j) {
    if (j < nv) {
      const int f = lane + 32 * j;
      const float4 gg = g4[f], bb = b4[f];
      float4 o;
      o.x = (v[j].x - mean) * rstd * gg.x + bb.x;
      o.y = (v[j].y - mean) * rstd * gg.y + bb.y;
      o.z = (v[j].z - mean) * rstd * gg.z + bb.z;
      o.w = (v[j].w - mean) * rstd * gg.w + bb.w;
      if (hr) hr[f] = o;
      if (hh) {
        // fp16 hi / lo planes: hi = fp16(v), lo = fp16(v - hi)
        const __half2 h0 = __floats2half2_rn(o.x, o.y), h1 = __floats2half2_rn(o.z, o.w);
        const float2 f0 = __half22float2(h0), f1 = __half22float2(h1);
        const __half2 l0 = __floats2half2_rn(o.x - f0.x, o.y - f0.y), l1 = __floats2half2_rn(o.z - f1.x, o.w - f1.y);
        big |= fabsf(o.x) >= 65504.f || fabsf(o.y) >= 65504.f || fabsf(o.z) >= 65504.f || fabsf(o.w) >= 65504.f;
        __half2* ph = reinterpret_cast<__half2*>(hh + (size_t)row * ldh + 4 * f);
        __half2* pl = reinterpret_cast<__half2*>(hl + (size_t)row * ldh + 4 * f);
        ph[0] = h0;
        ph[1] = h1;
        pl[0] = l0;
        pl[1] = l1;
      }
    }
  }
  if (big) flag_error(status, kErrShape);
}

cudaError_t launch_skipln(const Launch& L, float* x, const float* y, const float* g, const float* b, float eps,
                          int R, int d, float* h, __half* hh, __half* hl, int ldh) {
  if (R <= 0) return cudaSuccess;
  if (d % 128 != 0 || d > 16 * 128) return cudaErrorInvalidValue;
  return launch_k(L, skipln_kernel<16>, dim3((R + 7) / 8), dim3(256), 0, x, y, g, b, eps, R, d, h, hh, hl, ldh,
                  L.status);
}

// ---------------------------------------------------------------------------------
// RoPE (base 1e4, pairs (i, i + 32) of each 64-wide head, (a, b) -> (a cos - b sin,
// a sin + b cos)) on the q and k parts of each new qkv row, then the in-place append of
// post-RoPE k and of v at the row's position into the fixed-capacity cache
// ("MuScriptor Medium — optimized W4A32 ONNX Runtime", Model variant: past and present
// share one preallocated buffer).  Positions are implicit: len + i for the i-th new row
// ("MuScriptor small — ONNX conversion", muscriptor-small-lm.onnx).  The cache holds fp32
// (KV = 0) or, in the half-precision cache option, the IEEE half of each value (KV = 1).
// ---------------------------------------------------------------------------------
template <int KV>
__global__ void __launch_bounds__(128) rope_append_kernel(const float* __restrict__ qkv, int n, int H, int Hk,
                                                          const float* __restrict__ cosv,
                                                          const float* __restrict__ sinv, const int* __restrict__ dlen,
                                                          float* __restrict__ q_out, void* __restrict__ kc,
                                                          void* __restrict__ vc, int cap, unsigned* status) {
  pdl_wait();
  pdl_trigger();
  const int r = blockIdx.x;
  const int b = r / n, i = r - b * n;
  const int pos = *dlen + i;
  if (pos >= cap) {
    if (threadIdx.x == 0) flag_error(status, kErrShape);
    return;
  }
  const int nq = (H + 2 * Hk) * 64;
  const float* row = qkv + (size_t)r * nq;
  const float* cs = cosv + (size_t)pos * 32;
  const float* sn = sinv + (size_t)pos * 32;
  for (int idx = threadIdx.x; idx < (H + Hk) * 32; idx += blockDim.x) {
    const int hh = idx >> 5, j = idx & 31;
    const float a = row[hh * 64 + j], bb = row[hh * 64 + j + 32];
    const float c = cs[j], s = sn[j];
    const float a2 = a * c - bb * s;
    const float b2 = a * s + bb * c;
    if (hh < H) {
      float* dst = q_out + (size_t)r * H * 64 + hh * 64;
      dst[j] = a2;
      dst[j + 32] = b2;
    } else {
      const size_t e = (((size_t)b * Hk + (hh - H)) * cap + pos) * 64;
      kv_store<KV>(kc, e + j, a2);
      kv_store<KV>(kc, e + j + 32, b2);
    }
  }
  for (int idx = threadIdx.x; idx < Hk * 64; idx += blockDim.x) {
    const int g = idx >> 6, dd = idx & 63;
    kv_store<KV>(vc, (((size_t)b * Hk + g) * cap + pos) * 64 + dd, row[(H + Hk) * 64 + idx]);
  }
}

cudaError_t launch_rope_append(const Launch& L, const float* qkv, int B, int n, int H, int Hk, const float* cosv,
                               const float* sinv, const int* dlen, float* q_out, void* kc, void* vc, int cap,
                               int kv16) {
  if (B * n <= 0) return cudaSuccess;
  if (kv16)
    return launch_k(L, rope_append_kernel<1>, dim3(B * n), dim3(128), 0, qkv, n, H, Hk, cosv, sinv, dlen, q_out, kc,
                    vc, cap, L.status);
  return launch_k(L, rope_append_kernel<0>, dim3(B * n), dim3(128), 0, qkv, n, H, Hk, cosv, sinv, dlen, q_out, kc, vc,
                  cap, L.status);
}

// ---------------------------------------------------------------------------------
// Tile-packed copies of the backbone matrices for the persistent decode kernel, whose
// matrix-vector products run on warp-level tensor-core MMAs (m16n8k16 with the weights as
// the A operand).  A record covers one tile of 16 rows and one group of 32 columns (k =
// 32g .. 32g + 31); records are stored tile by tile, groups in order.  Lane l = 4 r + t of a
// warp needs, of rows r and r + 8 of the tile, the columns 2t + {0, 1, 8, 9, 16, 17, 24, 25}:
//   INT4 record (320 bytes): 64 words, words 2l and 2l + 1 holding those eight codes
//     (u = q + 8) of rows r and r + 8 as nibbles — columns 2t, 2t+8, 2t+16, 2t+24 in bits
//     0-3, 4-7, 8-11, 12-15 and 2t+1, 2t+9, 2t+17, 2t+25 in bits 16-19, 20-23, 24-27, 28-31,
//     so that one mask with 0x000F000F or 0x00F000F0 yields a pair of them as two halves;
//     then the group's fp32 scales as pairs (row r, row r + 8), r = 0..7.
//   FP16 record (1024 bytes): 32 chunks of 32 bytes, chunk l holding the pairs (r, 2t),
//     (r + 8, 2t), (r, 2t + 8), (r + 8, 2t + 8), then the same at columns + 16.
// ---------------------------------------------------------------------------------
__global__ void repack_int4_tiles_kernel(const uint8_t* __restrict__ rows, int ldq, int K, long long records,
                                         uint32_t* __restrict__ out) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= records * 80) return;
  const long long rec = i / 80;
  const int w = (int)(i - rec * 80);
  const int KG = K / 32;
  const long long t = rec / KG;
  const int g = (int)(rec - t * KG);
  if (w < 64) {
    const int l = w >> 1, r = (l >> 2) + 8 * (w & 1), tq = l & 3;
    const uint8_t* row = rows + (size_t)(t * 16 + r) * ldq;
    auto nib = [&](int k) -> uint32_t {
      const int kk = g * 32 + k;
      return (row[kk >> 1] >> (4 * (kk & 1))) & 15u;
    };
    const int c = 2 * tq;
    out[i] = nib(c) | nib(c + 8) << 4 | nib(c + 16) << 8 | nib(c + 24) << 12 | nib(c + 1) << 16 | nib(c + 9) << 20 |
             nib(c + 17) << 24 | nib(c + 25) << 28;
  } else {
    const int r = ((w - 64) >> 1) + 8 * ((w - 64) & 1);
    const float* sc = reinterpret_cast<const float*>(rows + (size_t)(t * 16 + r) * ldq + K / 2);
    out[i] = __float_as_uint(sc[g]);
  }
}

__global__ void repack_f16_tiles_kernel(const uint16_t* __restrict__ w, int K, long long records,
                                        uint32_t* __restrict__ out) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= records * 256) return;
  const long long rec = i / 256;
  const int j = (int)(i - rec * 256);
  const int l = j >> 3, reg = j & 3, step = (j >> 2) & 1;
  const int KG = K / 32;
  const long long t = rec / KG;
  const int g = (int)(rec - t * KG);
  const int r = (l >> 2) + ((reg & 1) ? 8 : 0), tq = l & 3;
  const uint16_t* row = w + (size_t)(t * 16 + r) * K + g * 32 + 2 * tq + ((reg & 2) ? 8 : 0) + 16 * step;
  out[i] = (uint32_t)row[0] | (uint32_t)row[1] << 16;
}

cudaError_t launch_repack_tiles(const WView& w, void* out, cudaStream_t s) {
  if (w.N % 16 != 0 || w.K % 32 != 0) return cudaErrorInvalidValue;
  const long long records = (long long)(w.N / 16) * (w.K / 32);
  if (w.fmt == kInt4) {
    if (!w.interleaved()) return cudaErrorInvalidValue;
    const long long n = records * 80;
    repack_int4_tiles_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(w.q, w.ldq, w.K, records,
                                                                         static_cast<uint32_t*>(out));
  } else {
    const long long n = records * 256;
    repack_f16_tiles_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(w.h, w.K, records,
                                                                        static_cast<uint32_t*>(out));
  }
  return cudaGetLastError();
}

size_t tile_packed_bytes(const WView& w) {
  const size_t records = (size_t)(w.N / 16) * (w.K / 32);
  return records * (w.fmt == kInt4 ? 320 : 1024);
}

}  // namespace ms
