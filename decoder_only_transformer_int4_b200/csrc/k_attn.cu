// Attention over the shared in-place KV cache ("MuScriptor Medium — optimized W4A32
// ONNX Runtime", Model variant: GroupQueryAttention nodes, fixed-capacity cache shared by
// past and present).  Causal, scale 1/sqrt(64), query head h reads kv head h / (H / Hk).
//
// Cache layout: K and V each [B][Hk][cap][64] per layer, so the keys of one (stream,
// kv head) are one contiguous run of 256-byte rows.
#include <cuda_fp16.h>
#include <math.h>
#include "ms_device.cuh"
#include "ms_launch.cuh"

namespace ms {

// ---------------------------------------------------------------------------------
// Decode: split-K flash-decoding.  Grid (splits, Hk, B).  Each CTA takes a contiguous
// run of positions of one (stream, kv head), computes the scores of all H/Hk query heads
// of the group against it (each key is read once for the whole group), keeps a running
// max / sum / weighted V sum, and writes its partial (m, l, o).  The last CTA of the
// (stream, kv head) to finish — an atomic ticket, nothing waits — merges the partials.
// The split count adapts to the current length read from the device, so one launch
// configuration (and one captured graph) serves every step.
// ---------------------------------------------------------------------------------
namespace {
constexpr int kDecThreads = 128;
constexpr int kDecSub = 64;        // positions staged in shared memory at a time
static_assert(kDecThreads == 2 * kDecSub && kDecSub == 64, "the score and PV loops map two thread halves onto 64 rows");
constexpr int kMinPerSplit = 16;   // smallest run of positions worth a CTA
constexpr int kDecTargetCtas = 6 * 148;   // several resident CTAs per SM overlap their K/V loads
constexpr int kMaxSplits = 128;    // partials one (stream, kv head) may have

struct AttnDecArgs {
  const float* q;
  const void* kc;   // fp32 or IEEE half elements (the kernel's KV parameter)
  const void* vc;
  int B, H, Hk, cap;
  const int* dlen;
  int add;
  int splits;
  float* part;
  unsigned* counters;
  __half* oh;       // if set, the result as fp16 hi / lo planes [B][ldo] instead of fp32 o
  __half* ol;
  int ldo;
  float* o;
};
}  // namespace

int attn_decode_splits(int B, int Hk, int cap) {
  int s = (kDecTargetCtas + B * Hk - 1) / (B * Hk);
  const int most = (cap + kMinPerSplit - 1) / kMinPerSplit;
  if (s > most) s = most;
  if (s > kMaxSplits) s = kMaxSplits;
  if (s < 1) s = 1;
  return s;
}

template <int HPG, int KV>
__global__ void __launch_bounds__(kDecThreads) attn_decode_kernel(AttnDecArgs a) {
  __shared__ __align__(16) float qs[HPG][64];
  __shared__ float Ks[kDecSub][65];
  __shared__ __align__(16) float Vs[kDecSub][64];
  __shared__ __align__(16) float sc[HPG][kDecSub];
  __shared__ float mh[HPG], lh[HPG], corr[HPG];
  __shared__ float mwbuf[HPG * kMaxSplits], lbuf[HPG * kMaxSplits];
  __shared__ unsigned last;
  constexpr int kSlots = (HPG * 64 + kDecThreads - 1) / kDecThreads;
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  pdl_wait();
  pdl_trigger();
  const int T = *a.dlen + a.add;
  int s_act = (T + kMinPerSplit - 1) / kMinPerSplit;
  if (s_act > (int)gridDim.x) s_act = gridDim.x;
  if (s_act < 1) s_act = 1;
  const int chunk = (T + s_act - 1) / s_act;
  s_act = (T + chunk - 1) / chunk;  // every active split gets at least one position
  if (split >= s_act) return;
  const int t0 = split * chunk;
  const int t1 = min(T, t0 + chunk);

  for (int i = tid; i < HPG * 64; i += kDecThreads)
    qs[i >> 6][i & 63] = a.q[((size_t)b * a.H + g * HPG + (i >> 6)) * 64 + (i & 63)] * 0.125f;
  if (tid < HPG) {
    mh[tid] = -INFINITY;
    lh[tid] = 0.f;
  }
  float oacc[kSlots];
#pragma unroll
  for (int k = 0; k < kSlots; ++k) oacc[k] = 0.f;

  const size_t head = ((size_t)b * a.Hk + g) * a.cap * 64;   // first element of the head's rows

  // K/V of the next run of positions are loaded into registers while the current run is
  // computed (each thread: elements 4f .. 4f + 3 of row p, i = tid + 128 j of the run, j < 8)
  constexpr int kPf = kDecSub * 16 / kDecThreads;
  float4 pk[kPf], pv[kPf];
  auto fetch = [&](int c0, int cn) {
#pragma unroll
    for (int j = 0; j < kPf; ++j) {
      const int i = tid + j * kDecThreads, p = i >> 4, f = i & 15;
      if (p < cn) {
        pk[j] = kv_load4<KV>(a.kc, head + (size_t)(c0 + p) * 64 + 4 * f);
        pv[j] = kv_load4<KV>(a.vc, head + (size_t)(c0 + p) * 64 + 4 * f);
      }
    }
  };
  if (t0 < t1) fetch(t0, min(kDecSub, t1 - t0));
  for (int c0 = t0; c0 < t1; c0 += kDecSub) {
    const int cn = min(kDecSub, t1 - c0);
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kPf; ++j) {
      const int i = tid + j * kDecThreads, p = i >> 4, f = i & 15;
      if (p < cn) {
        Ks[p][4 * f + 0] = pk[j].x;
        Ks[p][4 * f + 1] = pk[j].y;
        Ks[p][4 * f + 2] = pk[j].z;
        Ks[p][4 * f + 3] = pk[j].w;
        reinterpret_cast<float4*>(&Vs[p][0])[f] = pv[j];
      } else {
        reinterpret_cast<float4*>(&Vs[p][0])[f] = make_float4(0.f, 0.f, 0.f, 0.f);   // read as 0 x p = 0
      }
    }
    if (c0 + kDecSub < t1) fetch(c0 + kDecSub, min(kDecSub, t1 - c0 - kDecSub));
    __syncthreads();
    {
      // thread: position p = tid % 64, heads hg, hg + 2, ... (hg = tid / 64); each K element is
      // loaded once for all of them, q by broadcast float4 reads
      const int p = tid & (kDecSub - 1), hg = tid / kDecSub;
      float sacc[kSlots];
#pragma unroll
      for (int k = 0; k < kSlots; ++k) sacc[k] = 0.f;
#pragma unroll 4
      for (int dd = 0; dd < 64; dd += 4) {
        const float k0 = Ks[p][dd], k1 = Ks[p][dd + 1], k2 = Ks[p][dd + 2], k3 = Ks[p][dd + 3];
#pragma unroll
        for (int k = 0; k < kSlots; ++k) {
          const int h = hg + 2 * k;
          if (h < HPG) {
            const float4 q4 = *reinterpret_cast<const float4*>(&qs[h][dd]);
            sacc[k] = fmaf(q4.x, k0, fmaf(q4.y, k1, fmaf(q4.z, k2, fmaf(q4.w, k3, sacc[k]))));
          }
        }
      }
#pragma unroll
      for (int k = 0; k < kSlots; ++k) {
        const int h = hg + 2 * k;
        if (h < HPG) sc[h][p] = p < cn ? sacc[k] : -INFINITY;
      }
    }
    __syncthreads();
    for (int h = warp; h < HPG; h += kDecThreads / 32) {
      const float v0 = sc[h][lane], v1 = sc[h][lane + 32];
      const float mx = warp_max(fmaxf(v0, v1));
      const float mold = mh[h];
      const float mnew = fmaxf(mold, mx);
      const float e0 = lane < cn ? expf(v0 - mnew) : 0.f;
      const float e1 = lane + 32 < cn ? expf(v1 - mnew) : 0.f;
      sc[h][lane] = e0;
      sc[h][lane + 32] = e1;
      const float sum = warp_sum(e0 + e1);
      __syncwarp();
      if (lane == 0) {
        const float cf = expf(mold - mnew);
        corr[h] = cf;
        lh[h] = lh[h] * cf + sum;
        mh[h] = mnew;
      }
    }
    __syncthreads();
    {
      // thread: dimension dd = tid % 64 of heads hg, hg + 2, ...; each V element loaded once for
      // all of them, the probabilities by broadcast float4 reads (rows past cn hold 0 x 0)
      const int dd = tid & 63, hg = tid >> 6;
      const int cn4 = (cn + 3) & ~3;
#pragma unroll
      for (int k = 0; k < kSlots; ++k)
        if (hg + 2 * k < HPG) oacc[k] *= corr[hg + 2 * k];
      for (int p = 0; p < cn4; p += 4) {
        const float v0 = Vs[p][dd], v1 = Vs[p + 1][dd], v2 = Vs[p + 2][dd], v3 = Vs[p + 3][dd];
#pragma unroll
        for (int k = 0; k < kSlots; ++k) {
          const int h = hg + 2 * k;
          if (h < HPG) {
            const float4 p4 = *reinterpret_cast<const float4*>(&sc[h][p]);
            oacc[k] = fmaf(p4.x, v0, fmaf(p4.y, v1, fmaf(p4.z, v2, fmaf(p4.w, v3, oacc[k]))));
          }
        }
      }
    }
  }
  __syncthreads();

  float* pb = a.part + (((size_t)b * a.Hk + g) * a.splits + split) * HPG * 66;
#pragma unroll
  for (int k = 0; k < kSlots; ++k) {
    const int idx = tid + k * kDecThreads;
    if (idx < HPG * 64) pb[(idx >> 6) * 66 + 2 + (idx & 63)] = oacc[k];
  }
  if (tid < HPG) {
    pb[tid * 66 + 0] = mh[tid];
    pb[tid * 66 + 1] = lh[tid];
  }
  __threadfence();
  __syncthreads();
  unsigned* ctr = a.counters + (size_t)b * a.Hk + g;
  if (tid == 0) last = (atomicAdd(ctr, 1u) == (unsigned)(s_act - 1)) ? 1u : 0u;
  __syncthreads();
  if (!last) return;
  __threadfence();
  // Merge: weight of split s for head h is exp(m_s - M) with M the largest m_s; the
  // loads of every split go out together (one round trip per step of the merge).
  const float* p0 = a.part + ((size_t)b * a.Hk + g) * a.splits * HPG * 66;
  __shared__ float Linv[HPG];
  for (int i = tid; i < HPG * s_act; i += kDecThreads) {
    const int h = i / s_act, s = i - h * s_act;
    mwbuf[h * kMaxSplits + s] = __ldcg(p0 + ((size_t)s * HPG + h) * 66);
    lbuf[h * kMaxSplits + s] = __ldcg(p0 + ((size_t)s * HPG + h) * 66 + 1);
  }
  __syncthreads();
  for (int h = warp; h < HPG; h += kDecThreads / 32) {
    float mx = -INFINITY;
    for (int s = lane; s < s_act; s += 32) mx = fmaxf(mx, mwbuf[h * kMaxSplits + s]);
    mx = warp_max(mx);
    float l = 0.f;
    for (int s = lane; s < s_act; s += 32) {
      const float w = expf(mwbuf[h * kMaxSplits + s] - mx);
      mwbuf[h * kMaxSplits + s] = w;
      l = fmaf(w, lbuf[h * kMaxSplits + s], l);
    }
    l = warp_sum(l);
    if (lane == 0) Linv[h] = 1.0f / l;
  }
  __syncthreads();
  for (int idx = tid; idx < HPG * 64; idx += kDecThreads) {
    const int h = idx >> 6, dd = idx & 63;
    float O = 0.f;
#pragma unroll 8
    for (int s = 0; s < s_act; ++s) O = fmaf(mwbuf[h * kMaxSplits + s], __ldcg(p0 + ((size_t)s * HPG + h) * 66 + 2 + dd), O);
    const float r = O * Linv[h];
    if (a.oh) {
      const __half hi = __float2half_rn(r);
      a.oh[(size_t)b * a.ldo + (g * HPG + h) * 64 + dd] = hi;
      a.ol[(size_t)b * a.ldo + (g * HPG + h) * 64 + dd] = __float2half_rn(r - __half2float(hi));
    } else {
      a.o[((size_t)b * a.H + g * HPG + h) * 64 + dd] = r;
    }
  }
  if (tid == 0) *ctr = 0u;
}

template <int HPG>
static cudaError_t attn_dec_go(const Launch& L, const AttnDecArgs& a, int kv16) {
  if (kv16) return launch_k(L, attn_decode_kernel<HPG, 1>, dim3(a.splits, a.Hk, a.B), dim3(kDecThreads), 0, a);
  return launch_k(L, attn_decode_kernel<HPG, 0>, dim3(a.splits, a.Hk, a.B), dim3(kDecThreads), 0, a);
}

cudaError_t launch_attn_decode(const Launch& L, const float* q, const void* kc, const void* vc, int B, int H,
                               int Hk, int cap, const int* dlen, int add, const AttnDecodeWork& w, float* o,
                               int kv16, __half* oh, __half* ol, int ldo) {
  if (oh && (!ol || ldo < H * 64)) return cudaErrorInvalidValue;
  AttnDecArgs a;
  a.oh = oh;
  a.ol = ol;
  a.ldo = ldo;
  a.q = q;
  a.kc = kc;
  a.vc = vc;
  a.B = B;
  a.H = H;
  a.Hk = Hk;
  a.cap = cap;
  a.dlen = dlen;
  a.add = add;
  a.splits = w.splits;
  a.part = w.part;
  a.counters = w.counters;
  a.o = o;
  switch (H / Hk) {
    case 1: return attn_dec_go<1>(L, a, kv16);
    case 2: return attn_dec_go<2>(L, a, kv16);
    case 3: return attn_dec_go<3>(L, a, kv16);
    case 4: return attn_dec_go<4>(L, a, kv16);
    case 6: return attn_dec_go<6>(L, a, kv16);
    case 8: return attn_dec_go<8>(L, a, kv16);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace ms
