// Persistent decode kernel: greedy decode steps of the whole decoder (all layers, LM head,
// argmax, token feedback) in one cooperative launch, one CTA per SM.
//
// Why: at a few streams the decoder step is a chain of ~5 dependent matrix-vector phases
// per layer, each moving only a few MB; separate kernel launches pay a launch and drain per
// phase.  Here each phase ends in a grid barrier instead, and the weight bytes — which
// never depend on the previous phase — stream continuously: a producer warp per CTA walks
// the CTA's whole weight schedule (every slice of every layer of every step) and issues
// bulk copies into a shared-memory ring, limited only by free slots, while eight consumer
// warps compute.  The HBM stream therefore runs ahead across phase, layer and step
// boundaries.
//
// Phases of one step (token position pos, T = pos + 1 keys):
//   A  LN1 of x, QKV rows (raw q, k, v)                                 -> qkv
//   B  attention unit (stream, kv head, split): RoPE of q (and of the new k, which the
//      last split appends to the cache with v), scores over its run of positions, partial
//      (m, l, o); the last unit of a (stream, kv head) merges the partials  -> o
//   C  O rows, residual                                                  x += o Wo^T
//   D  LN2 of x, FC1 rows, GELU                                          -> u
//   E  FC2 rows, residual                                                x += u W2^T
//   after the last layer: LN_f of x, LM head rows, per-CTA argmax, last CTA picks the token,
//   records it in the token history and advances the cache length.
// The arithmetic per element is the same as the separate kernels' (fp32, INT4 codes
// converted exactly, one scale FMA per 32-element group).
//
// Every wait is bounded: the grid barrier's spin and the ring's mbarrier waits give up
// after a limit, set the status word's timeout bit and an abort word that makes every CTA
// leave; the producer then waits (bounded) for the copies it has in flight.
#include <float.h>
#include <limits.h>
#include "ms_device.cuh"
#include "ms_launch.cuh"
#include "ms_persistent.h"

namespace ms {

namespace {
constexpr int kConsumers = 256;
constexpr int kThreads = kConsumers + 32;
constexpr int kSlot = 16384;
constexpr long long kGridSpinLimit = 1ll << 24;  // polls of the barrier flag (~10 s)
constexpr int kAttSub = 64;
constexpr int kAttMaxSplits = 128;
constexpr int kMinPerSplit = 16;

__device__ __forceinline__ void consumer_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
// Named barrier of the consumer warps that also ORs a flag over them.
__device__ __forceinline__ bool consumer_bar_or(bool pred) {
  unsigned r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n barrier.cta.red.or.pred q, 1, 256, p;\n selp.u32 %0, 1, 0, q;\n}"
      : "=r"(r)
      : "r"((unsigned)pred)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_gpu(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned atom_add_release_gpu(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.add.release.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Rows [n0, n1) of an N-row matrix owned by CTA c of G (contiguous, balanced).
__device__ __forceinline__ void partition(int N, int c, int G, int& n0, int& n1) {
  n0 = (int)(((long long)N * c) / G);
  n1 = (int)(((long long)N * (c + 1)) / G);
}

struct Shape {
  int N[4], K[4], rowb[4];
};

__device__ __forceinline__ Shape shapes_of(const PersistArgs& a) {
  Shape s;
  const int d = a.d, H = a.H, Hk = a.Hk, F = a.F;
  s.N[0] = (H + 2 * Hk) * 64; s.K[0] = d;
  s.N[1] = d;                 s.K[1] = H * 64;
  s.N[2] = F;                 s.K[2] = d;
  s.N[3] = d;                 s.K[3] = F;
  for (int i = 0; i < 4; ++i) s.rowb[i] = a.fmt == kInt4 ? s.K[i] / 2 + s.K[i] / 8 : s.K[i] * 2;
  return s;
}

// Ring position shared by the producer and the consumers (each keeps its own copy).
struct RingPos {
  int slot = 0;
  uint32_t phase = 0;
  __device__ __forceinline__ void next(int nslot) {
    if (++slot == nslot) {
      slot = 0;
      phase ^= 1u;
    }
  }
};

struct Smem {
  uint64_t* full;
  uint64_t* empty;
  unsigned char* ring;
  float* act;      // activation rows / attention scratch
  float* red;      // 64 floats
};

__device__ __forceinline__ Smem carve(unsigned char* base, int nslot) {
  Smem s;
  s.full = reinterpret_cast<uint64_t*>(base);
  s.empty = s.full + 16;
  s.red = reinterpret_cast<float*>(s.empty + 16);
  s.ring = base + 1024;
  s.act = reinterpret_cast<float*>(s.ring + (size_t)nslot * kSlot);
  return s;
}

// ---------------------------------------------------------------------------------
// Producer: one lane issues every weight slice of the schedule in order.
// ---------------------------------------------------------------------------------
__device__ void producer(const PersistArgs& a, const Smem& sm) {
  const Shape sh = shapes_of(a);
  const int c = blockIdx.x, G = gridDim.x;
  RingPos rp;
  long long issued = 0;
  bool stop = false;
  auto issue = [&](const unsigned char* src, uint32_t bytes) {
    if (stop) return;
    long long it = 0;
    while (!mbar_try_wait(&sm.empty[rp.slot], rp.phase ^ 1u)) {
      if ((++it & 255) == 0 && (*reinterpret_cast<volatile unsigned*>(a.abort) || it > kSpinLimit)) {
        if (it > kSpinLimit) {
          flag_error(a.status, kErrTimeout);
          atomicExch(a.abort, 1u);
        }
        stop = true;
        return;
      }
    }
    mbar_expect_tx(&sm.full[rp.slot], bytes);
    bulk_g2s(sm.ring + (size_t)rp.slot * kSlot, src, bytes, &sm.full[rp.slot]);
    ++issued;
    rp.next(a.nslot);
  };
  for (int step = 0; step < a.n_steps && !stop; ++step) {
    for (int l = 0; l < a.L && !stop; ++l) {
      for (int mi = 0; mi < 4 && !stop; ++mi) {
        int n0, n1;
        partition(sh.N[mi], c, G, n0, n1);
        const int rb = sh.rowb[mi];
        const int rpp = kSlot / rb;
        const unsigned char* w = a.layers[l].w[mi];
        for (int p = n0; p < n1 && !stop; p += rpp) {
          const int rows = min(rpp, n1 - p);
          issue(w + (size_t)p * rb, (uint32_t)(rows * rb));
        }
      }
    }
    int v0, v1;
    partition(a.V, c, G, v0, v1);
    const int rb = a.d * 4;
    const int rpp = kSlot / rb;
    for (int p = v0; p < v1 && !stop; p += rpp) {
      const int rows = min(rpp, v1 - p);
      issue(reinterpret_cast<const unsigned char*>(a.lm_head) + (size_t)p * rb, (uint32_t)(rows * rb));
    }
  }
  if (stop) {
    // wait (bounded) for the copies that may still be in flight before leaving
    RingPos back = rp;
    const long long n = issued < a.nslot ? issued : a.nslot;
    for (long long i = 0; i < n; ++i) {
      back.slot = back.slot == 0 ? a.nslot - 1 : back.slot - 1;
      if (back.slot == a.nslot - 1) back.phase ^= 1u;
      for (long long it = 0; it < kSpinLimit; ++it)
        if (mbar_try_wait(&sm.full[back.slot], back.phase)) break;
    }
  }
}

// ---------------------------------------------------------------------------------
// Consumer helpers
// ---------------------------------------------------------------------------------
__device__ __forceinline__ float csum(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum(v);
  consumer_bar();
  if (lane == 0) red[warp] = v;
  consumer_bar();
  float t = lane < kConsumers / 32 ? red[lane] : 0.f;
  return warp_sum(t);
}

// Rows m < M of src (stride ld floats, read through L2) into act, de-interleaved by 8-element
// words (elements 8c..8c+3 in one float4 array, 8c+4..8c+7 in the next), optionally
// LayerNorm'd.  natural = true keeps plain row order (the LM head).
template <int M>
__device__ void load_act(float* act, float* red, const float* src, int ld, int K, const float* g, const float* b,
                         float eps, bool natural) {
  const int tid = threadIdx.x, KW = K / 8;
  float4* a4 = reinterpret_cast<float4*>(act);
  for (int m = 0; m < M; ++m) {
    const float4* s4 = reinterpret_cast<const float4*>(src + (size_t)m * ld);
    float4* d4 = a4 + (size_t)m * (K / 4);
    auto at = [&](int f) -> float4& { return natural ? d4[f] : d4[(f & 1) * KW + (f >> 1)]; };
    float s = 0.f;
    for (int f = tid; f < K / 4; f += kConsumers) {
      const float4 v = __ldcg(s4 + f);
      at(f) = v;
      s += (v.x + v.y) + (v.z + v.w);
    }
    if (g) {
      const float mean = csum(s, red) / K;
      float q = 0.f;
      for (int f = tid; f < K / 4; f += kConsumers) {
        const float4 v = at(f);
        const float p0 = v.x - mean, p1 = v.y - mean, p2 = v.z - mean, p3 = v.w - mean;
        q += (p0 * p0 + p1 * p1) + (p2 * p2 + p3 * p3);
      }
      const float rstd = 1.0f / sqrtf(csum(q, red) / K + eps);
      const float4* g4 = reinterpret_cast<const float4*>(g);
      const float4* b4 = reinterpret_cast<const float4*>(b);
      for (int f = tid; f < K / 4; f += kConsumers) {
        float4 v = at(f);
        const float4 gg = g4[f], bb = b4[f];
        v.x = (v.x - mean) * rstd * gg.x + bb.x;
        v.y = (v.y - mean) * rstd * gg.y + bb.y;
        v.z = (v.z - mean) * rstd * gg.z + bb.z;
        v.w = (v.w - mean) * rstd * gg.w + bb.w;
        at(f) = v;
      }
    }
  }
  consumer_bar();
}

// Dot products of one weight row (in shared memory) with the M activation rows.
template <int M, int FMT>
__device__ __forceinline__ void row_dot(const unsigned char* row, const float4* act, int K, float* acc) {
  const int lane = threadIdx.x & 31;
  const int KW = K / 8, JW = KW / 32;
#pragma unroll
  for (int m = 0; m < M; ++m) acc[m] = 0.f;
  if (FMT == kInt4) {
    const uint32_t* wr = reinterpret_cast<const uint32_t*>(row);
    const float* sr = reinterpret_cast<const float*>(row + K / 2);
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
        const float4 xa = act[(size_t)m * 2 * KW + c];
        const float4 xb = act[(size_t)m * 2 * KW + KW + c];
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
    const uint4* wr = reinterpret_cast<const uint4*>(row);
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
        const float4 xa = act[(size_t)m * 2 * KW + c];
        const float4 xb = act[(size_t)m * 2 * KW + KW + c];
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
}

// Consumer side of the ring: wait for a slot's bytes, hand it back when done.  Every
// consumer thread waits (bounded) on its own; release() ORs the outcome over all of them
// so that they either all carry on or all leave together (no thread is left waiting at
// a named barrier for one that gave up).
struct Consumer {
  const PersistArgs* a;
  Smem sm;
  RingPos rp;
  bool got = false;
  __device__ const unsigned char* acquire() {
    got = mbar_wait(&sm.full[rp.slot], rp.phase, a->status);
    if (!got) atomicExch(a->abort, 1u);
    return got ? sm.ring + (size_t)rp.slot * kSlot : nullptr;
  }
  __device__ bool release() {
    const bool failed = consumer_bar_or(!got);
    if (failed) return false;
    if (threadIdx.x == 0) mbar_arrive(&sm.empty[rp.slot]);
    rp.next(a->nslot);
    return true;
  }
};

// One matrix phase: rows [n0, n1) of matrix mi, piece by piece from the ring.
// epi(m, n, value) is called by lane m of the warp that computed row n.
template <int M, int FMT, typename Epi>
__device__ bool gemv_phase(Consumer& cs, const float4* act, int K, int rb, int n0, int n1, Epi epi) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rpp = kSlot / rb;
  for (int p = n0; p < n1; p += rpp) {
    const int rows = min(rpp, n1 - p);
    const unsigned char* buf = cs.acquire();
    for (int r = warp; buf && r < rows; r += kConsumers / 32) {
      float acc[M];
      row_dot<M, FMT>(buf + (size_t)r * rb, act, K, acc);
      if (lane < M) {
        float v = acc[0];
#pragma unroll
        for (int m = 1; m < M; ++m)
          if (lane == m) v = acc[m];
        epi(lane, p + r, v);
      }
    }
    if (!cs.release()) return false;
  }
  return true;
}

__device__ bool grid_sync(const PersistArgs& a, unsigned& epoch, int* ok_s) {
  consumer_bar();
  if (threadIdx.x == 0) {
    ++epoch;
    int ok = 1;
    __threadfence();
    const unsigned old = atom_add_release_gpu(a.bar_count, 1u);
    if (old == epoch * gridDim.x - 1) {
      st_release_gpu(a.bar_flag, epoch);
    } else {
      long long it = 0;
      while (ld_acquire_gpu(a.bar_flag) < epoch) {
        if ((++it & 1023) == 0) {
          if (*reinterpret_cast<volatile unsigned*>(a.abort)) {
            ok = 0;
            break;
          }
          if (it > kGridSpinLimit) {
            flag_error(a.status, kErrTimeout);
            atomicExch(a.abort, 1u);
            ok = 0;
            break;
          }
        }
      }
    }
    __threadfence();
    *ok_s = ok;
  }
  consumer_bar();
  return *ok_s != 0;
}

// Attention for one (stream b, kv head g, split) unit over keys [0, T) of layer slices
// kc/vc.  The split holding position pos = T - 1 first appends the new key (RoPE'd) and
// value.  Writes the split's partial; the last split of (b, g) to finish merges them into o.
__device__ void attention_unit(const PersistArgs& a, float* scratch, int b, int g, int split, int S, int T, int pos,
                               float* kc, float* vc, unsigned* ticket_s) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H = a.H, Hk = a.Hk, hpg = H / Hk;
  int s_act = (T + kMinPerSplit - 1) / kMinPerSplit;
  if (s_act > S) s_act = S;
  const int chunk = (T + s_act - 1) / s_act;
  s_act = (T + chunk - 1) / chunk;  // every active split gets at least one position
  if (split >= s_act) return;
  const int t0 = split * chunk, t1 = min(T, t0 + chunk);
  float* qs = scratch;                         // [8][64]
  float* Ks = qs + 8 * 64;                     // [64][65]
  float* Vs = Ks + kAttSub * 65;               // [64][64]
  float* sc = Vs + kAttSub * 64;               // [8][64]
  float* mh = sc + 8 * kAttSub;                // [8]
  float* lh = mh + 8;
  float* corr = lh + 8;
  float* mw = corr + 8;                        // [8][kAttMaxSplits]
  float* lw = mw + 8 * kAttMaxSplits;          // [8][kAttMaxSplits]
  float* linv = lw + 8 * kAttMaxSplits;        // [8]
  const int nq = (H + 2 * Hk) * 64;
  const float* row = a.qkv + (size_t)b * nq;
  const float* cs = a.cosv + (size_t)pos * 32;
  const float* sn = a.sinv + (size_t)pos * 32;
  for (int i = tid; i < hpg * 32; i += kConsumers) {
    const int h = i >> 5, j = i & 31;
    const float x0 = __ldcg(row + (g * hpg + h) * 64 + j), x1 = __ldcg(row + (g * hpg + h) * 64 + j + 32);
    const float c = cs[j], s = sn[j];
    qs[h * 64 + j] = (x0 * c - x1 * s) * 0.125f;
    qs[h * 64 + j + 32] = (x0 * s + x1 * c) * 0.125f;
  }
  const size_t head = ((size_t)b * Hk + g) * a.cap;
  float* kb = kc + head * 64;
  float* vb = vc + head * 64;
  if (t1 == T && tid < 64) {
    // append position pos: k gets RoPE, v is stored as computed
    if (tid < 32) {
      const float x0 = __ldcg(row + (H + g) * 64 + tid), x1 = __ldcg(row + (H + g) * 64 + tid + 32);
      const float c = cs[tid], s = sn[tid];
      kb[(size_t)pos * 64 + tid] = x0 * c - x1 * s;
      kb[(size_t)pos * 64 + tid + 32] = x0 * s + x1 * c;
    }
    vb[(size_t)pos * 64 + tid] = __ldcg(row + (H + Hk + g) * 64 + tid);
  }
  if (tid < 8) {
    mh[tid] = -INFINITY;
    lh[tid] = 0.f;
  }
  float oacc[2] = {0.f, 0.f};   // slots tid and tid + 256 of hpg * 64 (hpg <= 8)
  __threadfence();
  for (int c0 = t0; c0 < t1; c0 += kAttSub) {
    const int cn = min(kAttSub, t1 - c0);
    consumer_bar();
    for (int i = tid; i < cn * 16; i += kConsumers) {
      const int p = i >> 4, f = i & 15;
      const float4 kv = __ldcg(reinterpret_cast<const float4*>(kb + (size_t)(c0 + p) * 64) + f);
      Ks[p * 65 + 4 * f + 0] = kv.x;
      Ks[p * 65 + 4 * f + 1] = kv.y;
      Ks[p * 65 + 4 * f + 2] = kv.z;
      Ks[p * 65 + 4 * f + 3] = kv.w;
      reinterpret_cast<float4*>(Vs + p * 64)[f] = __ldcg(reinterpret_cast<const float4*>(vb + (size_t)(c0 + p) * 64) + f);
    }
    consumer_bar();
    for (int i = tid; i < hpg * kAttSub; i += kConsumers) {
      const int h = i / kAttSub, p = i - h * kAttSub;
      float s = -INFINITY;
      if (p < cn) {
        s = 0.f;
#pragma unroll 16
        for (int dd = 0; dd < 64; ++dd) s = fmaf(qs[h * 64 + dd], Ks[p * 65 + dd], s);
      }
      sc[h * kAttSub + p] = s;
    }
    consumer_bar();
    for (int h = warp; h < hpg; h += kConsumers / 32) {
      const float v0 = sc[h * kAttSub + lane], v1 = sc[h * kAttSub + lane + 32];
      const float mx = warp_max(fmaxf(v0, v1));
      const float mold = mh[h];
      const float mnew = fmaxf(mold, mx);
      const float e0 = lane < cn ? expf(v0 - mnew) : 0.f;
      const float e1 = lane + 32 < cn ? expf(v1 - mnew) : 0.f;
      sc[h * kAttSub + lane] = e0;
      sc[h * kAttSub + lane + 32] = e1;
      const float sum = warp_sum(e0 + e1);
      __syncwarp();
      if (lane == 0) {
        const float cf = expf(mold - mnew);
        corr[h] = cf;
        lh[h] = lh[h] * cf + sum;
        mh[h] = mnew;
      }
    }
    consumer_bar();
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int idx = tid + k * kConsumers;
      if (idx < hpg * 64) {
        const int h = idx >> 6, dd = idx & 63;
        float acc = oacc[k] * corr[h];
        for (int p = 0; p < cn; ++p) acc = fmaf(sc[h * kAttSub + p], Vs[p * 64 + dd], acc);
        oacc[k] = acc;
      }
    }
  }
  consumer_bar();
  float* pb = a.part + (((size_t)b * Hk + g) * a.att_splits + split) * hpg * 66;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int idx = tid + k * kConsumers;
    if (idx < hpg * 64) pb[(idx >> 6) * 66 + 2 + (idx & 63)] = oacc[k];
  }
  if (tid < hpg) {
    pb[tid * 66 + 0] = mh[tid];
    pb[tid * 66 + 1] = lh[tid];
  }
  __threadfence();
  consumer_bar();
  unsigned* ctr = a.att_counters + (size_t)b * Hk + g;
  if (tid == 0) *ticket_s = (atomicAdd(ctr, 1u) == (unsigned)(s_act - 1)) ? 1u : 0u;
  consumer_bar();
  if (!*ticket_s) return;
  __threadfence();
  const float* p0 = a.part + ((size_t)b * Hk + g) * a.att_splits * hpg * 66;
  for (int i = tid; i < hpg * s_act; i += kConsumers) {
    const int h = i / s_act, s = i - h * s_act;
    mw[h * kAttMaxSplits + s] = __ldcg(p0 + ((size_t)s * hpg + h) * 66);
    lw[h * kAttMaxSplits + s] = __ldcg(p0 + ((size_t)s * hpg + h) * 66 + 1);
  }
  consumer_bar();
  for (int h = warp; h < hpg; h += kConsumers / 32) {
    float mx = -INFINITY;
    for (int s = lane; s < s_act; s += 32) mx = fmaxf(mx, mw[h * kAttMaxSplits + s]);
    mx = warp_max(mx);
    float l = 0.f;
    for (int s = lane; s < s_act; s += 32) {
      const float w = expf(mw[h * kAttMaxSplits + s] - mx);
      mw[h * kAttMaxSplits + s] = w;
      l = fmaf(w, lw[h * kAttMaxSplits + s], l);
    }
    l = warp_sum(l);
    if (lane == 0) linv[h] = 1.0f / l;
  }
  consumer_bar();
  for (int idx = tid; idx < hpg * 64; idx += kConsumers) {
    const int h = idx >> 6, dd = idx & 63;
    float O = 0.f;
#pragma unroll 8
    for (int s = 0; s < s_act; ++s) O = fmaf(mw[h * kAttMaxSplits + s], __ldcg(p0 + ((size_t)s * hpg + h) * 66 + 2 + dd), O);
    a.o[((size_t)b * H + g * hpg + h) * 64 + dd] = O * linv[h];
  }
  if (tid == 0) *ctr = 0u;
}

__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

}  // namespace

template <int M, int FMT>
__global__ void __launch_bounds__(kThreads, 1) decode_persistent_kernel(PersistArgs a) {
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ int ok_s;
  __shared__ unsigned ticket_s;
  __shared__ float bval[8][8];
  __shared__ int bidx[8][8];
  const Smem sm = carve(smem, a.nslot);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < a.nslot; ++i) {
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.empty[i], 1);
    }
    mbar_fence_init();
  }
  __syncthreads();
  if (warp == kConsumers / 32) {
    if (lane == 0) producer(a, sm);
    return;
  }

  const Shape sh = shapes_of(a);
  const int c = blockIdx.x, G = gridDim.x;
  const int d = a.d, H = a.H, Hk = a.Hk, F = a.F, V = a.V, B = M;
  const int nq = (H + 2 * Hk) * 64;
  Consumer cs;
  cs.a = &a;
  cs.sm = sm;
  unsigned epoch = 0;
  const int len0 = *a.dlen;
  const float4* act4 = reinterpret_cast<const float4*>(sm.act);
  int nr0[4], nr1[4];
  for (int i = 0; i < 4; ++i) partition(sh.N[i], c, G, nr0[i], nr1[i]);
  int v0, v1;
  partition(V, c, G, v0, v1);
  const int units = B * Hk;
  int S = G / units;
  if (S < 1) S = 1;
  if (S > a.att_splits) S = a.att_splits;

  for (int step = 0; step < a.n_steps; ++step) {
    const int pos = len0 + step;
    const int T = pos + 1;
    __shared__ int tok_s[8];
    if (tid < M) {
      int t = (step == 0 && a.tokens_in) ? a.tokens_in[tid] : __ldcg(a.hist + (size_t)(pos - 1) * B + tid);
      if (t < 0 || t >= V) {
        flag_error(a.status, kErrToken);
        t = t < 0 ? 0 : V - 1;
      }
      tok_s[tid] = t;
    }
    consumer_bar();
    for (int l = 0; l < a.L; ++l) {
      const PLayer& ly = a.layers[l];
      float* kc = a.kc + (size_t)l * a.layer_stride;
      float* vc = a.vc + (size_t)l * a.layer_stride;
      // ---- A: LN1 + QKV -------------------------------------------------------------
      if (l == 0) {
        // x = E[token]; this CTA materialises its own residual rows
        for (int m = 0; m < M; ++m)
          for (int n = nr0[1] + tid; n < nr1[1]; n += kConsumers)
            a.x[(size_t)m * d + n] = a.tok_emb[(size_t)tok_s[m] * d + n];
        // LN1 reads the embedding rows directly (ld stride 0 between m handled per row)
        for (int m = 0; m < M; ++m)
          load_act<1>(sm.act + (size_t)m * d, sm.red, a.tok_emb + (size_t)tok_s[m] * d, 0, d, ly.ln1_g, ly.ln1_b,
                      a.eps, false);
      } else {
        load_act<M>(sm.act, sm.red, a.x, d, d, ly.ln1_g, ly.ln1_b, a.eps, false);
      }
      if (!gemv_phase<M, FMT>(cs, act4, d, sh.rowb[0], nr0[0], nr1[0],
                               [&](int m, int n, float v) { a.qkv[(size_t)m * nq + n] = v; }))
        return;
      if (!grid_sync(a, epoch, &ok_s)) return;
      // ---- B: attention -------------------------------------------------------------
      for (int u = c; u < units * S; u += G) {
        const int bg = u / S, split = u - bg * S;
        attention_unit(a, sm.act, bg / Hk, bg % Hk, split, S, T, pos, kc, vc, &ticket_s);
        consumer_bar();
      }
      if (!grid_sync(a, epoch, &ok_s)) return;
      // ---- C: O + residual ----------------------------------------------------------
      load_act<M>(sm.act, sm.red, a.o, H * 64, H * 64, nullptr, nullptr, 0.f, false);
      if (!gemv_phase<M, FMT>(cs, act4, H * 64, sh.rowb[1], nr0[1], nr1[1], [&](int m, int n, float v) {
            float* p = a.x + (size_t)m * d + n;
            *p = __ldcg(p) + v;
          }))
        return;
      if (!grid_sync(a, epoch, &ok_s)) return;
      // ---- D: LN2 + FC1 + GELU ------------------------------------------------------
      load_act<M>(sm.act, sm.red, a.x, d, d, ly.ln2_g, ly.ln2_b, a.eps, false);
      if (!gemv_phase<M, FMT>(cs, act4, d, sh.rowb[2], nr0[2], nr1[2],
                               [&](int m, int n, float v) { a.u[(size_t)m * F + n] = gelu_erf(v); }))
        return;
      if (!grid_sync(a, epoch, &ok_s)) return;
      // ---- E: FC2 + residual --------------------------------------------------------
      load_act<M>(sm.act, sm.red, a.u, F, F, nullptr, nullptr, 0.f, false);
      if (!gemv_phase<M, FMT>(cs, act4, F, sh.rowb[3], nr0[3], nr1[3], [&](int m, int n, float v) {
            float* p = a.x + (size_t)m * d + n;
            *p = __ldcg(p) + v;
          }))
        return;
      if (!grid_sync(a, epoch, &ok_s)) return;
    }
    // ---- LM head + argmax ------------------------------------------------------------
    load_act<M>(sm.act, sm.red, a.x, d, d, a.lnf_g, a.lnf_b, a.eps, true);
    float best[M];
    int bi[M];
#pragma unroll
    for (int m = 0; m < M; ++m) {
      best[m] = -FLT_MAX;
      bi[m] = INT_MAX;
    }
    {
      const int rb = d * 4, rpp = kSlot / rb;
      for (int p = v0; p < v1; p += rpp) {
        const int rows = min(rpp, v1 - p);
        const unsigned char* buf = cs.acquire();
        for (int r = warp; buf && r < rows; r += kConsumers / 32) {
          const float4* w4 = reinterpret_cast<const float4*>(buf + (size_t)r * rb);
          float acc[M];
#pragma unroll
          for (int m = 0; m < M; ++m) acc[m] = 0.f;
          for (int f = lane; f < d / 4; f += 32) {
            const float4 w = w4[f];
#pragma unroll
            for (int m = 0; m < M; ++m) {
              const float4 h = act4[(size_t)m * (d / 4) + f];
              acc[m] = fmaf(w.x, h.x, acc[m]);
              acc[m] = fmaf(w.y, h.y, acc[m]);
              acc[m] = fmaf(w.z, h.z, acc[m]);
              acc[m] = fmaf(w.w, h.w, acc[m]);
            }
          }
          const int v = p + r;
#pragma unroll
          for (int m = 0; m < M; ++m) {
            const float s = warp_sum(acc[m]);
            if (lane == 0 && a.logits) a.logits[(size_t)m * V + v] = s;
            if (better(s, v, best[m], bi[m])) {
              best[m] = s;
              bi[m] = v;
            }
          }
        }
        if (!cs.release()) return;
      }
    }
    if (lane == 0)
      for (int m = 0; m < M; ++m) {
        bval[warp][m] = best[m];
        bidx[warp][m] = bi[m];
      }
    consumer_bar();
    if (tid < M) {
      float bv = -FLT_MAX;
      int bx = INT_MAX;
      for (int w = 0; w < kConsumers / 32; ++w)
        if (better(bval[w][tid], bidx[w][tid], bv, bx)) {
          bv = bval[w][tid];
          bx = bidx[w][tid];
        }
      a.lm_val[(size_t)c * 64 + tid] = bv;
      a.lm_idx[(size_t)c * 64 + tid] = bx;
    }
    __threadfence();
    consumer_bar();
    if (tid == 0) ticket_s = (atomicAdd(a.lm_counter, 1u) == (unsigned)(G - 1)) ? 1u : 0u;
    consumer_bar();
    if (ticket_s) {
      __threadfence();
      for (int m = 0; m < M; ++m) {
        float bv = -FLT_MAX;
        int bx = INT_MAX;
        for (int k = tid; k < G; k += kConsumers) {
          const float v = __ldcg(a.lm_val + (size_t)k * 64 + m);
          const int i = __ldcg(a.lm_idx + (size_t)k * 64 + m);
          if (better(v, i, bv, bx)) {
            bv = v;
            bx = i;
          }
        }
        warp_argmax(bv, bx);
        if (lane == 0) {
          bval[warp][m] = bv;
          bidx[warp][m] = bx;
        }
      }
      consumer_bar();
      if (tid < M) {
        float bv = -FLT_MAX;
        int bx = INT_MAX;
        for (int w = 0; w < kConsumers / 32; ++w)
          if (better(bval[w][tid], bidx[w][tid], bv, bx)) {
            bv = bval[w][tid];
            bx = bidx[w][tid];
          }
        if (bx == INT_MAX) bx = 0;
        a.hist[(size_t)pos * B + tid] = bx;
        if (a.argmax_out && step == a.n_steps - 1) a.argmax_out[tid] = bx;
      }
      consumer_bar();
      if (tid == 0) {
        *a.lm_counter = 0u;
        *a.dlen = pos + 1;
      }
    }
    if (step + 1 < a.n_steps)
      if (!grid_sync(a, epoch, &ok_s)) return;
  }
}

// ---------------------------------------------------------------------------------
namespace {
size_t persist_region(int M, int d, int H, int F) {
  size_t act = (size_t)M * 4 * (size_t)max(max(d, H * 64), F);
  size_t att = sizeof(float) * (8 * 64 + kAttSub * 65 + kAttSub * 64 + 8 * kAttSub + 24 + 2 * 8 * kAttMaxSplits + 8);
  return align16(act > att ? act : att);
}
}  // namespace

int persistent_slots(int M, int d, int H, int F, size_t smem_optin) {
  const size_t region = persist_region(M, d, H, F);
  if (smem_optin < 1024 + region + 4 * (size_t)kSlot) return 0;
  size_t n = (smem_optin - 1024 - region) / kSlot;
  if (n > 16) n = 16;
  return (int)n;
}

size_t persistent_smem(int M, int d, int H, int F, int nslot) {
  return 1024 + (size_t)nslot * kSlot + persist_region(M, d, H, F);
}

template <int M, int FMT>
static cudaError_t go(const PersistArgs& a, int grid, size_t smem, cudaStream_t st) {
  auto k = decode_persistent_kernel<M, FMT>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, k, a);
  if (e == cudaSuccess) launch_counter().fetch_add(1, std::memory_order_relaxed);
  return e;
}

cudaError_t init_attrs_persistent() {
  cudaError_t e = cudaSuccess;
  if (e == cudaSuccess) e = allow_smem(decode_persistent_kernel<1, kInt4>, kMaxDynSmem);
  if (e == cudaSuccess) e = allow_smem(decode_persistent_kernel<2, kInt4>, kMaxDynSmem);
  if (e == cudaSuccess) e = allow_smem(decode_persistent_kernel<4, kInt4>, kMaxDynSmem);
  if (e == cudaSuccess) e = allow_smem(decode_persistent_kernel<8, kInt4>, kMaxDynSmem);
  if (e == cudaSuccess) e = allow_smem(decode_persistent_kernel<1, kFp16>, kMaxDynSmem);
  if (e == cudaSuccess) e = allow_smem(decode_persistent_kernel<2, kFp16>, kMaxDynSmem);
  if (e == cudaSuccess) e = allow_smem(decode_persistent_kernel<4, kFp16>, kMaxDynSmem);
  if (e == cudaSuccess) e = allow_smem(decode_persistent_kernel<8, kFp16>, kMaxDynSmem);
  return e;
}

cudaError_t launch_decode_persistent(const PersistArgs& a, int M, int grid, size_t smem, cudaStream_t st) {
  if (a.fmt == kInt4) {
    switch (M) {
      case 1: return go<1, kInt4>(a, grid, smem, st);
      case 2: return go<2, kInt4>(a, grid, smem, st);
      case 4: return go<4, kInt4>(a, grid, smem, st);
      case 8: return go<8, kInt4>(a, grid, smem, st);
    }
  } else {
    switch (M) {
      case 1: return go<1, kFp16>(a, grid, smem, st);
      case 2: return go<2, kFp16>(a, grid, smem, st);
      case 4: return go<4, kFp16>(a, grid, smem, st);
      case 8: return go<8, kFp16>(a, grid, smem, st);
    }
  }
  return cudaErrorInvalidValue;
}

int persistent_max_ctas(int M, int fmt, size_t smem) {
  int n = 0;
  cudaError_t e;
  if (fmt == kInt4) {
    if (M == 1) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_persistent_kernel<1, kInt4>, kThreads, smem);
    else if (M == 2) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_persistent_kernel<2, kInt4>, kThreads, smem);
    else if (M == 4) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_persistent_kernel<4, kInt4>, kThreads, smem);
    else e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_persistent_kernel<8, kInt4>, kThreads, smem);
  } else {
    if (M == 1) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_persistent_kernel<1, kFp16>, kThreads, smem);
    else if (M == 2) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_persistent_kernel<2, kFp16>, kThreads, smem);
    else if (M == 4) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_persistent_kernel<4, kFp16>, kThreads, smem);
    else e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_persistent_kernel<8, kFp16>, kThreads, smem);
  }
  return e == cudaSuccess ? n : 0;
}

}  // namespace ms
