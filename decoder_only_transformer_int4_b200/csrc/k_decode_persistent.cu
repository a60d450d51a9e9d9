// Persistent decode kernel: greedy decode steps of the whole decoder (all layers, LM head,
// argmax, token feedback) in one cooperative launch, one CTA per SM.
//
// Why: at a few streams the decoder step is a chain of ~5 dependent matrix-vector phases
// per layer, each moving only a few MB; separate kernel launches pay a launch and drain per
// phase, and even a grid barrier costs ~2 us on 148 SMs.  Here the weight bytes — which
// never depend on the previous phase — stream continuously: each CTA walks its whole weight
// schedule (every slice of every layer of every step) with bulk copies into a shared-memory
// ring; the slot the eight warps have just finished with is refilled at once with the slice
// nslot places ahead, so the copies run ahead of use across phase, layer and step
// boundaries.  And the hand-off between phases needs no barrier: every activation
// vector a phase produces (qkv, o, x, u) is written as 64-bit words {value, epoch}, each
// element stored once, and the next phase polls the words it needs until they carry the
// current epoch — the wait and the read are one round trip.  One grid barrier per step
// (after the LM head) orders the rest (cache append, token history).
//
// Phases of one step (token position pos, T = pos + 1 keys):
//   A  LN1 of x, QKV rows (raw q, k, v)                                 -> qkv
//   B  attention unit (stream, kv head, split): RoPE of q (and of the new k, which the
//      last split appends to the cache with v), scores over its run of positions, partial
//      (m, l, o); the last unit of a (stream, kv head) merges the partials  -> o
//   C  O rows, residual                                                  x += o Wo^T -> xc
//   D  LN2 of x, FC1 rows, GELU                                          -> u
//   E  FC2 rows, residual                                                x += u W2^T -> xe
// The residual rows a CTA owns (the same rows in C and E) stay in its shared memory; the
// other CTAs read them from the stamped copies.
//   after the last layer: LN_f of x, LM head rows, per-CTA argmax, last CTA picks the token,
//   records it in the token history and advances the cache length.
// The arithmetic per element is the same as the separate kernels' (fp32, INT4 codes
// converted exactly, one scale FMA per 32-element group).
//
// Every wait is bounded: the grid barrier's spin, the stamp polls and the ring's mbarrier
// waits give up after a limit, set the status word's timeout bit and an abort word that
// makes every CTA leave; a CTA that leaves first waits (bounded) for its copies in flight.
#include <float.h>
#include <limits.h>
#include "ms_device.cuh"
#include "ms_launch.cuh"
#include "ms_persistent.h"

namespace ms {

namespace {
constexpr int kConsumers = 256;
constexpr int kThreads = kConsumers;
constexpr int kSlot = 16384;
constexpr long long kGridSpinLimit = 1ll << 24;  // polls of the barrier flag (~10 s)
constexpr int kAttSub = 64;
constexpr int kAttMaxSplits = 128;
constexpr int kMinPerSplit = 16;
constexpr int kMaxOwnRows = 16;   // residual rows a CTA owns: ceil(d_model / CTAs) <= 16
constexpr int kMaxLayers = 64;    // layer table kept in shared memory

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

// No routine of this kernel is called out of line: with nearly all of the SM's unified L1
// given to shared memory, a call's register saves (local memory) would cost a round trip
// to L2.  Each routine has a single call site, so inlining does not grow the code.
__device__ __forceinline__ float ex(float x) { return expf(x); }
__device__ __forceinline__ float gelu_ool(float u) { return gelu_erf(u); }

// Rows [n0, n1) of an N-row matrix owned by CTA c of G (contiguous, balanced).
__device__ __forceinline__ void partition(int N, int c, int G, int& n0, int& n1) {
  n0 = (int)(((long long)N * c) / G);
  n1 = (int)(((long long)N * (c + 1)) / G);
}

// Shapes of matrix mi (0 QKV, 1 O, 2 FC1, 3 FC2) and of the LM head (mi 4), as scalar
// selects: a small array indexed at run time would live in local memory.
__device__ __forceinline__ int mat_N(const PersistArgs& a, int mi) {
  return mi == 0 ? (a.H + 2 * a.Hk) * 64 : mi == 2 ? a.F : mi == 4 ? a.V : a.d;
}
__device__ __forceinline__ int mat_K(const PersistArgs& a, int mi) {
  return mi == 1 ? a.H * 64 : mi == 3 ? a.F : a.d;
}
__device__ __forceinline__ int mat_rowb(const PersistArgs& a, int mi) {
  if (mi == 4) return a.d * 4;
  const int K = mat_K(a, mi);
  return a.fmt == kInt4 ? K / 2 + K / 8 : K * 2;
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
// Weight schedule: the CTA's slices in consumption order (per step: per layer the rows of
// QKV, O, FC1, FC2; then the LM head rows), one ring slot each.  Thread 0 keeps a cursor
// and issues the next slice whenever a slot comes free.
// ---------------------------------------------------------------------------------
struct Cursor {
  int step = 0, l = 0, stage = 0, p = -1;  // stage 0..3: matrices, 4: LM head
  const PLayer* layers = nullptr;          // the layer table (a shared-memory copy)
  __device__ bool next(const PersistArgs& a, int c, int G, const unsigned char** src, uint32_t* bytes) {
    for (;;) {
      if (step >= a.n_steps) return false;
      const int N = mat_N(a, stage);
      const int rb = mat_rowb(a, stage);
      int n0, n1;
      partition(N, c, G, n0, n1);
      const int rpp = kSlot / rb;
      p = p < 0 ? n0 : p + rpp;
      if (p < n1) {
        const int rows = min(rpp, n1 - p);
        const PLayer& ly = layers[l];
        const unsigned char* base = stage == 0   ? ly.w[0]
                                    : stage == 1 ? ly.w[1]
                                    : stage == 2 ? ly.w[2]
                                    : stage == 3 ? ly.w[3]
                                                 : reinterpret_cast<const unsigned char*>(a.lm_head);
        *src = base + (size_t)p * rb;
        *bytes = (uint32_t)(rows * rb);
        return true;
      }
      p = -1;
      if (stage < 3) {
        ++stage;
      } else if (stage == 3) {
        if (++l < a.L) stage = 0;
        else stage = 4;
      } else {
        stage = 0;
        l = 0;
        ++step;
      }
    }
  }
};

// ---------------------------------------------------------------------------------
// Consumer helpers
// ---------------------------------------------------------------------------------
constexpr long long kPollLimit = 1ll << 22;  // re-reads of one stamped word (>= 512 ns apart) before giving up

__device__ __forceinline__ float csum(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum(v);
  consumer_bar();
  if (lane == 0) red[warp] = v;
  consumer_bar();
  float t = lane < kConsumers / 32 ? red[lane] : 0.f;
  return warp_sum(t);
}

// {value, epoch} words: the value's bits in the low half, the epoch in the high half; one
// 64-bit store / load each, so a reader sees either the old or the new word whole.
__device__ __forceinline__ void st_stamp(uint64_t* p, float v, unsigned ep) {
  const uint64_t w = ((uint64_t)ep << 32) | (uint64_t)__float_as_uint(v);
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}
__device__ __forceinline__ uint64_t ld_stamp(const uint64_t* p) {
  uint64_t w;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(w) : "l"(p) : "memory");
  return w;
}

// Read element i of a stamped vector, waiting until it carries epoch ep.  Returns false
// if the wait ran out or another CTA gave up.
// Waiting threads back off (64 ns doubling to 512 ns) so that a CTA's spinning threads do
// not flood the L2 slices that hold the words being produced.
__device__ __forceinline__ bool poll_slow(const uint64_t* p, unsigned ep, float& v, const PersistArgs& a);
__device__ __forceinline__ bool poll_one(const uint64_t* p, unsigned ep, float& v, const PersistArgs& a) {
  const uint64_t w = ld_stamp(p);
  if ((unsigned)(w >> 32) == ep) {
    v = __uint_as_float((unsigned)w);
    return true;
  }
  return poll_slow(p, ep, v, a);
}
__device__ __forceinline__ bool poll_slow(const uint64_t* p, unsigned ep, float& v, const PersistArgs& a) {
  uint64_t w = ld_stamp(p);
  long long it = 0;
  unsigned ns = 64;
  while ((unsigned)(w >> 32) != ep) {
    __nanosleep(ns);
    if (ns < 512) ns <<= 1;
    if ((++it & 63) == 0) {
      if (*reinterpret_cast<volatile unsigned*>(a.abort)) return false;
      if (it > kPollLimit) {
        flag_error(a.status, kErrTimeout);
        atomicExch(a.abort, 1u);
        return false;
      }
    }
    w = ld_stamp(p);
  }
  v = __uint_as_float((unsigned)w);
  return true;
}

// Rows m < M of a stamped vector (row stride ld words) into act: de-interleaved by
// 8-element words (elements 8c..8c+3 in one float4 array, 8c+4..8c+7 in the next) or, with
// natural, in plain order; optionally LayerNorm'd.  All the loads of a thread go out before
// it waits on any of them.  Returns false (for every consumer thread) on a failed wait.
template <int M>
__device__ __forceinline__ bool poll_act(float* act, float* red, const uint64_t* src, int ld, int K, unsigned ep,
                                      const float* g, const float* b, float eps, bool natural, const PersistArgs& a) {
  const int tid = threadIdx.x, KW = K / 8;
  bool ok = true;
  for (int m = 0; m < M; ++m) {
    const uint64_t* s0 = src + (size_t)m * ld;
    float* dm = act + (size_t)m * K;
    auto slot = [&](int k) -> float& {
      if (natural) return dm[k];
      const int c = k >> 3, e = k & 7;
      return dm[((e >> 2) * KW + c) * 4 + (e & 3)];
    };
    constexpr int kBatch = 4;
    for (int k0 = tid; k0 < K; k0 += kConsumers * kBatch) {
      uint64_t w[kBatch];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int k = k0 + j * kConsumers;
        w[j] = k < K ? ld_stamp(s0 + k) : 0;
      }
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int k = k0 + j * kConsumers;
        if (k < K && ok) {
          float v = __uint_as_float((unsigned)w[j]);
          if ((unsigned)(w[j] >> 32) != ep) ok = poll_one(s0 + k, ep, v, a);
          slot(k) = v;
        }
      }
    }
  }
  if (consumer_bar_or(!ok)) return false;
  if (g) {
    for (int m = 0; m < M; ++m) {
      float* dm = act + (size_t)m * K;
      float s = 0.f;
      for (int k = tid; k < K; k += kConsumers) s += dm[k];  // order-free sum over the row
      const float mean = csum(s, red) / K;
      float q = 0.f;
      for (int k = tid; k < K; k += kConsumers) {
        const float t = dm[k] - mean;
        q += t * t;
      }
      const float rstd = 1.0f / sqrtf(csum(q, red) / K + eps);
      // normalise in place; the gamma/beta index is the element's position in the row
      for (int k = tid; k < K; k += kConsumers) {
        int e;  // element index of storage slot k
        if (natural) {
          e = k;
        } else {
          const int half = (k >> 2) / KW, c = (k >> 2) - half * KW;
          e = c * 8 + half * 4 + (k & 3);
        }
        dm[k] = (dm[k] - mean) * rstd * g[e] + b[e];
      }
    }
    consumer_bar();
  }
  return true;
}

// Plain fp32 rows (the token embedding) into act, de-interleaved, LayerNorm'd.
__device__ __forceinline__ void embed_act(float* act, float* red, const float* src, int K, const float* g, const float* b,
                                       float eps) {
  const int tid = threadIdx.x, KW = K / 8;
  float4* d4 = reinterpret_cast<float4*>(act);
  const float4* s4 = reinterpret_cast<const float4*>(src);
  float s = 0.f;
  for (int f = tid; f < K / 4; f += kConsumers) {
    const float4 v = s4[f];
    d4[(f & 1) * KW + (f >> 1)] = v;
    s += (v.x + v.y) + (v.z + v.w);
  }
  const float mean = csum(s, red) / K;
  float q = 0.f;
  for (int f = tid; f < K / 4; f += kConsumers) {
    const float4 v = d4[(f & 1) * KW + (f >> 1)];
    const float p0 = v.x - mean, p1 = v.y - mean, p2 = v.z - mean, p3 = v.w - mean;
    q += (p0 * p0 + p1 * p1) + (p2 * p2 + p3 * p3);
  }
  const float rstd = 1.0f / sqrtf(csum(q, red) / K + eps);
  const float4* g4 = reinterpret_cast<const float4*>(g);
  const float4* b4 = reinterpret_cast<const float4*>(b);
  for (int f = tid; f < K / 4; f += kConsumers) {
    float4 v = d4[(f & 1) * KW + (f >> 1)];
    const float4 gg = g4[f], bb = b4[f];
    v.x = (v.x - mean) * rstd * gg.x + bb.x;
    v.y = (v.y - mean) * rstd * gg.y + bb.y;
    v.z = (v.z - mean) * rstd * gg.z + bb.z;
    v.w = (v.w - mean) * rstd * gg.w + bb.w;
    d4[(f & 1) * KW + (f >> 1)] = v;
  }
  consumer_bar();
}

// Dot products of RB weight rows (rows r, r + 8, ... of the slot) with the M activation
// rows.  Lane l takes the 4-byte words l + 32 j of each row; two words are loaded ahead and
// each word's 8 products go into two chains, so a warp keeps several independent FMA
// chains in flight.
template <int M, int FMT>
__device__ __forceinline__ void word_fma(const unsigned char* row, int c, int K, const float4* xa, const float4* xb,
                                         float* acc) {
  float q[8];
  float sc = 1.f;
  if (FMT == kInt4) {
    const uint32_t wd = reinterpret_cast<const uint32_t*>(row)[c];
    sc = reinterpret_cast<const float*>(row + K / 2)[c >> 2];
#pragma unroll
    for (int e = 0; e < 8; ++e) q[e] = nib_to_q((wd >> (4 * e)) & 15u);
  } else {
    const uint4 hv = reinterpret_cast<const uint4*>(row)[c];
    const __half2* h2 = reinterpret_cast<const __half2*>(&hv);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f2 = __half22float2(h2[e]);
      q[2 * e] = f2.x;
      q[2 * e + 1] = f2.y;
    }
  }
#pragma unroll
  for (int m = 0; m < M; ++m) {
    float p0 = q[0] * xa[m].x, p1 = q[1] * xa[m].y;
    p0 = fmaf(q[2], xa[m].z, p0);
    p1 = fmaf(q[3], xa[m].w, p1);
    p0 = fmaf(q[4], xb[m].x, p0);
    p1 = fmaf(q[5], xb[m].y, p1);
    p0 = fmaf(q[6], xb[m].z, p0);
    p1 = fmaf(q[7], xb[m].w, p1);
    acc[m] = FMT == kInt4 ? fmaf(sc, p0 + p1, acc[m]) : acc[m] + (p0 + p1);
  }
}

template <int M, int FMT, int RB>
__device__ __forceinline__ void rows_dot(const unsigned char* buf, int rb, int r0, int nr, const float4* act, int K,
                                         float (&acc)[RB][M]) {
  const int lane = threadIdx.x & 31;
  const int KW = K / 8, JW = KW / 32;
  float acc2[RB][M];
#pragma unroll
  for (int i = 0; i < RB; ++i)
#pragma unroll
    for (int m = 0; m < M; ++m) acc[i][m] = acc2[i][m] = 0.f;
#pragma unroll 1
  for (int j = 0; j < JW; j += 2) {
    const int c0 = lane + 32 * j, c1 = c0 + 32;
    const bool two = j + 1 < JW;
    float4 xa0[M], xb0[M], xa1[M], xb1[M];
#pragma unroll
    for (int m = 0; m < M; ++m) {
      xa0[m] = act[(size_t)m * 2 * KW + c0];
      xb0[m] = act[(size_t)m * 2 * KW + KW + c0];
      xa1[m] = two ? act[(size_t)m * 2 * KW + c1] : make_float4(0.f, 0.f, 0.f, 0.f);
      xb1[m] = two ? act[(size_t)m * 2 * KW + KW + c1] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int i = 0; i < RB; ++i) {
      if (i < nr) {
        const unsigned char* row = buf + (size_t)(r0 + 8 * i) * rb;
        word_fma<M, FMT>(row, c0, K, xa0, xb0, acc[i]);
        if (two) word_fma<M, FMT>(row, c1, K, xa1, xb1, acc2[i]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < RB; ++i)
#pragma unroll
    for (int m = 0; m < M; ++m) acc[i][m] = warp_sum(acc[i][m] + acc2[i][m]);
}

// Consumer side of the ring: wait for a slot's bytes, hand it back when done.  Every
// consumer thread waits (bounded) on its own; release() ORs the outcome over all of them
// so that they either all carry on or all leave together (no thread is left waiting at
// a named barrier for one that gave up).
struct Consumer {
  const PersistArgs* a;
  Smem sm;
  RingPos rp;           // next slot to consume
  bool got = false;
  // thread 0 only: the schedule cursor and the number of slices issued
  Cursor cur;
  int c = 0, G = 1;
  long long issued = 0, consumed = 0;
  __device__ void issue_next() {
    const unsigned char* src;
    uint32_t bytes;
    if (!cur.next(*a, c, G, &src, &bytes)) return;
    const int slot = (int)(issued % a->nslot);
    mbar_expect_tx(&sm.full[slot], bytes);
    bulk_g2s(sm.ring + (size_t)slot * kSlot, src, bytes, &sm.full[slot]);
    ++issued;
  }
  __device__ void start() {
    if (threadIdx.x == 0)
      for (int i = 0; i < a->nslot; ++i) issue_next();
  }
  __device__ const unsigned char* acquire() {
    got = mbar_wait(&sm.full[rp.slot], rp.phase, a->status);
    if (!got) atomicExch(a->abort, 1u);
    return got ? sm.ring + (size_t)rp.slot * kSlot : nullptr;
  }
  // All consumers are done with the slot: refill it with the slice nslot places ahead.
  __device__ bool release() {
    const bool failed = consumer_bar_or(!got);
    if (failed) return false;
    ++consumed;
    // The named barrier above has every consumer's reads of the slot complete (their values
    // are in registers) before thread 0 hands the slot to the next bulk copy.
    if (threadIdx.x == 0) issue_next();
    rp.next(a->nslot);
    return true;
  }
  // Before leaving early: wait (bounded) for the copies still in flight.
  __device__ void drain() {
    if (threadIdx.x != 0) return;
    RingPos q = rp;
    for (long long i = consumed; i < issued; ++i) {
      for (long long it = 0; it < kSpinLimit; ++it)
        if (mbar_try_wait(&sm.full[q.slot], q.phase)) break;
      q.next(a->nslot);
    }
  }
};

// Where a matrix phase's outputs go.  mode: 0 store, 1 residual (x += value, kept in the
// CTA's own rows and published), 2 GELU.  Outputs are {value, epoch} words at out[m * ldo + n].
struct OutSpec {
  int mode;
  uint64_t* out;
  int ldo;
  unsigned ep;
  float* xown;   // residual rows of this CTA, [M][kMaxOwnRows], first row xr0
  int xr0;
};

// One matrix phase: rows [n0, n1) of a matrix, slot by slot from the ring.  Warp w takes
// rows w, w+8, w+16, w+24 of a slot together; lane m writes output m of each row.
template <int M, int FMT>
__device__ __forceinline__ bool gemv_phase(Consumer& cs, const float4* act, int K, int rb, int n0, int n1,
                                        const OutSpec e) {
  constexpr int RB = M <= 2 ? 2 : 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rpp = kSlot / rb;
  for (int p = n0; p < n1; p += rpp) {
    const int rows = min(rpp, n1 - p);
    const unsigned char* buf = cs.acquire();
    for (int r0 = warp; buf && r0 < rows; r0 += 8 * RB) {
      const int nr = min(RB, (rows - r0 + 7) / 8);
      float acc[RB][M];
      rows_dot<M, FMT, RB>(buf, rb, r0, nr, act, K, acc);
      if (lane < M) {
#pragma unroll
        for (int i = 0; i < RB; ++i) {
          if (i < nr) {
            float v = acc[i][0];
#pragma unroll
            for (int m = 1; m < M; ++m)
              if (lane == m) v = acc[i][m];
            const int n = p + r0 + 8 * i;
            if (e.mode == 1) {
              float* xo = e.xown + lane * kMaxOwnRows + (n - e.xr0);
              v += *xo;
              *xo = v;
            } else if (e.mode == 2) {
              v = gelu_ool(v);
            }
            st_stamp(e.out + (size_t)lane * e.ldo + n, v, e.ep);
          }
        }
      }
    }
    if (!cs.release()) return false;
  }
  return true;
}

// Grid barrier: one fire-and-forget release add per CTA, then poll the count (relaxed) and
// acquire once.  The count only grows, so the e-th barrier completes at e * G arrivals.
__device__ bool grid_sync(const PersistArgs& a, unsigned& epoch, int* ok_s) {
  consumer_bar();
  if (threadIdx.x == 0) {
    ++epoch;
    int ok = 1;
    __threadfence();  // the CTA's stores (seen through the named barrier) before the release
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(a.bar_count), "r"(1u) : "memory");
    const unsigned target = epoch * gridDim.x;
    long long it = 0;
    for (;;) {
      unsigned v;
      asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a.bar_count) : "memory");
      if (v >= target) break;
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
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
    *ok_s = ok;
  }
  consumer_bar();
  return *ok_s != 0;
}

// Attention for one (stream b, kv head g, split) unit over keys [0, T) of layer slices
// kc/vc; the new position pos = T - 1 comes from the stamped qkv words (epoch ep).  The
// split holding pos appends the new key (RoPE'd) and value to the cache and uses them
// directly.  Writes the split's partial; the last split of (b, g) to finish merges them into
// the stamped o words (epoch ep_out).  Returns false on a failed wait.
__device__ __forceinline__ bool attention_unit(const PersistArgs& a, float* scratch, int b, int g, int split, int S, int T,
                                            int pos, float* kc, float* vc, unsigned ep, unsigned ep_out,
                                            unsigned* ticket_s) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H = a.H, Hk = a.Hk, hpg = H / Hk;
  int s_act = (T + kMinPerSplit - 1) / kMinPerSplit;
  if (s_act > S) s_act = S;
  const int chunk = (T + s_act - 1) / s_act;
  s_act = (T + chunk - 1) / chunk;  // every active split gets at least one position
  if (split >= s_act) return true;
  const int t0 = split * chunk, t1 = min(T, t0 + chunk);
  const bool owner = t1 == T;  // this split holds the new position
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
  float* knew = linv + 8;                      // [64]
  float* vnew = knew + 64;                     // [64]
  const int nq = (H + 2 * Hk) * 64;
  const uint64_t* row = a.qkv_s + (size_t)b * nq;
  const float* cs = a.cosv + (size_t)pos * 32;
  const float* sn = a.sinv + (size_t)pos * 32;
  const size_t head = ((size_t)b * Hk + g) * a.cap;
  float* kb = kc + head * 64;
  float* vb = vc + head * 64;
  if (tid < 8) {
    mh[tid] = -INFINITY;
    lh[tid] = 0.f;
  }
  // first run of cached keys: issue these loads before waiting on this step's q
  auto stage = [&](int c0, int cn) {
    for (int i = tid; i < cn * 16; i += kConsumers) {
      const int p = i >> 4, f = i & 15;
      if (c0 + p == pos) continue;  // the new position comes from qkv
      const float4 kv = __ldcg(reinterpret_cast<const float4*>(kb + (size_t)(c0 + p) * 64) + f);
      Ks[p * 65 + 4 * f + 0] = kv.x;
      Ks[p * 65 + 4 * f + 1] = kv.y;
      Ks[p * 65 + 4 * f + 2] = kv.z;
      Ks[p * 65 + 4 * f + 3] = kv.w;
      reinterpret_cast<float4*>(Vs + p * 64)[f] = __ldcg(reinterpret_cast<const float4*>(vb + (size_t)(c0 + p) * 64) + f);
    }
  };
  stage(t0, min(kAttSub, t1 - t0));
  bool ok = true;
  for (int i = tid; i < hpg * 32; i += kConsumers) {
    const int h = i >> 5, j = i & 31;
    float x0 = 0.f, x1 = 0.f;
    ok = ok && poll_one(row + (g * hpg + h) * 64 + j, ep, x0, a);
    ok = ok && poll_one(row + (g * hpg + h) * 64 + j + 32, ep, x1, a);
    const float c = cs[j], s = sn[j];
    qs[h * 64 + j] = (x0 * c - x1 * s) * 0.125f;
    qs[h * 64 + j + 32] = (x0 * s + x1 * c) * 0.125f;
  }
  if (owner && tid < 64) {
    float v = 0.f;
    ok = ok && poll_one(row + (H + Hk + g) * 64 + tid, ep, v, a);
    vnew[tid] = v;
    vb[(size_t)pos * 64 + tid] = v;
    if (tid < 32) {
      float x0 = 0.f, x1 = 0.f;
      ok = ok && poll_one(row + (H + g) * 64 + tid, ep, x0, a);
      ok = ok && poll_one(row + (H + g) * 64 + tid + 32, ep, x1, a);
      const float c = cs[tid], s = sn[tid];
      const float k0 = x0 * c - x1 * s, k1 = x0 * s + x1 * c;
      knew[tid] = k0;
      knew[tid + 32] = k1;
      kb[(size_t)pos * 64 + tid] = k0;
      kb[(size_t)pos * 64 + tid + 32] = k1;
    }
  }
  if (consumer_bar_or(!ok)) return false;
  float oacc[2] = {0.f, 0.f};   // slots tid and tid + 256 of hpg * 64 (hpg <= 8)
  for (int c0 = t0; c0 < t1; c0 += kAttSub) {
    const int cn = min(kAttSub, t1 - c0);
    if (c0 != t0) {
      consumer_bar();
      stage(c0, cn);
    }
    if (owner && pos >= c0 && pos < c0 + cn && tid < 64) {
      const int p = pos - c0;
      Ks[p * 65 + tid] = knew[tid];
      Vs[p * 64 + tid] = vnew[tid];
    }
    consumer_bar();
    for (int i = tid; i < hpg * kAttSub; i += kConsumers) {
      const int h = i / kAttSub, p = i - h * kAttSub;
      float s = -INFINITY;
      if (p < cn) {
        s = 0.f;
#pragma unroll 4
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
      const float e0 = lane < cn ? ex(v0 - mnew) : 0.f;
      const float e1 = lane + 32 < cn ? ex(v1 - mnew) : 0.f;
      sc[h * kAttSub + lane] = e0;
      sc[h * kAttSub + lane + 32] = e1;
      const float sum = warp_sum(e0 + e1);
      __syncwarp();
      if (lane == 0) {
        const float cf = ex(mold - mnew);
        corr[h] = cf;
        lh[h] = lh[h] * cf + sum;
        mh[h] = mnew;
      }
    }
    consumer_bar();
    for (int k = 0; k < 2; ++k) {
      const int idx = tid + k * kConsumers;
      if (idx < hpg * 64) {
        const int h = idx >> 6, dd = idx & 63;
        float acc = oacc[k] * corr[h];
#pragma unroll 4
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
  if (!*ticket_s) return true;
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
      const float w = ex(mw[h * kAttMaxSplits + s] - mx);
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
    for (int s0 = 0; s0 < s_act; s0 += 8) {
      float v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        v[j] = s0 + j < s_act ? __ldcg(p0 + ((size_t)(s0 + j) * hpg + h) * 66 + 2 + dd) : 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (s0 + j < s_act) O = fmaf(mw[h * kAttMaxSplits + s0 + j], v[j], O);
    }
    st_stamp(a.o_s + ((size_t)b * H + g * hpg + h) * 64 + dd, O * linv[h], ep_out);
  }
  if (tid == 0) *ctr = 0u;
  return true;
}

__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

}  // namespace

template <int M, int FMT>
__device__ __forceinline__ bool decode_steps(const PersistArgs& a, Consumer& cs, const Smem& sm, const PLayer* layers);

template <int M, int FMT>
__global__ void __launch_bounds__(kThreads, 1) decode_persistent_kernel(const __grid_constant__ PersistArgs a) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const Smem sm = carve(smem, a.nslot);
  __shared__ PLayer layers_s[kMaxLayers];
  if (threadIdx.x == 0) {
    for (int i = 0; i < a.nslot; ++i) mbar_init(&sm.full[i], 1);
    mbar_fence_init();
  }
  for (int i = threadIdx.x; i < a.L * (int)(sizeof(PLayer) / 8); i += kThreads)
    reinterpret_cast<uint64_t*>(layers_s)[i] = reinterpret_cast<const uint64_t*>(a.layers)[i];
  __syncthreads();
  Consumer cs;
  cs.cur.layers = layers_s;
  cs.a = &a;
  cs.sm = sm;
  cs.c = blockIdx.x;
  cs.G = gridDim.x;
  cs.start();
  if (!decode_steps<M, FMT>(a, cs, sm, layers_s)) cs.drain();
}

template <int M, int FMT>
__device__ __forceinline__ bool decode_steps(const PersistArgs& a, Consumer& cs, const Smem& sm, const PLayer* layers) {
  __shared__ int ok_s;
  __shared__ unsigned ticket_s;
  __shared__ float bval[8][8];
  __shared__ int bidx[8][8];
  __shared__ int tok_s[8];
  __shared__ float xown[8][kMaxOwnRows];   // this CTA's residual rows (same rows in C and E)
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x, G = gridDim.x;
  const int d = a.d, H = a.H, Hk = a.Hk, F = a.F, V = a.V, B = M;
  const int nq = (H + 2 * Hk) * 64;
  unsigned epoch = 0;
  const int len0 = *a.dlen;
  const float4* act4 = reinterpret_cast<const float4*>(sm.act);
  int xr0, xr1;  // residual rows owned (the O and FC2 phases both have d rows)
  partition(d, c, G, xr0, xr1);
  int v0, v1;
  partition(V, c, G, v0, v1);
  const int units = B * Hk;
  int S = G / units;
  if (S < 1) S = 1;
  if (S > a.att_splits) S = a.att_splits;
  const unsigned per_step = 5u * a.L;

  for (int step = 0; step < a.n_steps; ++step) {
    const int pos = len0 + step;
    const int T = pos + 1;
    const unsigned ep0 = a.epoch_base + 1u + (unsigned)step * per_step;
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
      const PLayer& ly = layers[l];
      float* kc = a.kc + (size_t)l * a.layer_stride;
      float* vc = a.vc + (size_t)l * a.layer_stride;
      const unsigned epA = ep0 + 5u * l;
      if (l == 0) {
        for (int m = 0; m < M; ++m)
          for (int n = xr0 + tid; n < xr1; n += kConsumers) xown[m][n - xr0] = a.tok_emb[(size_t)tok_s[m] * d + n];
        for (int m = 0; m < M; ++m)
          embed_act(sm.act + (size_t)m * d, sm.red, a.tok_emb + (size_t)tok_s[m] * d, d, ly.ln1_g, ly.ln1_b, a.eps);
      }
      // phases A (QKV), B (attention), C (O + residual), D (FC1 + GELU), E (FC2 + residual)
      for (int ph = 0; ph < 5; ++ph) {
        const unsigned ep = epA + ph;
        if (ph == 1) {
          for (int u = c; u < units * S; u += G) {
            const int bg = u / S, split = u - bg * S;
            if (!attention_unit(a, sm.act, bg / Hk, bg % Hk, split, S, T, pos, kc, vc, epA, ep, &ticket_s))
              return false;
            consumer_bar();
          }
          continue;
        }
        const int mi = ph == 0 ? 0 : ph - 1;  // matrix of the phase
        const int K = mat_K(a, mi);
        if (!(ph == 0 && l == 0)) {
          const uint64_t* src = ph == 0 ? a.xe_s : ph == 2 ? a.o_s : ph == 3 ? a.xc_s : a.u_s;
          const float* g = ph == 0 ? ly.ln1_g : ph == 3 ? ly.ln2_g : nullptr;
          const float* bb = ph == 0 ? ly.ln1_b : ph == 3 ? ly.ln2_b : nullptr;
          if (!poll_act<M>(sm.act, sm.red, src, K, K, ep - 1, g, bb, a.eps, false, a)) return false;
        }
        OutSpec e;
        e.mode = (ph == 2 || ph == 4) ? 1 : ph == 3 ? 2 : 0;
        e.out = ph == 0 ? a.qkv_s : ph == 2 ? a.xc_s : ph == 3 ? a.u_s : a.xe_s;
        e.ldo = ph == 0 ? nq : ph == 3 ? F : d;
        e.ep = ep;
        e.xown = &xown[0][0];
        e.xr0 = xr0;
        int n0, n1;
        partition(mat_N(a, mi), c, G, n0, n1);
        if (!gemv_phase<M, FMT>(cs, act4, K, mat_rowb(a, mi), n0, n1, e)) return false;
      }
    }
    // ---- LM head + argmax ------------------------------------------------------------
    if (!poll_act<M>(sm.act, sm.red, a.xe_s, d, d, ep0 + per_step - 1, a.lnf_g, a.lnf_b, a.eps, true, a)) return false;
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
        if (!cs.release()) return false;
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
    // orders the cache append, the token history and the counters for the next step
    if (step + 1 < a.n_steps)
      if (!grid_sync(a, epoch, &ok_s)) return false;
  }
  return true;
}

// ---------------------------------------------------------------------------------
namespace {
size_t persist_region(int M, int d, int H, int F) {
  size_t act = (size_t)M * 4 * (size_t)max(max(d, H * 64), F);
  size_t att = sizeof(float) * (8 * 64 + kAttSub * 65 + kAttSub * 64 + 8 * kAttSub + 24 + 2 * 8 * kAttMaxSplits + 8 + 128);
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

size_t persistent_static_smem(int M, int fmt) {
  cudaFuncAttributes fa;
  cudaError_t e;
  if (fmt == kInt4)
    e = M == 1 ? cudaFuncGetAttributes(&fa, decode_persistent_kernel<1, kInt4>)
        : M == 2 ? cudaFuncGetAttributes(&fa, decode_persistent_kernel<2, kInt4>)
        : M == 4 ? cudaFuncGetAttributes(&fa, decode_persistent_kernel<4, kInt4>)
                 : cudaFuncGetAttributes(&fa, decode_persistent_kernel<8, kInt4>);
  else
    e = M == 1 ? cudaFuncGetAttributes(&fa, decode_persistent_kernel<1, kFp16>)
        : M == 2 ? cudaFuncGetAttributes(&fa, decode_persistent_kernel<2, kFp16>)
        : M == 4 ? cudaFuncGetAttributes(&fa, decode_persistent_kernel<4, kFp16>)
                 : cudaFuncGetAttributes(&fa, decode_persistent_kernel<8, kFp16>);
  return e == cudaSuccess ? fa.sharedSizeBytes : (size_t)-1;
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
