// Persistent decode kernel: greedy decode steps of the whole decoder (all layers, LM head,
// argmax, token feedback) in one cooperative launch, one CTA per SM.
//
// Why: at a few streams the decoder step is a chain of ~6 dependent phases per layer, each
// moving only a few MB; separate kernel launches pay a launch and drain per phase, and even a
// grid barrier costs ~2 us on 148 SMs.  Here the weight bytes — which never depend on the
// previous phase — stream continuously: each CTA builds the table of its weight slices for
// one step (its records of every matrix of every layer, then its LM head rows) and copies
// them with cp.async.bulk into a ring of shared-memory slots, nslot slices ahead of use
// across phase, layer and step boundaries; the last warp to finish a slot refills it, with no
// CTA barrier per slot.  The hand-off between phases needs no barrier either: every vector a
// phase produces (QKV, O, FC1 and FC2 outputs, attention output and partials) is written once
// as 64-bit words {value, epoch}; the consumer loads all the words it needs at once and
// re-reads only the stale ones, all together — the wait and the read are one L2 round trip.
// One grid barrier per step (after the LM head) orders the rest (cache append, token
// history).
//
// Phases of one step (token position pos, T = pos + 1 keys):
//   A  x += FC2 parts of the previous layer (or x = the token embedding), LN1, QKV rows
//   B  attention unit (stream, kv head, split): RoPE of q (and of the new k, which the
//      split holding pos appends to the cache with v), scores over its run of positions,
//      partial (m, l, o); one CTA per head then merges the splits' partials  -> o
//   C  O rows
//   D  x += O parts, LN2, FC1 rows (GELU applied by the producer when FC1's tiles are whole)
//   E  GELU of the FC1 parts' sum when FC1 is split along K, FC2 rows
// Every CTA keeps its own copy of the residual rows x (each thread its own elements) and
// adds the published partial sums itself, so no CTA owns output rows.
//   after the last layer: x, LN_f, LM head rows, per-CTA argmax (guided for stream pairs
//   when classifier-free guidance is on), the last CTA picks the token, records it in the
//   token history and advances the cache length.
//
// Matrix-vector products.  The weights are a tile-packed copy of each matrix: records of 16
// rows x 32 columns (one quantisation group), each lane's MMA fragment words adjacent.  Each
// tile's K range is cut into S = 1, 2 or 4 work units, spread evenly over the CTAs; the eight
// warps split each slice's records.  Per record a warp runs two m16n8k16 tensor-core MMAs
// with the 16 weight rows as A (INT4 codes turned into exact fp16 integers with one mask and
// one fp16 op per pair) and the activations as B: the fp32 input vector, scaled by a power of
// two so that its largest element is below 2^14, is written once per phase as an fp16 pair
// hi + lo (hi = fp16(x), lo = fp16(x - hi): 22 significant bits), columns 2m and 2m + 1 for
// stream m.  The products are exact, the sums fp32, and each record's result is multiplied
// by its group's fp32 scales.
//
// Every wait is bounded: the grid barrier's spin, the stamped-word settles and the ring's
// mbarrier waits give up after a limit, set the status word's timeout bit and an abort word
// that makes every CTA leave; a CTA that leaves first waits (bounded) for its copies in
// flight.
#include <float.h>
#include <limits.h>
#include "ms_device.cuh"
#include "ms_launch.cuh"
#include "ms_persistent.h"

namespace ms {

namespace {
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kSlot = 16384;
constexpr int kAttSub = 64;
constexpr int kAttMaxSplits = 128;
constexpr int kMinPerSplit = 16;
constexpr int kTile = 16;                 // weight rows per tile (the MMA's M)
constexpr int kMaxUnits = 4;              // work units (a tile's K range) of one matrix per CTA
constexpr int kMaxLayers = 64;            // layer table kept in shared memory
constexpr int kPairBatch = 8;             // element pairs a thread has in flight per round
constexpr int kRecInt4 = 320;             // tile-packed record: 64 code words + 16 scales
constexpr int kRecF16 = 1024;             // tile-packed record: 32 x 32 bytes of halves
constexpr int kUnroll = 4;                // records a warp has in flight (2 for more than 4 streams)

// Attention scratch (floats): q, scores, per-head running stats, the new k and v; then either
// the staged keys/values or, for a merge, the splits' partials.
constexpr int kAttQs = 0;
constexpr int kAttSc = kAttQs + 8 * 64;
constexpr int kAttSmall = kAttSc + 8 * kAttSub;   // mh[8] lh[8] corr[8] pad[8] knew[64] vnew[64]
constexpr int kAttU = kAttSmall + 160;
constexpr int kAttKs = kAttU;                     // [64][65]
constexpr int kAttVs = kAttKs + kAttSub * 65;     // [64][64]
constexpr int kMrgMw = kAttU;                     // [128]
constexpr int kMrgLw = kMrgMw + kAttMaxSplits;    // [128]
constexpr int kMrgOv = kMrgLw + kAttMaxSplits;    // [128][64]
constexpr int kMrgP4 = kMrgOv + kAttMaxSplits * 64;  // [4][64]
constexpr int kMrgLin = kMrgP4 + 256;
constexpr int kAttFloats = (kAttVs + kAttSub * 64 > kMrgLin + 4 ? kAttVs + kAttSub * 64 : kMrgLin + 4);
static_assert((kAttVs * 4) % 16 == 0 && (kMrgOv * 4) % 16 == 0, "float4 alignment of the attention scratch");

__device__ __forceinline__ void consumer_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
// Named barrier of the CTA's threads that also ORs a flag over them.
__device__ __forceinline__ bool consumer_bar_or(bool pred) {
  unsigned r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n barrier.cta.red.or.pred q, 1, 256, p;\n selp.u32 %0, 1, 0, q;\n}"
      : "=r"(r)
      : "r"((unsigned)pred)
      : "memory");
  return r != 0;
}

// No routine of this kernel is called out of line: with nearly all of the SM's unified L1
// given to shared memory, a call's register saves (local memory) would cost a round trip
// to L2.
__device__ __forceinline__ float ex(float x) { return expf(x); }
__device__ __forceinline__ float gelu_ool(float u) { return gelu_erf(u); }

// Shapes of matrix mi (0 QKV, 1 O, 2 FC1, 3 FC2), as scalar selects: a small array indexed
// at run time would live in local memory.
__device__ __forceinline__ int mat_N(const PersistArgs& a, int mi) {
  return mi == 0 ? (a.H + 2 * a.Hk) * 64 : mi == 2 ? a.F : a.d;
}
__device__ __forceinline__ int mat_K(const PersistArgs& a, int mi) {
  return mi == 1 ? a.H * 64 : mi == 3 ? a.F : a.d;
}

// Ring position (each consumer thread keeps its own copy).
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

// One weight slice of the schedule: a contiguous run of records (or LM head rows).
struct Slice {
  const unsigned char* src;
  uint32_t bytes;
  uint32_t pad;
};

struct Smem {
  uint64_t* full;          // ring mbarriers [16]
  float* red;              // reduction slots [2][8][4]
  unsigned* cnt;           // warps done with each slot, counted up [16]
  unsigned* niss;          // copies issued into each slot [16]
  int* ntab;               // slices per step
  Slice* tab;              // the CTA's slices of one step, in consumption order
  unsigned char* ring;
  unsigned char* region;   // activation planes, staging, partial sums / attention scratch / LM head input
};

__host__ __device__ __forceinline__ size_t tab_bytes(int cap) { return ((size_t)cap * sizeof(Slice) + 1023) & ~(size_t)1023; }

__device__ __forceinline__ Smem carve(unsigned char* base, int nslot, int cap) {
  Smem s;
  s.full = reinterpret_cast<uint64_t*>(base);
  s.red = reinterpret_cast<float*>(base + 128);
  s.cnt = reinterpret_cast<unsigned*>(base + 384);
  s.niss = reinterpret_cast<unsigned*>(base + 448);
  s.ntab = reinterpret_cast<int*>(base + 512);
  s.tab = reinterpret_cast<Slice*>(base + 1024);
  s.ring = base + 1024 + tab_bytes(cap);
  s.region = s.ring + (size_t)nslot * kSlot;
  return s;
}

// Shared-memory region of the matrix phases: A planes (2M rows of K halves, row stride
// K/2 + 16 words so that rows 2m and 2m + 1 fall in different banks), the thread-private
// staging of the loaded vector, and the warps' partial sums [tile][warp][m][8].
__host__ __device__ __forceinline__ size_t plane_bytes(int M, int kmax) {
  return align16((size_t)2 * M * (2 * kmax + 64));
}
__host__ __device__ __forceinline__ size_t xin_bytes(int kmax) { return align16((size_t)kmax * 4); }
__host__ __device__ __forceinline__ size_t part_bytes(int M) { return (size_t)kMaxUnits * kWarps * M * kTile * 4; }
__host__ __device__ __forceinline__ size_t gb_bytes(int d) { return align16((size_t)d * 8); }

// Work units of a matrix: each 16-row tile's K range cut into S equal parts (S = 1, 2 or
// 4), units spread evenly over the G CTAs.  S is the smallest that minimises the busiest
// CTA's records, counting each extra part as 10 % more work (its consumers read one more
// partial sum per element); at most kMaxUnits units per CTA.
__host__ __device__ __forceinline__ int choose_split(int nt, int KG, int G) {
  int best = 1;
  long long best_cost = -1;
  for (int S = 1; S <= 4; S *= 2) {
    if (KG % S != 0) continue;
    const long long units = ((long long)nt * S + G - 1) / G;
    if (units > kMaxUnits) continue;
    const long long cost = units * (KG / S) * (10 + (S - 1));
    if (best_cost < 0 || cost < best_cost) {
      best = S;
      best_cost = cost;
    }
  }
  return best;
}
// First record of unit u (tile u / S, part u % S) in the tile-packed matrix.
__host__ __device__ __forceinline__ int unit_rec(int u, int S, int KG) { return (u / S) * KG + (KG * (u % S)) / S; }

// Bytes of the region's aliased part: the matrix phases' planes, staging and partial sums,
// the attention scratch, or the LM head's input, whichever is largest.  The zero row follows.
__host__ __device__ __forceinline__ size_t persist_main(int M, int d, int H, int F) {
  const int kmax = max(max(d, H * 64), F);
  const size_t mv = plane_bytes(M, kmax) + xin_bytes(kmax) + gb_bytes(d) + part_bytes(M);
  const size_t att = align16(sizeof(float) * (size_t)kAttFloats);
  const size_t lm = align16((size_t)M * d * 4);
  const size_t r = mv > att ? mv : att;
  return r > lm ? r : lm;
}

struct Region {
  uint32_t* planes;
  float2* xin;    // staged input pairs (each thread reads back only the pairs it wrote)
  float4* gb;     // staged LayerNorm (gamma, gamma, beta, beta) per pair, likewise
  float* part;
  const uint32_t* zero;   // a row of zeros: the B columns of streams that do not exist
};

// ---------------------------------------------------------------------------------
// Stamped words and reductions
// ---------------------------------------------------------------------------------

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
// Two consecutive words (16-byte aligned); each element is read whole.
__device__ __forceinline__ void ld_stamp2(const uint64_t* p, uint64_t& w0, uint64_t& w1) {
  asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(w0), "=l"(w1) : "l"(p) : "memory");
}

// Waits until every word a thread has loaded carries epoch ep: the stale ones are read
// again together (all in flight), with one backoff per round — never one round trip per
// word.  Pairs (two consecutive words per load) and single words.  Returns false if the
// wait ran out or another CTA gave up.
__device__ __forceinline__ bool stale2(uint64_t w0, uint64_t w1, unsigned ep) {
  return ((unsigned)(w0 >> 32) != ep) | ((unsigned)(w1 >> 32) != ep);
}
__device__ __forceinline__ bool settle_wait(long long it, unsigned& ns, const PersistArgs& a) {
  if ((it & 15) == 15) {
    if (*reinterpret_cast<volatile unsigned*>(a.abort)) return false;
    if (it > a.settle_limit) {
      flag_error(a.status, kErrTimeout);
      atomicExch(a.abort, 1u);
      return false;
    }
  }
  __nanosleep(ns);
  if (ns < 256) ns <<= 1;
  return true;
}
template <int N>
__device__ __forceinline__ bool settle_pairs(uint64_t (&w0)[N], uint64_t (&w1)[N], const uint64_t* const (&pp)[N],
                                             const bool (&use)[N], unsigned ep, const PersistArgs& a) {
  unsigned ns = 64;
  for (long long it = 0;; ++it) {
    bool stale = false;
#pragma unroll
    for (int j = 0; j < N; ++j) stale |= use[j] && stale2(w0[j], w1[j], ep);
    if (!stale) return true;
    if (!settle_wait(it, ns, a)) return false;
#pragma unroll
    for (int j = 0; j < N; ++j)
      if (use[j] && stale2(w0[j], w1[j], ep)) ld_stamp2(pp[j], w0[j], w1[j]);
  }
}
template <int N>
__device__ __forceinline__ bool settle_words(uint64_t (&w)[N], const uint64_t* const (&pp)[N], const bool (&use)[N],
                                             unsigned ep, const PersistArgs& a) {
  unsigned ns = 64;
  for (long long it = 0;; ++it) {
    bool stale = false;
#pragma unroll
    for (int j = 0; j < N; ++j) stale |= use[j] && (unsigned)(w[j] >> 32) != ep;
    if (!stale) return true;
    if (!settle_wait(it, ns, a)) return false;
#pragma unroll
    for (int j = 0; j < N; ++j)
      if (use[j] && (unsigned)(w[j] >> 32) != ep) w[j] = ld_stamp(pp[j]);
  }
}

// Block-wide reduction with one barrier: x summed, y and z maxed.  The slots alternate
// between two halves, so a reduction's slots are never rewritten before every thread has
// passed the next reduction's barrier (and so has read them).
struct Red {
  float* buf;
  int par;
};
__device__ __forceinline__ float3 block_red(float x, float y, float z, Red& r) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    x += __shfl_xor_sync(0xffffffffu, x, o);
    y = fmaxf(y, __shfl_xor_sync(0xffffffffu, y, o));
    z = fmaxf(z, __shfl_xor_sync(0xffffffffu, z, o));
  }
  float* slot = r.buf + r.par * 32;
  if (lane == 0) *reinterpret_cast<float4*>(slot + warp * 4) = make_float4(x, y, z, 0.f);
  consumer_bar();
  float X = 0.f, Y = 0.f, Z = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const float4 v = *reinterpret_cast<const float4*>(slot + w * 4);
    X += v.x;
    Y = fmaxf(Y, v.y);
    Z = fmaxf(Z, v.z);
  }
  r.par ^= 1;
  return make_float3(X, Y, Z);
}

// e such that bound * 2^e < 2^14 (fp16 hi/lo pairs then stay far from overflow and keep
// ~22 significant bits); clamped so that 2^e and 2^-e are normal floats.
__device__ __forceinline__ int act_exp(float bound) {
  const unsigned bits = __float_as_uint(bound);
  if ((bits & 0x7F800000u) == 0) return 100;  // zero or subnormal bound
  const int E = (int)((bits >> 23) & 0xFFu) - 126;   // bound < 2^E
  return min(max(14 - E, -100), 100);
}
__device__ __forceinline__ float exp2i(int e) { return __uint_as_float((unsigned)(127 + e) << 23); }
// Two floats to an fp16 pair (lo in the low half), round to nearest even.
__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ float half_lo(uint32_t h) {
  float f;
  asm("{ .reg .b16 l, u;\n mov.b32 {l, u}, %1;\n cvt.f32.f16 %0, l; }" : "=f"(f) : "r"(h));
  return f;
}
__device__ __forceinline__ float half_hi(uint32_t h) {
  float f;
  asm("{ .reg .b16 l, u;\n mov.b32 {l, u}, %1;\n cvt.f32.f16 %0, u; }" : "=f"(f) : "r"(h));
  return f;
}
// Word of pair p (elements 2p, 2p + 1) in a plane row: within each 32-element group, lane
// quad t's four pairs (2t + 8i, i = 0..3) are adjacent, so one 16-byte load fetches a lane's
// A fragments of both k16 steps.
__device__ __forceinline__ int plane_word(int p) {
  const int q = p & 15;
  return (p >> 4) * 16 + (q & 3) * 4 + (q >> 2);
}

// Source of a phase's input row: S stamped slices (st + h * stride, h < S, added in order)
// carrying epoch ep, or plain floats (pl, the token embedding); then, with res, the CTA's
// copy of the residual row added to the sum (res := x), or GELU applied.
struct VecSrc {
  const uint64_t* st;
  long long stride;
  const float* pl;
  unsigned ep;
  float2* res;   // residual pairs of this row (each thread's own pairs), or null
  bool gelu;
};

// Loads one vector row of K elements, optionally LayerNorm'd (g != null), into shared
// memory: as the fp16 hi/lo A rows phi/plo scaled by 2^e (PLANES; *inv = 2^-e), or as plain
// fp32 at act.  Every load of a round is in flight before the thread waits on any; the
// values (and gamma, beta) are staged in shared memory, each thread reading back only the
// pairs it wrote.  Returns false (this thread) on a failed wait; the caller ORs the outcome
// over the CTA.
// Only pairs [p0, P) are loaded (a phase whose work units all lie in one K range needs no
// more); a LayerNorm'd row is always loaded whole.
template <bool PLANES, int S>
__device__ __forceinline__ bool load_row(const VecSrc& src, int K, int p0, int P, const float* g, const float* bt,
                                         float eps, uint32_t* phi, uint32_t* plo, float* inv, float* act,
                                         const Region& rg, Red& red, const PersistArgs& a) {
  constexpr int PR = kPairBatch / S;   // pairs per round per thread
  const int tid = threadIdx.x;
  float2* xin = rg.xin;
  bool ok = true;
#pragma unroll 1
  for (int base = p0; base < P; base += kThreads * PR) {
    uint64_t w0[kPairBatch], w1[kPairBatch];
    const uint64_t* pp[kPairBatch];
    bool use[kPairBatch];
#pragma unroll
    for (int j = 0; j < kPairBatch; ++j) {
      const int pj = j / S, hj = j % S;
      const int p = base + tid + pj * kThreads;
      use[j] = p < P;
      pp[j] = src.st + hj * src.stride + 2 * (use[j] ? p : 0);
      w0[j] = w1[j] = 0;
      if (use[j]) {
        if (src.st) {
          ld_stamp2(pp[j], w0[j], w1[j]);
        } else {
          const float2 f = reinterpret_cast<const float2*>(src.pl)[p];
          w0[j] = __float_as_uint(f.x);
          w1[j] = __float_as_uint(f.y);
        }
      }
    }
    if (g)
      for (int p = base + tid; p < min(P, base + kThreads * PR); p += kThreads) {
        const float2 gv = reinterpret_cast<const float2*>(g)[p], bv = reinterpret_cast<const float2*>(bt)[p];
        rg.gb[p] = make_float4(gv.x, gv.y, bv.x, bv.y);
      }
    if (src.st && ok) ok = settle_pairs<kPairBatch>(w0, w1, pp, use, src.ep, a);
#pragma unroll
    for (int pj = 0; pj < PR; ++pj) {
      const int p = base + tid + pj * kThreads;
      if (use[pj * S]) {
        float v0 = 0.f, v1 = 0.f;
#pragma unroll
        for (int h = 0; h < S; ++h) {
          v0 += __uint_as_float((unsigned)w0[pj * S + h]);
          v1 += __uint_as_float((unsigned)w1[pj * S + h]);
        }
        if (src.res) {
          if (!src.pl) {
            const float2 r = src.res[p];
            v0 = r.x + v0;
            v1 = r.y + v1;
          }
          src.res[p] = make_float2(v0, v1);
        }
        if (src.gelu) {
          v0 = gelu_ool(v0);
          v1 = gelu_ool(v1);
        }
        xin[p] = make_float2(v0, v1);
      }
    }
  }
  float mean = 0.f, rstd = 1.f, bound = 0.f;
  if (g) {
    float s = 0.f;
    for (int p = p0 + tid; p < P; p += kThreads) {
      const float2 x = xin[p];
      s += x.x + x.y;
    }
    mean = block_red(s, 0.f, 0.f, red).x / K;
    float q = 0.f, am = 0.f, bm = 0.f;
    for (int p = p0 + tid; p < P; p += kThreads) {
      const float2 x = xin[p];
      const float4 gb = rg.gb[p];
      const float d0 = x.x - mean, d1 = x.y - mean;
      q += d0 * d0 + d1 * d1;
      am = fmaxf(am, fmaxf(fabsf(d0) * fabsf(gb.x), fabsf(d1) * fabsf(gb.y)));
      bm = fmaxf(bm, fmaxf(fabsf(gb.z), fabsf(gb.w)));
    }
    const float3 r = block_red(q, am, bm, red);
    rstd = 1.0f / sqrtf(r.x / K + eps);
    bound = rstd * r.y + r.z;   // |LN(x)_k| <= rstd |x_k - mean| |g_k| + |b_k|
  } else if (PLANES) {
    float am = 0.f;
    for (int p = p0 + tid; p < P; p += kThreads) {
      const float2 x = xin[p];
      am = fmaxf(am, fmaxf(fabsf(x.x), fabsf(x.y)));
    }
    bound = block_red(0.f, am, 0.f, red).y;
  }
  float sc = 1.f;
  if (PLANES) {
    const int e = act_exp(bound);
    sc = exp2i(e);
    if (tid == 0) *inv = exp2i(-e);
  }
  for (int p = p0 + tid; p < P; p += kThreads) {
    const float2 x = xin[p];
    float y0 = x.x, y1 = x.y;
    if (g) {
      const float4 gb = rg.gb[p];
      y0 = (x.x - mean) * rstd * gb.x + gb.z;
      y1 = (x.y - mean) * rstd * gb.y + gb.w;
    }
    if (PLANES) {
      y0 *= sc;
      y1 *= sc;
      const uint32_t hi = pack_half2(y0, y1);
      const int wd = plane_word(p);
      phi[wd] = hi;
      plo[wd] = pack_half2(y0 - half_lo(hi), y1 - half_hi(hi));
    } else {
      reinterpret_cast<float2*>(act)[p] = make_float2(y0, y1);
    }
  }
  return ok;
}

// ---------------------------------------------------------------------------------
// Matrix phases
// ---------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t b, uint32_t c) {  // (a & b) | c
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}
// Codes u (= q + 8) in bits 0-3 and 16-19 -> halves q: 0x6400 | u is 1024 + u, minus 1032.
__device__ __forceinline__ uint32_t q_pair_a(uint32_t w) {
  const uint32_t h = lop3_and_or(w, 0x000F000Fu, 0x64006400u);
  uint32_t r;
  asm("sub.f16x2 %0, %1, %2;" : "=r"(r) : "r"(h), "r"(0x64086408u));
  return r;
}
// Codes in bits 4-7 and 20-23 -> halves q: 0x6400 | (u << 4) is 1024 + 16u; / 16 - 72.
__device__ __forceinline__ uint32_t q_pair_b(uint32_t w) {
  const uint32_t h = lop3_and_or(w, 0x00F000F0u, 0x64006400u);
  uint32_t r;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(h), "r"(0x2C002C00u), "r"(0xD480D480u));
  return r;
}
// D += A B for one m16n8k16 step (A rows = activation planes, B columns = weight rows).
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One record (tile, group g) of the warp's share, added into acc (use = false: read but
// not added).  A = the 16 weight rows (INT4 codes turned into exact fp16 integers, two
// halves per mask and fp16 op), B = the activation planes (column 2m + j: stream m, hi or
// lo).  Lane (r = lane / 4, t = lane % 4) holds acc[0], acc[1] = rows r of columns 2t, 2t + 1
// (stream t, hi and lo), acc[2], acc[3] = row r + 8 of the same; acc[4..7] the same for
// streams 4 + t.  The group's INT4 scales multiply each record's sums.
// Shared-memory loads by 32-bit shared address (the record and plane pointers reach the loop
// as generic pointers; explicit ld.shared avoids the generic path's extra latency).
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}

// rec, blo, bhi: shared addresses of the record and of this lane's activation plane words.
template <int M, int FMT>
__device__ __forceinline__ void mv_record(uint32_t rec, uint32_t blo, uint32_t bhi, int g, bool use,
                                          float (&acc)[8]) {
  const int lane = threadIdx.x & 31, gid = lane >> 2;
  const uint4 b = lds128(blo + g * 64);
  uint4 b2 = make_uint4(0u, 0u, 0u, 0u);
  if (M > 4) b2 = lds128(bhi + g * 64);
  uint32_t a[8];
  float s0, s1;
  if (FMT == kInt4) {
    const uint2 w = lds64(rec + lane * 8);
    const uint2 sr = lds64(rec + 256 + gid * 8);
    const float2 s = make_float2(__uint_as_float(sr.x), __uint_as_float(sr.y));
    s0 = use ? s.x : 0.f;
    s1 = use ? s.y : 0.f;
    const uint32_t x8 = w.x >> 8, y8 = w.y >> 8;
    a[0] = q_pair_a(w.x);
    a[1] = q_pair_a(w.y);
    a[2] = q_pair_b(w.x);
    a[3] = q_pair_b(w.y);
    a[4] = q_pair_a(x8);
    a[5] = q_pair_a(y8);
    a[6] = q_pair_b(x8);
    a[7] = q_pair_b(y8);
  } else {
    const uint4 x0 = lds128(rec + lane * 32);
    const uint4 x1 = lds128(rec + lane * 32 + 16);
    s0 = s1 = use ? 1.f : 0.f;
    a[0] = x0.x;
    a[1] = x0.y;
    a[2] = x0.z;
    a[3] = x0.w;
    a[4] = x1.x;
    a[5] = x1.y;
    a[6] = x1.z;
    a[7] = x1.w;
  }
  float d[4] = {0.f, 0.f, 0.f, 0.f};
  mma16816(d, a[0], a[1], a[2], a[3], b.x, b.y);
  mma16816(d, a[4], a[5], a[6], a[7], b.z, b.w);
  acc[0] = fmaf(s0, d[0], acc[0]);
  acc[1] = fmaf(s0, d[1], acc[1]);
  acc[2] = fmaf(s1, d[2], acc[2]);
  acc[3] = fmaf(s1, d[3], acc[3]);
  if (M > 4) {
    float e[4] = {0.f, 0.f, 0.f, 0.f};
    mma16816(e, a[0], a[1], a[2], a[3], b2.x, b2.y);
    mma16816(e, a[4], a[5], a[6], a[7], b2.z, b2.w);
    acc[4] = fmaf(s0, e[0], acc[4]);
    acc[5] = fmaf(s0, e[1], acc[5]);
    acc[6] = fmaf(s1, e[2], acc[6]);
    acc[7] = fmaf(s1, e[3], acc[7]);
  }
}

// Adds a warp's sums for tile tl (hi + lo) into its partial slots [tile][warp][m][16].
template <int M>
__device__ __forceinline__ void flush_tile(float (&acc)[8], float* part, int tl) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, gid = lane >> 2, tq = lane & 3;
  float* pp = part + (size_t)(tl * kWarps + warp) * M * kTile;
  if (tq < M) {
    pp[tq * kTile + gid] += acc[0] + acc[1];
    pp[tq * kTile + gid + 8] += acc[2] + acc[3];
  }
  if (M > 4 && tq + 4 < M) {
    pp[(tq + 4) * kTile + gid] += acc[4] + acc[5];
    pp[(tq + 4) * kTile + gid + 8] += acc[6] + acc[7];
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
}

// A matrix phase's share: units [u0, u1) of the matrix's S-part split, i.e. records
// [rbeg, rend); outputs (partial sums) go to slice (unit % S) of out, words
// out[h * stride + m * N + n], with epoch ep.
struct MvJob {
  int K, N, S, u0, u1, rbeg, rend;
  uint64_t* out;
  long long stride;
  unsigned ep;
  bool gelu;   // publish GELU of the sums (only when the tiles are not split along K)
};

__device__ __forceinline__ unsigned atom_add_acq_rel_shared(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(smem_u32(p)), "r"(v) : "memory");
  return old;
}

// The weight ring.  Every thread consumes the slices in order (slice i in slot i % nslot);
// a warp that is done with a slice counts itself out of the slot (acquire-release), and the
// last of the eight warps refills the slot with slice i + nslot at once — no CTA barrier per
// slot.  It refills only if its own wait saw the slice's bytes arrive (so no copy into the
// slot is still in flight).  Waits are bounded; a thread whose wait ran out raises the
// abort word and the CTA leaves at the end of the phase.
struct Ring {
  const PersistArgs* a;
  Smem sm;
  long long i = 0;       // next slice to consume
  long long total = 0;   // slices of the launch
  int E = 1;             // slices per step
  bool got = false;
  __device__ void issue(long long j) {
    if (j >= total) return;
    const Slice sl = sm.tab[j % E];
    const int slot = (int)(j % a->nslot);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    mbar_expect_tx(&sm.full[slot], sl.bytes);
    bulk_g2s(sm.ring + (size_t)slot * kSlot, sl.src, sl.bytes, &sm.full[slot]);
    sm.niss[slot] += 1u;
  }
  __device__ void start() {
    if (threadIdx.x == 0)
      for (int k = 0; k < a->nslot; ++k) issue(k);
  }
  // The slot of slice i (its bytes valid only if got).
  __device__ const unsigned char* acquire() {
    const int slot = (int)(i % a->nslot);
    got = mbar_wait(&sm.full[slot], (uint32_t)((i / a->nslot) & 1), a->status);
    if (!got) atomicExch(a->abort, 1u);
    return sm.ring + (size_t)slot * kSlot;
  }
  __device__ void release() {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) {
      const int slot = (int)(i % a->nslot);
      const unsigned old = atom_add_acq_rel_shared(&sm.cnt[slot], 1u);
      if (old % kWarps == kWarps - 1 && got) issue(i + a->nslot);
    }
    __syncwarp();
    ++i;
  }
  // Before leaving early: wait (bounded) for the last copy issued into each slot.
  __device__ void drain() {
    if (threadIdx.x != 0) return;
    for (int k = 0; k < a->nslot; ++k) {
      const unsigned n = sm.niss[k];
      if (n == 0) continue;
      for (long long it = 0; it < kSpinLimit; ++it)
        if (mbar_try_wait(&sm.full[k], (n - 1u) & 1u)) break;
    }
  }
};

// One matrix phase over the CTA's records, slice by slice from the ring; the A planes hold
// the phase's input.  Each warp takes a contiguous run of each slice's records, unit segment
// by unit segment (kUnroll records in flight, branch-free); a segment's sums go to the
// warp's partial slots; the CTA then adds the eight warps' partials in a fixed order, scales
// by the input's 2^-e and publishes each unit's 16 rows as {value, epoch} words.
template <int M, int FMT>
__device__ __forceinline__ bool mv_phase(Ring& ring, const Region& rg, const MvJob& jb, const float* inv_s) {
  constexpr int RB = FMT == kInt4 ? kRecInt4 : kRecF16;
  constexpr int PER = kSlot / RB;
  constexpr int U = M > 4 ? kUnroll / 2 : kUnroll;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, gid = lane >> 2, tq = lane & 3;
  const int K = jb.K, S = jb.S, KG = K >> 5;
  const int nu = jb.u1 - jb.u0;
  const int pw = (K >> 1) + 16;
  // this lane's B rows: plane row gid (the zero row past the streams) and, for 8 streams, gid + 8
  const uint32_t blo = smem_u32((gid < 2 * M ? rg.planes + gid * pw : rg.zero) + tq * 4);
  const uint32_t bhi = smem_u32(rg.planes + (M > 4 ? (gid + 8) * pw : 0) + tq * 4);
  for (int i = lane; i < nu * M * kTile; i += 32) {
    const int ul = i / (M * kTile);
    rg.part[(size_t)(ul * kWarps + warp) * M * kTile + (i - ul * M * kTile)] = 0.f;
  }
  __syncwarp();
  bool ok = true;
  for (int p = jb.rbeg; p < jb.rend; p += PER) {
    const int n = min(PER, jb.rend - p);
    const uint32_t buf = smem_u32(ring.acquire());
    ok = ok && ring.got;
    if (ring.got) {
      const int c0 = (n * warp) >> 3, c1 = (n * (warp + 1)) >> 3;
      int i = c0;
      while (i < c1) {
        const int r = p + i;                                 // record index in the matrix
        const int t = r / KG, g = r - t * KG;
        const int h = ((g + 1) * S - 1) / KG;                // part of the tile holding group g
        const int rend_u = t * KG + (KG * (h + 1)) / S;       // the unit's end
        const int s1 = min(c1, i + (rend_u - r));
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int gi = g; i < s1; i += U, gi += U) {
#pragma unroll
          for (int j = 0; j < U; ++j) {
            const int ij = min(i + j, s1 - 1);  // past the segment's end: re-read its last record, not added
            mv_record<M, FMT>(buf + (uint32_t)(ij * RB), blo, bhi, gi + (ij - i), i + j < s1, acc);
          }
        }
        i = s1;   // the next segment starts exactly where this one ends
        flush_tile<M>(acc, rg.part, t * S + h - jb.u0);
      }
    }
    ring.release();
  }
  if (consumer_bar_or(!ok)) return false;
  for (int o = threadIdx.x; o < nu * kTile * M; o += kThreads) {
    const int ul = o / (kTile * M), rem = o - ul * kTile * M, m = rem / kTile, rr = rem - m * kTile;
    const float* pp = rg.part + (size_t)ul * kWarps * M * kTile + m * kTile + rr;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) v += pp[w * M * kTile];
    const int u = jb.u0 + ul, t = u / S, h = u - t * S;
    v *= inv_s[m];
    if (jb.gelu) v = gelu_ool(v);
    st_stamp(jb.out + h * jb.stride + (size_t)m * jb.N + t * kTile + rr, v, jb.ep);
  }
  consumer_bar();  // the region is reused by the next phase
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
    const unsigned target = epoch * gridDim.x + (a.test_stall == 2 ? 1u : 0u);
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
        if (it > a.grid_limit) {
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

// Active splits of a (stream, kv head) over T keys (at least kMinPerSplit positions each, no
// empty split) and the positions per split.
__device__ __forceinline__ void att_split_count(int T, int S, int& s_act, int& chunk) {
  s_act = (T + kMinPerSplit - 1) / kMinPerSplit;
  if (s_act > S) s_act = S;
  chunk = (T + s_act - 1) / s_act;
  s_act = (T + chunk - 1) / chunk;
}

// Attention for one (stream b, kv head g, split) unit over keys [0, T) of layer slices
// kc/vc; the new position pos = T - 1 comes from the stamped qkv words (epoch ep).  The
// split holding pos appends the new key (RoPE'd) and value to the cache and uses them
// directly.  With one active split it writes the normalised output o; otherwise its partial
// (m, l, o) per head as stamped words (epoch ep_out) for the merge.  Returns false on a
// failed wait.
__device__ __forceinline__ bool attention_unit(const PersistArgs& a, float* scratch, int b, int g, int split, int S,
                                            int s_act, int chunk, int T, int pos, void* kc, void* vc, unsigned ep,
                                            unsigned ep_out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H = a.H, Hk = a.Hk, hpg = H / Hk;
  if (split >= s_act) return true;
  const int t0 = split * chunk, t1 = min(T, t0 + chunk);
  const bool owner = t1 == T;  // this split holds the new position
  float* qs = scratch + kAttQs;    // [8][64]
  float* sc = scratch + kAttSc;    // [8][64]
  float* mh = scratch + kAttSmall; // [8]
  float* lh = mh + 8;
  float* corr = lh + 8;
  float* knew = corr + 16;         // [64]
  float* vnew = knew + 64;         // [64]
  float* Ks = scratch + kAttKs;    // [64][65]
  float* Vs = scratch + kAttVs;    // [64][64]
  const int nq = (H + 2 * Hk) * 64;
  const uint64_t* row = a.vs[0] + (size_t)b * nq;   // QKV is one slice
  const float* cs = a.cosv + (size_t)pos * 32;
  const float* sn = a.sinv + (size_t)pos * 32;
  const size_t head = ((size_t)b * Hk + g) * a.cap * 64;   // first element of the head's rows
  const bool h16 = a.kv16 != 0;
  if (tid < 8) {
    mh[tid] = -INFINITY;
    lh[tid] = 0.f;
  }
  // a run of up to 64 cached positions into Ks / Vs: every load of the thread (4 of K, 4 of
  // V) is in flight before its first store, so a run costs one memory round trip.  The first
  // run is issued before the wait on this step's q.
  auto stage = [&](int c0, int cn) {
    float4 kr[kAttSub * 16 / kThreads], vr[kAttSub * 16 / kThreads];
#pragma unroll
    for (int j = 0; j < kAttSub * 16 / kThreads; ++j) {
      const int i = tid + j * kThreads, p = i >> 4, f = i & 15;
      if (p < cn && c0 + p != pos) {   // the new position comes from qkv
        const size_t e = head + (size_t)(c0 + p) * 64 + 4 * f;
        kr[j] = h16 ? kv_load4<1>(kc, e) : kv_load4<0>(kc, e);
        vr[j] = h16 ? kv_load4<1>(vc, e) : kv_load4<0>(vc, e);
      }
    }
#pragma unroll
    for (int j = 0; j < kAttSub * 16 / kThreads; ++j) {
      const int i = tid + j * kThreads, p = i >> 4, f = i & 15;
      if (p < cn && c0 + p != pos) {
        Ks[p * 65 + 4 * f + 0] = kr[j].x;
        Ks[p * 65 + 4 * f + 1] = kr[j].y;
        Ks[p * 65 + 4 * f + 2] = kr[j].z;
        Ks[p * 65 + 4 * f + 3] = kr[j].w;
        reinterpret_cast<float4*>(Vs + p * 64)[f] = vr[j];
      }
    }
  };
  stage(t0, min(kAttSub, t1 - t0));
  // this thread's words of q (pair j, j + 32 of head tid / 32; hpg * 32 <= 256 threads)
  // and, in the split that holds pos, of the new v and k: all loaded, then settled together
  const int qh = tid >> 5, qj = tid & 31;
  const float c_r = cs[qj], s_r = sn[qj];   // this thread's RoPE pair, read before the wait
  uint64_t w[5];
  const uint64_t* pp[5];
  bool use[5];
  pp[0] = row + (g * hpg + (tid < hpg * 32 ? qh : 0)) * 64 + qj;
  pp[1] = pp[0] + 32;
  pp[2] = row + (H + Hk + g) * 64 + (tid & 63);
  pp[3] = row + (H + g) * 64 + qj;
  pp[4] = pp[3] + 32;
  use[0] = use[1] = tid < hpg * 32;
  use[2] = owner && tid < 64;
  use[3] = use[4] = owner && tid < 32;
#pragma unroll
  for (int k = 0; k < 5; ++k) w[k] = use[k] ? ld_stamp(pp[k]) : 0;
  // (a test may make this wait for an epoch that no phase writes)
  const bool ok = settle_words<5>(w, pp, use, a.test_stall == 1 ? (ep ^ 0x80000000u) : ep, a);
  if (use[0]) {
    const float x0 = __uint_as_float((unsigned)w[0]), x1 = __uint_as_float((unsigned)w[1]);
    qs[qh * 64 + qj] = (x0 * c_r - x1 * s_r) * 0.125f;
    qs[qh * 64 + qj + 32] = (x0 * s_r + x1 * c_r) * 0.125f;
  }
  if (use[2]) {
    // the new row: appended to the cache, and used by this step in the cache's precision
    const size_t e = head + (size_t)pos * 64;
    float v = __uint_as_float((unsigned)w[2]);
    if (h16) {
      v = __half2float(__float2half_rn(v));
      kv_store<1>(vc, e + tid, v);
    } else {
      kv_store<0>(vc, e + tid, v);
    }
    vnew[tid] = v;
    if (use[3]) {
      const float x0 = __uint_as_float((unsigned)w[3]), x1 = __uint_as_float((unsigned)w[4]);
      float k0 = x0 * c_r - x1 * s_r, k1 = x0 * s_r + x1 * c_r;   // tid < 32: qj == tid
      if (h16) {
        k0 = __half2float(__float2half_rn(k0));
        k1 = __half2float(__float2half_rn(k1));
        kv_store<1>(kc, e + tid, k0);
        kv_store<1>(kc, e + tid + 32, k1);
      } else {
        kv_store<0>(kc, e + tid, k0);
        kv_store<0>(kc, e + tid + 32, k1);
      }
      knew[tid] = k0;
      knew[tid + 32] = k1;
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
    for (int i = tid; i < hpg * kAttSub; i += kThreads) {
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
    for (int h = warp; h < hpg; h += kWarps) {
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
      const int idx = tid + k * kThreads;
      if (idx < hpg * 64) {
        const int h = idx >> 6, dd = idx & 63;
        float acc = oacc[k] * corr[h];
#pragma unroll 4
        for (int p = 0; p < cn; ++p) acc = fmaf(sc[h * kAttSub + p], Vs[p * 64 + dd], acc);
        oacc[k] = acc;
      }
    }
  }
  if (s_act == 1) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int idx = tid + k * kThreads;
      if (idx < hpg * 64) {
        const int h = idx >> 6, dd = idx & 63;
        st_stamp(a.o_s + ((size_t)b * H + g * hpg + h) * 64 + dd, oacc[k] * (1.0f / lh[h]), ep_out);
      }
    }
  } else {
    uint64_t* pb = a.part_s + (((size_t)b * Hk + g) * S + split) * hpg * 66;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int idx = tid + k * kThreads;
      if (idx < hpg * 64) st_stamp(pb + (idx >> 6) * 66 + 2 + (idx & 63), oacc[k], ep_out);
    }
    if (tid < hpg) {
      st_stamp(pb + tid * 66 + 0, mh[tid], ep_out);
      st_stamp(pb + tid * 66 + 1, lh[tid], ep_out);
    }
  }
  consumer_bar();  // scratch reuse
  return true;
}

// Merges head hl of (stream b, kv head g) from the s_act splits' stamped partials (epoch
// ep): o = sum_s w_s o_s / sum_s w_s l_s, w_s = exp(m_s - max m).  Every load is in flight
// before the first wait.  Returns false on a failed wait.
__device__ __forceinline__ bool merge_head(const PersistArgs& a, float* scratch, int b, int g, int hl, int S, int s_act,
                                        unsigned ep) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H = a.H, Hk = a.Hk, hpg = H / Hk;
  float* mw = scratch + kMrgMw;
  float* lw = scratch + kMrgLw;
  float* ov = scratch + kMrgOv;
  float* p4 = scratch + kMrgP4;
  float* lin = scratch + kMrgLin;
  const uint64_t* p0 = a.part_s + ((size_t)b * Hk + g) * S * hpg * 66;
  const int npairs = s_act * 33;
  bool ok = true;
#pragma unroll 1
  for (int base = 0; base < npairs; base += kThreads * kPairBatch) {
    uint64_t w0[kPairBatch], w1[kPairBatch];
    const uint64_t* pp[kPairBatch];
    bool use[kPairBatch];
#pragma unroll
    for (int j = 0; j < kPairBatch; ++j) {
      const int q = base + tid + j * kThreads;
      use[j] = q < npairs;
      const int qq = use[j] ? q : 0;
      const int s = qq / 33, e2 = qq - s * 33;
      pp[j] = p0 + ((size_t)s * hpg + hl) * 66 + 2 * e2;
      w0[j] = w1[j] = 0;
      if (use[j]) ld_stamp2(pp[j], w0[j], w1[j]);
    }
    if (ok) ok = settle_pairs<kPairBatch>(w0, w1, pp, use, ep, a);
#pragma unroll
    for (int j = 0; j < kPairBatch; ++j) {
      const int q = base + tid + j * kThreads;
      if (use[j]) {
        const int s = q / 33, e2 = q - s * 33;
        const float v0 = __uint_as_float((unsigned)w0[j]), v1 = __uint_as_float((unsigned)w1[j]);
        if (e2 == 0) {
          mw[s] = v0;
          lw[s] = v1;
        } else {
          ov[s * 64 + 2 * e2 - 2] = v0;
          ov[s * 64 + 2 * e2 - 1] = v1;
        }
      }
    }
  }
  if (consumer_bar_or(!ok)) return false;
  if (warp == 0) {
    float mx = -INFINITY;
    for (int s = lane; s < s_act; s += 32) mx = fmaxf(mx, mw[s]);
    mx = warp_max(mx);
    float l = 0.f;
    for (int s = lane; s < s_act; s += 32) {
      const float w = ex(mw[s] - mx);
      mw[s] = w;
      l = fmaf(w, lw[s], l);
    }
    l = warp_sum(l);
    if (lane == 0) *lin = 1.0f / l;
  }
  consumer_bar();
  {
    const int dd = tid & 63, qq = tid >> 6;
    float acc = 0.f;
    for (int s = qq; s < s_act; s += 4) acc = fmaf(mw[s], ov[s * 64 + dd], acc);
    p4[qq * 64 + dd] = acc;
  }
  consumer_bar();
  if (tid < 64) {
    const float O = (p4[tid] + p4[64 + tid]) + (p4[128 + tid] + p4[192 + tid]);
    st_stamp(a.o_s + ((size_t)b * H + g * hpg + hl) * 64 + tid, O * *lin, ep);
  }
  consumer_bar();  // scratch reuse
  return true;
}

__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

}  // namespace

// The CTA's share of each stage: sched[s] .. sched[5 + s] = records of matrix s < 4 (units
// sched[10 + s] .. sched[14 + s] of an sched[18 + s]-part split), LM head rows for s = 4.
template <int M, int FMT>
__device__ __forceinline__ bool decode_steps(const PersistArgs& a, Ring& ring, const Smem& sm, const PLayer* layers,
                                             const int* sched);

__device__ __forceinline__ int mat_KG(const PersistArgs& a, int s) { return mat_K(a, s) / 32; }

template <int M, int FMT>
__global__ void __launch_bounds__(kThreads, 1) decode_persistent_kernel(const __grid_constant__ PersistArgs a) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const Smem sm = carve(smem, a.nslot, a.sched_cap);
  __shared__ PLayer layers_s[kMaxLayers];
  __shared__ int sched_s[22];
  const int kmax = max(max(a.d, a.H * 64), a.F);
  if (threadIdx.x == 0) {
    for (int i = 0; i < a.nslot; ++i) {
      mbar_init(&sm.full[i], 1);
      sm.cnt[i] = 0u;
      sm.niss[i] = 0u;
    }
    mbar_fence_init();
    const int c = blockIdx.x, G = gridDim.x;
    for (int s = 0; s < 4; ++s) {
      const int nt = mat_N(a, s) / kTile, KG = mat_KG(a, s);
      // QKV stays whole per tile: the attention reads q, k and v as one slice
      const int S = s == 0 ? 1 : choose_split(nt, KG, G);
      const int U = nt * S, u0 = U * c / G, u1 = U * (c + 1) / G;
      sched_s[s] = unit_rec(u0, S, KG);
      sched_s[5 + s] = unit_rec(u1, S, KG);
      sched_s[10 + s] = u0;
      sched_s[14 + s] = u1;
      sched_s[18 + s] = S;
    }
    sched_s[4] = a.V * c / G;
    sched_s[9] = a.V * (c + 1) / G;
  }
  for (int i = threadIdx.x; i < a.L * (int)(sizeof(PLayer) / 8); i += kThreads)
    reinterpret_cast<uint64_t*>(layers_s)[i] = reinterpret_cast<const uint64_t*>(a.layers)[i];
  // the zero row (B columns of streams that do not exist); never written again
  {
    uint32_t* z = reinterpret_cast<uint32_t*>(sm.region + persist_main(M, a.d, a.H, a.F));
    for (int i = threadIdx.x; i < kmax / 2 + 16; i += kThreads) z[i] = 0u;
  }
  __syncthreads();
  // the slice table of one step (the same every step)
  if (threadIdx.x == 0) {
    const int rb = a.fmt == kInt4 ? kRecInt4 : kRecF16;
    const int per = kSlot / rb, rpp = kSlot / (a.d * 4);
    int E = 0;
    bool fits = true;
    for (int l = 0; l < a.L; ++l)
      for (int s = 0; s < 4; ++s)
        for (int p = sched_s[s]; p < sched_s[5 + s]; p += per) {
          if (E < a.sched_cap)
            sm.tab[E] = Slice{layers_s[l].w[s] + (size_t)p * rb, (uint32_t)(min(per, sched_s[5 + s] - p) * rb), 0u};
          else fits = false;
          ++E;
        }
    for (int p = sched_s[4]; p < sched_s[9]; p += rpp) {
      if (E < a.sched_cap)
        sm.tab[E] = Slice{reinterpret_cast<const unsigned char*>(a.lm_head) + (size_t)p * a.d * 4,
                          (uint32_t)(min(rpp, sched_s[9] - p) * a.d * 4), 0u};
      else fits = false;
      ++E;
    }
    if (!fits || E == 0) {
      flag_error(a.status, kErrShapeBit);
      atomicExch(a.abort, 1u);
      E = 0;
    }
    *sm.ntab = E;
  }
  __syncthreads();
  Ring ring;
  ring.a = &a;
  ring.sm = sm;
  ring.E = *sm.ntab;
  if (ring.E == 0) return;
  ring.total = (long long)a.n_steps * ring.E;
  ring.start();
  if (!decode_steps<M, FMT>(a, ring, sm, layers_s, sched_s)) ring.drain();
}

template <int M, int FMT>
__device__ __forceinline__ bool decode_steps(const PersistArgs& a, Ring& ring, const Smem& sm, const PLayer* layers,
                                             const int* sched) {
  __shared__ int ok_s;
  __shared__ unsigned ticket_s;
  __shared__ float bval[8][8];
  __shared__ int bidx[8][8];
  __shared__ int tok_s[8];
  __shared__ float inv_s[8];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x, G = gridDim.x;
  const int d = a.d, H = a.H, Hk = a.Hk, F = a.F, V = a.V, B = M;
  const int hpg = H / Hk;
  const int nq = (H + 2 * Hk) * 64;
  const int kmax = max(max(d, H * 64), F);
  Region rg;
  rg.planes = reinterpret_cast<uint32_t*>(sm.region);
  rg.xin = reinterpret_cast<float2*>(sm.region + plane_bytes(M, kmax));
  rg.gb = reinterpret_cast<float4*>(sm.region + plane_bytes(M, kmax) + xin_bytes(kmax));
  rg.part = reinterpret_cast<float*>(sm.region + plane_bytes(M, kmax) + xin_bytes(kmax) + gb_bytes(d));
  rg.zero = reinterpret_cast<const uint32_t*>(sm.region + persist_main(M, d, H, F));
  // the CTA's copy of the residual rows (each thread's own pairs), [M][d / 2] pairs
  float2* xres = reinterpret_cast<float2*>(sm.region + persist_main(M, d, H, F) + align16((size_t)kmax * 2 + 64));
  float* scratch = reinterpret_cast<float*>(sm.region);
  Red red{sm.red, 0};
  unsigned epoch = 0;
  const int len0 = *a.dlen;
  const int units = B * Hk;
  int S = G / units;
  if (S < 1) S = 1;
  if (S > a.att_splits) S = a.att_splits;
  const unsigned per_step = 5u * a.L;

  // The phase input: row m of a vector into A planes rows 2m, 2m + 1.  st: the S slices of
  // the vector (stride between slices, ld between rows) or null for the token embedding;
  // res: add and update the residual copy; gelu: GELU of the sum.
  auto load_planes = [&](const uint64_t* st, long long stride, int S, int ld, int K, int p0, int p1, unsigned ep,
                         const float* g, const float* bt, bool res, bool gelu) -> bool {
    bool ok = true;
    const int pw = (K >> 1) + 16;
#pragma unroll 1
    for (int m = 0; m < M; ++m) {
      const VecSrc src{st ? st + (size_t)m * ld : nullptr, stride, st ? nullptr : a.tok_emb + (size_t)tok_s[m] * d, ep,
                       res ? xres + (size_t)m * (d / 2) : nullptr, gelu};
      uint32_t* phi = rg.planes + (2 * m) * pw;
      uint32_t* plo = rg.planes + (2 * m + 1) * pw;
      if (S == 1) ok = load_row<true, 1>(src, K, p0, p1, g, bt, a.eps, phi, plo, &inv_s[m], nullptr, rg, red, a) && ok;
      else if (S == 2) ok = load_row<true, 2>(src, K, p0, p1, g, bt, a.eps, phi, plo, &inv_s[m], nullptr, rg, red, a) && ok;
      else ok = load_row<true, 4>(src, K, p0, p1, g, bt, a.eps, phi, plo, &inv_s[m], nullptr, rg, red, a) && ok;
    }
    return !consumer_bar_or(!ok);
  };

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
    int s_act, chunk;
    att_split_count(T, S, s_act, chunk);
    for (int l = 0; l < a.L; ++l) {
      const PLayer& ly = layers[l];
      const size_t es = a.kv16 ? 2 : 4;
      void* kc = static_cast<char*>(a.kc) + (size_t)l * a.layer_stride * es;
      void* vc = static_cast<char*>(a.vc) + (size_t)l * a.layer_stride * es;
      const unsigned epA = ep0 + 5u * l;
      // phases A (LN1 + QKV), B (attention), C (O + residual), D (LN2 + FC1 + GELU),
      // E (FC2 + residual); one call site for the four matrix phases
#pragma unroll 1
      for (int ph = 0; ph < 5; ++ph) {
        if (ph == 1) {
          for (int u = c; u < units * S; u += G) {
            const int bg = u / S, split = u - bg * S;
            if (!attention_unit(a, scratch, bg / Hk, bg % Hk, split, S, s_act, chunk, T, pos, kc, vc, epA, epA + 1))
              return false;
          }
          if (s_act > 1)
            for (int u = c; u < units * S; u += G) {
              const int bg = u / S, split = u - bg * S;
              if (split < s_act)
                for (int hl = split; hl < hpg; hl += s_act)
                  if (!merge_head(a, scratch, bg / Hk, bg % Hk, hl, S, s_act, epA + 1)) return false;
            }
          continue;
        }
        const int mi = ph == 0 ? 0 : ph - 1;   // matrix of the phase
        const int K = mat_K(a, mi);
        // the input: the token embedding (layer 0), or the previous matrix's output slices;
        // A and D add them to the residual copy, E applies GELU to FC1's sum
        const bool emb = ph == 0 && l == 0;
        const int pm = ph == 0 ? 3 : ph == 2 ? -1 : ph == 3 ? 1 : 2;   // producing matrix (-1: attention)
        const uint64_t* src = emb ? nullptr : pm < 0 ? a.o_s : a.vs[pm];
        const long long stride = pm < 0 ? 0 : a.vstride[pm];
        const int S_in = (emb || pm < 0) ? 1 : sched[18 + pm];   // the embedding and o are single vectors
        const float* g = ph == 0 ? ly.ln1_g : ph == 3 ? ly.ln2_g : nullptr;
        const float* bt = ph == 0 ? ly.ln1_b : ph == 3 ? ly.ln2_b : nullptr;
        // GELU of FC1's output: applied by FC1's producers when its tiles are whole, else by
        // the consumers after adding the K-range parts
        const bool fc1_whole = sched[18 + 2] == 1;
        // O and FC2 (no LayerNorm on their input): load only the K range of this CTA's units
        // when they all lie in one part of a K-split matrix, nothing when it has none
        int p0 = 0, p1 = K >> 1;
        if (mi == 1 || mi == 3) {
          const int Sm = sched[18 + mi], u0 = sched[10 + mi], u1 = sched[14 + mi], KG = K >> 5;
          if (u1 <= u0) {
            p1 = 0;
          } else if (Sm > 1) {
            const int h0 = u0 % Sm, h1 = (u1 - 1) % Sm;
            if (u1 - u0 <= Sm && h0 <= h1) {
              p0 = (KG * h0 / Sm) * 16;
              p1 = (KG * (h1 + 1) / Sm) * 16;
            }
          }
        }
        if (!load_planes(src, stride, S_in, K, K, p0, p1, epA + ph - 1, g, bt, ph == 0 || ph == 3,
                         ph == 4 && !fc1_whole))
          return false;
        MvJob jb;
        jb.K = K;
        jb.N = mat_N(a, mi);
        jb.S = sched[18 + mi];
        jb.u0 = sched[10 + mi];
        jb.u1 = sched[14 + mi];
        jb.rbeg = sched[mi];
        jb.rend = sched[5 + mi];
        jb.out = a.vs[mi];
        jb.stride = a.vstride[mi];
        jb.ep = epA + ph;
        jb.gelu = mi == 2 && fc1_whole;
        if (!mv_phase<M, FMT>(ring, rg, jb, inv_s)) return false;
      }
    }
    // ---- LM head + argmax ------------------------------------------------------------
    float* act = reinterpret_cast<float*>(sm.region);
    {
      bool ok = true;
#pragma unroll 1
      for (int m = 0; m < M; ++m) {
        const VecSrc src{a.vs[3] + (size_t)m * d, a.vstride[3], nullptr, ep0 + per_step - 1, xres + (size_t)m * (d / 2),
                         false};
        const int S3 = sched[18 + 3];
        if (S3 == 1)
          ok = load_row<false, 1>(src, d, 0, d >> 1, a.lnf_g, a.lnf_b, a.eps, nullptr, nullptr, nullptr, act + (size_t)m * d, rg,
                                  red, a) && ok;
        else if (S3 == 2)
          ok = load_row<false, 2>(src, d, 0, d >> 1, a.lnf_g, a.lnf_b, a.eps, nullptr, nullptr, nullptr, act + (size_t)m * d, rg,
                                  red, a) && ok;
        else
          ok = load_row<false, 4>(src, d, 0, d >> 1, a.lnf_g, a.lnf_b, a.eps, nullptr, nullptr, nullptr, act + (size_t)m * d, rg,
                                  red, a) && ok;
      }
      if (consumer_bar_or(!ok)) return false;
    }
    const float4* act4 = reinterpret_cast<const float4*>(act);
    float best[M];
    int bi[M];
#pragma unroll
    for (int m = 0; m < M; ++m) {
      best[m] = -FLT_MAX;
      bi[m] = INT_MAX;
    }
    bool lm_ok = true;
    {
      const int rb = d * 4, rpp = kSlot / rb;
      for (int p = sched[4]; p < sched[9]; p += rpp) {
        const int rows = min(rpp, sched[9] - p);
        const unsigned char* buf = ring.acquire();
        lm_ok = lm_ok && ring.got;
        for (int r = warp; ring.got && r < rows; r += kWarps) {
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
          float sv[M];
#pragma unroll
          for (int m = 0; m < M; ++m) {
            sv[m] = warp_sum(acc[m]);
            if (lane == 0 && a.logits) a.logits[(size_t)m * V + v] = sv[m];
          }
#pragma unroll
          for (int m = 0; m < M; ++m) {
            // classifier-free guidance: both streams of a pair choose by u + scale (k - u)
            float gv = sv[m];
            if (M >= 2 && a.guidance != 0.f) {
              const int c2 = m & ~1;
              gv = sv[c2 + 1] + a.guidance * (sv[c2] - sv[c2 + 1]);
            }
            if (better(gv, v, best[m], bi[m])) {
              best[m] = gv;
              bi[m] = v;
            }
          }
        }
        ring.release();
      }
    }
    if (lane == 0)
      for (int m = 0; m < M; ++m) {
        bval[warp][m] = best[m];
        bidx[warp][m] = bi[m];
      }
    if (consumer_bar_or(!lm_ok)) return false;
    if (tid < M) {
      float bv = -FLT_MAX;
      int bx = INT_MAX;
      for (int w = 0; w < kWarps; ++w)
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
        for (int k = tid; k < G; k += kThreads) {
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
        for (int w = 0; w < kWarps; ++w)
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
int persistent_sched_cap(int L, int d, int H, int Hk, int F, int V, int G, int fmt) {
  const int rb = fmt == kInt4 ? kRecInt4 : kRecF16;
  const int per = kSlot / rb;
  const int Ns[4] = {(H + 2 * Hk) * 64, d, F, d};
  const int Ks[4] = {d, H * 64, d, F};
  long long per_layer = 0;
  for (int s = 0; s < 4; ++s) {
    const int nt = Ns[s] / kTile, KG = Ks[s] / 32;
    const int S = s == 0 ? 1 : choose_split(nt, KG, G);
    const long long umax = ((long long)nt * S + G - 1) / G;
    per_layer += (umax * (KG / S) + per - 1) / per;
  }
  const long long rows = (V + G - 1) / G, rpp = kSlot / (d * 4);
  const long long cap = (long long)L * per_layer + (rows + rpp - 1) / rpp;
  return cap > (1 << 20) ? (1 << 20) : (int)cap;
}

static size_t region_bytes(int M, int d, int H, int F) {
  const int kmax = max(max(d, H * 64), F);
  // + the zero row + the residual copy
  return persist_main(M, d, H, F) + align16((size_t)kmax * 2 + 64) + align16((size_t)M * d * 4);
}

int persistent_slots(int M, int L, int d, int H, int Hk, int F, int V, int G, int fmt, size_t smem_optin) {
  const size_t fixed = 1024 + tab_bytes(persistent_sched_cap(L, d, H, Hk, F, V, G, fmt)) + region_bytes(M, d, H, F);
  if (smem_optin < fixed + 4 * (size_t)kSlot) return 0;
  size_t n = (smem_optin - fixed) / kSlot;
  if (n > 16) n = 16;
  return (int)n;
}

size_t persistent_smem(int M, int L, int d, int H, int Hk, int F, int V, int G, int fmt, int nslot) {
  return 1024 + tab_bytes(persistent_sched_cap(L, d, H, Hk, F, V, G, fmt)) + (size_t)nslot * kSlot +
         region_bytes(M, d, H, F);
}

bool persistent_shapes_ok(int M, int d, int H, int Hk, int F, int V, int G, const char** why) {
  auto no = [&](const char* m) {
    if (why) *why = m;
    return false;
  };
  if (M != 1 && M != 2 && M != 4 && M != 8) return no("batch must be 1, 2, 4 or 8");
  if (G < 1) return no("no CTAs");
  const int Ns[4] = {(H + 2 * Hk) * 64, d, F, d};
  const int Ks[4] = {d, H * 64, d, F};
  for (int s = 0; s < 4; ++s) {
    const int nt = Ns[s] / kTile, KG = Ks[s] / 32;
    const int S = s == 0 ? 1 : choose_split(nt, KG, G);
    if (Ns[s] % kTile != 0 || Ks[s] % 32 != 0 || ((long long)nt * S + G - 1) / G > kMaxUnits)
      return no("a matrix needs more than 4 work units per CTA");
  }
  if (d % 64 != 0 || F % 64 != 0) return no("d_model and d_ff must be multiples of 64");
  if (d > 2 * kThreads * kPairBatch) return no("d_model above 4096");
  if ((size_t)d * 4 > (size_t)kSlot) return no("an LM head row does not fit a ring slot");
  if (H % Hk != 0 || H / Hk > 8) return no("more than 8 query heads per kv head");
  if (V < 1) return no("empty vocabulary");
  return true;
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
