// Causal prefill attention on the 5th-generation tensor cores ("MuScriptor Medium — optimized
// W4A32 ONNX Runtime", Model variant: GroupQueryAttention over the shared fixed-capacity cache;
// "MuScriptor small — ONNX conversion", muscriptor-small-lm.onnx: new rows attend to every
// cached position and to the earlier new rows).
//
// For the n new rows of each stream at positions len .. len + n - 1 and every query head h of
// kv group g:  o_h[i] = sum_{j <= len + i} softmax_j(q_h[i] . k_g[j] / 8) v_g[j].
//
// One CTA per (128-row tile, kv group, stream).  A tile stacks the hpg = H / Hk query heads of
// the group: row r = hh * prows + p is head g * hpg + hh at new row i0 + p (prows = 128 / hpg
// rounded down), so every key tile staged in shared memory serves all of the group's heads.
// Per key tile of 64 positions (the next tile's K and V loads in flight meanwhile):
//   S = Q K^T on the tensor cores (M = 128 rows, N = 64 keys, K = 64) into TMEM;
//   online softmax on the CUDA cores: the two threads of a row (warps w and w + 4 read the same
//   TMEM lane quarter) each read their 32 scores, exchange their maxima through shared memory,
//   exponentiate their 32 and write them as the A operand of the next product;
//   O_tile = P V (M = 128, N = 64 head dims, K = 64 keys) into TMEM, with V read as an MN-major
//   operand straight from its row-per-key tile; each thread adds its 32 columns into registers
//   after scaling them by the softmax correction.
// Precision: every fp32 operand enters as an fp16 pair hi + lo (22-bit significand) and each
// product is three MMAs (hi*hi + hi*lo + lo*hi) with fp32 accumulation.  Q, K and V are scaled
// by 8 and P by 2^14 before the split (exact powers of two, undone on the fp32 results) so that
// small values keep their lo halves out of the fp16 subnormal range; a |value| that would not
// fit an fp16 after scaling flags the status word.
// Waits are bounded; a wait that runs out flags the status word and the CTA leaves the loop,
// waits (bounded) for the MMAs it issued and frees its TMEM.
#include "ms_device.cuh"
#include "ms_kernels.h"
#include "ms_launch.cuh"
#include "ms_tc.cuh"

namespace ms {

namespace {

constexpr int kAtRows = 128;    // query rows per CTA (MMA M)
constexpr int kAtKeys = 64;     // keys per tile
constexpr int kAtThreads = 256;
constexpr int kAtQh = 0, kAtQl = 16384;          // [128 rows][64] K-major, 128-byte swizzle
constexpr int kAtKh = 32768, kAtKl = 40960;      // [64 keys][64] K-major
constexpr int kAtVh = 49152, kAtVl = 57344;      // [64 keys][64 dims]: MN-major B of P V
constexpr int kAtPh = 65536, kAtPl = 81920;      // [128 rows][64 keys] K-major
constexpr size_t kAtSmem = 98304 + 1024;         // + alignment slack
constexpr float kAtPScale = 16384.f;             // P * 2^14
constexpr float kAtIn = 8.f;                     // Q, K, V * 8

struct AttnTcArgs {
  const float* q;        // [B * n][H * 64], post-RoPE
  const void* kc;        // layer slices [B][Hk][cap][64], fp32 or half
  const void* vc;
  int B, n, H, Hk, cap, hpg, prows;
  const int* dlen;       // cache length before these rows
  float* o;              // [B * n][H * 64] or null
  __half* oh;            // fp16 hi / lo planes [B * n][ldo] or null
  __half* ol;
  int ldo;
  unsigned* status;
};

// 4 consecutive fp32 values (times s) into the hi and lo tiles at row r, elements 4f .. 4f+3.
__device__ __forceinline__ bool put4(unsigned char* hi_tile, unsigned char* lo_tile, int r, int f, float4 v, float s) {
  v.x *= s, v.y *= s, v.z *= s, v.w *= s;
  const bool big = fabsf(v.x) >= 65504.f || fabsf(v.y) >= 65504.f || fabsf(v.z) >= 65504.f || fabsf(v.w) >= 65504.f;
  uint32_t h0, l0, h1, l1;
  split_h2(v.x, v.y, h0, l0);
  split_h2(v.z, v.w, h1, l1);
  const uint32_t off = sw128(r, f >> 1) + (uint32_t)(f & 1) * 8;
  *reinterpret_cast<uint2*>(hi_tile + off) = make_uint2(h0, h1);
  *reinterpret_cast<uint2*>(lo_tile + off) = make_uint2(l0, l1);
  return big;
}

}  // namespace

template <int KV>
__global__ void __launch_bounds__(kAtThreads, 2) attn_prefill_tc_kernel(const AttnTcArgs a) {
  extern __shared__ __align__(1024) unsigned char dsm[];
  __shared__ uint64_t bar_s, bar_o, bar_end;
  __shared__ uint32_t tmem_base_s;
  __shared__ float red[2][kAtRows], red_m[2][kAtRows];
  unsigned char* base = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(dsm) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x, g = blockIdx.y, b = blockIdx.z;

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_s)),
                 "r"(128)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    mbar_init(&bar_s, 1);
    mbar_init(&bar_o, 1);
    mbar_init(&bar_end, 1);
    mbar_fence_init();
  }
  pdl_wait();
  pdl_trigger();
  const int pos0 = *a.dlen;
  const int i0 = tile * a.prows;
  const int pvalid = min(a.prows, a.n - i0);
  const int rows = a.hpg * a.prows;
  const int kend = pos0 + i0 + pvalid;                        // keys [0, kend) are needed
  const size_t head = ((size_t)b * a.Hk + g) * a.cap * 64;   // first element of the group's cache rows
  bool big = false;

  // Q tile (scaled by 8; the score scale 1/8 and the 8 of K are applied to S)
  for (int idx = tid; idx < kAtRows * 16; idx += kAtThreads) {
    const int r = idx >> 4, f = idx & 15;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < rows) {
      const int hh = r / a.prows, p = r - hh * a.prows;
      if (p < pvalid)
        v = __ldg(reinterpret_cast<const float4*>(a.q + ((size_t)b * a.n + i0 + p) * a.H * 64 +
                                                  (size_t)(g * a.hpg + hh) * 64) + f);
    }
    big |= put4(base + kAtQh, base + kAtQl, r, f, v, kAtIn);
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tm = tmem_base_s;
  const uint32_t tS = tm, tO = tm + 64;

  // this thread's row and half of the columns
  const int q4 = warp & 3, half = warp >> 2;
  const int r = q4 * 32 + lane;
  int qpos = -1;
  if (r < rows) {
    const int hh = r / a.prows, p = r - hh * a.prows;
    if (p < pvalid) qpos = pos0 + i0 + p;
  }
  const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
  float m_i = -INFINITY, l_i = 0.f;
  float acc[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) acc[j] = 0.f;
  const uint32_t sb = smem_u32(base);
  const int nkt = (kend + kAtKeys - 1) / kAtKeys;
  bool ok = true;

  // K and V of a key tile travel in registers: each thread holds 4 float4 of K and of V
  // (key = (tid + 256 i) / 16, elements 4 f .. 4 f + 3 with f = (tid + 256 i) % 16); the next
  // tile's loads are issued right after the current one is staged, so they are in flight
  // during the current tile's products and softmax.
  float4 pk[4], pv[4];
  auto load_kv = [&](int c0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int idx = tid + kAtThreads * i, key = idx >> 4, f = idx & 15;
      pk[i] = pv[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c0 + key < kend) {
        pk[i] = kv_load4<KV>(a.kc, head + (size_t)(c0 + key) * 64 + 4 * f);
        pv[i] = kv_load4<KV>(a.vc, head + (size_t)(c0 + key) * 64 + 4 * f);
      }
    }
  };
  load_kv(0);

  for (int kt = 0; kt < nkt; ++kt) {
    const int c0 = kt * kAtKeys;
    if (__syncthreads_or(!ok)) break;   // also: the previous tile's P V has been read by every thread
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int idx = tid + kAtThreads * i, key = idx >> 4, f = idx & 15;
      big |= put4(base + kAtKh, base + kAtKl, key, f, pk[i], kAtIn);
      big |= put4(base + kAtVh, base + kAtVl, key, f, pv[i], kAtIn);
    }
    if (kt + 1 < nkt) load_kv(c0 + kAtKeys);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (tid == 0) {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t id = idesc_f16_mn(kAtRows, kAtKeys, false);
      const uint64_t qh = desc_sw128(sb + kAtQh), ql = desc_sw128(sb + kAtQl);
      const uint64_t kh = desc_sw128(sb + kAtKh), kl = desc_sw128(sb + kAtKl);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t adv = (uint64_t)kk * 2;   // 16 halves = 32 bytes along the row
        mma_f16(tS, qh + adv, kh + adv, id, kk > 0 ? 1u : 0u);
        mma_f16(tS, qh + adv, kl + adv, id, 1u);
        mma_f16(tS, ql + adv, kh + adv, id, 1u);
      }
      mma_commit(&bar_s);
    }
    // a wait that runs out clears ok; the thread still takes every barrier of the iteration
    ok = mbar_wait(&bar_s, (uint32_t)(kt & 1), a.status) && ok;
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    // this thread's half of the row's scores; the row maximum through the partner thread
    uint32_t s_own[32];
    tmem_ld32(tS + lane_base + (uint32_t)(half * 32), s_own);
    tmem_ld_wait();
    const float sc = 1.f / 512.f;   // (8 q) . (8 k) / 64 / 8
    const int cb = c0 + half * 32;
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (cb + j <= qpos) mx = fmaxf(mx, __uint_as_float(s_own[j]) * sc);
    red_m[half][r] = mx;
    __syncthreads();
    const float m_new = fmaxf(m_i, fmaxf(red_m[0][r], red_m[1][r]));
    const float alpha = m_new == -INFINITY ? 1.f : expf(m_i - m_new);
    m_i = m_new;
    float psum = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {   // chunk c: keys cb + 8c .. cb + 8c + 7
      uint32_t ph[4], pl[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = 8 * c + 2 * e;
        const float p0 = cb + j <= qpos ? expf(__uint_as_float(s_own[j]) * sc - m_new) : 0.f;
        const float p1 = cb + j + 1 <= qpos ? expf(__uint_as_float(s_own[j + 1]) * sc - m_new) : 0.f;
        psum += p0 + p1;
        split_h2(p0 * kAtPScale, p1 * kAtPScale, ph[e], pl[e]);
      }
      const uint32_t off = sw128(r, half * 4 + c);
      *reinterpret_cast<uint4*>(base + kAtPh + off) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
      *reinterpret_cast<uint4*>(base + kAtPl + off) = make_uint4(pl[0], pl[1], pl[2], pl[3]);
    }
    red[half][r] = psum;
#pragma unroll
    for (int j = 0; j < 32; ++j) acc[j] *= alpha;
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (tid == 0) {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t id = idesc_f16_mn(kAtRows, 64, true);
      const uint64_t ph_d = desc_sw128(sb + kAtPh), pl_d = desc_sw128(sb + kAtPl);
      const uint64_t vh = desc_sw128(sb + kAtVh), vl = desc_sw128(sb + kAtVl);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t adv_a = (uint64_t)kk * 2;           // 16 keys along the P row
        const uint64_t adv_b = (uint64_t)kk * (2048 >> 4); // 16 key rows of V
        mma_f16(tO, ph_d + adv_a, vh + adv_b, id, kk > 0 ? 1u : 0u);
        mma_f16(tO, ph_d + adv_a, vl + adv_b, id, 1u);
        mma_f16(tO, pl_d + adv_a, vh + adv_b, id, 1u);
      }
      mma_commit(&bar_o);
    }
    l_i = l_i * alpha + red[0][r] + red[1][r];
    ok = mbar_wait(&bar_o, (uint32_t)(kt & 1), a.status) && ok;
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    uint32_t ov[32];
    tmem_ld32(tO + lane_base + half * 32, ov);
    tmem_ld_wait();
#pragma unroll
    for (int j = 0; j < 32; ++j) acc[j] += __uint_as_float(ov[j]);
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  }

  if (__syncthreads_or(!ok || big)) {
    if (tid == 0) flag_error(a.status, !ok ? kErrTimeout : kErrShape);
  }
  if (ok && qpos >= 0) {
    const int hh = r / a.prows, p = r - hh * a.prows;
    const size_t row = (size_t)b * a.n + i0 + p;
    const int col = (g * a.hpg + hh) * 64 + half * 32;
    const float inv = 1.f / (l_i * (kAtPScale * kAtIn));
    if (a.o) {
      float4* dst = reinterpret_cast<float4*>(a.o + row * a.H * 64 + col);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        dst[j] = make_float4(acc[4 * j] * inv, acc[4 * j + 1] * inv, acc[4 * j + 2] * inv, acc[4 * j + 3] * inv);
    }
    if (a.oh) {
      uint32_t hv[16], lv[16];
#pragma unroll
      for (int j = 0; j < 32; j += 2) split_h2(acc[j] * inv, acc[j + 1] * inv, hv[j >> 1], lv[j >> 1]);
      uint4* dh = reinterpret_cast<uint4*>(a.oh + row * a.ldo + col);
      uint4* dl = reinterpret_cast<uint4*>(a.ol + row * a.ldo + col);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        dh[c] = make_uint4(hv[4 * c], hv[4 * c + 1], hv[4 * c + 2], hv[4 * c + 3]);
        dl[c] = make_uint4(lv[4 * c], lv[4 * c + 1], lv[4 * c + 2], lv[4 * c + 3]);
      }
    }
  }
  // every MMA this CTA issued has completed before its TMEM is freed
  if (tid == 0) mma_commit(&bar_end);
  for (long long it = 0; it < kSpinLimit; ++it)
    if (mbar_try_wait(&bar_end, 0u)) break;
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tm), "r"(128) : "memory");
}

cudaError_t init_attrs_attn_tc() {
  cudaError_t e = allow_smem(attn_prefill_tc_kernel<0>, kAtSmem);
  if (e == cudaSuccess) e = allow_smem(attn_prefill_tc_kernel<1>, kAtSmem);
  return e;
}

bool attn_prefill_tc_fits(int H, int Hk) { return Hk > 0 && H % Hk == 0 && H / Hk <= kAtRows; }

cudaError_t launch_attn_prefill_tc(const Launch& L, const float* q, const void* kc, const void* vc, int B, int n,
                                   int H, int Hk, int cap, const int* dlen, float* o, __half* oh, __half* ol, int ldo,
                                   int kv16) {
  if (n <= 0 || B <= 0) return cudaSuccess;
  if (!attn_prefill_tc_fits(H, Hk) || (oh && (ldo % 8 != 0 || !ol)) || (!o && !oh)) return cudaErrorInvalidValue;
  AttnTcArgs a;
  a.q = q;
  a.kc = kc;
  a.vc = vc;
  a.B = B;
  a.n = n;
  a.H = H;
  a.Hk = Hk;
  a.cap = cap;
  a.hpg = H / Hk;
  a.prows = kAtRows / a.hpg;
  a.dlen = dlen;
  a.o = o;
  a.oh = oh;
  a.ol = ol;
  a.ldo = ldo;
  a.status = L.status;
  const dim3 grid((n + a.prows - 1) / a.prows, Hk, B);
  if (kv16) return launch_k(L, attn_prefill_tc_kernel<1>, grid, dim3(kAtThreads), kAtSmem, a);
  return launch_k(L, attn_prefill_tc_kernel<0>, grid, dim3(kAtThreads), kAtSmem, a);
}

}  // namespace ms
