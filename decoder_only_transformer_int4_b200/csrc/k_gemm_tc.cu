// Dequant-GEMM on the 5th-generation tensor cores (tcgen05, accumulator in TMEM):
// y[m][n] (+)= sum_k x[m][k] W[n][k] for prefill and batched decode, where the MatMul is a
// real dense contraction ("MuScriptor Medium — optimized W4A32 ONNX Runtime", Model
// variant: MatMulNBits with INT4 g32 weights; the fp16-weight variant of "MuScriptor for
// Core AI (.aimodel)", file table).
//
// Shape of the work: swap-AB.  The weight rows are the MMA's M = 128 side (operand A), the
// activation rows (tokens or streams) its N side (operand B, 16..128 per tile), so a batch
// of 16 or 64 streams fills whole MMA tiles and prefill tiles tokens the same way.  One CTA
// computes a 128 x BN tile of y^T in TMEM.
//
// Precision: the activations and the model are fp32.  Each fp32 operand is split into a
// tf32 "big" part (low 13 mantissa bits cleared) and the exact remainder "small", and the
// three products big*big + big*small + small*big are accumulated in fp32 (the 3xTF32
// method); the dropped small*small term and the tensor core's truncation of "small" leave
// an error of about 2^-21 relative per product.  The weight value is the fp32 product q*s
// (INT4) or the half value (fp16).
//
// Pipeline per 32-wide K block (one quantisation group): cp.async stages the raw block
// (nibbles and scale of 128 weight rows, BN activation rows) three blocks ahead; 256 threads
// dequantise and split it into the four operand tiles in the canonical K-major
// 128-byte-swizzled layout; a proxy fence and a CTA barrier hand them to the elected thread,
// which issues 3 x 4 tcgen05.mma (K = 8 each) and commits them to the stage's mbarrier.  Three
// operand stages (two for 16-wide tiles): the conversion of block k+1 overlaps the MMAs of
// blocks k and k-1.  Every wait is
// bounded; TMEM is freed on every path.
//
// Split-K: when the output tiles are too few to fill the GPU (batched decode: 8 to 32 tiles of
// 128 weight rows), the S <= 8 CTAs of a tile form a thread-block cluster (1, 1, S), each over
// a contiguous run of K blocks.  Each leaves its fp32 partial tile in its own shared memory;
// after a cluster barrier every CTA adds, for its 1/S of the tile, the S partials in rank
// order by reading its peers' shared memory (distributed shared memory), and applies the
// epilogue; a second cluster barrier keeps each CTA's shared memory alive until its peers
// are done reading it.  Every CTA of the cluster passes both barriers on every path.
#include "ms_device.cuh"
#include "ms_launch.cuh"

namespace ms {

namespace {

constexpr int TM = 128;      // weight rows per tile (MMA M)
constexpr int TK = 32;       // K per block (one quantisation group, one 128-byte row of fp32)
constexpr int kTileBytes = TM * TK * 4;  // 16 KiB per 128-row operand tile

struct TcArgs {
  const uint8_t* wq;
  const float* ws;
  const uint16_t* wh;
  int N, K, ldq, lds;
  const float* x;
  int ldx, M;
  float* y;
  int ldy;
  unsigned* status;
  int splits;          // CTAs per output tile along K (gridDim.z = the cluster's size)
};

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ float ld_peer(uint32_t local_saddr, uint32_t rank) {
  uint32_t ra;
  float v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(local_saddr), "r"(rank));
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(ra) : "memory");
  return v;
}

__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
  // K-major, 128-byte swizzle: rows of 128 bytes, 8-row atoms 1024 bytes apart (SBO),
  // LBO unused (1), descriptor version 1, layout type 2 (SWIZZLE_128B).
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor, kind::tf32: D fp32, A and B tf32, both K-major, M = 128, N = bn.
__device__ __forceinline__ uint32_t idesc_tf32(int bn) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(bn >> 3) << 17) | ((uint32_t)(TM >> 4) << 24);
}

__device__ __forceinline__ void mma_tf32(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n}" ::"r"(
          tmem_d),
      "l"(da), "l"(db), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Byte offset of float4 chunk j (K elements 4j..4j+3) of row r in a K-major SW128 tile.
__device__ __forceinline__ uint32_t sw128_off(int r, int j) {
  return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((j ^ (r & 7)) << 4));
}

__device__ __forceinline__ void split4(const float4 v, float4& big, float4& small) {
  big.x = __uint_as_float(__float_as_uint(v.x) & 0xFFFFE000u);
  big.y = __uint_as_float(__float_as_uint(v.y) & 0xFFFFE000u);
  big.z = __uint_as_float(__float_as_uint(v.z) & 0xFFFFE000u);
  big.w = __uint_as_float(__float_as_uint(v.w) & 0xFFFFE000u);
  small.x = v.x - big.x;
  small.y = v.y - big.y;
  small.z = v.z - big.z;
  small.w = v.w - big.w;
}

}  // namespace

// Raw blocks are staged by cp.async kStages - 1 blocks ahead of use (weights: 16 nibble
// bytes and one scale per row, or 64 half bytes; activations: 128 bytes per row); 256
// threads then convert a staged block into the MMA operand tiles.
constexpr int kStages = 4;
// Operand stages: block k's conversion waits for the MMAs of block k - NS.  Three for wide
// tiles; two for BN = 16, whose smaller CTAs then fit two to an SM.
template <int BN>
constexpr int op_stages() { return BN >= 32 ? 3 : 2; }

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(valid ? 4 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <int BN, int FMT>
struct TcLayout {
  static constexpr int kBBytes = BN * TK * 4;                      // one activation operand tile
  static constexpr int kOpStage = 2 * kTileBytes + 2 * kBBytes;    // A big/small + B big/small
  static constexpr int kRawW = FMT == kInt4 ? TM * 16 : TM * 64;   // staged weight bytes per block
  static constexpr int kRawS = FMT == kInt4 ? TM * 4 : 0;          // staged scales
  static constexpr int kRawX = BN * TK * 4;                        // staged activations
  static constexpr int kRawStage = kRawW + kRawS + kRawX;
  static constexpr size_t kBytes = 1024 + op_stages<BN>() * (size_t)kOpStage + (size_t)kStages * kRawStage;
};

template <int BN, int FMT>
__device__ __forceinline__ void stage_block(const TcArgs& a, unsigned char* raw, int n0, int m0, int kb) {
  using LY = TcLayout<BN, FMT>;
  const int tid = threadIdx.x;
  const int k0 = kb * TK;
  if (FMT == kInt4) {
    if (tid < TM) {
      const int n = n0 + tid;
      const bool v = n < a.N;
      const size_t row = (size_t)(v ? n : 0) * a.ldq;
      cp_async16(raw + tid * 16, a.wq + row + k0 / 2, v);
      cp_async4(raw + LY::kRawW + tid * 4, a.ws + (size_t)(v ? n : 0) * a.lds + k0 / 32, v);
    }
  } else {
    for (int i = tid; i < TM * 4; i += 256) {
      const int r = i >> 2, j = i & 3;
      const int n = n0 + r;
      const bool v = n < a.N;
      cp_async16(raw + r * 64 + j * 16, a.wh + (size_t)(v ? n : 0) * a.K + k0 + j * 8, v);
    }
  }
  unsigned char* rx = raw + LY::kRawW + LY::kRawS;
  for (int i = tid; i < BN * 8; i += 256) {
    const int r = i >> 3, j = i & 7;
    const int m = m0 + r;
    const bool v = m < a.M;
    cp_async16(rx + r * 128 + j * 16, a.x + (size_t)(v ? m : 0) * a.ldx + k0 + 4 * j, v);
  }
}

// Stage layout (dynamic shared memory, 1024-byte aligned): kOpStages operand stages (A_big,
// A_small for 128 weight rows, B_big, B_small for BN activation rows), then kStages raw
// staging slots.
template <int BN, int FMT, int EPI>
__global__ void __launch_bounds__(256, 1) gemm_tc_kernel(TcArgs a) {
  using LY = TcLayout<BN, FMT>;
  constexpr int kOpStages = op_stages<BN>();
  extern __shared__ __align__(1024) unsigned char dsm[];
  __shared__ uint64_t bars[kOpStages];
  __shared__ uint32_t tmem_base_s;
  __shared__ int fail_s;
  constexpr int kCols = BN < 32 ? 32 : BN;
  unsigned char* base = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(dsm) + 1023) & ~uintptr_t(1023));
  unsigned char* raw0 = base + kOpStages * LY::kOpStage;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.x * TM;   // weight rows
  const int m0 = blockIdx.y * BN;   // activation rows

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_s)),
                 "r"(kCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    for (int i = 0; i < kOpStages; ++i) mbar_init(&bars[i], 1);
    mbar_fence_init();
    fail_s = 0;
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem_d = tmem_base_s;
  pdl_wait();

  const int nk_all = a.K / TK;
  const int z = a.splits > 1 ? (int)cluster_rank() : 0;   // this CTA's K slice
  const int kb0 = nk_all * z / a.splits, kb1 = nk_all * (z + 1) / a.splits;
  const int nk = kb1 - kb0;   // this CTA's K blocks: kb0 + 0 .. kb0 + nk - 1
  const uint32_t idesc = idesc_tf32(BN);
  uint32_t phases = 0u;   // bit s: the parity of operand stage s's next MMA completion
  bool ok = true;
  // prologue: stage the first kStages - 1 blocks
#pragma unroll
  for (int i = 0; i < kStages - 1; ++i) {
    if (i < nk) stage_block<BN, FMT>(a, raw0 + i * LY::kRawStage, n0, m0, kb0 + i);
    cp_async_commit();
  }
  for (int kb = 0; kb < nk; ++kb) {
    const int s = kb % kOpStages;
    unsigned char* st = base + s * LY::kOpStage;
    // keep the copy engine kStages - 1 blocks ahead
    if (kb + kStages - 1 < nk)
      stage_block<BN, FMT>(a, raw0 + ((kb + kStages - 1) % kStages) * LY::kRawStage, n0, m0, kb0 + kb + kStages - 1);
    cp_async_commit();
    cp_async_wait<kStages - 1>();  // this thread's copies of block kb have landed
    // the MMAs that read this operand stage kOpStages blocks ago must be done before it is
    // rewritten
    if (kb >= kOpStages) {
      if (!mbar_wait(&bars[s], (phases >> s) & 1u, a.status)) ok = false;
      phases ^= 1u << s;
    }
    if (__syncthreads_or(!ok)) break;  // also: every thread's copies of block kb are visible
    const unsigned char* raw = raw0 + (kb % kStages) * LY::kRawStage;
    // ---- weights: thread t converts half a row (16 values) ----
    {
      const int r = tid >> 1, hf = tid & 1;
      float w[16];
      if (FMT == kInt4) {
        const uint2 p = *reinterpret_cast<const uint2*>(raw + r * 16 + hf * 8);
        const float sc = *reinterpret_cast<const float*>(raw + LY::kRawW + r * 4);
        const uint32_t wd[2] = {p.x, p.y};
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
          for (int e = 0; e < 8; ++e) w[8 * i + e] = nib_to_q((wd[i] >> (4 * e)) & 15u) * sc;
      } else {
        const uint4* h4 = reinterpret_cast<const uint4*>(raw + r * 64 + hf * 32);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const uint4 hv = h4[i];
          const __half2* h2 = reinterpret_cast<const __half2*>(&hv);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __half22float2(h2[e]);
            w[8 * i + 2 * e] = f.x;
            w[8 * i + 2 * e + 1] = f.y;
          }
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float4 big, small;
        split4(make_float4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]), big, small);
        *reinterpret_cast<float4*>(st + sw128_off(r, hf * 4 + j)) = big;
        *reinterpret_cast<float4*>(st + kTileBytes + sw128_off(r, hf * 4 + j)) = small;
      }
    }
    // ---- activations: BN rows x 8 chunks ----
    {
      const unsigned char* rx = raw + LY::kRawW + LY::kRawS;
      for (int i = tid; i < BN * 8; i += 256) {
        const int r = i >> 3, j = i & 7;
        const float4 v = *reinterpret_cast<const float4*>(rx + r * 128 + j * 16);
        float4 big, small;
        split4(v, big, small);
        *reinterpret_cast<float4*>(st + 2 * kTileBytes + sw128_off(r, j)) = big;
        *reinterpret_cast<float4*>(st + 2 * kTileBytes + LY::kBBytes + sw128_off(r, j)) = small;
      }
    }
    // hand the tiles to the tensor core (async proxy)
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    if (tid == 0) {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t sa = smem_u32(st);
      const uint64_t abig = smem_desc_sw128(sa), asmall = smem_desc_sw128(sa + kTileBytes);
      const uint64_t bbig = smem_desc_sw128(sa + 2 * kTileBytes);
      const uint64_t bsmall = smem_desc_sw128(sa + 2 * kTileBytes + LY::kBBytes);
#pragma unroll
      for (int kk = 0; kk < TK / 8; ++kk) {
        const uint64_t adv = (uint64_t)((kk * 32) >> 4);  // 8 tf32 = 32 bytes along the swizzled row
        const uint32_t first = (kb == 0 && kk == 0) ? 0u : 1u;
        mma_tf32(tmem_d, abig + adv, bbig + adv, idesc, first);
        mma_tf32(tmem_d, abig + adv, bsmall + adv, idesc, 1u);
        mma_tf32(tmem_d, asmall + adv, bbig + adv, idesc, 1u);
      }
      mma_commit(&bars[s]);
    }
  }
  cp_async_wait<0>();
  // wait for the MMAs still outstanding: the latest commit of each stage in use.  Also on
  // the failure path (bounded), so that TMEM is never freed under a running MMA.
  {
    const int used = nk < kOpStages ? nk : kOpStages;
    for (int s = 0; s < used; ++s)
      if (!mbar_wait(&bars[s], (phases >> s) & 1u, a.status)) ok = false;
  }
  if (__syncthreads_or(!ok)) fail_s = 1;
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  pdl_trigger();
  if (a.splits > 1) {
    // ---- split-K: partial tile [col][row] into this CTA's shared memory (operand stage 0,
    // free now that every MMA has completed), then this CTA's 1/S of the tile summed over the
    // cluster in rank order ----
    const int q = warp & 3, hh = warp >> 2;
    constexpr int kHalf = BN / 2;
    float* P = reinterpret_cast<float*>(base);
#pragma unroll
    for (int c0 = 0; c0 < (fail_s ? 0 : kHalf); c0 += 8) {
      uint32_t r[8];
      const int col = hh * kHalf + c0;
      const uint32_t taddr = tmem_d + ((uint32_t)(q * 32) << 16) + (uint32_t)col;
      asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                   : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                   : "r"(taddr)
                   : "memory");
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
      for (int j = 0; j < 8; ++j) P[(col + j) * TM + q * 32 + lane] = __uint_as_float(r[j]);
    }
    cluster_sync_all();
    const int S = a.splits, E = BN * TM;
    const int e0 = E * z / S, e1 = E * (z + 1) / S;
    const uint32_t pbase = smem_u32(P);
    for (int e = e0 + tid; e < e1; e += 256) {
      float part[8];
#pragma unroll
      for (int zz = 0; zz < 8; ++zz) part[zz] = zz < S ? ld_peer(pbase + 4u * (uint32_t)e, (uint32_t)zz) : 0.f;
      float v = 0.f;
#pragma unroll
      for (int zz = 0; zz < 8; ++zz)
        if (zz < S) v += part[zz];
      const int col = e / TM, row = e - col * TM;
      const int n = n0 + row, m = m0 + col;
      if (!fail_s && n < a.N && m < a.M) {
        float* yp = a.y + (size_t)m * a.ldy + n;
        if (EPI == kAdd) v += *yp;
        else if (EPI == kGelu) v = gelu_erf(v);
        *yp = v;
      }
    }
    cluster_sync_all();   // the peers have read this CTA's partial
  } else if (!fail_s) {
    // ---- epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31 (weight rows); warps 0-3 take
    // the first half of the BN columns, warps 4-7 the second ----
    const int q = warp & 3, hh = warp >> 2;
    const int n = n0 + q * 32 + lane;
    constexpr int kHalf = BN / 2;
#pragma unroll
    for (int c0 = 0; c0 < kHalf; c0 += 8) {
      uint32_t r[8];
      const int col = hh * kHalf + c0;
      const uint32_t taddr = tmem_d + ((uint32_t)(q * 32) << 16) + (uint32_t)col;
      asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                   : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                   : "r"(taddr)
                   : "memory");
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
      if (n < a.N) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int m = m0 + col + j;
          if (m < a.M) {
            float v = __uint_as_float(r[j]);
            float* yp = a.y + (size_t)m * a.ldy + n;
            if (EPI == kAdd) v += *yp;
            else if (EPI == kGelu) v = gelu_erf(v);
            *yp = v;
          }
        }
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_d), "r"(kCols) : "memory");
}

namespace {
template <int BN, int FMT>
cudaError_t tc_go(const Launch& L, TcArgs a, int epi, const GemmWork* gw) {
  const int tiles = ((a.N + TM - 1) / TM) * ((a.M + BN - 1) / BN);
  // split K when the tiles leave SMs idle: as many parts (<= 8, a portable cluster) as keep
  // the grid to one wave (one CTA per SM), at least 2 K blocks each
  a.splits = 1;
  if (gw && 2 * tiles <= gw->sms) {
    int s = gw->sms / tiles;
    const int nk = a.K / TK;
    if (s > nk / 2) s = nk / 2;
    if (s > 8) s = 8;
    if (s > 1) a.splits = s;
  }
  const dim3 grid((a.N + TM - 1) / TM, (a.M + BN - 1) / BN, a.splits);
  const size_t smem = TcLayout<BN, FMT>::kBytes;
  void (*k)(TcArgs) = epi == kAdd    ? gemm_tc_kernel<BN, FMT, kAdd>
                      : epi == kGelu ? gemm_tc_kernel<BN, FMT, kGelu>
                                     : gemm_tc_kernel<BN, FMT, kStore>;
  // TMEM is allocated at kernel start: launches stay stream-ordered (no PDL)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = L.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = (unsigned)a.splits;
  cfg.attrs = attr;
  cfg.numAttrs = a.splits > 1 ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, k, a);
  if (e == cudaSuccess) launch_counter().fetch_add(1, std::memory_order_relaxed);
  return e;
}

template <int BN>
cudaError_t tc_attrs_bn() {
  cudaError_t e = cudaSuccess;
  const size_t si = TcLayout<BN, kInt4>::kBytes, sh = TcLayout<BN, kFp16>::kBytes;
  if (e == cudaSuccess) e = allow_smem(gemm_tc_kernel<BN, kInt4, kStore>, si);
  if (e == cudaSuccess) e = allow_smem(gemm_tc_kernel<BN, kInt4, kAdd>, si);
  if (e == cudaSuccess) e = allow_smem(gemm_tc_kernel<BN, kInt4, kGelu>, si);
  if (e == cudaSuccess) e = allow_smem(gemm_tc_kernel<BN, kFp16, kStore>, sh);
  if (e == cudaSuccess) e = allow_smem(gemm_tc_kernel<BN, kFp16, kAdd>, sh);
  if (e == cudaSuccess) e = allow_smem(gemm_tc_kernel<BN, kFp16, kGelu>, sh);
  return e;
}
}  // namespace

cudaError_t init_attrs_gemm_tc() {
  cudaError_t e = tc_attrs_bn<16>();
  if (e == cudaSuccess) e = tc_attrs_bn<32>();
  if (e == cudaSuccess) e = tc_attrs_bn<64>();
  return e;
}

cudaError_t launch_gemm_tc(const Launch& L, const WView& w, const float* x, int ldx, int M, float* y, int ldy,
                           int epi, const GemmWork* gw) {
  if (M <= 0) return cudaSuccess;
  if (w.K % TK != 0 || ldx % 4 != 0) return cudaErrorInvalidValue;
  TcArgs a;
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
  a.status = L.status;
  a.splits = 1;
  const bool h = w.fmt == kFp16;
  if (M <= 16) return h ? tc_go<16, kFp16>(L, a, epi, gw) : tc_go<16, kInt4>(L, a, epi, gw);
  if (M <= 32) return h ? tc_go<32, kFp16>(L, a, epi, gw) : tc_go<32, kInt4>(L, a, epi, gw);
  return h ? tc_go<64, kFp16>(L, a, epi, gw) : tc_go<64, kInt4>(L, a, epi, gw);
}

}  // namespace ms
