// Dequant-GEMM on the 5th-generation tensor cores for prefill and batched decode, where the
// MatMul is a real dense contraction ("MuScriptor Medium — optimized W4A32 ONNX Runtime",
// Model variant: MatMulNBits with symmetric INT4 g32 weights; the fp16-weight variant of
// "MuScriptor for Core AI (.aimodel)", file table):  y[m][n] (+)= sum_k x[m][k] W[n][k].
//
// Shape: swap-AB.  128 weight rows are the MMA's M side (operand A), BN activation rows its N
// side (operand B); one CTA owns a 128 x BN tile of y^T in TMEM (fp32).
//
// Precision.  kind::f16 MMAs with fp32 accumulation, each fp32 operand carried as an fp16
// pair hi + lo (hi = fp16(v), lo = fp16(v - hi): a 22-bit significand):
//   - weights: the dequantised value q * s (one fp32 product, as the pages' MatMulNBits
//     dequantisation defines it) times 2^e_n, a per-row power of two chosen at model creation
//     so that the row's largest |q s| lands in [2^13, 2^14); the epilogue multiplies by 2^-e_n
//     (exact).  Half weights (the fp16 variant) are exact: one operand, no lo part.
//   - activations: split by their producer (LayerNorm, attention, the previous GEMM's
//     epilogue) into fp16 hi and lo arrays.
// Three products per step (hi*hi + hi*lo + lo*hi; two for half weights); the dropped lo*lo
// term is below 2^-22 of each product.
//
// Roles (320 threads), no CTA barrier inside the K loop:
//   warp 0   producer: per 64-wide K stage one bulk copy of the stage's tile-packed INT4
//            block (codes + scales of 128 rows, 5120 bytes; or a TMA tile of half weights)
//            and two TMA tiles (128-byte swizzle) of the activation hi / lo planes, all
//            completing on the stage's `full` mbarrier;
//   warps 2-9 converters: dequantise the staged block into the A hi / lo operand tiles
//            (canonical K-major 128-byte-swizzled layout) and arrive on `conv`;
//   warp 1   one elected thread issues the tcgen05.mma of the stage and commits them to the
//            stage's `empty` mbarrier, which frees the stage for the producer;
//   warps 2-9 then read the accumulator from TMEM (epilogue): scale, store / add / GELU, and
//            optionally write the result as fp16 hi / lo planes for the next GEMM.
// Split-K: when the output tiles alone would leave SMs idle, the S <= 8 CTAs of one tile form
// a thread-block cluster over disjoint K ranges; each leaves its partial tile in its shared
// memory and each sums 1/S of the tile over the cluster (distributed shared memory) in rank
// order before the epilogue.
//
// Every wait is bounded; a wait that runs out flags the status word, the CTA stops issuing,
// waits (bounded) for the copies it issued and frees TMEM after its MMAs have completed.
#include <cuda.h>

#include "ms_device.cuh"
#include "ms_launch.cuh"
#include "ms_tc.cuh"

namespace ms {

namespace {

constexpr int GM = 128;                   // weight rows per tile (MMA M)
constexpr int GK = 64;                    // K per stage: one 128-byte row of halves
constexpr int kATile = GM * GK * 2;       // 16 KiB, one fp16 operand tile of weights
constexpr int kRawA = GM * 32 + GM * 8;   // 5120: the stage's INT4 codes and two scales per row
constexpr int kGThreads = 320;
constexpr int kConv0 = 64;                // first converter / epilogue thread

struct GArgs {
  const unsigned char* wt;   // INT4: tile-packed blocks [N/128][K/64][5120]; null for halves
  const float* rinv;         // INT4: 2^-e_n per weight row [N/128 * 128]; null for halves
  int N, K, M;
  float* y;                  // fp32 output [M][ldy], or null
  int ldy;
  __half* yh;                // fp16 hi / lo output planes [M][ldyh], or null
  __half* yl;
  int ldyh;
  unsigned* status;
  int splits;                // CTAs per output tile along K (the cluster's size)
};

template <int BN, int FMT>
struct GLayout {
  static constexpr int kBTile = BN * 128;                       // one activation operand tile
  static constexpr int kA = FMT == kInt4 ? 2 * kATile : kATile; // A hi (+ lo)
  static constexpr int kRaw = FMT == kInt4 ? kRawA : 0;
  static constexpr int kStage = kA + 2 * kBTile + kRaw;         // a multiple of 1024
  static constexpr int kStages = (BN >= 256 ? 2 : BN >= 128 ? 3 : 4);
  static constexpr size_t kBytes = 1024 + (size_t)kStages * kStage;
  static constexpr uint32_t kTx = (FMT == kInt4 ? kRawA : kATile) + 2 * kBTile;
  static_assert(kStage % 1024 == 0, "stages stay 1024-byte aligned");
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

// Instruction descriptor, kind::f16: D fp32, A and B fp16, both K-major, M = 128, N = bn.
__device__ __forceinline__ uint32_t idesc_f16(int bn) { return idesc_f16_mn(GM, bn, false); }

}  // namespace

template <int BN, int FMT, int EPI>
__global__ void __launch_bounds__(kGThreads, 1)
    gemm_f16_kernel(const GArgs a, const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmBh,
                    const __grid_constant__ CUtensorMap tmBl) {
  using LY = GLayout<BN, FMT>;
  constexpr int NS = LY::kStages;
  extern __shared__ __align__(1024) unsigned char dsm[];
  __shared__ uint64_t full[NS], conv[NS], empty[NS], accb;
  __shared__ uint32_t tmem_base_s;
  __shared__ int fail_s;
  constexpr int kCols = BN < 32 ? 32 : BN;
  unsigned char* base = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(dsm) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x;
  const int n0 = tile * GM, m0 = blockIdx.y * BN;

  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_s)),
                 "r"(kCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&conv[i], kGThreads - kConv0);
      mbar_init(&empty[i], 1);
    }
    mbar_init(&accb, 1);
    mbar_fence_init();
    fail_s = 0;
    if (FMT == kFp16) prefetch_map(&tmA);
    prefetch_map(&tmBh);
    prefetch_map(&tmBl);
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem_d = tmem_base_s;

  const int nkb_all = a.K / GK;
  const int z = a.splits > 1 ? (int)cluster_rank() : 0;
  const int kb0 = nkb_all * z / a.splits, kb1 = nkb_all * (z + 1) / a.splits;
  const int nk = kb1 - kb0;
  bool ok = true;

  pdl_trigger();
  if (warp == 0) {
    // ---- producer ----
    if (lane == 0) {
      auto load_weights = [&](int kb) {
        unsigned char* st = base + (size_t)(kb % NS) * LY::kStage;
        if (FMT == kInt4)
          bulk_g2s(st + LY::kA + 2 * LY::kBTile, a.wt + ((size_t)tile * nkb_all + kb0 + kb) * kRawA, kRawA,
                   &full[kb % NS]);
        else
          tma_load_2d(st, &tmA, (kb0 + kb) * GK, n0, &full[kb % NS]);
      };
      auto load_acts = [&](int kb) {
        unsigned char* st = base + (size_t)(kb % NS) * LY::kStage;
        tma_load_2d(st + LY::kA, &tmBh, (kb0 + kb) * GK, m0, &full[kb % NS]);
        tma_load_2d(st + LY::kA + LY::kBTile, &tmBl, (kb0 + kb) * GK, m0, &full[kb % NS]);
      };
      // the weights are constants: the first stages' weight copies go out before the wait for
      // the kernel that produces the activations (programmatic dependent launch)
      const int pre = nk < NS ? nk : NS;
      for (int kb = 0; kb < pre; ++kb) {
        mbar_expect_tx(&full[kb], LY::kTx);
        load_weights(kb);
      }
      pdl_wait();
      for (int kb = 0; kb < pre; ++kb) load_acts(kb);
      int issued = pre;
      for (int kb = pre; kb < nk && ok; ++kb) {
        const int s = kb % NS;
        if (!mbar_wait(&empty[s], (uint32_t)(((kb / NS) - 1) & 1), a.status)) {
          ok = false;
          break;
        }
        mbar_expect_tx(&full[s], LY::kTx);
        load_weights(kb);
        load_acts(kb);
        ++issued;
      }
      // before leaving: the last copy issued into each stage has landed
      for (int s = 0; s < NS && s < issued; ++s) {
        const int uses = (issued - s + NS - 1) / NS;
        for (long long it = 0; it < kSpinLimit; ++it)
          if (mbar_try_wait(&full[s], (uint32_t)((uses - 1) & 1))) break;
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer ----
    if (lane == 0) {
      const uint32_t idesc = idesc_f16(BN);
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % NS;
        const uint32_t par = (uint32_t)((kb / NS) & 1);
        if (!mbar_wait(FMT == kInt4 ? &conv[s] : &full[s], par, a.status)) {
          ok = false;
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t sa = smem_u32(base + (size_t)s * LY::kStage);
        const uint64_t ahi = desc_sw128(sa), alo = desc_sw128(sa + kATile);
        const uint64_t bhi = desc_sw128(sa + LY::kA), blo = desc_sw128(sa + LY::kA + LY::kBTile);
#pragma unroll
        for (int kk = 0; kk < GK / 16; ++kk) {
          const uint64_t adv = (uint64_t)((kk * 32) >> 4);   // 16 halves = 32 bytes along the row
          mma_f16(tmem_d, ahi + adv, bhi + adv, idesc, (kb == 0 && kk == 0) ? 0u : 1u);
          mma_f16(tmem_d, ahi + adv, blo + adv, idesc, 1u);
          if (FMT == kInt4) mma_f16(tmem_d, alo + adv, bhi + adv, idesc, 1u);
        }
        mma_commit(&empty[s]);
      }
      mma_commit(&accb);   // every MMA issued above, also on the failure path
    }
  } else if (FMT == kInt4) {
    // ---- converters: thread (row r, half hf) dequantises 32 weights per stage ----
    const int ct = tid - kConv0, r = ct >> 1, hf = ct & 1;
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % NS;
      if (!mbar_wait(&full[s], (uint32_t)((kb / NS) & 1), a.status)) {
        ok = false;
        break;
      }
      unsigned char* st = base + (size_t)s * LY::kStage;
      const unsigned char* raw = st + LY::kA + 2 * LY::kBTile;
      const uint4 codes = *reinterpret_cast<const uint4*>(raw + r * 32 + hf * 16);
      const float sc = *reinterpret_cast<const float*>(raw + GM * 32 + r * 8 + hf * 4);
      const uint32_t wd[4] = {codes.x, codes.y, codes.z, codes.w};
#pragma unroll
      for (int c = 0; c < 4; ++c) {   // chunk c: 8 weights = word wd[c]
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const float w0 = nib_to_q((wd[c] >> (8 * p)) & 15u) * sc;
          const float w1 = nib_to_q((wd[c] >> (8 * p + 4)) & 15u) * sc;
          hi[p] = pack_h2(w0, w1);
          const float2 hf2 = unpack_h2(hi[p]);
          lo[p] = pack_h2(w0 - hf2.x, w1 - hf2.y);
        }
        const uint32_t off = sw128(r, hf * 4 + c);
        *reinterpret_cast<uint4*>(st + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(st + kATile + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(&conv[s]);
    }
  }

  // ---- epilogue (warps 2-9) ----
  pdl_wait();   // before any global read or write of activations (returns at once by now)
  if (__syncthreads_or(!ok)) {
    if (tid == 0) flag_error(a.status, kErrTimeout);
  }
  const bool epi_warp = warp >= 2;
  const int q = warp & 3;            // TMEM lane quarter this warp may read
  const int hh = (warp - 2) >> 2;    // column half
  bool acc_ok = true;
  if (epi_warp) {
    acc_ok = mbar_wait(&accb, 0u, a.status);
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  }
  const int failed = __syncthreads_or(!acc_ok || !ok);
  constexpr int kHalf = BN / 2;
  auto emit = [&](int n, int m, float v) {
    if (n >= a.N || m >= a.M) return;
    if (a.rinv) v *= a.rinv[n];
    if (a.y) {
      float* yp = a.y + (size_t)m * a.ldy + n;
      if (EPI == kAdd) v += *yp;
      else if (EPI == kGelu) v = gelu_erf(v);
      *yp = v;
    } else if (EPI == kGelu) {
      v = gelu_erf(v);
    }
    if (a.yh) {
      const __half h = __float2half_rn(v);
      a.yh[(size_t)m * a.ldyh + n] = h;
      a.yl[(size_t)m * a.ldyh + n] = __float2half_rn(v - __half2float(h));
    }
  };
  if (a.splits > 1) {
    float* P = reinterpret_cast<float*>(base);   // stage memory is free: every MMA has completed
    if (epi_warp && !failed) {
#pragma unroll 1
      for (int c0 = 0; c0 < kHalf; c0 += 8) {
        uint32_t rr[8];
        const int col = hh * kHalf + c0;
        const uint32_t taddr = tmem_d + ((uint32_t)(q * 32) << 16) + (uint32_t)col;
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                     : "=r"(rr[0]), "=r"(rr[1]), "=r"(rr[2]), "=r"(rr[3]), "=r"(rr[4]), "=r"(rr[5]), "=r"(rr[6]),
                       "=r"(rr[7])
                     : "r"(taddr)
                     : "memory");
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
        for (int j = 0; j < 8; ++j) P[(col + j) * GM + q * 32 + lane] = __uint_as_float(rr[j]);
      }
    }
    cluster_sync_all();
    const int S = a.splits, E = BN * GM;
    const int e0 = E * z / S, e1 = E * (z + 1) / S;
    const uint32_t pbase = smem_u32(P);
    for (int e = e0 + tid; e < e1; e += kGThreads) {
      float v = 0.f;
      for (int zz = 0; zz < S; ++zz) v += ld_peer(pbase + 4u * (uint32_t)e, (uint32_t)zz);
      const int col = e / GM, row = e - col * GM;
      if (!failed) emit(n0 + row, m0 + col, v);
    }
    cluster_sync_all();   // the peers have read this CTA's partial
  } else if (epi_warp && !failed) {
    const int n = n0 + q * 32 + lane;
#pragma unroll 1
    for (int c0 = 0; c0 < kHalf; c0 += 8) {
      uint32_t rr[8];
      const int col = hh * kHalf + c0;
      const uint32_t taddr = tmem_d + ((uint32_t)(q * 32) << 16) + (uint32_t)col;
      asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                   : "=r"(rr[0]), "=r"(rr[1]), "=r"(rr[2]), "=r"(rr[3]), "=r"(rr[4]), "=r"(rr[5]), "=r"(rr[6]),
                     "=r"(rr[7])
                   : "r"(taddr)
                   : "memory");
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
      for (int j = 0; j < 8; ++j) emit(n, m0 + col + j, __uint_as_float(rr[j]));
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_d), "r"(kCols) : "memory");
}

// ---- weight repack for the GEMM ------------------------------------------------------------
// Per weight row n: e_n such that 7 max_g s[n][g] 2^e_n lies in [2^13, 2^14) (0 for an all-zero
// row); rinv[n] = 2^-e_n.  Rows past N (up to the tile) get rinv 0.
__global__ void gemm_row_exp_kernel(WView w, int Npad, float* __restrict__ rexp, float* __restrict__ rinv) {
  const int n = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (n >= Npad) return;
  float m = 0.f;
  if (n < w.N)
    for (int g = lane; g < w.K / 32; g += 32) m = fmaxf(m, fabsf(w.s[(size_t)n * w.lds + g]));
  m = warp_max(m) * 7.0f;
  if (lane == 0) {
    int e = 0;
    const unsigned bits = __float_as_uint(m);
    if ((bits & 0x7F800000u) != 0) {
      const int E = (int)((bits >> 23) & 0xFFu) - 127;   // m in [2^E, 2^(E+1))
      e = min(max(13 - E, -100), 100);
    }
    rexp[n] = __uint_as_float((unsigned)(127 + e) << 23);
    rinv[n] = n < w.N ? __uint_as_float((unsigned)(127 - e) << 23) : 0.f;
  }
}

// Block (tile t, stage kb): [128 rows x 32 bytes of codes][128 rows x 2 scales times 2^e_n].
// Codes keep their order (element 2j in the low nibble of byte j); rows past N hold code 8
// (q = 0) and scale 0.
__global__ void gemm_repack_int4_kernel(WView w, int nkb, const float* __restrict__ rexp,
                                        unsigned char* __restrict__ out) {
  const int blk = blockIdx.x, t = blk / nkb, kb = blk - t * nkb;
  unsigned char* o = out + (size_t)blk * kRawA;
  for (int i = threadIdx.x; i < GM * 2; i += blockDim.x) {   // 16-byte pieces of codes
    const int r = i >> 1, hf = i & 1, n = t * GM + r;
    uint4 v = make_uint4(0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u);
    if (n < w.N) v = *reinterpret_cast<const uint4*>(w.q + (size_t)n * w.ldq + kb * 32 + hf * 16);
    *reinterpret_cast<uint4*>(o + r * 32 + hf * 16) = v;
  }
  float* so = reinterpret_cast<float*>(o + GM * 32);
  for (int i = threadIdx.x; i < GM * 2; i += blockDim.x) {
    const int r = i >> 1, g = i & 1, n = t * GM + r;
    so[i] = n < w.N ? w.s[(size_t)n * w.lds + kb * 2 + g] * rexp[n] : 0.f;
  }
}

// fp32 rows -> fp16 hi / lo planes (hi = fp16(v), lo = fp16(v - hi)); |v| >= 65504 flags the
// status word (the planes would not hold it).
__global__ void split_f16_kernel(const float* __restrict__ x, int ldx, int M, int K, __half* __restrict__ xh,
                                 __half* __restrict__ xl, int ldh, unsigned* status) {
  pdl_wait();
  pdl_trigger();
  const int per_row = K / 4;
  const long long total = (long long)M * per_row;
  bool big = false;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (long long)gridDim.x * blockDim.x) {
    const int m = (int)(i / per_row), k = (int)(i - (long long)m * per_row) * 4;
    const float4 v = *reinterpret_cast<const float4*>(x + (size_t)m * ldx + k);
    big |= fabsf(v.x) >= 65504.f || fabsf(v.y) >= 65504.f || fabsf(v.z) >= 65504.f || fabsf(v.w) >= 65504.f;
    const uint32_t h0 = pack_h2(v.x, v.y), h1 = pack_h2(v.z, v.w);
    const float2 f0 = unpack_h2(h0), f1 = unpack_h2(h1);
    const uint32_t l0 = pack_h2(v.x - f0.x, v.y - f0.y), l1 = pack_h2(v.z - f1.x, v.w - f1.y);
    *reinterpret_cast<uint2*>(xh + (size_t)m * ldh + k) = make_uint2(h0, h1);
    *reinterpret_cast<uint2*>(xl + (size_t)m * ldh + k) = make_uint2(l0, l1);
  }
  if (big) flag_error(status, kErrShape);
}

namespace {

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encoder() {
  static EncodeTiled fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<EncodeTiled>(p);
  }();
  return fn;
}

}  // namespace

cudaError_t encode_map_2d(CUtensorMap* m, CUtensorMapDataType type, const void* ptr, uint64_t cols, uint64_t rows,
                          uint64_t stride_bytes, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
  EncodeTiled enc = encoder();
  if (!enc) return cudaErrorNotSupported;
  if ((reinterpret_cast<uintptr_t>(ptr) & 15) || stride_bytes % 16 != 0) return cudaErrorInvalidValue;
  const cuuint64_t dim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t stride[1] = {(cuuint64_t)stride_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t es[2] = {1, 1};
  const CUresult r = enc(m, type, 2, const_cast<void*>(ptr), dim, stride, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

namespace {

// 2-D fp16 tensor [rows][cols] (row stride ld halves) in boxes of 64 columns x box_rows rows,
// 128-byte swizzle; out-of-range rows read as zero.
cudaError_t map_f16(CUtensorMap* m, const void* ptr, int rows, int cols, int ld, int box_rows) {
  EncodeTiled enc = encoder();
  if (!enc) return cudaErrorNotSupported;
  if ((reinterpret_cast<uintptr_t>(ptr) & 15) || (ld * 2) % 16 != 0 || cols % GK != 0) return cudaErrorInvalidValue;
  const cuuint64_t dim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t stride[1] = {(cuuint64_t)ld * 2};
  const cuuint32_t box[2] = {(cuuint32_t)GK, (cuuint32_t)box_rows};
  const cuuint32_t es[2] = {1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(ptr), dim, stride, box, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int BN, int FMT>
cudaError_t gf_go(const Launch& L, GArgs a, int epi, const GemmWork* gw, const CUtensorMap& tA, const __half* xh,
                  const __half* xl, int ldx) {
  CUtensorMap tBh, tBl;
  cudaError_t e = map_f16(&tBh, xh, a.M, a.K, ldx, BN);
  if (e == cudaSuccess) e = map_f16(&tBl, xl, a.M, a.K, ldx, BN);
  if (e != cudaSuccess) return e;
  const int ntile = (a.N + GM - 1) / GM;
  const int tiles = ntile * ((a.M + BN - 1) / BN);
  a.splits = 1;
  if (gw && 2 * tiles <= gw->sms) {
    int s = gw->sms / tiles;
    const int nk = a.K / GK;
    if (s > nk / 2) s = nk / 2;
    if (s > 8) s = 8;
    while (s & (s - 1)) s &= s - 1;   // a power of two: 3- and 6-CTA clusters measured slower
    if (s > 1) a.splits = s;
  }
  const dim3 grid(ntile, (a.M + BN - 1) / BN, a.splits);
  void (*k)(const GArgs, const CUtensorMap, const CUtensorMap, const CUtensorMap) =
      epi == kAdd ? gemm_f16_kernel<BN, FMT, kAdd> : epi == kGelu ? gemm_f16_kernel<BN, FMT, kGelu>
                                                                 : gemm_f16_kernel<BN, FMT, kStore>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kGThreads);
  cfg.dynamicSmemBytes = GLayout<BN, FMT>::kBytes;
  cfg.stream = L.stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (a.splits > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 1;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = (unsigned)a.splits;
    ++na;
  }
  if (L.pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  e = cudaLaunchKernelEx(&cfg, k, a, tA, tBh, tBl);
  if (e == cudaSuccess) launch_counter().fetch_add(1, std::memory_order_relaxed);
  return e;
}

template <int BN>
cudaError_t gf_attrs_bn() {
  cudaError_t e = cudaSuccess;
  const size_t si = GLayout<BN, kInt4>::kBytes, sh = GLayout<BN, kFp16>::kBytes;
  if (e == cudaSuccess) e = allow_smem(gemm_f16_kernel<BN, kInt4, kStore>, si);
  if (e == cudaSuccess) e = allow_smem(gemm_f16_kernel<BN, kInt4, kAdd>, si);
  if (e == cudaSuccess) e = allow_smem(gemm_f16_kernel<BN, kInt4, kGelu>, si);
  if (e == cudaSuccess) e = allow_smem(gemm_f16_kernel<BN, kFp16, kStore>, sh);
  if (e == cudaSuccess) e = allow_smem(gemm_f16_kernel<BN, kFp16, kAdd>, sh);
  if (e == cudaSuccess) e = allow_smem(gemm_f16_kernel<BN, kFp16, kGelu>, sh);
  return e;
}

}  // namespace

cudaError_t init_attrs_gemm_f16() {
  cudaError_t e = gf_attrs_bn<32>();
  if (e == cudaSuccess) e = gf_attrs_bn<64>();
  if (e == cudaSuccess) e = gf_attrs_bn<128>();
  if (e == cudaSuccess) e = gf_attrs_bn<256>();
  return e;
}

size_t gemm_tiles_bytes(const WView& w) {
  if (w.fmt != kInt4) return 0;
  return (size_t)((w.N + GM - 1) / GM) * (w.K / GK) * kRawA;
}
size_t gemm_rows_padded(const WView& w) { return (size_t)((w.N + GM - 1) / GM) * GM; }

cudaError_t launch_gemm_repack(const WView& w, GemmWeights& g, float* rexp_scratch, cudaStream_t s) {
  if (w.fmt != kInt4) return cudaSuccess;
  if (w.K % GK != 0) return cudaErrorInvalidValue;
  const int npad = (int)gemm_rows_padded(w), nkb = w.K / GK;
  gemm_row_exp_kernel<<<(npad + 7) / 8, 256, 0, s>>>(w, npad, rexp_scratch, const_cast<float*>(g.rinv));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  gemm_repack_int4_kernel<<<(npad / GM) * nkb, 256, 0, s>>>(w, nkb, rexp_scratch, const_cast<unsigned char*>(g.wt));
  return cudaGetLastError();
}

cudaError_t launch_split_f16(const Launch& L, const float* x, int ldx, int M, int K, __half* xh, __half* xl, int ldh) {
  if (M <= 0) return cudaSuccess;
  if (K % 4 != 0 || ldx % 4 != 0 || ldh % 4 != 0) return cudaErrorInvalidValue;
  long long n4 = (long long)M * (K / 4);
  int grid = (int)((n4 + 255) / 256);
  if (grid > 148 * 8) grid = 148 * 8;
  return launch_k(L, split_f16_kernel, dim3(grid), dim3(256), 0, x, ldx, M, K, xh, xl, ldh, L.status);
}

cudaError_t launch_gemm_f16(const Launch& L, const WView& w, const GemmWeights& g, const __half* xh, const __half* xl,
                            int ldx, int M, float* y, int ldy, __half* yh, __half* yl, int ldyh, int epi,
                            const GemmWork* gw) {
  if (M <= 0) return cudaSuccess;
  if (w.K % GK != 0 || (w.fmt == kInt4 && (!g.wt || !g.rinv))) return cudaErrorInvalidValue;
  if (epi == kAdd && !y) return cudaErrorInvalidValue;
  GArgs a;
  a.wt = g.wt;
  a.rinv = w.fmt == kInt4 ? g.rinv : nullptr;
  a.N = w.N;
  a.K = w.K;
  a.M = M;
  a.y = y;
  a.ldy = ldy;
  a.yh = yh;
  a.yl = yl;
  a.ldyh = ldyh;
  a.status = L.status;
  a.splits = 1;
  const bool h = w.fmt == kFp16;
  CUtensorMap tA;
  memset(&tA, 0, sizeof(tA));
  if (h) {
    cudaError_t e = map_f16(&tA, w.h, w.N, w.K, w.K, GM);
    if (e != cudaSuccess) return e;
  }
  // tile width by rows; 256 only when even those tiles fill every SM twice
  const int ntile = (w.N + GM - 1) / GM;
  auto tiles = [&](int bn) { return ntile * ((M + bn - 1) / bn); };
  const int sms = gw ? gw->sms : 148;
  // 128 rather than 64 unless it pads more rows: 128-row activation tiles halve the weight
  // tiles each CTA dequantises (measured faster at 504 rows even with SMs left idle; slower at
  // 130, where the second 128-row tile is nearly empty)
  auto padded = [&](int b) { return (M + b - 1) / b * b; };
  int bn = 32;
  if (M > 32) bn = 64;
  if (M > 64 && padded(128) <= padded(64)) bn = 128;
  if (M > 128 && tiles(256) >= 2 * sms) bn = 256;
  switch (bn) {
    case 32: return h ? gf_go<32, kFp16>(L, a, epi, gw, tA, xh, xl, ldx) : gf_go<32, kInt4>(L, a, epi, gw, tA, xh, xl, ldx);
    case 64: return h ? gf_go<64, kFp16>(L, a, epi, gw, tA, xh, xl, ldx) : gf_go<64, kInt4>(L, a, epi, gw, tA, xh, xl, ldx);
    case 128:
      return h ? gf_go<128, kFp16>(L, a, epi, gw, tA, xh, xl, ldx) : gf_go<128, kInt4>(L, a, epi, gw, tA, xh, xl, ldx);
    default:
      return h ? gf_go<256, kFp16>(L, a, epi, gw, tA, xh, xl, ldx) : gf_go<256, kInt4>(L, a, epi, gw, tA, xh, xl, ldx);
  }
}

}  // namespace ms
