// W4A8 dequant-GEMM on the 5th-generation tensor cores ("MuScriptor Medium — optimized W4A32
// ONNX Runtime", Model variant: MatMulNBits with accuracy_level=4 quantises the activations to
// INT8 at run time and accumulates in INT32):  y[m][n] = sum over 32-wide blocks b of
// sa[m][b] * sw[n][b] * sum_{k in b} qa[m][k] * qw[n][k], with qw the INT4 codes of the weights
// and qa the INT8 codes of the activations (the quantiser in k_w4a8.cu).
//
// Shape: swap-AB, 128 weight rows on the MMA's M side and 64 activation rows on its N side; K
// in stages of 128 (one 128-byte swizzled row of int8).  Each 32-wide block is one
// tcgen05.mma kind::i8 (signed x signed, int32 result) into a TMEM region of its own, since the
// two block scales differ from block to block; the 8 regions (two stages of four blocks, 512
// columns) let the MMAs of one stage run while the previous stage's results are drained.
// Roles (320 threads):
//   warp 0   producer: per stage one bulk copy of two tile-packed INT4 blocks (the tcgen05 f16
//            GEMM's copy: codes and the per-row scales times 2^e_n), a TMA tile of the
//            activation codes (128-byte swizzle) and a TMA tile of their block scales;
//   warps 2-9 converters: INT4 codes -> signed bytes in the A tile; then, one stage behind,
//            drain the four int32 block results from TMEM, scale each by sa * sw and add into
//            fp32 registers; finally store / residual add / GELU with the factor 2^-e_n;
//   warp 1   one thread issues the four MMAs of a stage and commits them.
// The integer block sums are exact; the scaling and the sum over blocks are fp32, like the dp4a
// kernels.  Every wait is bounded.
#include <cuda.h>

#include "ms_device.cuh"
#include "ms_kernels.h"
#include "ms_launch.cuh"
#include "ms_tc.cuh"

namespace ms {

namespace {

constexpr int QM = 128;                               // weight rows per tile (MMA M)
constexpr int QK = 128;                               // K per stage
constexpr int QBN = 64;                               // activation rows per tile (MMA N)
constexpr int QNS = 4;                                // stages
constexpr int kQA = QM * QK;                          // int8 weight tile
constexpr int kQB = QBN * QK;                         // int8 activation tile
constexpr int kQBlk = 5120;                           // one tile-packed 64-wide INT4 block
constexpr int kQRaw = 2 * kQBlk;
constexpr int kQSa = QBN * 4 * 4;                     // [QBN][4] activation block scales
constexpr int kQStage = kQA + kQB + kQRaw + kQSa;     // 35 KiB
constexpr size_t kQBytes = 1024 + (size_t)QNS * kQStage;
constexpr uint32_t kQTx = kQRaw + kQB + kQSa;
constexpr int kQThreads = 320, kQConv0 = 64;
constexpr int kQCols = 512;                           // 2 stages x 4 blocks x QBN int32 columns
static_assert(kQStage % 1024 == 0, "stages stay 1024-byte aligned");

struct QArgs {
  const unsigned char* wt;   // tile-packed INT4 blocks [N/128][K/64][5120]
  const float* rinv;         // 2^-e_n per weight row
  int N, K, M;
  float* y;
  int ldy;
  unsigned* status;
};

// kind::i8: D s32, A and B signed 8-bit, both K-major, M = 128, N = n.
__device__ __forceinline__ uint32_t idesc_i8(int n) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(QM >> 4) << 24);
}
__device__ __forceinline__ void mma_i8(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n}" ::"r"(
          tmem_d),
      "l"(da), "l"(db), "r"(idesc), "r"(0u)
      : "memory");
}
// Eight INT4 codes (four bytes, element 2j in the low nibble of byte j) -> two words of four
// signed bytes in element order.
__device__ __forceinline__ void codes_to_s8(uint32_t w, uint32_t& e0123, uint32_t& e4567) {
  const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
  e0123 = __vsub4(__byte_perm(lo, hi, 0x5140), 0x08080808u);
  e4567 = __vsub4(__byte_perm(lo, hi, 0x7362), 0x08080808u);
}

}  // namespace

template <int EPI>
__global__ void __launch_bounds__(kQThreads, 1)
    gemm_w4a8_tc_kernel(const QArgs a, const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmS) {
  extern __shared__ __align__(1024) unsigned char dsm[];
  __shared__ uint64_t full[QNS], conv[QNS], empty[QNS], accfull[2], accfree[2], fin;
  __shared__ uint32_t tmem_base_s;
  unsigned char* base = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(dsm) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x;
  const int n0 = tile * QM, m0 = blockIdx.y * QBN;

  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_s)),
                 "r"(kQCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    for (int i = 0; i < QNS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&conv[i], kQThreads - kQConv0);
      mbar_init(&empty[i], 1 + 8);   // the MMAs' commit and the eight draining warps
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&accfull[i], 1);
      mbar_init(&accfree[i], 8);
    }
    mbar_init(&fin, 1);
    mbar_fence_init();
    prefetch_map(&tmQ);
    prefetch_map(&tmS);
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = tmem_base_s;
  pdl_trigger();
  const int nk = a.K / QK, nkb64 = a.K / 64;
  bool ok = true;

  // epilogue mapping (warps 2-9): TMEM lane quarter q, column half hh
  const int q = warp & 3, hh = (warp - 2) >> 2, n_local = q * 32 + lane;
  float acc[QBN / 2];
#pragma unroll
  for (int j = 0; j < QBN / 2; ++j) acc[j] = 0.f;

  if (warp == 0) {
    // ---- producer ----
    if (lane == 0) {
      pdl_wait();
      int issued = 0;
      for (int kb = 0; kb < nk && ok; ++kb) {
        const int s = kb % QNS;
        if (kb >= QNS && !mbar_wait(&empty[s], (uint32_t)(((kb / QNS) - 1) & 1), a.status)) {
          ok = false;
          break;
        }
        unsigned char* st = base + (size_t)s * kQStage;
        mbar_expect_tx(&full[s], kQTx);
        bulk_g2s(st + kQA + kQB, a.wt + ((size_t)tile * nkb64 + 2 * kb) * kQBlk, kQRaw, &full[s]);
        tma_load_2d(st + kQA, &tmQ, kb * QK, m0, &full[s]);
        tma_load_2d(st + kQA + kQB + kQRaw, &tmS, kb * 4, m0, &full[s]);
        ++issued;
      }
      for (int s = 0; s < QNS && s < issued; ++s) {   // the last copy into each stage has landed
        const int uses = (issued - s + QNS - 1) / QNS;
        for (long long it = 0; it < kSpinLimit; ++it)
          if (mbar_try_wait(&full[s], (uint32_t)((uses - 1) & 1))) break;
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer ----
    if (lane == 0) {
      const uint32_t id = idesc_i8(QBN);
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % QNS, set = kb & 1;
        if (!mbar_wait(&conv[s], (uint32_t)((kb / QNS) & 1), a.status)) {
          ok = false;
          break;
        }
        if (kb >= 2 && !mbar_wait(&accfree[set], (uint32_t)(((kb >> 1) - 1) & 1), a.status)) {
          ok = false;
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t sa = smem_u32(base + (size_t)s * kQStage);
        const uint64_t ad = desc_sw128(sa), bd = desc_sw128(sa + kQA);
#pragma unroll
        for (int blk = 0; blk < 4; ++blk)   // 32 bytes = 32 int8 along the row per block
          mma_i8(tmem + (uint32_t)((set * 4 + blk) * QBN), ad + (uint64_t)(2 * blk), bd + (uint64_t)(2 * blk), id);
        mma_commit(&accfull[set]);
        mma_commit(&empty[s]);
      }
      mma_commit(&fin);   // every MMA issued above, also on the failure path
    }
  } else {
    // ---- converters, and the drain of the previous stage ----
    const int ct = tid - kQConv0, r = ct >> 1, hf = ct & 1;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    auto drain = [&](int kb) -> bool {
      const int s = kb % QNS, set = kb & 1;
      if (!mbar_wait(&accfull[set], (uint32_t)((kb >> 1) & 1), a.status)) return false;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const unsigned char* st = base + (size_t)s * kQStage;
      const float* sat = reinterpret_cast<const float*>(st + kQA + kQB + kQRaw);   // [QBN][4]
#pragma unroll 1
      for (int blk = 0; blk < 4; ++blk) {
        uint32_t d[32];
        tmem_ld32(tmem + lane_base + (uint32_t)((set * 4 + blk) * QBN + hh * 32), d);
        tmem_ld_wait();
        const float sw = *reinterpret_cast<const float*>(st + kQA + kQB + (blk >> 1) * kQBlk + QM * 32 + n_local * 8 +
                                                         (blk & 1) * 4);
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[j] = fmaf((float)(int)d[j], sat[(hh * 32 + j) * 4 + blk] * sw, acc[j]);
      }
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&accfree[set]);
        mbar_arrive(&empty[s]);
      }
      return true;
    };
    for (int kb = 0; kb < nk && ok; ++kb) {
      const int s = kb % QNS;
      if (!mbar_wait(&full[s], (uint32_t)((kb / QNS) & 1), a.status)) {
        ok = false;
        break;
      }
      unsigned char* st = base + (size_t)s * kQStage;
      const unsigned char* raw = st + kQA + kQB + hf * kQBlk;
      const uint4 c0 = *reinterpret_cast<const uint4*>(raw + r * 32);
      const uint4 c1 = *reinterpret_cast<const uint4*>(raw + r * 32 + 16);
      const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
      for (int c = 0; c < 4; ++c) {   // 16 elements per 16-byte chunk
        uint32_t e0, e1, e2, e3;
        codes_to_s8(cw[2 * c], e0, e1);
        codes_to_s8(cw[2 * c + 1], e2, e3);
        *reinterpret_cast<uint4*>(st + sw128(r, hf * 4 + c)) = make_uint4(e0, e1, e2, e3);
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(&conv[s]);
      if (kb >= 1 && !drain(kb - 1)) {
        ok = false;
        break;
      }
    }
    if (ok && nk >= 1 && !drain(nk - 1)) ok = false;
  }

  // ---- epilogue ----
  if (__syncthreads_or(!ok)) {
    if (tid == 0) flag_error(a.status, kErrTimeout);
  }
  bool fin_ok = true;
  if (warp >= 2) {
    fin_ok = mbar_wait(&fin, 0u, a.status);
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  }
  const int failed = __syncthreads_or(!fin_ok || !ok);
  if (warp >= 2 && !failed) {
    const int n = n0 + n_local;
    if (n < a.N) {
      const float ri = a.rinv[n];
#pragma unroll
      for (int j = 0; j < QBN / 2; ++j) {
        const int m = m0 + hh * 32 + j;
        if (m < a.M) {
          float* yp = a.y + (size_t)m * a.ldy + n;
          float v = acc[j] * ri;
          if (EPI == kAdd) v += *yp;
          else if (EPI == kGelu) v = gelu_erf(v);
          *yp = v;
        }
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kQCols) : "memory");
}

cudaError_t init_attrs_w4a8_tc() {
  cudaError_t e = allow_smem(gemm_w4a8_tc_kernel<kStore>, kQBytes);
  if (e == cudaSuccess) e = allow_smem(gemm_w4a8_tc_kernel<kAdd>, kQBytes);
  if (e == cudaSuccess) e = allow_smem(gemm_w4a8_tc_kernel<kGelu>, kQBytes);
  return e;
}

bool w4a8_tc_fits(const WView& w, int M, int ldqa, int ldsa) {
  return w.fmt == kInt4 && M >= 128 && w.K % QK == 0 && ldqa % 16 == 0 && (ldsa * 4) % 16 == 0;
}

cudaError_t launch_matmul_w4a8_tc(const Launch& L, const WView& w, const GemmWeights& g, const int8_t* qa, int ldqa,
                                  const float* sa, int ldsa, int M, float* y, int ldy, int epi) {
  if (M <= 0) return cudaSuccess;
  if (!w4a8_tc_fits(w, M, ldqa, ldsa) || !g.wt || !g.rinv || !y) return cudaErrorInvalidValue;
  CUtensorMap tQ, tS;
  memset(&tQ, 0, sizeof(tQ));
  memset(&tS, 0, sizeof(tS));
  cudaError_t e = encode_map_2d(&tQ, CU_TENSOR_MAP_DATA_TYPE_UINT8, qa, (uint64_t)w.K, (uint64_t)M, (uint64_t)ldqa, QK,
                                QBN, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e == cudaSuccess)
    e = encode_map_2d(&tS, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, sa, (uint64_t)(w.K / 32), (uint64_t)M, (uint64_t)ldsa * 4,
                      4, QBN, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (e != cudaSuccess) return e;
  QArgs a;
  a.wt = g.wt;
  a.rinv = g.rinv;
  a.N = w.N;
  a.K = w.K;
  a.M = M;
  a.y = y;
  a.ldy = ldy;
  a.status = L.status;
  void (*k)(const QArgs, const CUtensorMap, const CUtensorMap) =
      epi == kAdd ? gemm_w4a8_tc_kernel<kAdd> : epi == kGelu ? gemm_w4a8_tc_kernel<kGelu> : gemm_w4a8_tc_kernel<kStore>;
  return launch_k(L, k, dim3((w.N + QM - 1) / QM, (M + QBN - 1) / QBN), dim3(kQThreads), kQBytes, a, tQ, tS);
}

}  // namespace ms
