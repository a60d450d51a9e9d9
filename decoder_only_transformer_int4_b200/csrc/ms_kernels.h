// Host-side launchers of the decoder kernels (internal to the library).
#pragma once
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ms {

// Bits of the per-cache device status word.
constexpr unsigned kErrTokenBit = 1u;    // a token id was outside [0, vocab) and was clamped
constexpr unsigned kErrTimeoutBit = 2u;  // a bounded wait ran out
constexpr unsigned kErrShapeBit = 4u;    // a device-side size check failed

enum WFmt { kInt4 = 0, kFp16 = 1 };
enum Epi { kStore = 0, kAdd = 1, kGelu = 2 };

// Where a kernel runs and what it reports into.
struct Launch {
  cudaStream_t stream;
  bool pdl;           // launch with programmatic stream serialisation
  unsigned* status;   // device status word (may be null)
};

// A backbone matrix [N][K] (row n = output feature n).  INT4: row n's nibbles start at
// q + n * ldq (bytes) and its K/32 scales at s + n * lds (floats).  The model keeps each
// row as [K/2 nibble bytes | K/32 fp32 scales] (ldq = 5K/8, s = q + K/2, lds = ldq / 4),
// so one contiguous copy moves a slice of rows with their scales; the single-operation
// entry points pass the C ABI's separate arrays (ldq = K/2, lds = K/32).  FP16: row n at
// h + n * K.
struct WView {
  const uint8_t* q;
  const float* s;
  const uint16_t* h;
  int N, K;
  int fmt;            // WFmt
  int ldq;            // bytes between INT4 rows
  int lds;            // floats between scale rows
  bool interleaved() const {
    return fmt == kInt4 && reinterpret_cast<const uint8_t*>(s) == q + K / 2 && lds * 4 == ldq;
  }
};

// Sets the message ms_last_error() returns on the calling thread.
void set_last_error(const char* msg);

// Opt every kernel that needs it into large dynamic shared memory on the current device.
cudaError_t init_attrs_gemv();

cudaError_t launch_quantize_int4(const float* w, int N, int K, uint8_t* packed, float* scales,
                                 cudaStream_t s);

// x[b][i] rows of a prefill: prefix rows then embedded tokens; tokens int64 [B][S].
cudaError_t launch_embed_prefill(const Launch& L, const int64_t* tokens, int S, const float* prefix,
                                 int P, const float* tok_emb, int V, int d, int B, float* x);
// x[b] = tok_emb[token[b]]; token from `tokens` (int32 [B]) or, if null, from
// hist[(len - 1) * B + b] with len read from `dlen`.
cudaError_t launch_embed_decode(const Launch& L, const int32_t* tokens, const int32_t* hist,
                                const int* dlen, const float* tok_emb, int V, int d, int B, float* x);

// x <- x + y (y may be null), h = LN(x) * g + b, per row.  h (fp32 [R][d]) may be null;
// with hh, the result is also written as fp16 hi / lo planes hh, hl [R][ldh] (the tcgen05
// GEMM's operand form).
cudaError_t launch_skipln(const Launch& L, float* x, const float* y, const float* g, const float* b,
                          float eps, int R, int d, float* h, __half* hh = nullptr, __half* hl = nullptr,
                          int ldh = 0);

// RoPE on the q and k parts of qkv rows (row r = b * n + i at position len + i, len read
// from dlen) and append post-RoPE k and v to the layer's cache slices.
// The cache elements are fp32, or IEEE halves with kv16 (every kernel that touches the cache
// takes the same flag).
cudaError_t launch_rope_append(const Launch& L, const float* qkv, int B, int n, int H, int Hk,
                               const float* cosv, const float* sinv, const int* dlen, float* q_out,
                               void* kc, void* vc, int cap, int kv16);

// Smallest-M path (decode): M <= 8.  Optional LayerNorm of x in the prologue (ln_g != null).
cudaError_t launch_gemv(const Launch& L, const WView& w, const float* x, int ldx, int M,
                        const float* ln_g, const float* ln_b, float eps, float* y, int ldy, int epi);
bool gemv_fits(const WView& w, int M);

// Launch policy of the tcgen05 GEMM: with gw, K is split over a cluster of CTAs per output
// tile when the tiles alone would leave SMs idle.
struct GemmWork {
  int sms;             // SMs of the device
};

// The warp-specialised tcgen05 GEMM on fp16 hi / lo operand planes (kind::f16, three
// products).  INT4 weights come from a tile-packed copy made once (launch_gemm_repack): per
// 128-row tile and 64-wide K stage, 128 x 32 bytes of codes then 128 x 2 scales, the scales
// of row n multiplied by 2^e_n, with rinv[n] = 2^-e_n; half weights are read in place.
struct GemmWeights {
  const unsigned char* wt;   // INT4 tile-packed blocks, gemm_tiles_bytes(w) bytes
  const float* rinv;         // [gemm_rows_padded(w)]
};
size_t gemm_tiles_bytes(const WView& w);
size_t gemm_rows_padded(const WView& w);
// rexp_scratch: gemm_rows_padded(w) floats of device memory.
cudaError_t launch_gemm_repack(const WView& w, GemmWeights& g, float* rexp_scratch, cudaStream_t s);
// y (fp32 [M][ldy], store / add / GELU) and / or yh, yl (fp16 planes [M][ldyh] of the result)
// from activation planes xh, xl [M][ldx] (ldx a multiple of 8, 16-byte aligned).
cudaError_t launch_gemm_f16(const Launch& L, const WView& w, const GemmWeights& g, const __half* xh,
                            const __half* xl, int ldx, int M, float* y, int ldy, __half* yh, __half* yl,
                            int ldyh, int epi, const GemmWork* gw);
// fp32 rows [M][ldx] -> planes xh, xl [M][ldh] (|v| >= 65504 flags kErrShapeBit).
cudaError_t launch_split_f16(const Launch& L, const float* x, int ldx, int M, int K, __half* xh, __half* xl,
                             int ldh);
cudaError_t init_attrs_gemm_f16();

// W4A8 (accuracy_level=4 reading): INT8 activation codes per 32-element block (q [M][ldq],
// scales [M][lds]) and the MatMul on them (dp4a GEMV for M in {1, 2, 4, 8}, dp4a tiled GEMM
// otherwise); INT4 weights only, K a multiple of 128, ldqa a multiple of 16.
cudaError_t launch_quantize_act_int8(const Launch& L, const float* x, int ldx, int M, int K, int8_t* q, int ldq,
                                     float* s, int lds);
cudaError_t launch_matmul_w4a8(const Launch& L, const WView& w, const int8_t* qa, int ldqa, const float* sa, int ldsa,
                               int M, float* y, int ldy, int epi, int sms);
cudaError_t init_attrs_w4a8();
// The same MatMul on tcgen05 (kind::i8, one int32 TMEM result per 32-wide block, scaled while
// the next stage's MMAs run) for M >= 128, reading the weights from the tcgen05 f16 GEMM's
// tile-packed copy (g); qa and sa 16-byte aligned, ldqa a multiple of 16, ldsa of 4.
bool w4a8_tc_fits(const WView& w, int M, int ldqa, int ldsa);
cudaError_t launch_matmul_w4a8_tc(const Launch& L, const WView& w, const GemmWeights& g, const int8_t* qa, int ldqa,
                                  const float* sa, int ldsa, int M, float* y, int ldy, int epi);
cudaError_t init_attrs_w4a8_tc();

// Causal prefill attention on the tensor cores (tcgen05, fp16 hi / lo operands, three products):
// q [B * n][H * 64] post-RoPE, the layer's cache slices, positions len .. len + n - 1 with len
// read from dlen; the result as fp32 rows o [B * n][H * 64] and / or fp16 hi / lo planes
// oh, ol [B * n][ldo] (ldo a multiple of 8).  H / Hk query heads per kv head, at most 128.
bool attn_prefill_tc_fits(int H, int Hk);
cudaError_t init_attrs_attn_tc();
cudaError_t launch_attn_prefill_tc(const Launch& L, const float* q, const void* kc, const void* vc, int B, int n,
                                   int H, int Hk, int cap, const int* dlen, float* o, __half* oh, __half* ol, int ldo,
                                   int kv16);

// Conditioner front-end: the log-mel spectrogram of centred, reflection-padded frames (one
// CTA per frame and stream, double-precision FFT), and the prefix rows after the projection.
constexpr int kCondMaxFft = 4096;
struct CondDev {
  const double* window;    // [n_fft]
  const double2* twiddle;  // [n_fft]: e^{-2 pi i k / n_fft}
  const int* band_lo;      // [n_mels]: first bin of band m's non-zero range
  const int* band_off;     // [n_mels + 1]: band m's weights are band_w[band_off[m] .. band_off[m+1])
  const float* band_w;
  int n_fft, hop, n_mels;
  int kp;                  // columns of the fp16 planes: n_mels rounded up to 64, zero-filled
};
size_t log_mel_smem_bytes(int n_fft);
cudaError_t init_attrs_cond();
// out (fp32 [B * frames][n_mels]) and / or the planes xh, xl ([B * frames][kp]); either may be null.
cudaError_t launch_log_mel(const Launch& L, const float* audio, int n_samples, int B, const CondDev& c, int frames,
                           float* out, __half* xh, __half* xl);
// prefix [B][frames + 1 + K][d]: y rows * yscale + bias, then ds_emb[dataset[b]], then
// inst_emb[instruments[b][k]] (ids out of range are clamped and flag kErrTokenBit).
cudaError_t launch_cond_assemble(const Launch& L, const float* y, float yscale, const float* bias,
                                 const float* ds_emb, int n_ds, const float* inst_emb, int n_inst,
                                 const int32_t* dataset, const int32_t* instruments, int K, int frames, int d, int B,
                                 float* prefix);

// Split-K decode attention over positions [0, len + add) of each (stream, kv head), with
// the combine done by the last CTA of each (stream, kv head); the result as fp32 rows o, or
// (oh set) as fp16 hi / lo planes [B][ldo] for the O GEMM.
struct AttnDecodeWork {
  float* part;        // [B][Hk][splits][hpg][66]
  unsigned* counters; // [B][Hk], zero between launches
  int splits;         // grid splits (max)
};
cudaError_t launch_attn_decode(const Launch& L, const float* q, const void* kc, const void* vc,
                               int B, int H, int Hk, int cap, const int* dlen, int add,
                               const AttnDecodeWork& w, float* o, int kv16, __half* oh = nullptr,
                               __half* ol = nullptr, int ldo = 0);
int attn_decode_splits(int B, int Hk, int cap);

// LM head + argmax over rows x[m * ldx], m < M.  Writes logits (may be null), argmax
// (may be null), hist[(len + hist_off) * B + m] (may be null) and, in its last CTA,
// *dlen += len_add.
struct LmHeadWork {
  float* part_val;    // [grid][64]
  int* part_idx;      // [grid][64]
  unsigned* counter;  // one word, zero between launches
};
// guidance != 0 (M even): rows (2p, 2p+1) are (conditional, unconditional) pairs and both
// take the argmax of u + guidance (k - u); logits stay per row.
cudaError_t launch_lm_head(const Launch& L, const float* x, int ldx, int M, int d, const float* ln_g,
                           const float* ln_b, float eps, const float* W, int V, float* logits,
                           int32_t* argmax, int32_t* hist, int hist_B, int hist_off, int* dlen,
                           int len_add, const LmHeadWork& w, float guidance = 0.f);
int lm_head_grid(int V);

// Tile-packed copy of a backbone matrix (records of 16 rows x 32 columns, laid out for the
// persistent decode kernel's warp MMAs); N % 16 == 0, K % 32 == 0, INT4 rows interleaved.
cudaError_t launch_repack_tiles(const WView& w, void* out, cudaStream_t s);
size_t tile_packed_bytes(const WView& w);

}  // namespace ms
