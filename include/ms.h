/*
 * ms.h — C ABI of the MuScriptor KV-cached INT4 decoder step on NVIDIA B200 (sm_100a).
 *
 * The decoder is the one the pages describe:
 *   - "MuScriptor small — ONNX conversion", section "muscriptor-small-lm.onnx": one
 *     branch-free call takes tokens [1,S], the conditioner prefix [1,P,d] (P = 0 after
 *     the first call) and the KV cache, and returns last-position logits [1,1393] and
 *     the grown cache; positions are implicit in the cache length.
 *   - "MuScriptor Medium — optimized W4A32 ONNX Runtime", section "Model variant":
 *     backbone MatMuls in symmetric RTN INT4 with group size 32, activations, KV cache,
 *     embeddings and LM head in fp32, a fixed-capacity cache shared in place between
 *     past and present; section "Quick smoke test": capacity chosen by the caller.
 *   - "MuScriptor — small (≈100M)" model card, "Model description": greedy (argmax)
 *     decoding; "Model variants": the three shapes.
 *
 * Conventions for every call:
 *   - Return value: MS_OK or an error code.  On error nothing was launched and no state
 *     changed, unless the description says otherwise; ms_last_error() gives a message
 *     for the calling thread.
 *   - "device" pointers are CUDA device memory of the model's device; "host" pointers
 *     are ordinary host memory; "any" pointers may be either (the library copies with
 *     cudaMemcpyDefault).  The caller keeps ownership of everything it passes in.
 *   - stream is a cudaStream_t passed as void* (NULL = the legacy default stream).  Calls
 *     that take a stream are asynchronous on it; device-side errors (a token id out of
 *     range, a wait that ran out) are recorded in a status word read by ms_device_status.
 *   - Calls on one ms_cache must not overlap on the GPU (they share its work buffers);
 *     different caches of one model may run on different streams.
 *
 * Error behaviour common to all calls: a NULL handle or required pointer gives
 * MS_ERR_INVALID_ARG; a size that does not fit the model or the cache gives MS_ERR_SHAPE;
 * a call that would grow the cache past its capacity gives MS_ERR_CACHE_FULL and changes
 * nothing; a failed CUDA runtime call gives MS_ERR_CUDA (the message names the call).
 */
#ifndef MS_H
#define MS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct ms_model ms_model;
typedef struct ms_cache ms_cache;

typedef enum {
  MS_OK = 0,
  MS_ERR_INVALID_ARG = 1,
  MS_ERR_SHAPE = 2,
  MS_ERR_CACHE_FULL = 3,
  MS_ERR_TOKEN_RANGE = 4,
  MS_ERR_OOM = 5,
  MS_ERR_CUDA = 6,
  MS_ERR_TIMEOUT = 7,
  MS_ERR_UNSUPPORTED = 8
} ms_status;

/* Backbone weight storage.  INT4_G32: the W4A32 page's format.  FP16: the same matrices
 * rounded to IEEE half ("MuScriptor for Core AI (.aimodel)", file table: the large model
 * with weights cast to half), fp32 accumulation. */
typedef enum { MS_W_INT4_G32 = 0, MS_W_FP16 = 1 } ms_weight_format;

/* Model shape.  head_dim must be 64; vocab is 1393 for MuScriptor but any value >= 1 is
 * accepted.  d_model must be a multiple of 256, d_ff a multiple of 256, n_heads a
 * multiple of n_kv_heads, n_heads * 64 a multiple of 256. */
typedef struct {
  int n_layers;
  int d_model;
  int n_heads;
  int n_kv_heads;
  int head_dim;
  int d_ff;
  int vocab;
  float rope_base; /* 1e4 */
  float ln_eps;    /* 1e-5 */
  int weight_format; /* ms_weight_format */
} ms_config;

/* One layer's weights ("any" pointers, copied at ms_model_create).
 * Matrix order in w/s/w16: 0 = fused QKV [(H + 2 Hk) * 64][d], 1 = O [d][H * 64],
 * 2 = FC1 [d_ff][d], 3 = FC2 [d][d_ff]; each matrix is [N][K] with row n = output
 * feature n.  INT4: w[i] is uint8 [N][K/2], nibble u = q + 8, element 2j in the low
 * nibble of byte j; s[i] is fp32 [N][K/32], one scale per 32 consecutive K elements.
 * FP16: w16[i] is IEEE half bits [N][K].  The unused format's pointers may be NULL. */
typedef struct {
  const float* ln1_g;
  const float* ln1_b;
  const float* ln2_g;
  const float* ln2_b;
  const uint8_t* w[4];
  const float* s[4];
  const uint16_t* w16[4];
} ms_layer_weights;

typedef struct {
  const float* tok_emb;  /* fp32 [vocab][d] */
  const float* lm_head;  /* fp32 [vocab][d], logits = LN_f(x) . lm_head^T */
  const float* ln_f_g;   /* fp32 [d] */
  const float* ln_f_b;   /* fp32 [d] */
  const ms_layer_weights* layers; /* host array of n_layers entries */
} ms_weights;

/* ---- INT4 quantiser -------------------------------------------------------------
 * Symmetric round-to-nearest INT4, group 32 along K ("MuScriptor Medium — optimized
 * W4A32 ONNX Runtime", Model variant): per group scale = absmax / 7 and
 * q = clamp(rint(w / scale), -7, 7), both divisions IEEE fp32, ties to even; an all-zero
 * group gets scale 0 and q = 0.  w: device fp32 [N][K] row-major; packed: device uint8
 * [N][K/2]; scales: device fp32 [N][K/32].  K must be a multiple of 32, N >= 1.
 * Asynchronous on stream. */
ms_status ms_quantize_int4_g32(const float* w, int N, int K, uint8_t* packed, float* scales,
                               void* stream);

/* ---- model -------------------------------------------------------------------------
 * Copies the weights to `device` in the library's own layout.  Synchronous.  Returns
 * MS_ERR_SHAPE for an unsupported shape, MS_ERR_OOM when device memory runs out. */
ms_status ms_model_create(const ms_config* cfg, const ms_weights* weights, int device,
                          ms_model** out);
ms_status ms_model_destroy(ms_model* model);
/* Bytes of device memory the model's weights occupy; 0 on NULL. */
size_t ms_model_weight_bytes(const ms_model* model);

/* Element format of the KV cache.  F32 is the pages' ("MuScriptor Medium — optimized W4A32
 * ONNX Runtime", Model variant: fp32 KV cache).  F16 stores each post-RoPE key and value as
 * its IEEE half (round to nearest even) and halves the bytes every decode step reads; all
 * arithmetic stays fp32 (the attention converts each half back to fp32). */
typedef enum { MS_KV_F32 = 0, MS_KV_F16 = 1 } ms_kv_format;

/* ---- cache -------------------------------------------------------------------------
 * A fixed-capacity fp32 KV cache for `batch` independent streams that advance together
 * (every call appends the same number of positions to each stream), plus the work
 * buffers one call needs.  Layout on the device: K and V each [L][batch][Hk][capacity][64].
 * Allocates device memory; length starts at 0.  Synchronous. */
ms_status ms_cache_create(ms_model* model, int batch, int capacity, ms_cache** out);
/* The same with the cache's element format (ms_kv_format); ms_cache_create is
 * ms_cache_create_ex(..., MS_KV_F32, ...).  MS_ERR_INVALID_ARG for an unknown format. */
ms_status ms_cache_create_ex(ms_model* model, int batch, int capacity, int kv_format, ms_cache** out);
/* The cache's element format (ms_kv_format), -1 on NULL. */
int ms_cache_kv_format(const ms_cache* cache);
ms_status ms_cache_reset(ms_cache* cache); /* length = 0; no device work */
int ms_cache_length(const ms_cache* cache);   /* positions held (host view), -1 on NULL */
int ms_cache_capacity(const ms_cache* cache); /* positions per stream, -1 on NULL */
int ms_cache_batch(const ms_cache* cache);    /* streams, -1 on NULL */
ms_status ms_cache_destroy(ms_cache* cache);
/* Bytes of K plus V for a cache of this shape (no allocation): 2 * L * batch * Hk *
 * capacity * 64 * 4.  For the medium model with Hk = 16 and capacity 2504 this is the
 * W4A32 page's "about 469.5 MiB". Returns 0 on an invalid argument. */
size_t ms_cache_kv_bytes(const ms_config* cfg, int batch, int capacity);
/* The same for a cache of the given element format (half the bytes for MS_KV_F16). */
size_t ms_cache_kv_bytes_ex(const ms_config* cfg, int batch, int capacity, int kv_format);

/* ---- one decoder call ----------------------------------------------------------------
 * Prefill: appends P prefix rows followed by S token rows to every stream (positions
 * len .. len + P + S - 1), then returns the logits of the last new position and their
 * argmax.  tokens: device int64 [batch][S] (S >= 0); prefix: device fp32 [batch][P][d]
 * or NULL with P = 0; P + S >= 1.  logits: device fp32 [batch][vocab] or NULL; argmax:
 * device int32 [batch] or NULL.  Token ids are device data: an id outside [0, vocab) is
 * clamped on the device and flagged in the status word (ms_device_status then returns
 * MS_ERR_TOKEN_RANGE).  MS_ERR_CACHE_FULL if len + P + S > capacity. */
ms_status ms_prefill(ms_model* model, ms_cache* cache, const int64_t* tokens, int S,
                     const float* prefix, int P, float* logits, int32_t* argmax, void* stream);

/* Decode step: appends one token per stream (device int32 [batch]; may alias the
 * previous call's argmax buffer) and returns the new position's logits and argmax
 * (either may be NULL).  The cache is updated in place. */
ms_status ms_decode_step(ms_model* model, ms_cache* cache, const int32_t* tokens, float* logits,
                         int32_t* argmax, void* stream);

/* Greedy loop: n_steps decode steps, each feeding the previous argmax back (the first
 * step takes the argmax of the last prefill or decode call on this cache).  out_tokens:
 * device int32 [n_steps][batch] receives every step's argmax; logits: device fp32
 * [batch][vocab] receives the last step's logits, or NULL.  On the persistent path it
 * runs up to 128 steps per kernel launch (the argmax feeds the next step on the device);
 * on the per-operation path it replays a CUDA graph of one step, captured on first use.
 * No host synchronisation either way. */
ms_status ms_generate(ms_model* model, ms_cache* cache, int n_steps, int32_t* out_tokens,
                      float* logits, void* stream);

/* Decode path for ms_decode_step and ms_generate on this cache: 0 = automatic (the
 * persistent kernel when it fits, else one kernel per operation), 1 = the persistent
 * kernel (MS_ERR_UNSUPPORTED when it does not fit: batch not 1, 2, 4 or 8, or its shared
 * memory does not fit), 2 = one kernel per operation.  Both compute the same decoder and
 * differ only in rounding: the persistent kernel's matrix products take each activation
 * as an exact fp16 pair hi + lo (22 significant bits, products exact, sums fp32), the
 * other path multiplies in fp32; their logits agree to about 1e-4.  Host state only. */
ms_status ms_cache_set_decode_path(ms_cache* cache, int path);
/* The path the next decode call will take: 1 persistent kernel, 2 one kernel per
 * operation; -1 on NULL. */
int ms_cache_decode_path(const ms_cache* cache);

/* Classifier-free guidance ("MuScriptor — small (≈100M)" model card, Model description:
 * generation with classifier-free guidance; the pages give no formula, this library reads it
 * as the usual u + scale (k - u)).  With scale != 0 the streams of the cache form pairs
 * (2p, 2p + 1) = (conditional, unconditional): every greedy choice — the argmax returned by
 * ms_prefill / ms_decode_step, recorded in the token history and fed back by ms_generate —
 * takes, for both streams of a pair, the lowest index maximising
 *     u[v] + scale * (k[v] - u[v]),  k = conditional logits, u = unconditional logits,
 * in fp32.  The logits returned stay each stream's own.  scale = 0 (the default) turns it
 * off.  MS_ERR_SHAPE for a non-zero scale on an odd batch, MS_ERR_INVALID_ARG for a
 * non-finite scale.  Host state only; applies to the next call. */
ms_status ms_cache_set_guidance(ms_cache* cache, float scale);
/* The current guidance scale (0 when off or on NULL). */
float ms_cache_guidance(const ms_cache* cache);

/* W4A8 ("MuScriptor Medium — optimized W4A32 ONNX Runtime", Model variant: MatMulNBits with
 * accuracy_level=4, activations quantised to INT8 at run time, INT32 accumulation).  With
 * on != 0 the four backbone MatMuls of every layer, in prefill and decode, take their fp32
 * input as INT8 codes: per 32-element block of a row, scale = absmax / 127 and
 * q = clamp(rint(x / scale), -127, 127) (fp32 IEEE divisions, ties to even; an all-zero block
 * has scale 0), the block's integer sum with the INT4 codes is exact and is multiplied by
 * both scales, the blocks summed in fp32.  (The page does not state the block or the rule;
 * this is the weight quantiser's rule at 127 levels.)  Attention, LayerNorm and the LM head
 * stay fp32.  Decoding then runs one kernel per operation (ms_cache_set_decode_path(1) is
 * refused).  MS_ERR_UNSUPPORTED for half weights or when the persistent path was requested.
 * Host state only; applies to the next call. */
ms_status ms_cache_set_act_int8(ms_cache* cache, int on);
/* 1 when INT8 activations are on, 0 when off, -1 on NULL. */
int ms_cache_act_int8(const ms_cache* cache);

/* Wait limits of the persistent decode kernel, for tests of its failure path.  No passage of
 * the pages corresponds to this call.  Every wait of that kernel (a stamped activation word
 * from another CTA, the grid barrier between steps) gives up after a limit, sets the timeout
 * bit of the status word (ms_device_status then returns MS_ERR_TIMEOUT) and makes every CTA
 * leave; the launch then returns with the cache's contents undefined (reset it or use
 * another cache).  polls: the limit in polls (0 restores the defaults, about ten seconds of
 * waiting).  stall (tests only, 0 in normal use): 1 makes the attention units wait for an
 * activation word that no phase writes, 2 makes the grid barrier wait for one arrival more
 * than the grid makes; either wait then runs out after `polls`.  Host state only; applies to
 * the next persistent launch on this cache.  MS_ERR_INVALID_ARG for a negative limit or an
 * unknown stall. */
ms_status ms_cache_set_wait_limits(ms_cache* cache, long long polls, int stall);

/* ---- cache transfer (host pointers, synchronous) --------------------------------------
 * Export in the pages' layout [L][batch][T][Hk][64] (T = current length);
 * import T positions in the same layout and set the length to T.  Always fp32 on the host: a
 * half-precision cache converts on the way (import rounds to nearest even). */
ms_status ms_cache_export(const ms_cache* cache, float* k, float* v);
ms_status ms_cache_import(ms_cache* cache, const float* k, const float* v, int T);

/* ---- status -------------------------------------------------------------------------
 * Synchronises `stream`, reads and clears the device-side status word of `cache` and
 * returns MS_ERR_TOKEN_RANGE or MS_ERR_TIMEOUT if a kernel recorded one, else MS_OK. */
ms_status ms_device_status(ms_cache* cache, void* stream);
/* Number of CUDA kernels the calls on this cache have launched so far: direct launches
 * plus, for every replay of a captured graph, the kernels in that graph.  Host counter,
 * no device work; 0 on NULL. */
uint64_t ms_cache_kernel_launches(const ms_cache* cache);
/* Message of the last error on the calling thread ("" if none). */
const char* ms_last_error(void);

/* ---- single operations (the kernels the calls above are made of) ----------------------
 * For kernel-level tests and for callers that assemble their own pipeline.  All
 * pointers are device pointers of the current device; all calls are asynchronous. */

/* One backbone MatMul ("MuScriptor Medium — optimized W4A32 ONNX Runtime", Model
 * variant: symmetric INT4 g32 weights, fp32 activations): y[m][n] = sum_k x[m][k] * W[n][k]
 * with W[n][k] = q[n][k] * s[n][k/32].  x fp32 [M][K] and y fp32 [M][N], row-major;
 * packed and scales as ms_quantize_int4_g32 writes them.  M in {1, 2, 4, 8} runs the
 * decode GEMV (fp32) when a CTA's slice of rows fits its shared memory; any other M runs the
 * tcgen05 GEMM (fp16 hi + lo operand pairs, three products, fp32 accumulation), after making
 * the weights' tile-packed copy and the activation planes in stream-ordered temporaries
 * (cudaMallocAsync / cudaFreeAsync on `stream`).  K a multiple of 256.  MS_ERR_INVALID_ARG
 * for a NULL pointer, MS_ERR_SHAPE for other sizes; nothing is launched then. */
ms_status ms_op_matmul_w4(const float* x, int M, int K, const uint8_t* packed, const float* scales,
                          int N, float* y, void* stream);
/* The same with IEEE half weights w16 [N][K] (the half-precision weight variant of
 * "MuScriptor for Core AI (.aimodel)", file table), same size rules. */
ms_status ms_op_matmul_f16(const float* x, int M, int K, const uint16_t* w16, int N, float* y,
                           void* stream);
/* The operand form of the tcgen05 GEMM: each fp32 value v of x (rows of K at stride ldx)
 * as an IEEE half pair, x_hi = fp16(v) and x_lo = fp16(v - x_hi) (round to nearest even,
 * a 22-bit significand together), written to x_hi and x_lo (rows at stride ldh halves).
 * K, ldx and ldh multiples of 4 (ldx, ldh >= K); x 16-byte aligned, the planes 8-byte
 * aligned.  A |v| of 65504 or more does not fit a half: the pair is then inf and the call
 * cannot report it (the calls of a cache flag it in the status word, MS_ERR_SHAPE). */
ms_status ms_op_split_f16(const float* x, int ldx, int M, int K, uint16_t* x_hi, uint16_t* x_lo, int ldh,
                          void* stream);

/* The INT8 activation codes of the W4A8 reading (see ms_cache_set_act_int8): x fp32 rows of K
 * at stride ldx -> q int8 [M][K] and scales fp32 [M][K/32].  K a multiple of 32. */
ms_status ms_op_quantize_act_int8(const float* x, int ldx, int M, int K, int8_t* q, float* scales, void* stream);
/* The W4A8 MatMul: y[m][n] = sum over blocks b of (sa[m][b] * s[n][b]) * (sum_{k in b}
 * qa[m][k] * q[n][k]), y fp32 [M][N]; qa, sa as ms_op_quantize_act_int8 writes them, packed
 * and scales as ms_quantize_int4_g32 writes them.  A dp4a GEMV for M in {1, 2, 4, 8}, a dp4a
 * tiled GEMM otherwise.  K a multiple of 128; qa and packed 16-byte aligned. */
ms_status ms_op_matmul_w4a8(const int8_t* qa, const float* sa, int M, int K, const uint8_t* packed,
                            const float* scales, int N, float* y, void* stream);

/* Backbone MatMul `which` (0 QKV, 1 O, 2 FC1, 3 FC2) of layer `layer` of the model, on M
 * activation rows given as ms_op_split_f16 planes (row stride ldx halves, a multiple of 8,
 * 16-byte aligned): y[m][n] = sum_k (x_hi + x_lo)[m][k] W[n][k], y fp32 [M][ldy].  This is
 * the tcgen05 GEMM the prefill and batched decode run ("MuScriptor Medium — optimized W4A32
 * ONNX Runtime", Model variant: MatMulNBits), with the model's own tile-packed weights.
 * MS_ERR_INVALID_ARG for no such matrix or a NULL pointer, MS_ERR_SHAPE for other sizes. */
ms_status ms_model_matmul(const ms_model* model, int layer, int which, const uint16_t* x_hi,
                          const uint16_t* x_lo, int ldx, int M, float* y, int ldy, void* stream);

/* SkipLayerNorm ("MuScriptor Medium — optimized W4A32 ONNX Runtime", Model variant):
 * s = x + y (y may be NULL: plain LayerNorm), x <- s, h = (s - mean) / sqrt(var + eps)
 * * gamma + beta with the biased variance, per row of d.  x, y, h fp32 [R][d]. */
ms_status ms_op_skip_layernorm(float* x, const float* y, const float* gamma, const float* beta,
                               float eps, int R, int d, float* h, void* stream);
/* LM head and greedy choice ("MuScriptor small — ONNX conversion", muscriptor-small-lm.onnx:
 * fp32 logits over the vocabulary; "MuScriptor — small (≈100M)" model card, Model
 * description: greedy argmax): logits[m][v] = LN(x_m) . W[v] (LN skipped when gamma and
 * beta are NULL), argmax[m] = lowest index of the largest logit.  x fp32 rows at stride
 * ldx floats (ldx >= d, a multiple of 4), W fp32 [V][d], d a multiple of 128, 1 <= M <= 64.
 * logits or argmax may be NULL.  The first call on a device allocates a scratch buffer
 * (ms_op_lm_head_argmax_static does not).  MS_ERR_INVALID_ARG for a NULL x or W or for
 * only one of gamma and beta, MS_ERR_SHAPE for other sizes.  The call is asynchronous, so
 * a device-side failure cannot change its return value: if the kernel's bounded wait for
 * its weight rows ran out, argmax[m] is -1 for every row (and those logits are unwritten). */
ms_status ms_op_lm_head_argmax(const float* x, int ldx, int M, int d, const float* gamma,
                               const float* beta, float eps, const float* W, int V, float* logits,
                               int32_t* argmax, void* stream);

/* The same LM head and greedy choice for callers that cannot allocate device memory.
 * No passage of the pages corresponds to this entry point; it exists for callers such as
 * code that runs while a CUDA stream is being captured into a graph (cudaMalloc is not
 * allowed there), code whose device memory is owned by another allocator that must see
 * every allocation, and latency-critical paths where an allocation could synchronise
 * the device.  ms_op_lm_head_argmax allocates a scratch buffer on its first call; this
 * variant instead uses a fixed scratch array compiled into the library (about 128 KiB:
 * per-CTA results for up to 256 CTAs and 64 rows, plus a counter), which every GPU that
 * loads the library holds until the process exits.  Arguments and results are those of
 * ms_op_lm_head_argmax.  Limits: M <= 64 and V small enough for 256 CTAs (always the
 * case for vocabularies that fit the kernel's shared memory); larger sizes return
 * MS_ERR_SHAPE with a message.  The first call on a device looks up the array's device
 * address (with that device current), so make that first call before any stream
 * capture.  Every call shares the one array and keeps the last call's contents; the
 * counter that must start at zero is cleared on the stream before each launch.  Calls
 * that overlap on the GPU (different streams, or different host threads) race on the
 * array: order them on one stream.  It calls no cudaMalloc or cudaFree.  A wait that ran
 * out on the device shows as argmax -1, as for ms_op_lm_head_argmax. */
ms_status ms_op_lm_head_argmax_static(const float* x, int ldx, int M, int d, const float* gamma,
                                      const float* beta, float eps, const float* W, int V,
                                      float* logits, int32_t* argmax, void* stream);

/* ---- conditioner front-end ------------------------------------------------------------
 * "MuScriptor small — ONNX conversion", the conditioner graph muscriptor-small-cond.onnx:
 * audio fp32 [1, N] at 16 kHz, instrument ids [1, K] and a dataset id -> the decoder's prefix
 * [1, frames + 1 + K, d]; the spectrogram is computed inside that graph from a window and a mel
 * filterbank stored with the checkpoint.  MuScriptor model card, Model description: STFT with
 * n_fft 2048 and hop 160, 512 mel bands, log features, a projection to d_model.
 * The conditioner computes, per stream b:
 *   frame t (t = 0 .. frames-1, frames = 1 + n_samples / hop) = samples t*hop - n_fft/2 ..
 *     t*hop + n_fft/2 - 1 of the signal extended by reflection at both ends (sample -i is
 *     sample i, sample N-1+i is sample N-1-i; the edge sample is not repeated), times window;
 *   mag[t][k] = |DFT(frame t)[k]|, k = 0 .. n_fft/2;
 *   logmel[t][m] = ln(max(sum_k mel_fb[m][k] * mag[t][k], 1e-6));
 *   prefix[b][t] = logmel[t] . proj_w^T + proj_b (t < frames);
 *   prefix[b][frames] = ds_emb[dataset[b]];  prefix[b][frames + 1 + k] = inst_emb[instruments[b][k]].
 * Which of these steps the pages leave open and how they are read here: centred frames with
 * reflection, the magnitude (not the power), the natural log, and the row order (frames,
 * dataset, instruments), which gives the decoder's 503 prefix rows for 501 frames and one
 * instrument.
 * Arithmetic: window, DFT, magnitudes, mel sums and log in double precision, rounded to fp32;
 * the projection on the tensor cores with the features and the weights each as an fp16 hi + lo
 * pair (the weights scaled by a power of two first) and fp32 accumulation; bias in fp32. */
typedef struct ms_cond ms_cond;

typedef struct {
  int n_samples;      /* audio samples per stream (80000: 5 s at 16 kHz); > n_fft / 2 */
  int n_fft;          /* a power of two, 16 .. 4096 (2048) */
  int hop;            /* frame step in samples, >= 1 (160) */
  int n_mels;         /* mel bands, 1 .. 4096 (512) */
  int d_model;        /* width of the prefix rows (the decoder's d_model), a multiple of 4 */
  int n_instruments;  /* rows of the instrument table, >= 1 (130) */
  int n_datasets;     /* rows of the dataset table, >= 1 (2) */
  int max_batch;      /* most streams one call may take, >= 1 (work buffers are sized for it) */
} ms_cond_config;

typedef struct {              /* host or device pointers; copied at create; caller keeps ownership */
  const float* window;        /* [n_fft] */
  const float* mel_fb;        /* [n_mels][n_fft/2 + 1], row m = band m's weight of each bin */
  const float* proj_w;        /* [d_model][n_mels] */
  const float* proj_b;        /* [d_model] */
  const float* inst_emb;      /* [n_instruments][d_model] */
  const float* ds_emb;        /* [n_datasets][d_model] */
} ms_cond_weights;

/* Copies the weights to `device` and allocates the work buffers for max_batch streams
 * (about max_batch * frames * (4 * n_mels + 4 * d_model) bytes).  MS_ERR_INVALID_ARG for NULL
 * pointers or a config outside the ranges above, MS_ERR_OOM, MS_ERR_CUDA. */
ms_status ms_cond_create(const ms_cond_config* cfg, const ms_cond_weights* w, int device, ms_cond** out);
ms_status ms_cond_destroy(ms_cond* cond);
/* frames = 1 + n_samples / hop (501 for 5 s at 16 kHz and hop 160); 0 on NULL. */
int ms_cond_frames(const ms_cond* cond);
/* The prefix of B streams (1 <= B <= max_batch): audio fp32 [B][n_samples], dataset int32 [B],
 * instruments int32 [B][K] (K >= 0; may be NULL when K = 0) -> prefix fp32
 * [B][frames + 1 + K][d_model], 16-byte aligned.  Device pointers of the cond's device;
 * asynchronous on `stream`.  An id outside its table is clamped on the device and flagged:
 * ms_cond_device_status then returns MS_ERR_TOKEN_RANGE.  Calls on one cond share its work
 * buffers: order them on one stream. */
ms_status ms_condition(ms_cond* cond, const float* audio, int B, const int32_t* dataset,
                       const int32_t* instruments, int K, float* prefix, void* stream);
/* The log-mel features alone: audio fp32 [B][n_samples] -> out fp32 [B][frames][n_mels]. */
ms_status ms_cond_log_mel(ms_cond* cond, const float* audio, int B, float* out, void* stream);
/* Synchronises `stream`, reads and clears the cond's device status word. */
ms_status ms_cond_device_status(ms_cond* cond, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MS_H */
