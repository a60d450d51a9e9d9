// Host runtime of the C ABI in include/ms.h: owns the device copy of the weights, the
// fixed-capacity KV cache and its work buffers, and sequences the kernels of one
// decoder call (prefill, decode step, greedy loop from a captured CUDA graph).
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <cmath>
#include <mutex>
#include <new>
#include <string>
#include <vector>

#include "../../include/ms.h"
#include "ms_kernels.h"
#include "ms_launch.cuh"
#include "ms_persistent.h"

namespace ms {
std::atomic<unsigned long long>& launch_counter() {
  static std::atomic<unsigned long long> n{0};
  return n;
}
}  // namespace ms

namespace {

thread_local std::string g_err;

ms_status fail(ms_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return s;
}

#define CUDA_TRY(call)                                                              \
  do {                                                                              \
    cudaError_t e_ = (call);                                                        \
    if (e_ != cudaSuccess) {                                                        \
      if (e_ == cudaErrorMemoryAllocation) {                                        \
        cudaGetLastError();                                                         \
        return fail(MS_ERR_OOM, "%s: %s", #call, cudaGetErrorString(e_));           \
      }                                                                             \
      return fail(MS_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_));            \
    }                                                                               \
  } while (0)

// Makes `dev` current for the duration of a call and restores the caller's device.
struct DeviceGuard {
  int prev = -1;
  bool ok = true;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
    if (prev != dev) ok = cudaSetDevice(dev) == cudaSuccess;
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Bump allocator over one cudaMalloc'd arena (256-byte aligned pieces).
struct Arena {
  char* base = nullptr;
  size_t size = 0, used = 0;
  template <typename T>
  T* take(size_t count) {
    size_t off = round_up(used, 256);
    used = off + count * sizeof(T);
    return base ? reinterpret_cast<T*>(base + off) : nullptr;
  }
};

struct DevLayer {
  float *ln1_g, *ln1_b, *ln2_g, *ln2_b;
  ms::WView w[4];
  uint8_t* wt[4];  // tile-packed copies for the persistent decode kernel
  ms::GemmWeights gw[4];  // tile-packed INT4 copies for the tcgen05 GEMM (prefill, batched decode)
};

bool shape_ok(const ms_config* c, std::string* why) {
  char b[256];
  auto bad = [&](const char* m) {
    snprintf(b, sizeof(b), "%s", m);
    *why = b;
    return false;
  };
  if (c->n_layers < 0) return bad("n_layers < 0");
  if (c->head_dim != 64) return bad("head_dim must be 64");
  if (c->d_model <= 0 || c->d_model % 256 != 0) return bad("d_model must be a positive multiple of 256");
  if (c->d_model > 2048) return bad("d_model above 2048 is not supported");
  if (c->d_ff <= 0 || c->d_ff % 256 != 0) return bad("d_ff must be a positive multiple of 256");
  if (c->n_heads <= 0 || c->n_kv_heads <= 0 || c->n_heads % c->n_kv_heads != 0)
    return bad("n_heads must be a positive multiple of n_kv_heads");
  const int hpg = c->n_heads / c->n_kv_heads;
  if (hpg != 1 && hpg != 2 && hpg != 3 && hpg != 4 && hpg != 6 && hpg != 8)
    return bad("n_heads / n_kv_heads must be 1, 2, 3, 4, 6 or 8");
  if ((c->n_heads * 64) % 256 != 0) return bad("n_heads * 64 must be a multiple of 256");
  if (c->vocab < 1) return bad("vocab < 1");
  if (c->weight_format != MS_W_INT4_G32 && c->weight_format != MS_W_FP16) return bad("unknown weight_format");
  if (!(c->ln_eps > 0.f) || !(c->rope_base > 0.f)) return bad("ln_eps and rope_base must be positive");
  return true;
}

void mat_nk(const ms_config& c, int i, int* N, int* K) {
  const int d = c.d_model, H = c.n_heads, Hk = c.n_kv_heads, F = c.d_ff;
  switch (i) {
    case 0: *N = (H + 2 * Hk) * 64; *K = d; break;
    case 1: *N = d; *K = H * 64; break;
    case 2: *N = F; *K = d; break;
    default: *N = d; *K = F; break;
  }
}

// Library-owned scratch for the single-operation entry points (per device).
struct OpScratch {
  float* part_val = nullptr;
  int* part_idx = nullptr;
  unsigned* counter = nullptr;
};
std::mutex g_scratch_mu;
std::vector<OpScratch> g_scratch;

// Kernel attributes are set once per device, outside any stream capture.
std::mutex g_attr_mu;
std::vector<char> g_attr_done;

cudaError_t ensure_kernel_attributes() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(g_attr_mu);
  if ((int)g_attr_done.size() <= dev) g_attr_done.resize(dev + 1, 0);
  if (g_attr_done[dev]) return cudaSuccess;
  e = ms::init_attrs_gemv();
  if (e == cudaSuccess) e = ms::init_attrs_persistent();
  if (e == cudaSuccess) e = ms::init_attrs_gemm_f16();
  if (e == cudaSuccess) e = ms::init_attrs_w4a8();
  if (e == cudaSuccess) e = ms::init_attrs_cond();
  if (e == cudaSuccess) e = ms::init_attrs_attn_tc();
  if (e == cudaSuccess) e = ms::init_attrs_w4a8_tc();
  if (e == cudaSuccess) g_attr_done[dev] = 1;
  return e;
}

}  // namespace

namespace ms {
void set_last_error(const char* msg) { g_err = msg; }
}  // namespace ms

struct ms_model {
  ms_config cfg;
  int device = 0;
  Arena arena;
  float *tok_emb = nullptr, *lm_head = nullptr, *ln_f_g = nullptr, *ln_f_b = nullptr;
  std::vector<DevLayer> layers;
  ms::PLayer* d_players = nullptr;  // the same pointers, on the device, for the persistent kernel
  float* rexp = nullptr;             // per-row powers of two while the GEMM copies are made
};

struct ms_cache {
  ms_model* m = nullptr;
  int B = 0, cap = 0, len = 0;
  bool has_next = false;  // hist holds the argmax of position len - 1
  Arena arena;
  void *k = nullptr, *v = nullptr;         // [L][B][Hk][cap][64] fp32, or IEEE half with kv16
  int kv16 = 0;                            // the cache holds IEEE halves
  float *cosv = nullptr, *sinv = nullptr;  // [cap][32]
  int* dlen = nullptr;
  int32_t* hist = nullptr;                 // [cap][B]
  unsigned* status = nullptr;
  unsigned* att_counters = nullptr;        // [B][Hk]
  float* att_part = nullptr;
  int splits = 1;
  float* lm_val = nullptr;
  int* lm_idx = nullptr;
  unsigned* lm_counter = nullptr;
  float *x = nullptr, *h = nullptr, *y = nullptr, *qkv = nullptr, *q = nullptr, *o = nullptr, *u = nullptr;
  __half *hh = nullptr, *hl = nullptr;     // GEMM operand planes [rows][kh] (LayerNorm or attention output)
  __half *uh = nullptr, *ul = nullptr;     // FC1's GELU output as planes [rows][d_ff] (they share u's memory)
  int kh = 0;                              // row stride of hh / hl: max(d, H * 64)
  int act_int8 = 0;                        // W4A8: backbone MatMuls on INT8 activation codes
  int8_t* qa = nullptr;                    // INT8 activation codes [rows][ka]
  float* sa = nullptr;                     // their block scales [rows][ka / 32]
  int ka = 0;                              // max(d, H * 64, d_ff)
  float* logits = nullptr;                 // [B][V] internal
  size_t rows_cap = 0;
  cudaGraphExec_t gen_exec = nullptr;
  size_t gen_nodes = 0;
  cudaStream_t gen_stream = nullptr;     // used when the caller passes the legacy stream
  cudaEvent_t ev_in = nullptr, ev_out = nullptr;
  // persistent decode kernel
  unsigned* sync3 = nullptr;             // grid barrier count, completed epoch, abort word
  uint64_t* vs[4] = {nullptr, nullptr, nullptr, nullptr};
  long long vstride[4] = {0, 0, 0, 0};
  uint64_t *o_s = nullptr, *part_s = nullptr;
  size_t stamp_bytes = 0;                // the five stamped vectors, contiguous
  unsigned epoch_next = 0;               // first unused epoch of the stamped vectors
  int persist_grid = 0, persist_nslot = 0;
  size_t persist_smem = 0;
  int persist_sched_cap = 0;
  float guidance = 0.f;              // classifier-free guidance scale (0: off)
  long long wait_limit = 0;          // persistent kernel's wait limits (0: the defaults)
  int test_stall = 0;                // tests only: an injected wait nothing satisfies
  int nsm = 148;                     // SMs of the device
  int path_request = 0;                  // 0 auto, 1 persistent kernel, 2 one kernel per operation
  unsigned long long launches = 0;  // kernels launched for this cache
};

namespace {

size_t layer_stride(const ms_cache* c) {
  return (size_t)c->B * c->m->cfg.n_kv_heads * c->cap * 64;
}

ms::Launch launch_of(ms_cache* c, cudaStream_t s, bool pdl) { return ms::Launch{s, pdl, c->status}; }

// Layer l of a cache buffer (K or V): fp32 or half elements.
void* kv_layer(const ms_cache* c, void* base, int l) {
  return static_cast<char*>(base) + (size_t)l * layer_stride(c) * (c->kv16 ? sizeof(__half) : sizeof(float));
}

// W4A8: quantise fp32 rows x [R][ldx] (K columns) to the cache's INT8 codes, then MatMul i.
cudaError_t w4a8(const ms::Launch& L, ms_cache* c, const ms::WView& w, const ms::GemmWeights& g, const float* x, int ldx,
                 int R, float* y, int ldy, int epi) {
  cudaError_t e = ms::launch_quantize_act_int8(L, x, ldx, R, w.K, c->qa, c->ka, c->sa, c->ka / 32);
  if (e != cudaSuccess) return e;
  if (g.wt && ms::w4a8_tc_fits(w, R, c->ka, c->ka / 32))
    return ms::launch_matmul_w4a8_tc(L, w, g, c->qa, c->ka, c->sa, c->ka / 32, R, y, ldy, epi);
  return ms::launch_matmul_w4a8(L, w, c->qa, c->ka, c->sa, c->ka / 32, R, y, ldy, epi, c->nsm);
}

// ---- one decoder call, kernel by kernel ----------------------------------------------
// Prefill of n = P + S rows per stream.  Rows of stream b are b * n + i.
cudaError_t run_prefill(ms_model* m, ms_cache* c, const int64_t* tokens, int S, const float* prefix, int P,
                        float* logits, int32_t* argmax, cudaStream_t st) {
  const ms::GemmWork gw{c->nsm};
  const ms_config& g = m->cfg;
  const int n = P + S, B = c->B, R = B * n, d = g.d_model, H = g.n_heads, Hk = g.n_kv_heads;
  const int nq = (H + 2 * Hk) * 64;
  ms::Launch L0 = launch_of(c, st, false), L = launch_of(c, st, true);
  cudaError_t e = ms::launch_embed_prefill(L0, tokens, S, prefix, P, m->tok_emb, g.vocab, d, B, c->x);
  const int kh = c->kh, F = g.d_ff;
  for (int l = 0; l < g.n_layers && e == cudaSuccess && c->act_int8; ++l) {
    // W4A8: each backbone MatMul on the INT8 codes of its fp32 input
    const DevLayer& ly = m->layers[l];
    void* kc = kv_layer(c, c->k, l);
    void* vc = kv_layer(c, c->v, l);
    if (e == cudaSuccess) e = ms::launch_skipln(L, c->x, l == 0 ? nullptr : c->y, ly.ln1_g, ly.ln1_b, g.ln_eps, R, d, c->h);
    if (e == cudaSuccess) e = w4a8(L, c, ly.w[0], ly.gw[0], c->h, d, R, c->qkv, nq, ms::kStore);
    if (e == cudaSuccess)
      e = ms::launch_rope_append(L, c->qkv, B, n, H, Hk, c->cosv, c->sinv, c->dlen, c->q, kc, vc, c->cap, c->kv16);
    if (e == cudaSuccess)
      e = ms::launch_attn_prefill_tc(L, c->q, kc, vc, B, n, H, Hk, c->cap, c->dlen, c->o, nullptr, nullptr, 0, c->kv16);
    if (e == cudaSuccess) e = w4a8(L, c, ly.w[1], ly.gw[1], c->o, H * 64, R, c->y, d, ms::kStore);
    if (e == cudaSuccess) e = ms::launch_skipln(L, c->x, c->y, ly.ln2_g, ly.ln2_b, g.ln_eps, R, d, c->h);
    if (e == cudaSuccess) e = w4a8(L, c, ly.w[2], ly.gw[2], c->h, d, R, c->u, F, ms::kGelu);
    if (e == cudaSuccess) e = w4a8(L, c, ly.w[3], ly.gw[3], c->u, F, R, c->y, d, ms::kStore);
  }
  for (int l = 0; l < g.n_layers && e == cudaSuccess && !c->act_int8; ++l) {
    const DevLayer& ly = m->layers[l];
    void* kc = kv_layer(c, c->k, l);
    void* vc = kv_layer(c, c->v, l);
    // LN1 -> planes -> QKV -> RoPE + append -> attention -> planes -> O -> SkipLN2 -> planes
    // -> FC1 + GELU -> planes -> FC2
    if (e == cudaSuccess)
      e = ms::launch_skipln(L, c->x, l == 0 ? nullptr : c->y, ly.ln1_g, ly.ln1_b, g.ln_eps, R, d, nullptr, c->hh, c->hl,
                            kh);
    if (e == cudaSuccess)
      e = ms::launch_gemm_f16(L, ly.w[0], ly.gw[0], c->hh, c->hl, kh, R, c->qkv, nq, nullptr, nullptr, 0, ms::kStore, &gw);
    if (e == cudaSuccess)
      e = ms::launch_rope_append(L, c->qkv, B, n, H, Hk, c->cosv, c->sinv, c->dlen, c->q, kc, vc, c->cap, c->kv16);
    if (e == cudaSuccess)
      e = ms::launch_attn_prefill_tc(L, c->q, kc, vc, B, n, H, Hk, c->cap, c->dlen, nullptr, c->hh, c->hl, kh, c->kv16);
    if (e == cudaSuccess)
      e = ms::launch_gemm_f16(L, ly.w[1], ly.gw[1], c->hh, c->hl, kh, R, c->y, d, nullptr, nullptr, 0, ms::kStore, &gw);
    if (e == cudaSuccess)
      e = ms::launch_skipln(L, c->x, c->y, ly.ln2_g, ly.ln2_b, g.ln_eps, R, d, nullptr, c->hh, c->hl, kh);
    if (e == cudaSuccess)
      e = ms::launch_gemm_f16(L, ly.w[2], ly.gw[2], c->hh, c->hl, kh, R, nullptr, 0, c->uh, c->ul, F, ms::kGelu, &gw);
    if (e == cudaSuccess)
      e = ms::launch_gemm_f16(L, ly.w[3], ly.gw[3], c->uh, c->ul, F, R, c->y, d, nullptr, nullptr, 0, ms::kStore, &gw);
  }
  if (e == cudaSuccess)
    e = ms::launch_skipln(L, c->x, g.n_layers > 0 ? c->y : nullptr, m->ln_f_g, m->ln_f_b, g.ln_eps, R, d, c->h);
  ms::LmHeadWork w{c->lm_val, c->lm_idx, c->lm_counter};
  if (e == cudaSuccess)
    e = ms::launch_lm_head(L, c->h + (size_t)(n - 1) * d, n * d, B, d, nullptr, nullptr, g.ln_eps, m->lm_head, g.vocab,
                           logits, argmax, c->hist, B, n - 1, c->dlen, n, w, c->guidance);
  return e;
}

// One decode step: one row per stream.  tokens == nullptr reads the previous argmax from
// the cache's token history (the greedy loop).
cudaError_t run_decode(ms_model* m, ms_cache* c, const int32_t* tokens, float* logits, int32_t* argmax,
                       cudaStream_t st, bool first_pdl) {
  const ms::GemmWork gw{c->nsm};
  const ms_config& g = m->cfg;
  const int B = c->B, d = g.d_model, H = g.n_heads, Hk = g.n_kv_heads, F = g.d_ff;
  const int nq = (H + 2 * Hk) * 64;
  ms::Launch L0 = launch_of(c, st, first_pdl), L = launch_of(c, st, true);
  const bool small = (B == 1 || B == 2 || B == 4 || B == 8);
  ms::AttnDecodeWork aw{c->att_part, c->att_counters, c->splits};
  cudaError_t e = ms::launch_embed_decode(L0, tokens, c->hist, c->dlen, m->tok_emb, g.vocab, d, B, c->x);
  for (int l = 0; l < g.n_layers && e == cudaSuccess; ++l) {
    const DevLayer& ly = m->layers[l];
    void* kc = kv_layer(c, c->k, l);
    void* vc = kv_layer(c, c->v, l);
    const bool gv = small && ms::gemv_fits(ly.w[0], B) && ms::gemv_fits(ly.w[1], B) && ms::gemv_fits(ly.w[2], B) &&
                    ms::gemv_fits(ly.w[3], B);
    if (c->act_int8) {
      // W4A8: each backbone MatMul on the INT8 codes of its fp32 input
      e = ms::launch_skipln(L, c->x, nullptr, ly.ln1_g, ly.ln1_b, g.ln_eps, B, d, c->h);
      if (e == cudaSuccess) e = w4a8(L, c, ly.w[0], ly.gw[0], c->h, d, B, c->qkv, nq, ms::kStore);
      if (e == cudaSuccess)
        e = ms::launch_rope_append(L, c->qkv, B, 1, H, Hk, c->cosv, c->sinv, c->dlen, c->q, kc, vc, c->cap, c->kv16);
      if (e == cudaSuccess)
        e = ms::launch_attn_decode(L, c->q, kc, vc, B, H, Hk, c->cap, c->dlen, 1, aw, c->o, c->kv16);
      if (e == cudaSuccess) e = w4a8(L, c, ly.w[1], ly.gw[1], c->o, H * 64, B, c->x, d, ms::kAdd);
      if (e == cudaSuccess) e = ms::launch_skipln(L, c->x, nullptr, ly.ln2_g, ly.ln2_b, g.ln_eps, B, d, c->h);
      if (e == cudaSuccess) e = w4a8(L, c, ly.w[2], ly.gw[2], c->h, d, B, c->u, F, ms::kGelu);
      if (e == cudaSuccess) e = w4a8(L, c, ly.w[3], ly.gw[3], c->u, F, B, c->x, d, ms::kAdd);
      continue;
    }
    if (gv) {
      e = ms::launch_gemv(L, ly.w[0], c->x, d, B, ly.ln1_g, ly.ln1_b, g.ln_eps, c->qkv, nq, ms::kStore);
    } else {
      e = ms::launch_skipln(L, c->x, nullptr, ly.ln1_g, ly.ln1_b, g.ln_eps, B, d, nullptr, c->hh, c->hl, c->kh);
      if (e == cudaSuccess)
        e = ms::launch_gemm_f16(L, ly.w[0], ly.gw[0], c->hh, c->hl, c->kh, B, c->qkv, nq, nullptr, nullptr, 0, ms::kStore,
                                &gw);
    }
    if (e == cudaSuccess)
      e = ms::launch_rope_append(L, c->qkv, B, 1, H, Hk, c->cosv, c->sinv, c->dlen, c->q, kc, vc, c->cap, c->kv16);
    if (e == cudaSuccess)
      e = ms::launch_attn_decode(L, c->q, kc, vc, B, H, Hk, c->cap, c->dlen, 1, aw, c->o, c->kv16, gv ? nullptr : c->hh,
                                 gv ? nullptr : c->hl, c->kh);
    if (gv) {
      if (e == cudaSuccess) e = ms::launch_gemv(L, ly.w[1], c->o, H * 64, B, nullptr, nullptr, 0.f, c->x, d, ms::kAdd);
      if (e == cudaSuccess) e = ms::launch_gemv(L, ly.w[2], c->x, d, B, ly.ln2_g, ly.ln2_b, g.ln_eps, c->u, F, ms::kGelu);
      if (e == cudaSuccess) e = ms::launch_gemv(L, ly.w[3], c->u, F, B, nullptr, nullptr, 0.f, c->x, d, ms::kAdd);
    } else {
      if (e == cudaSuccess)
        e = ms::launch_gemm_f16(L, ly.w[1], ly.gw[1], c->hh, c->hl, c->kh, B, c->x, d, nullptr, nullptr, 0, ms::kAdd, &gw);
      if (e == cudaSuccess)
        e = ms::launch_skipln(L, c->x, nullptr, ly.ln2_g, ly.ln2_b, g.ln_eps, B, d, nullptr, c->hh, c->hl, c->kh);
      if (e == cudaSuccess)
        e = ms::launch_gemm_f16(L, ly.w[2], ly.gw[2], c->hh, c->hl, c->kh, B, nullptr, 0, c->uh, c->ul, F, ms::kGelu, &gw);
      if (e == cudaSuccess)
        e = ms::launch_gemm_f16(L, ly.w[3], ly.gw[3], c->uh, c->ul, F, B, c->x, d, nullptr, nullptr, 0, ms::kAdd, &gw);
    }
  }
  ms::LmHeadWork w{c->lm_val, c->lm_idx, c->lm_counter};
  if (e == cudaSuccess)
    e = ms::launch_lm_head(L, c->x, d, B, d, m->ln_f_g, m->ln_f_b, g.ln_eps, m->lm_head, g.vocab, logits, argmax,
                           c->hist, B, 0, c->dlen, 1, w, c->guidance);
  return e;
}

bool use_persistent(const ms_cache* c) {
  if (c->path_request == 2 || c->act_int8) return false;
  return c->persist_grid > 0;
}

// n_steps greedy steps in one launch of the persistent kernel.  tokens: the first step's
// tokens (device int32 [B]) or null to continue from the token history.
cudaError_t run_persistent(ms_model* m, ms_cache* c, const int32_t* tokens, int n_steps, float* logits,
                           int32_t* argmax, cudaStream_t st) {
  const ms_config& g = m->cfg;
  cudaError_t e = cudaMemsetAsync(c->sync3, 0, 3 * sizeof(unsigned), st);
  // the last-CTA ticket of the LM head starts at zero (a launch that gave up may have left it set)
  if (e == cudaSuccess) e = cudaMemsetAsync(c->lm_counter, 0, sizeof(unsigned), st);
  if (e != cudaSuccess) return e;
  // epochs of the stamped vectors: fresh for every launch; restart from zeroed words
  // before the 32-bit counter would wrap
  const unsigned long long need = (unsigned long long)n_steps * 5ull * (unsigned long long)g.n_layers + 2ull;
  if ((unsigned long long)c->epoch_next + need >= 0xFFFFFFF0ull) {
    e = cudaMemsetAsync(c->vs[0], 0, c->stamp_bytes, st);
    if (e != cudaSuccess) return e;
    c->epoch_next = 0;
  }
  ms::PersistArgs a;
  a.L = g.n_layers;
  a.d = g.d_model;
  a.H = g.n_heads;
  a.Hk = g.n_kv_heads;
  a.F = g.d_ff;
  a.V = g.vocab;
  a.fmt = g.weight_format == MS_W_FP16 ? ms::kFp16 : ms::kInt4;
  a.eps = g.ln_eps;
  a.tok_emb = m->tok_emb;
  a.lm_head = m->lm_head;
  a.lnf_g = m->ln_f_g;
  a.lnf_b = m->ln_f_b;
  a.layers = m->d_players;
  a.cap = c->cap;
  a.kc = c->k;
  a.vc = c->v;
  a.kv16 = c->kv16;
  a.layer_stride = layer_stride(c);
  a.cosv = c->cosv;
  a.sinv = c->sinv;
  a.dlen = c->dlen;
  a.hist = c->hist;
  a.status = c->status;
  for (int i = 0; i < 4; ++i) {
    a.vs[i] = c->vs[i];
    a.vstride[i] = c->vstride[i];
  }
  a.o_s = c->o_s;
  a.epoch_base = c->epoch_next;
  c->epoch_next += (unsigned)need;
  a.part_s = c->part_s;
  a.att_splits = c->splits;
  a.lm_val = c->lm_val;
  a.lm_idx = c->lm_idx;
  a.lm_counter = c->lm_counter;
  a.bar_count = c->sync3;
  a.bar_flag = c->sync3 + 1;
  a.abort = c->sync3 + 2;
  a.tokens_in = tokens;
  a.logits = logits;
  a.argmax_out = argmax;
  a.n_steps = n_steps;
  a.nslot = c->persist_nslot;
  a.sched_cap = c->persist_sched_cap;
  a.guidance = c->guidance;
  a.settle_limit = c->wait_limit > 0 ? c->wait_limit : ms::kDefaultSettleLimit;
  a.grid_limit = c->wait_limit > 0 ? c->wait_limit : ms::kDefaultGridLimit;
  a.test_stall = c->test_stall;
  return ms::launch_decode_persistent(a, c->B, c->persist_grid, c->persist_smem, st);
}

ms_status check_launch(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return MS_OK;
  return fail(MS_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

}  // namespace

// =====================================================================================
// C ABI
// =====================================================================================
extern "C" {

const char* ms_last_error(void) { return g_err.c_str(); }

ms_status ms_quantize_int4_g32(const float* w, int N, int K, uint8_t* packed, float* scales, void* stream) {
  if (!w || !packed || !scales) return fail(MS_ERR_INVALID_ARG, "ms_quantize_int4_g32: null pointer");
  if (N < 1 || K < 32 || K % 32 != 0) return fail(MS_ERR_SHAPE, "ms_quantize_int4_g32: need N >= 1 and K a multiple of 32");
  if ((reinterpret_cast<uintptr_t>(w) & 15) || (reinterpret_cast<uintptr_t>(packed) & 15))
    return fail(MS_ERR_INVALID_ARG, "ms_quantize_int4_g32: w and packed must be 16-byte aligned");
  return check_launch(ms::launch_quantize_int4(w, N, K, packed, scales, (cudaStream_t)stream), "quantize kernel");
}

size_t ms_cache_kv_bytes(const ms_config* cfg, int batch, int capacity) {
  return ms_cache_kv_bytes_ex(cfg, batch, capacity, MS_KV_F32);
}

size_t ms_cache_kv_bytes_ex(const ms_config* cfg, int batch, int capacity, int kv_format) {
  if (!cfg || batch < 1 || capacity < 1 || cfg->n_layers < 0 || cfg->n_kv_heads < 1) return 0;
  if (kv_format != MS_KV_F32 && kv_format != MS_KV_F16) return 0;
  const size_t es = kv_format == MS_KV_F16 ? 2 : 4;
  return (size_t)2 * cfg->n_layers * batch * cfg->n_kv_heads * (size_t)capacity * 64 * es;
}

ms_status ms_model_create(const ms_config* cfg, const ms_weights* wt, int device, ms_model** out) {
  if (!cfg || !wt || !out) return fail(MS_ERR_INVALID_ARG, "ms_model_create: null argument");
  *out = nullptr;
  std::string why;
  if (!shape_ok(cfg, &why)) return fail(MS_ERR_SHAPE, "ms_model_create: %s", why.c_str());
  const ms_config& c = *cfg;
  if (!wt->tok_emb || !wt->lm_head || !wt->ln_f_g || !wt->ln_f_b || (c.n_layers > 0 && !wt->layers))
    return fail(MS_ERR_INVALID_ARG, "ms_model_create: null weight pointer");
  for (int l = 0; l < c.n_layers; ++l) {
    const ms_layer_weights& lw = wt->layers[l];
    if (!lw.ln1_g || !lw.ln1_b || !lw.ln2_g || !lw.ln2_b)
      return fail(MS_ERR_INVALID_ARG, "ms_model_create: layer %d: null LayerNorm pointer", l);
    for (int i = 0; i < 4; ++i) {
      if (c.weight_format == MS_W_INT4_G32 && (!lw.w[i] || !lw.s[i]))
        return fail(MS_ERR_INVALID_ARG, "ms_model_create: layer %d matrix %d: null INT4 pointer", l, i);
      if (c.weight_format == MS_W_FP16 && !lw.w16[i])
        return fail(MS_ERR_INVALID_ARG, "ms_model_create: layer %d matrix %d: null fp16 pointer", l, i);
    }
  }
  int ndev = 0;
  CUDA_TRY(cudaGetDeviceCount(&ndev));
  if (device < 0 || device >= ndev) return fail(MS_ERR_INVALID_ARG, "ms_model_create: no device %d", device);
  DeviceGuard dg(device);
  if (!dg.ok) return fail(MS_ERR_CUDA, "ms_model_create: cudaSetDevice(%d) failed", device);

  {
    cudaError_t ea = ensure_kernel_attributes();
    if (ea != cudaSuccess) return fail(MS_ERR_CUDA, "ms_model_create: kernel attributes: %s", cudaGetErrorString(ea));
  }
  ms_model* m = new (std::nothrow) ms_model;
  if (!m) return fail(MS_ERR_OOM, "ms_model_create: host allocation failed");
  m->cfg = c;
  m->device = device;
  const int d = c.d_model, V = c.vocab;
  // pass 1: sizes; pass 2: pointers
  for (int pass = 0; pass < 2; ++pass) {
    Arena& a = m->arena;
    a.used = 0;
    m->tok_emb = a.take<float>((size_t)V * d);
    m->lm_head = a.take<float>((size_t)V * d);
    m->ln_f_g = a.take<float>(d);
    m->ln_f_b = a.take<float>(d);
    m->d_players = a.take<ms::PLayer>(c.n_layers > 0 ? c.n_layers : 1);
    m->layers.assign(c.n_layers, DevLayer{});
    for (int l = 0; l < c.n_layers; ++l) {
      DevLayer& L = m->layers[l];
      L.ln1_g = a.take<float>(d);
      L.ln1_b = a.take<float>(d);
      L.ln2_g = a.take<float>(d);
      L.ln2_b = a.take<float>(d);
      for (int i = 0; i < 4; ++i) {
        int N, K;
        mat_nk(c, i, &N, &K);
        ms::WView& w = L.w[i];
        w.N = N;
        w.K = K;
        w.fmt = c.weight_format == MS_W_FP16 ? ms::kFp16 : ms::kInt4;
        w.q = nullptr;
        w.s = nullptr;
        w.h = nullptr;
        if (w.fmt == ms::kInt4) {
          // each row: K/2 nibble bytes then K/32 fp32 scales
          w.ldq = K / 2 + K / 8;
          w.lds = w.ldq / 4;
          w.q = a.take<uint8_t>((size_t)N * w.ldq);
          w.s = w.q ? reinterpret_cast<const float*>(w.q + K / 2) : nullptr;
        } else {
          w.ldq = 0;
          w.lds = 0;
          w.h = a.take<uint16_t>((size_t)N * K);
        }
        L.wt[i] = a.take<uint8_t>(ms::tile_packed_bytes(w));
        L.gw[i].wt = w.fmt == ms::kInt4 ? a.take<unsigned char>(ms::gemm_tiles_bytes(w)) : nullptr;
        L.gw[i].rinv = w.fmt == ms::kInt4 ? a.take<float>(ms::gemm_rows_padded(w)) : nullptr;
      }
    }
    {
      size_t rmax = 1;
      for (int i = 0; i < 4; ++i) {
        int N, K;
        mat_nk(c, i, &N, &K);
        rmax = std::max(rmax, (size_t)(N + 127) / 128 * 128);
      }
      m->rexp = a.take<float>(rmax);
    }
    if (pass == 0) {
      a.size = round_up(a.used, 256);
      cudaError_t e = cudaMalloc(&a.base, a.size);
      if (e != cudaSuccess) {
        cudaGetLastError();
        delete m;
        return fail(e == cudaErrorMemoryAllocation ? MS_ERR_OOM : MS_ERR_CUDA, "ms_model_create: cudaMalloc(%zu): %s",
                    a.size, cudaGetErrorString(e));
      }
    }
  }
  auto cp = [&](void* dst, const void* src, size_t bytes) -> cudaError_t {
    return cudaMemcpy(dst, src, bytes, cudaMemcpyDefault);
  };
  cudaError_t e = cudaSuccess;
  if (e == cudaSuccess) e = cp(m->tok_emb, wt->tok_emb, (size_t)V * d * 4);
  if (e == cudaSuccess) e = cp(m->lm_head, wt->lm_head, (size_t)V * d * 4);
  if (e == cudaSuccess) e = cp(m->ln_f_g, wt->ln_f_g, (size_t)d * 4);
  if (e == cudaSuccess) e = cp(m->ln_f_b, wt->ln_f_b, (size_t)d * 4);
  for (int l = 0; l < c.n_layers && e == cudaSuccess; ++l) {
    const ms_layer_weights& lw = wt->layers[l];
    DevLayer& L = m->layers[l];
    if (e == cudaSuccess) e = cp(L.ln1_g, lw.ln1_g, (size_t)d * 4);
    if (e == cudaSuccess) e = cp(L.ln1_b, lw.ln1_b, (size_t)d * 4);
    if (e == cudaSuccess) e = cp(L.ln2_g, lw.ln2_g, (size_t)d * 4);
    if (e == cudaSuccess) e = cp(L.ln2_b, lw.ln2_b, (size_t)d * 4);
    for (int i = 0; i < 4 && e == cudaSuccess; ++i) {
      const ms::WView& w = L.w[i];
      if (w.fmt == ms::kInt4) {
        e = cudaMemcpy2D(const_cast<uint8_t*>(w.q), w.ldq, lw.w[i], w.K / 2, w.K / 2, w.N, cudaMemcpyDefault);
        if (e == cudaSuccess)
          e = cudaMemcpy2D(const_cast<uint8_t*>(w.q) + w.K / 2, w.ldq, lw.s[i], w.K / 8, w.K / 8, w.N,
                           cudaMemcpyDefault);
      } else {
        e = cp(const_cast<uint16_t*>(w.h), lw.w16[i], (size_t)w.N * w.K * 2);
      }
    }
  }
  // tile-packed copies, made on the device from the rows just copied
  for (int l = 0; l < c.n_layers && e == cudaSuccess; ++l)
    for (int i = 0; i < 4 && e == cudaSuccess; ++i) e = ms::launch_repack_tiles(m->layers[l].w[i], m->layers[l].wt[i], 0);
  for (int l = 0; l < c.n_layers && e == cudaSuccess; ++l)
    for (int i = 0; i < 4 && e == cudaSuccess; ++i)
      e = ms::launch_gemm_repack(m->layers[l].w[i], m->layers[l].gw[i], m->rexp, 0);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess && c.n_layers > 0) {
    std::vector<ms::PLayer> pl(c.n_layers);
    for (int l = 0; l < c.n_layers; ++l) {
      const DevLayer& L = m->layers[l];
      pl[l].ln1_g = L.ln1_g;
      pl[l].ln1_b = L.ln1_b;
      pl[l].ln2_g = L.ln2_g;
      pl[l].ln2_b = L.ln2_b;
      for (int i = 0; i < 4; ++i) pl[l].w[i] = L.wt[i];
    }
    e = cudaMemcpy(m->d_players, pl.data(), pl.size() * sizeof(ms::PLayer), cudaMemcpyHostToDevice);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    cudaFree(m->arena.base);
    delete m;
    return fail(MS_ERR_CUDA, "ms_model_create: weight copy: %s", cudaGetErrorString(e));
  }
  *out = m;
  return MS_OK;
}

ms_status ms_model_destroy(ms_model* m) {
  if (!m) return fail(MS_ERR_INVALID_ARG, "ms_model_destroy: null model");
  DeviceGuard dg(m->device);
  cudaFree(m->arena.base);
  delete m;
  return MS_OK;
}

size_t ms_model_weight_bytes(const ms_model* m) { return m ? m->arena.used : 0; }

ms_status ms_cache_create(ms_model* m, int batch, int capacity, ms_cache** out) {
  return ms_cache_create_ex(m, batch, capacity, MS_KV_F32, out);
}

int ms_cache_kv_format(const ms_cache* c) { return c ? (c->kv16 ? MS_KV_F16 : MS_KV_F32) : -1; }

ms_status ms_cache_create_ex(ms_model* m, int batch, int capacity, int kv_format, ms_cache** out) {
  if (!m || !out) return fail(MS_ERR_INVALID_ARG, "ms_cache_create: null argument");
  *out = nullptr;
  if (batch < 1 || batch > 64) return fail(MS_ERR_SHAPE, "ms_cache_create: batch must be in [1, 64]");
  if (capacity < 1) return fail(MS_ERR_SHAPE, "ms_cache_create: capacity must be >= 1");
  if (kv_format != MS_KV_F32 && kv_format != MS_KV_F16)
    return fail(MS_ERR_INVALID_ARG, "ms_cache_create_ex: unknown kv_format %d", kv_format);
  DeviceGuard dg(m->device);
  const ms_config& g = m->cfg;
  ms_cache* c = new (std::nothrow) ms_cache;
  if (!c) return fail(MS_ERR_OOM, "ms_cache_create: host allocation failed");
  c->m = m;
  c->kv16 = kv_format == MS_KV_F16;
  c->B = batch;
  c->cap = capacity;
  c->splits = ms::attn_decode_splits(batch, g.n_kv_heads, capacity);
  c->rows_cap = (size_t)batch * capacity;
  cudaDeviceGetAttribute(&c->nsm, cudaDevAttrMultiProcessorCount, m->device);
  if (c->nsm < 1) c->nsm = 1;
  {
    // persistent decode kernel: one CTA per SM if its shared memory fits
    int dev = m->device, nsm = 0, optin = 0, coop = 0;
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev);
    const bool shapes = nsm > 0 && ms::persistent_shapes_ok(batch, g.d_model, g.n_heads, g.n_kv_heads, g.d_ff,
                                                            g.vocab, nsm, nullptr);
    if (shapes && coop && g.n_layers > 0 && g.n_layers <= 64) {
      // the ring gets what the kernel's static shared memory and its other regions leave
      const int fmt = g.weight_format == MS_W_FP16 ? ms::kFp16 : ms::kInt4;
      const size_t st_smem = ms::persistent_static_smem(batch, fmt);
      const int ns = st_smem < (size_t)optin
                         ? ms::persistent_slots(batch, g.n_layers, g.d_model, g.n_heads, g.n_kv_heads, g.d_ff, g.vocab,
                                                nsm, fmt, (size_t)optin - st_smem - 256)
                         : 0;
      if (ns >= 4) {
        const size_t sm_bytes = ms::persistent_smem(batch, g.n_layers, g.d_model, g.n_heads, g.n_kv_heads, g.d_ff,
                                                    g.vocab, nsm, fmt, ns);
        if (ms::persistent_max_ctas(batch, fmt, sm_bytes) >= 1) {
          c->persist_grid = nsm;
          c->persist_nslot = ns;
          c->persist_smem = sm_bytes;
          c->persist_sched_cap =
              ms::persistent_sched_cap(g.n_layers, g.d_model, g.n_heads, g.n_kv_heads, g.d_ff, g.vocab, nsm, fmt);
          int s = nsm / (batch * g.n_kv_heads);
          if (s > 128) s = 128;
          if (s > c->splits) c->splits = s;
        }
      }
    }
    cudaGetLastError();
  }
  const int hpg = g.n_heads / g.n_kv_heads;
  const size_t R = c->rows_cap;
  int lmg = ms::lm_head_grid(g.vocab);
  if (lmg < 1024) lmg = 1024;  // room for the persistent kernel's one entry per CTA
  for (int pass = 0; pass < 2; ++pass) {
    Arena& a = c->arena;
    a.used = 0;
    const size_t es = c->kv16 ? sizeof(__half) : sizeof(float);
    c->k = a.take<unsigned char>(((size_t)g.n_layers * layer_stride(c) + 64) * es);
    c->v = a.take<unsigned char>(((size_t)g.n_layers * layer_stride(c) + 64) * es);
    c->cosv = a.take<float>((size_t)capacity * 32);
    c->sinv = a.take<float>((size_t)capacity * 32);
    c->dlen = a.take<int>(4);
    c->status = a.take<unsigned>(4);
    c->lm_counter = a.take<unsigned>(4);
    c->sync3 = a.take<unsigned>(4);
    {
      // persistent kernel: the four matrices' output slices (up to 4 each), the attention
      // output and the attention partials, all {value, epoch} words in one block
      const size_t n_qkv = (size_t)batch * (g.n_heads + 2 * g.n_kv_heads) * 64;
      const size_t n_o = (size_t)batch * g.n_heads * 64;
      const size_t n_x = (size_t)batch * g.d_model;
      const size_t n_u = (size_t)batch * g.d_ff;
      const size_t n_p = (size_t)batch * g.n_kv_heads * c->splits * hpg * 66;  // attention partials
      const size_t total = 4 * (n_qkv + n_x + n_u + n_x) + n_o + n_p;
      c->vs[0] = a.take<uint64_t>(total);
      c->vstride[0] = (long long)n_qkv;
      c->vstride[1] = (long long)n_x;
      c->vstride[2] = (long long)n_u;
      c->vstride[3] = (long long)n_x;
      if (c->vs[0]) {
        c->vs[1] = c->vs[0] + 4 * n_qkv;
        c->vs[2] = c->vs[1] + 4 * n_x;
        c->vs[3] = c->vs[2] + 4 * n_u;
        c->o_s = c->vs[3] + 4 * n_x;
        c->part_s = c->o_s + n_o;
      }
      c->stamp_bytes = total * sizeof(uint64_t);
    }
    c->att_counters = a.take<unsigned>((size_t)batch * g.n_kv_heads);
    c->hist = a.take<int32_t>((size_t)capacity * batch);
    c->att_part = a.take<float>((size_t)batch * g.n_kv_heads * c->splits * hpg * 66);
    c->lm_val = a.take<float>((size_t)lmg * 64);
    c->lm_idx = a.take<int>((size_t)lmg * 64);
    c->x = a.take<float>(R * g.d_model);
    c->h = a.take<float>(R * g.d_model);
    c->y = a.take<float>(R * g.d_model);
    c->qkv = a.take<float>(R * (g.n_heads + 2 * g.n_kv_heads) * 64);
    c->q = a.take<float>(R * g.n_heads * 64);
    c->o = a.take<float>(R * g.n_heads * 64);
    c->u = a.take<float>(R * g.d_ff);
    c->kh = std::max(g.d_model, g.n_heads * 64);
    c->hh = a.take<__half>(R * c->kh);
    c->hl = a.take<__half>(R * c->kh);
    c->ka = std::max(c->kh, g.d_ff);
    c->qa = a.take<int8_t>(R * c->ka);
    c->sa = a.take<float>(R * (c->ka / 32));
    c->uh = reinterpret_cast<__half*>(c->u);
    c->ul = c->uh ? c->uh + R * g.d_ff : nullptr;
    c->logits = a.take<float>((size_t)batch * g.vocab);
    if (pass == 0) {
      a.size = round_up(a.used, 256);
      cudaError_t e = cudaMalloc(&a.base, a.size);
      if (e != cudaSuccess) {
        cudaGetLastError();
        delete c;
        return fail(e == cudaErrorMemoryAllocation ? MS_ERR_OOM : MS_ERR_CUDA, "ms_cache_create: cudaMalloc(%zu): %s",
                    a.size, cudaGetErrorString(e));
      }
    }
  }
  // RoPE table: angle = pos * base^(-2i/64), computed in double, stored fp32.
  std::vector<float> cs((size_t)capacity * 32), sn((size_t)capacity * 32);
  for (int p = 0; p < capacity; ++p)
    for (int i = 0; i < 32; ++i) {
      const double th = std::pow((double)g.rope_base, -2.0 * i / 64.0);
      const double ang = (double)p * th;
      cs[(size_t)p * 32 + i] = (float)std::cos(ang);
      sn[(size_t)p * 32 + i] = (float)std::sin(ang);
    }
  cudaError_t e = cudaMemset(c->arena.base, 0, c->arena.size);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&c->gen_stream, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->ev_in, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->ev_out, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaMemcpy(c->cosv, cs.data(), cs.size() * 4, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(c->sinv, sn.data(), sn.size() * 4, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    cudaGetLastError();
    if (c->gen_stream) cudaStreamDestroy(c->gen_stream);
    if (c->ev_in) cudaEventDestroy(c->ev_in);
    if (c->ev_out) cudaEventDestroy(c->ev_out);
    cudaFree(c->arena.base);
    delete c;
    return fail(MS_ERR_CUDA, "ms_cache_create: init: %s", cudaGetErrorString(e));
  }
  *out = c;
  return MS_OK;
}

ms_status ms_cache_destroy(ms_cache* c) {
  if (!c) return fail(MS_ERR_INVALID_ARG, "ms_cache_destroy: null cache");
  DeviceGuard dg(c->m->device);
  if (c->gen_exec) cudaGraphExecDestroy(c->gen_exec);
  if (c->gen_stream) {
    cudaStreamSynchronize(c->gen_stream);
    cudaStreamDestroy(c->gen_stream);
  }
  if (c->ev_in) cudaEventDestroy(c->ev_in);
  if (c->ev_out) cudaEventDestroy(c->ev_out);
  cudaDeviceSynchronize();
  cudaFree(c->arena.base);
  delete c;
  return MS_OK;
}

ms_status ms_cache_reset(ms_cache* c) {
  if (!c) return fail(MS_ERR_INVALID_ARG, "ms_cache_reset: null cache");
  DeviceGuard dg(c->m->device);
  CUDA_TRY(cudaDeviceSynchronize());
  int zero = 0;
  CUDA_TRY(cudaMemcpy(c->dlen, &zero, sizeof(int), cudaMemcpyHostToDevice));
  c->len = 0;
  c->has_next = false;
  return MS_OK;
}

int ms_cache_length(const ms_cache* c) { return c ? c->len : -1; }
uint64_t ms_cache_kernel_launches(const ms_cache* c) { return c ? c->launches : 0; }

ms_status ms_cache_set_decode_path(ms_cache* c, int path) {
  if (!c) return fail(MS_ERR_INVALID_ARG, "ms_cache_set_decode_path: null cache");
  if (path < 0 || path > 2) return fail(MS_ERR_INVALID_ARG, "ms_cache_set_decode_path: path must be 0, 1 or 2");
  if (path == 1 && c->persist_grid == 0)
    return fail(MS_ERR_UNSUPPORTED, "ms_cache_set_decode_path: the persistent kernel does not fit this model/batch");
  if (path == 1 && c->act_int8)
    return fail(MS_ERR_UNSUPPORTED, "ms_cache_set_decode_path: INT8 activations run one kernel per operation");
  c->path_request = path;
  return MS_OK;
}

ms_status ms_cache_set_guidance(ms_cache* c, float scale) {
  if (!c) return fail(MS_ERR_INVALID_ARG, "ms_cache_set_guidance: null cache");
  if (!std::isfinite(scale)) return fail(MS_ERR_INVALID_ARG, "ms_cache_set_guidance: scale must be finite");
  if (scale != 0.f && c->B % 2 != 0)
    return fail(MS_ERR_SHAPE, "ms_cache_set_guidance: guidance pairs streams (2p, 2p+1); batch %d is odd", c->B);
  c->guidance = scale;
  return MS_OK;
}

float ms_cache_guidance(const ms_cache* c) { return c ? c->guidance : 0.f; }

ms_status ms_cache_set_act_int8(ms_cache* c, int on) {
  if (!c) return fail(MS_ERR_INVALID_ARG, "ms_cache_set_act_int8: null cache");
  if (on && c->m->cfg.weight_format != MS_W_INT4_G32)
    return fail(MS_ERR_UNSUPPORTED, "ms_cache_set_act_int8: INT8 activations go with INT4 weights");
  if (on && c->path_request == 1)
    return fail(MS_ERR_UNSUPPORTED, "ms_cache_set_act_int8: the persistent decode path was requested on this cache");
  if (!!on != !!c->act_int8 && c->gen_exec) {
    // the captured decode graph belongs to the other arithmetic
    cudaGraphExecDestroy(c->gen_exec);
    c->gen_exec = nullptr;
  }
  c->act_int8 = on ? 1 : 0;
  return MS_OK;
}

int ms_cache_act_int8(const ms_cache* c) { return c ? c->act_int8 : -1; }

ms_status ms_cache_set_wait_limits(ms_cache* c, long long polls, int stall) {
  if (!c) return fail(MS_ERR_INVALID_ARG, "ms_cache_set_wait_limits: null cache");
  if (polls < 0 || stall < 0 || stall > 2)
    return fail(MS_ERR_INVALID_ARG, "ms_cache_set_wait_limits: need polls >= 0 and stall in {0, 1, 2}");
  c->wait_limit = polls;
  c->test_stall = stall;
  return MS_OK;
}

int ms_cache_decode_path(const ms_cache* c) {
  if (!c) return -1;
  return use_persistent(c) ? 1 : 2;
}
int ms_cache_capacity(const ms_cache* c) { return c ? c->cap : -1; }
int ms_cache_batch(const ms_cache* c) { return c ? c->B : -1; }

ms_status ms_prefill(ms_model* m, ms_cache* c, const int64_t* tokens, int S, const float* prefix, int P,
                     float* logits, int32_t* argmax, void* stream) {
  if (!m || !c) return fail(MS_ERR_INVALID_ARG, "ms_prefill: null model or cache");
  if (c->m != m) return fail(MS_ERR_INVALID_ARG, "ms_prefill: cache belongs to another model");
  if (S < 0 || P < 0 || P + S < 1) return fail(MS_ERR_SHAPE, "ms_prefill: need S >= 0, P >= 0, P + S >= 1");
  if (S > 0 && !tokens) return fail(MS_ERR_INVALID_ARG, "ms_prefill: null tokens with S > 0");
  if (P > 0 && !prefix) return fail(MS_ERR_INVALID_ARG, "ms_prefill: null prefix with P > 0");
  if ((long long)c->len + P + S > c->cap)
    return fail(MS_ERR_CACHE_FULL, "ms_prefill: %d + %d positions exceed capacity %d", c->len, P + S, c->cap);
  DeviceGuard dg(m->device);
  const unsigned long long before = ms::launch_counter().load();
  cudaError_t e = run_prefill(m, c, tokens, S, prefix, P, logits, argmax, (cudaStream_t)stream);
  c->launches += ms::launch_counter().load() - before;
  if (e != cudaSuccess) return check_launch(e, "ms_prefill launch");
  c->len += P + S;
  c->has_next = true;
  return MS_OK;
}

ms_status ms_decode_step(ms_model* m, ms_cache* c, const int32_t* tokens, float* logits, int32_t* argmax,
                         void* stream) {
  if (!m || !c) return fail(MS_ERR_INVALID_ARG, "ms_decode_step: null model or cache");
  if (c->m != m) return fail(MS_ERR_INVALID_ARG, "ms_decode_step: cache belongs to another model");
  if (!tokens) return fail(MS_ERR_INVALID_ARG, "ms_decode_step: null tokens");
  if (c->len + 1 > c->cap) return fail(MS_ERR_CACHE_FULL, "ms_decode_step: cache full (%d)", c->cap);
  DeviceGuard dg(m->device);
  const unsigned long long before = ms::launch_counter().load();
  cudaError_t e = use_persistent(c) ? run_persistent(m, c, tokens, 1, logits, argmax, (cudaStream_t)stream)
                                    : run_decode(m, c, tokens, logits, argmax, (cudaStream_t)stream, false);
  c->launches += ms::launch_counter().load() - before;
  if (e != cudaSuccess) return check_launch(e, "ms_decode_step launch");
  c->len += 1;
  c->has_next = true;
  return MS_OK;
}

ms_status ms_generate(ms_model* m, ms_cache* c, int n_steps, int32_t* out_tokens, float* logits, void* stream) {
  if (!m || !c) return fail(MS_ERR_INVALID_ARG, "ms_generate: null model or cache");
  if (c->m != m) return fail(MS_ERR_INVALID_ARG, "ms_generate: cache belongs to another model");
  if (n_steps < 0) return fail(MS_ERR_SHAPE, "ms_generate: n_steps < 0");
  if (n_steps == 0) return MS_OK;
  if (!out_tokens) return fail(MS_ERR_INVALID_ARG, "ms_generate: null out_tokens");
  if (!c->has_next) return fail(MS_ERR_INVALID_ARG, "ms_generate: no previous argmax on this cache (prefill first)");
  if ((long long)c->len + n_steps > c->cap)
    return fail(MS_ERR_CACHE_FULL, "ms_generate: %d + %d positions exceed capacity %d", c->len, n_steps, c->cap);
  DeviceGuard dg(m->device);
  if (use_persistent(c)) {
    cudaStream_t ps = (cudaStream_t)stream;
    const int len0 = c->len;
    const int chunk = 128;  // steps per launch
    for (int done = 0; done < n_steps;) {
      const int k = n_steps - done < chunk ? n_steps - done : chunk;
      const unsigned long long before = ms::launch_counter().load();
      cudaError_t e = run_persistent(m, c, nullptr, k, c->logits, nullptr, ps);
      c->launches += ms::launch_counter().load() - before;
      if (e != cudaSuccess) return check_launch(e, "ms_generate persistent launch");
      done += k;
    }
    CUDA_TRY(cudaMemcpyAsync(out_tokens, c->hist + (size_t)len0 * c->B, (size_t)n_steps * c->B * sizeof(int32_t),
                             cudaMemcpyDeviceToDevice, ps));
    if (logits)
      CUDA_TRY(cudaMemcpyAsync(logits, c->logits, (size_t)c->B * m->cfg.vocab * sizeof(float), cudaMemcpyDeviceToDevice,
                               ps));
    c->len += n_steps;
    return MS_OK;
  }
  const bool legacy = stream == nullptr;
  cudaStream_t st = legacy ? c->gen_stream : (cudaStream_t)stream;
  const int len0 = c->len;
  if (legacy) {
    // the graph runs on the cache's own stream, ordered after and before the legacy stream
    CUDA_TRY(cudaEventRecord(c->ev_in, nullptr));
    CUDA_TRY(cudaStreamWaitEvent(st, c->ev_in, 0));
  }
  {
    if (!c->gen_exec) {
      cudaGraph_t graph = nullptr;
      CUDA_TRY(cudaStreamBeginCapture(st, cudaStreamCaptureModeThreadLocal));
      cudaError_t e = run_decode(m, c, nullptr, c->logits, nullptr, st, false);
      cudaError_t e2 = cudaStreamEndCapture(st, &graph);
      if (e != cudaSuccess || e2 != cudaSuccess) {
        if (graph) cudaGraphDestroy(graph);
        cudaGetLastError();
        return fail(MS_ERR_CUDA, "ms_generate: capture: %s", cudaGetErrorString(e != cudaSuccess ? e : e2));
      }
      size_t nodes = 0;
      cudaGraphGetNodes(graph, nullptr, &nodes);
      c->gen_nodes = nodes;
      e = cudaGraphInstantiate(&c->gen_exec, graph, 0);
      cudaGraphDestroy(graph);
      if (e != cudaSuccess) {
        c->gen_exec = nullptr;
        return fail(MS_ERR_CUDA, "ms_generate: instantiate: %s", cudaGetErrorString(e));
      }
    }
    for (int i = 0; i < n_steps; ++i) {
      CUDA_TRY(cudaGraphLaunch(c->gen_exec, st));
      c->launches += c->gen_nodes;
    }
  }
  CUDA_TRY(cudaMemcpyAsync(out_tokens, c->hist + (size_t)len0 * c->B, (size_t)n_steps * c->B * sizeof(int32_t),
                           cudaMemcpyDeviceToDevice, st));
  if (logits)
    CUDA_TRY(cudaMemcpyAsync(logits, c->logits, (size_t)c->B * m->cfg.vocab * sizeof(float), cudaMemcpyDeviceToDevice, st));
  if (legacy) {
    CUDA_TRY(cudaEventRecord(c->ev_out, st));
    CUDA_TRY(cudaStreamWaitEvent(nullptr, c->ev_out, 0));
  }
  c->len += n_steps;
  return MS_OK;
}

// Host-side conversion between fp32 and IEEE half (round to nearest even), for the cache
// transfer calls of a half-precision cache.
namespace {
uint16_t f32_to_f16_bits(float f) { return __half_as_ushort(__float2half_rn(f)); }
float f16_bits_to_f32(uint16_t h) { return __half2float(__ushort_as_half(h)); }
}  // namespace

ms_status ms_cache_export(const ms_cache* c, float* k, float* v) {
  if (!c || !k || !v) return fail(MS_ERR_INVALID_ARG, "ms_cache_export: null argument");
  DeviceGuard dg(c->m->device);
  CUDA_TRY(cudaDeviceSynchronize());
  const ms_config& g = c->m->cfg;
  const int T = c->len, Hk = g.n_kv_heads;
  const size_t es = c->kv16 ? sizeof(__half) : sizeof(float);
  std::vector<unsigned char> buf((size_t)T * 64 * es);
  for (int which = 0; which < 2; ++which) {
    void* src = which ? c->v : c->k;
    float* dst = which ? v : k;
    for (int l = 0; l < g.n_layers; ++l)
      for (int b = 0; b < c->B; ++b)
        for (int gg = 0; gg < Hk; ++gg) {
          const char* s = static_cast<const char*>(kv_layer(c, src, l)) + (((size_t)b * Hk + gg) * c->cap) * 64 * es;
          if (T > 0) CUDA_TRY(cudaMemcpy(buf.data(), s, (size_t)T * 64 * es, cudaMemcpyDeviceToHost));
          for (int t = 0; t < T; ++t) {
            float* o = dst + ((((size_t)l * c->B + b) * T + t) * Hk + gg) * 64;
            if (c->kv16) {
              const uint16_t* hb = reinterpret_cast<const uint16_t*>(buf.data()) + (size_t)t * 64;
              for (int e = 0; e < 64; ++e) o[e] = f16_bits_to_f32(hb[e]);
            } else {
              memcpy(o, buf.data() + (size_t)t * 64 * 4, 64 * 4);
            }
          }
        }
  }
  return MS_OK;
}

ms_status ms_cache_import(ms_cache* c, const float* k, const float* v, int T) {
  if (!c || (T > 0 && (!k || !v))) return fail(MS_ERR_INVALID_ARG, "ms_cache_import: null argument");
  if (T < 0 || T > c->cap) return fail(MS_ERR_CACHE_FULL, "ms_cache_import: T = %d outside [0, %d]", T, c->cap);
  DeviceGuard dg(c->m->device);
  CUDA_TRY(cudaDeviceSynchronize());
  const ms_config& g = c->m->cfg;
  const int Hk = g.n_kv_heads;
  const size_t es = c->kv16 ? sizeof(__half) : sizeof(float);
  std::vector<unsigned char> buf((size_t)T * 64 * es);
  for (int which = 0; which < 2; ++which) {
    void* dst = which ? c->v : c->k;
    const float* src = which ? v : k;
    for (int l = 0; l < g.n_layers; ++l)
      for (int b = 0; b < c->B; ++b)
        for (int gg = 0; gg < Hk; ++gg) {
          for (int t = 0; t < T; ++t) {
            const float* in = src + ((((size_t)l * c->B + b) * T + t) * Hk + gg) * 64;
            if (c->kv16) {
              uint16_t* hb = reinterpret_cast<uint16_t*>(buf.data()) + (size_t)t * 64;
              for (int e = 0; e < 64; ++e) hb[e] = f32_to_f16_bits(in[e]);
            } else {
              memcpy(buf.data() + (size_t)t * 64 * 4, in, 64 * 4);
            }
          }
          char* d = static_cast<char*>(kv_layer(c, dst, l)) + (((size_t)b * Hk + gg) * c->cap) * 64 * es;
          if (T > 0) CUDA_TRY(cudaMemcpy(d, buf.data(), (size_t)T * 64 * es, cudaMemcpyHostToDevice));
        }
  }
  CUDA_TRY(cudaMemcpy(c->dlen, &T, sizeof(int), cudaMemcpyHostToDevice));
  c->len = T;
  c->has_next = false;
  return MS_OK;
}

ms_status ms_device_status(ms_cache* c, void* stream) {
  if (!c) return fail(MS_ERR_INVALID_ARG, "ms_device_status: null cache");
  DeviceGuard dg(c->m->device);
  CUDA_TRY(cudaStreamSynchronize((cudaStream_t)stream));
  unsigned w = 0;
  CUDA_TRY(cudaMemcpy(&w, c->status, sizeof(unsigned), cudaMemcpyDeviceToHost));
  const unsigned zero = 0;
  CUDA_TRY(cudaMemcpy(c->status, &zero, sizeof(unsigned), cudaMemcpyHostToDevice));
  if (w & ms::kErrTimeoutBit) return fail(MS_ERR_TIMEOUT, "a device-side wait ran out (status 0x%x)", w);
  if (w & ms::kErrTokenBit) return fail(MS_ERR_TOKEN_RANGE, "a token id was outside [0, vocab) (status 0x%x)", w);
  if (w & ms::kErrShapeBit) return fail(MS_ERR_SHAPE, "a device-side size check failed (status 0x%x)", w);
  return MS_OK;
}

// ---- single operations ---------------------------------------------------------------
}  // extern "C"

namespace {
// The tcgen05 GEMM for a single-operation call on caller arrays: the weights' tile-packed copy
// and the activation planes are made in stream-ordered temporaries (cudaMallocAsync) that are
// released on the stream after the GEMM; the launch policy is the model's own.
ms_status op_gemm(const ms::WView& w, const float* x, int M, float* y, cudaStream_t st, const char* who) {
  int dev = 0, nsm = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  CUDA_TRY(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev));
  const ms::GemmWork gw{nsm > 0 ? nsm : 1};
  ms::Launch L{st, false, nullptr};
  const size_t tiles = ms::gemm_tiles_bytes(w), rows = ms::gemm_rows_padded(w);
  const size_t planes = (size_t)M * w.K * sizeof(__half);
  const size_t bytes = round_up(tiles, 256) + 2 * round_up(rows * 4, 256) + 2 * round_up(planes, 256);
  char* tmp = nullptr;
  CUDA_TRY(cudaMallocAsync(reinterpret_cast<void**>(&tmp), bytes, st));
  char* p = tmp;
  ms::GemmWeights g{nullptr, nullptr};
  float* rexp = nullptr;
  if (w.fmt == ms::kInt4) {
    g.wt = reinterpret_cast<unsigned char*>(p);
    p += round_up(tiles, 256);
    g.rinv = reinterpret_cast<float*>(p);
    p += round_up(rows * 4, 256);
    rexp = reinterpret_cast<float*>(p);
    p += round_up(rows * 4, 256);
  }
  __half* xh = reinterpret_cast<__half*>(p);
  __half* xl = reinterpret_cast<__half*>(p + round_up(planes, 256));
  cudaError_t e = cudaSuccess;
  if (w.fmt == ms::kInt4) e = ms::launch_gemm_repack(w, g, rexp, st);
  if (e == cudaSuccess) e = ms::launch_split_f16(L, x, w.K, M, w.K, xh, xl, w.K);
  if (e == cudaSuccess) e = ms::launch_gemm_f16(L, w, g, xh, xl, w.K, M, y, w.N, nullptr, nullptr, 0, ms::kStore, &gw);
  const cudaError_t ef = cudaFreeAsync(tmp, st);
  if (e != cudaSuccess) return fail(MS_ERR_CUDA, "%s: gemm: %s", who, cudaGetErrorString(e));
  if (ef != cudaSuccess) return fail(MS_ERR_CUDA, "%s: cudaFreeAsync: %s", who, cudaGetErrorString(ef));
  return MS_OK;
}
}  // namespace

extern "C" {

ms_status ms_op_matmul_w4(const float* x, int M, int K, const uint8_t* packed, const float* scales, int N, float* y,
                          void* stream) {
  if (!x || !packed || !scales || !y) return fail(MS_ERR_INVALID_ARG, "ms_op_matmul_w4: null pointer");
  if (M < 1 || N < 1 || K < 256 || K % 256 != 0) return fail(MS_ERR_SHAPE, "ms_op_matmul_w4: need M, N >= 1, K a multiple of 256");
  CUDA_TRY(ensure_kernel_attributes());
  ms::WView w{packed, scales, nullptr, N, K, ms::kInt4, K / 2, K / 32};
  ms::Launch L{(cudaStream_t)stream, false, nullptr};
  if ((M == 1 || M == 2 || M == 4 || M == 8) && ms::gemv_fits(w, M))
    return check_launch(ms::launch_gemv(L, w, x, K, M, nullptr, nullptr, 0.f, y, N, ms::kStore), "gemv");
  return op_gemm(w, x, M, y, (cudaStream_t)stream, "ms_op_matmul_w4");
}

ms_status ms_op_matmul_f16(const float* x, int M, int K, const uint16_t* w16, int N, float* y, void* stream) {
  if (!x || !w16 || !y) return fail(MS_ERR_INVALID_ARG, "ms_op_matmul_f16: null pointer");
  if (M < 1 || N < 1 || K < 256 || K % 256 != 0) return fail(MS_ERR_SHAPE, "ms_op_matmul_f16: need M, N >= 1, K a multiple of 256");
  CUDA_TRY(ensure_kernel_attributes());
  ms::WView w{nullptr, nullptr, w16, N, K, ms::kFp16, 0, 0};
  ms::Launch L{(cudaStream_t)stream, false, nullptr};
  if ((M == 1 || M == 2 || M == 4 || M == 8) && ms::gemv_fits(w, M))
    return check_launch(ms::launch_gemv(L, w, x, K, M, nullptr, nullptr, 0.f, y, N, ms::kStore), "gemv");
  return op_gemm(w, x, M, y, (cudaStream_t)stream, "ms_op_matmul_f16");
}

ms_status ms_op_quantize_act_int8(const float* x, int ldx, int M, int K, int8_t* q, float* scales, void* stream) {
  if (!x || !q || !scales) return fail(MS_ERR_INVALID_ARG, "ms_op_quantize_act_int8: null pointer");
  if (M < 0 || K < 32 || K % 32 != 0 || ldx < K) return fail(MS_ERR_SHAPE, "ms_op_quantize_act_int8: need K a multiple of 32, ldx >= K");
  ms::Launch L{(cudaStream_t)stream, false, nullptr};
  return check_launch(ms::launch_quantize_act_int8(L, x, ldx, M, K, q, K, scales, K / 32), "quantize_act_int8");
}

ms_status ms_op_matmul_w4a8(const int8_t* qa, const float* sa, int M, int K, const uint8_t* packed, const float* scales,
                            int N, float* y, void* stream) {
  if (!qa || !sa || !packed || !scales || !y) return fail(MS_ERR_INVALID_ARG, "ms_op_matmul_w4a8: null pointer");
  if (M < 1 || N < 1 || K < 128 || K % 128 != 0) return fail(MS_ERR_SHAPE, "ms_op_matmul_w4a8: need M, N >= 1, K a multiple of 128");
  if ((reinterpret_cast<uintptr_t>(qa) & 15) || (reinterpret_cast<uintptr_t>(packed) & 15))
    return fail(MS_ERR_INVALID_ARG, "ms_op_matmul_w4a8: qa and packed must be 16-byte aligned");
  CUDA_TRY(ensure_kernel_attributes());
  int dev = 0, nsm = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  CUDA_TRY(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev));
  ms::WView w{packed, scales, nullptr, N, K, ms::kInt4, K / 2, K / 32};
  ms::Launch L{(cudaStream_t)stream, false, nullptr};
  if (ms::w4a8_tc_fits(w, M, K, K / 32) && !(reinterpret_cast<uintptr_t>(sa) & 15)) {
    // the tcgen05 kernel reads the tile-packed copy, made in stream-ordered temporaries
    const size_t tiles = ms::gemm_tiles_bytes(w), rows = ms::gemm_rows_padded(w);
    char* tmp = nullptr;
    CUDA_TRY(cudaMallocAsync(reinterpret_cast<void**>(&tmp), round_up(tiles, 256) + 2 * round_up(rows * 4, 256),
                             (cudaStream_t)stream));
    ms::GemmWeights g{reinterpret_cast<unsigned char*>(tmp), reinterpret_cast<float*>(tmp + round_up(tiles, 256))};
    float* rexp = reinterpret_cast<float*>(tmp + round_up(tiles, 256) + round_up(rows * 4, 256));
    cudaError_t e = ms::launch_gemm_repack(w, g, rexp, (cudaStream_t)stream);
    if (e == cudaSuccess) e = ms::launch_matmul_w4a8_tc(L, w, g, qa, K, sa, K / 32, M, y, N, ms::kStore);
    const cudaError_t ef = cudaFreeAsync(tmp, (cudaStream_t)stream);
    if (e != cudaSuccess) return check_launch(e, "matmul_w4a8 (tcgen05)");
    CUDA_TRY(ef);
    return MS_OK;
  }
  return check_launch(ms::launch_matmul_w4a8(L, w, qa, K, sa, K / 32, M, y, N, ms::kStore, nsm > 0 ? nsm : 1),
                      "matmul_w4a8");
}

ms_status ms_op_split_f16(const float* x, int ldx, int M, int K, uint16_t* x_hi, uint16_t* x_lo, int ldh,
                          void* stream) {
  if (!x || !x_hi || !x_lo) return fail(MS_ERR_INVALID_ARG, "ms_op_split_f16: null pointer");
  if (M < 0 || K < 4 || K % 4 != 0 || ldx < K || ldx % 4 != 0 || ldh < K || ldh % 4 != 0)
    return fail(MS_ERR_SHAPE, "ms_op_split_f16: need K a multiple of 4, ldx and ldh >= K and multiples of 4");
  if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(x_hi) & 7) ||
      (reinterpret_cast<uintptr_t>(x_lo) & 7))
    return fail(MS_ERR_INVALID_ARG, "ms_op_split_f16: x must be 16-byte and the planes 8-byte aligned");
  ms::Launch L{(cudaStream_t)stream, false, nullptr};
  return check_launch(ms::launch_split_f16(L, x, ldx, M, K, reinterpret_cast<__half*>(x_hi),
                                           reinterpret_cast<__half*>(x_lo), ldh),
                      "split_f16");
}

ms_status ms_model_matmul(const ms_model* m, int layer, int which, const uint16_t* x_hi, const uint16_t* x_lo,
                          int ldx, int M, float* y, int ldy, void* stream) {
  if (!m || !x_hi || !x_lo || !y) return fail(MS_ERR_INVALID_ARG, "ms_model_matmul: null argument");
  if (layer < 0 || layer >= m->cfg.n_layers || which < 0 || which > 3)
    return fail(MS_ERR_INVALID_ARG, "ms_model_matmul: no matrix %d of layer %d", which, layer);
  const DevLayer& ly = m->layers[layer];
  const ms::WView& w = ly.w[which];
  if (M < 1 || ldx < w.K || ldx % 8 != 0 || ldy < w.N)
    return fail(MS_ERR_SHAPE, "ms_model_matmul: need M >= 1, ldx >= K (a multiple of 8), ldy >= N");
  if ((reinterpret_cast<uintptr_t>(x_hi) & 15) || (reinterpret_cast<uintptr_t>(x_lo) & 15))
    return fail(MS_ERR_INVALID_ARG, "ms_model_matmul: the planes must be 16-byte aligned");
  DeviceGuard dg(m->device);
  int nsm = 0;
  CUDA_TRY(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, m->device));
  const ms::GemmWork gw{nsm > 0 ? nsm : 1};
  ms::Launch L{(cudaStream_t)stream, false, nullptr};
  return check_launch(ms::launch_gemm_f16(L, w, ly.gw[which], reinterpret_cast<const __half*>(x_hi),
                                          reinterpret_cast<const __half*>(x_lo), ldx, M, y, ldy, nullptr, nullptr, 0,
                                          ms::kStore, &gw),
                      "model matmul");
}

ms_status ms_op_skip_layernorm(float* x, const float* y, const float* gamma, const float* beta, float eps, int R, int d,
                               float* h, void* stream) {
  if (!x || !gamma || !beta || !h) return fail(MS_ERR_INVALID_ARG, "ms_op_skip_layernorm: null pointer");
  if (R < 0 || d < 128 || d % 128 != 0 || d > 2048) return fail(MS_ERR_SHAPE, "ms_op_skip_layernorm: d must be a multiple of 128 up to 2048");
  ms::Launch L{(cudaStream_t)stream, false, nullptr};
  return check_launch(ms::launch_skipln(L, x, y, gamma, beta, eps, R, d, h), "skip_layernorm");
}

ms_status ms_op_lm_head_argmax(const float* x, int ldx, int M, int d, const float* gamma, const float* beta, float eps,
                               const float* W, int V, float* logits, int32_t* argmax, void* stream) {
  if (!x || !W) return fail(MS_ERR_INVALID_ARG, "ms_op_lm_head_argmax: null pointer");
  if ((gamma == nullptr) != (beta == nullptr)) return fail(MS_ERR_INVALID_ARG, "ms_op_lm_head_argmax: gamma and beta go together");
  if (M < 1 || M > 64 || V < 1 || d < 128 || d % 128 != 0 || ldx < d || ldx % 4 != 0)
    return fail(MS_ERR_SHAPE, "ms_op_lm_head_argmax: bad sizes");
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  CUDA_TRY(ensure_kernel_attributes());
  OpScratch sc;
  {
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if ((int)g_scratch.size() <= dev) g_scratch.resize(dev + 1);
    OpScratch& s = g_scratch[dev];
    if (!s.counter) {
      // sized for the largest grid any V can give (one CTA per SM's worth of rows)
      CUDA_TRY(cudaMalloc(&s.part_val, 1024 * 64 * sizeof(float)));
      CUDA_TRY(cudaMalloc(&s.part_idx, 1024 * 64 * sizeof(int)));
      CUDA_TRY(cudaMalloc(&s.counter, 256));
      CUDA_TRY(cudaMemset(s.counter, 0, 256));
    }
    sc = s;
  }
  if (ms::lm_head_grid(V) > 1024) return fail(MS_ERR_SHAPE, "ms_op_lm_head_argmax: V too large");
  ms::Launch L{(cudaStream_t)stream, false, nullptr};
  ms::LmHeadWork w{sc.part_val, sc.part_idx, sc.counter};
  return check_launch(ms::launch_lm_head(L, x, ldx, M, d, gamma, beta, eps, W, V, logits, argmax, nullptr, M, 0, nullptr,
                                         0, w),
                      "lm_head");
}

}  // extern "C"

// ---- conditioner front-end --------------------------------------------------------------

struct ms_cond {
  ms_cond_config cfg;
  int device = 0;
  int frames = 0, kp = 0;
  float yscale = 1.f;        // 2^-s: the projection weights are stored times 2^s
  char* base = nullptr;
  ms::CondDev dev{};
  uint16_t *wh = nullptr, *wl = nullptr;
  float *bias = nullptr, *inst = nullptr, *ds = nullptr, *y = nullptr;
  __half *xh = nullptr, *xl = nullptr;
  unsigned* status = nullptr;
  ~ms_cond() {
    if (base) cudaFree(base);
  }
};

namespace {

bool cond_config_ok(const ms_cond_config& c) {
  const bool pow2 = c.n_fft >= 16 && c.n_fft <= ms::kCondMaxFft && (c.n_fft & (c.n_fft - 1)) == 0;
  return pow2 && c.hop >= 1 && c.n_samples > c.n_fft / 2 && c.n_mels >= 1 && c.n_mels <= 4096 && c.d_model >= 4 &&
         c.d_model % 4 == 0 && c.n_instruments >= 1 && c.n_datasets >= 1 && c.max_batch >= 1 &&
         c.max_batch <= 65535 && 1 + c.n_samples / c.hop <= (1 << 24);
}

ms::WView cond_view(const ms_cond* c, const uint16_t* h) {
  ms::WView w{};
  w.h = h;
  w.N = c->cfg.d_model;
  w.K = c->kp;
  w.fmt = ms::kFp16;
  return w;
}

}  // namespace

extern "C" {

ms_status ms_cond_create(const ms_cond_config* cfg, const ms_cond_weights* wt, int device, ms_cond** out) {
  if (!cfg || !wt || !out) return fail(MS_ERR_INVALID_ARG, "ms_cond_create: null argument");
  *out = nullptr;
  if (!wt->window || !wt->mel_fb || !wt->proj_w || !wt->proj_b || !wt->inst_emb || !wt->ds_emb)
    return fail(MS_ERR_INVALID_ARG, "ms_cond_create: null weight pointer");
  const ms_cond_config c = *cfg;
  if (!cond_config_ok(c))
    return fail(MS_ERR_INVALID_ARG,
                "ms_cond_create: need n_fft a power of two in 16..%d, hop >= 1, n_samples > n_fft / 2, "
                "n_mels 1..4096, d_model a positive multiple of 4, tables and max_batch >= 1",
                ms::kCondMaxFft);
  DeviceGuard dg(device);
  if (!dg.ok) return fail(MS_ERR_CUDA, "ms_cond_create: cannot select device %d", device);
  {
    cudaError_t ea = ensure_kernel_attributes();
    if (ea != cudaSuccess) return fail(MS_ERR_CUDA, "ms_cond_create: kernel attributes: %s", cudaGetErrorString(ea));
  }
  const int d = c.d_model, nf = c.n_fft / 2 + 1, half = c.n_fft / 2;
  const int frames = 1 + c.n_samples / c.hop, kp = (c.n_mels + 63) / 64 * 64;
  // host copies of what the preprocessing reads (the pointers may be host or device)
  std::vector<float> fb((size_t)c.n_mels * nf), pw((size_t)d * c.n_mels);
  CUDA_TRY(cudaMemcpy(fb.data(), wt->mel_fb, fb.size() * 4, cudaMemcpyDefault));
  CUDA_TRY(cudaMemcpy(pw.data(), wt->proj_w, pw.size() * 4, cudaMemcpyDefault));
  std::vector<float> win32(c.n_fft);
  CUDA_TRY(cudaMemcpy(win32.data(), wt->window, win32.size() * 4, cudaMemcpyDefault));
  const std::vector<double> win(win32.begin(), win32.end());
  // each filterbank row compressed to its non-zero range
  std::vector<int> lo(c.n_mels), off(c.n_mels + 1, 0);
  std::vector<float> bw;
  for (int m = 0; m < c.n_mels; ++m) {
    const float* row = fb.data() + (size_t)m * nf;
    int first = -1, last = -1;
    for (int k = 0; k < nf; ++k)
      if (row[k] != 0.f) {
        if (first < 0) first = k;
        last = k;
      }
    lo[m] = first < 0 ? 0 : first;
    if (first >= 0) bw.insert(bw.end(), row + first, row + last + 1);
    off[m + 1] = (int)bw.size();
  }
  if (bw.empty()) bw.push_back(0.f);
  // twiddles e^{-2 pi i k / n_fft}, k < n_fft, in double on the host; the window in double
  std::vector<double2> tw(c.n_fft);
  const double two_pi = 6.283185307179586476925286766559;
  for (int k = 0; k < c.n_fft; ++k) {
    const double a = two_pi * (double)k / (double)c.n_fft;
    tw[k] = make_double2(std::cos(a), -std::sin(a));
  }
  // projection weights times 2^s (largest magnitude below 2^15), split into fp16 hi and lo
  float amax = 0.f;
  for (float v : pw) amax = std::max(amax, std::fabs(v));
  int e2 = 0;
  if (amax > 0.f) std::frexp(amax, &e2);     // amax < 2^e2
  const int sh = std::max(-60, std::min(60, 15 - e2));
  std::vector<uint16_t> wh((size_t)d * kp, 0), wl((size_t)d * kp, 0);
  for (int n = 0; n < d; ++n)
    for (int k = 0; k < c.n_mels; ++k) {
      const float v = std::ldexp(pw[(size_t)n * c.n_mels + k], sh);
      const __half hi = __float2half_rn(v);
      const __half lo16 = __float2half_rn(v - __half2float(hi));
      wh[(size_t)n * kp + k] = __half_as_ushort(hi);
      wl[(size_t)n * kp + k] = __half_as_ushort(lo16);
    }

  ms_cond* q = new (std::nothrow) ms_cond;
  if (!q) return fail(MS_ERR_OOM, "ms_cond_create: host allocation failed");
  q->cfg = c;
  q->device = device;
  q->frames = frames;
  q->kp = kp;
  q->yscale = std::ldexp(1.f, -sh);
  const size_t rows = (size_t)c.max_batch * frames;
  Arena a;
  for (int pass = 0; pass < 2; ++pass) {
    a.used = 0;
    q->dev.window = a.take<double>(c.n_fft);
    q->dev.twiddle = a.take<double2>(c.n_fft);
    q->dev.band_lo = a.take<int>(c.n_mels);
    q->dev.band_off = a.take<int>(c.n_mels + 1);
    q->dev.band_w = a.take<float>(bw.size());
    q->wh = a.take<uint16_t>((size_t)d * kp);
    q->wl = a.take<uint16_t>((size_t)d * kp);
    q->bias = a.take<float>(d);
    q->inst = a.take<float>((size_t)c.n_instruments * d);
    q->ds = a.take<float>((size_t)c.n_datasets * d);
    q->xh = a.take<__half>(rows * kp);
    q->xl = a.take<__half>(rows * kp);
    q->y = a.take<float>(rows * d);
    q->status = a.take<unsigned>(1);
    if (pass == 0) {
      a.size = round_up(a.used, 256);
      cudaError_t e = cudaMalloc(&a.base, a.size);
      if (e != cudaSuccess) {
        cudaGetLastError();
        delete q;
        return fail(e == cudaErrorMemoryAllocation ? MS_ERR_OOM : MS_ERR_CUDA, "ms_cond_create: cudaMalloc(%zu): %s",
                    a.size, cudaGetErrorString(e));
      }
      q->base = a.base;
    }
  }
  q->dev.n_fft = c.n_fft;
  q->dev.hop = c.hop;
  q->dev.n_mels = c.n_mels;
  q->dev.kp = kp;
  auto cp = [&](const void* dst, const void* src, size_t bytes) -> cudaError_t {
    return cudaMemcpy(const_cast<void*>(dst), src, bytes, cudaMemcpyDefault);
  };
  cudaError_t e = cp(q->dev.window, win.data(), win.size() * sizeof(double));
  if (e == cudaSuccess) e = cp(q->dev.twiddle, tw.data(), tw.size() * sizeof(double2));
  if (e == cudaSuccess) e = cp(q->dev.band_lo, lo.data(), lo.size() * 4);
  if (e == cudaSuccess) e = cp(q->dev.band_off, off.data(), off.size() * 4);
  if (e == cudaSuccess) e = cp(q->dev.band_w, bw.data(), bw.size() * 4);
  if (e == cudaSuccess) e = cp(q->wh, wh.data(), wh.size() * 2);
  if (e == cudaSuccess) e = cp(q->wl, wl.data(), wl.size() * 2);
  if (e == cudaSuccess) e = cp(q->bias, wt->proj_b, (size_t)d * 4);
  if (e == cudaSuccess) e = cp(q->inst, wt->inst_emb, (size_t)c.n_instruments * d * 4);
  if (e == cudaSuccess) e = cp(q->ds, wt->ds_emb, (size_t)c.n_datasets * d * 4);
  if (e == cudaSuccess) e = cudaMemset(q->status, 0, sizeof(unsigned));
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    delete q;
    return fail(MS_ERR_CUDA, "ms_cond_create: copy: %s", cudaGetErrorString(e));
  }
  *out = q;
  return MS_OK;
}

ms_status ms_cond_destroy(ms_cond* cond) {
  if (!cond) return MS_OK;
  DeviceGuard dg(cond->device);
  delete cond;
  return MS_OK;
}

int ms_cond_frames(const ms_cond* cond) { return cond ? cond->frames : 0; }

ms_status ms_cond_log_mel(ms_cond* cond, const float* audio, int B, float* out, void* stream) {
  if (!cond || !audio || !out) return fail(MS_ERR_INVALID_ARG, "ms_cond_log_mel: null argument");
  if (B < 1 || B > cond->cfg.max_batch)
    return fail(MS_ERR_SHAPE, "ms_cond_log_mel: B = %d outside 1..%d", B, cond->cfg.max_batch);
  DeviceGuard dg(cond->device);
  ms::Launch L{(cudaStream_t)stream, false, cond->status};
  return check_launch(ms::launch_log_mel(L, audio, cond->cfg.n_samples, B, cond->dev, cond->frames, out, nullptr,
                                         nullptr),
                      "log_mel");
}

ms_status ms_condition(ms_cond* cond, const float* audio, int B, const int32_t* dataset, const int32_t* instruments,
                       int K, float* prefix, void* stream) {
  if (!cond || !audio || !dataset || !prefix || (K > 0 && !instruments))
    return fail(MS_ERR_INVALID_ARG, "ms_condition: null argument");
  if (B < 1 || B > cond->cfg.max_batch || K < 0 || K > 65536)
    return fail(MS_ERR_SHAPE, "ms_condition: B = %d outside 1..%d or K = %d outside 0..65536", B,
                cond->cfg.max_batch, K);
  if (reinterpret_cast<uintptr_t>(prefix) & 15) return fail(MS_ERR_INVALID_ARG, "ms_condition: prefix must be 16-byte aligned");
  DeviceGuard dg(cond->device);
  int nsm = 0;
  CUDA_TRY(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, cond->device));
  const ms::GemmWork gw{nsm > 0 ? nsm : 1};
  const ms::GemmWeights none{nullptr, nullptr};
  ms::Launch L{(cudaStream_t)stream, false, cond->status};
  const int M = B * cond->frames, d = cond->cfg.d_model;
  cudaError_t e = ms::launch_log_mel(L, audio, cond->cfg.n_samples, B, cond->dev, cond->frames, nullptr, cond->xh,
                                     cond->xl);
  if (e == cudaSuccess)
    e = ms::launch_gemm_f16(L, cond_view(cond, cond->wh), none, cond->xh, cond->xl, cond->kp, M, cond->y, d, nullptr,
                            nullptr, 0, ms::kStore, &gw);
  if (e == cudaSuccess)
    e = ms::launch_gemm_f16(L, cond_view(cond, cond->wl), none, cond->xh, cond->xl, cond->kp, M, cond->y, d, nullptr,
                            nullptr, 0, ms::kAdd, &gw);
  if (e == cudaSuccess)
    e = ms::launch_cond_assemble(L, cond->y, cond->yscale, cond->bias, cond->ds, cond->cfg.n_datasets, cond->inst,
                                 cond->cfg.n_instruments, dataset, instruments, K, cond->frames, d, B, prefix);
  return check_launch(e, "ms_condition");
}

ms_status ms_cond_device_status(ms_cond* cond, void* stream) {
  if (!cond) return fail(MS_ERR_INVALID_ARG, "ms_cond_device_status: null cond");
  DeviceGuard dg(cond->device);
  CUDA_TRY(cudaStreamSynchronize((cudaStream_t)stream));
  unsigned w = 0;
  CUDA_TRY(cudaMemcpy(&w, cond->status, sizeof(unsigned), cudaMemcpyDeviceToHost));
  const unsigned zero = 0;
  CUDA_TRY(cudaMemcpy(cond->status, &zero, sizeof(unsigned), cudaMemcpyHostToDevice));
  if (w & ms::kErrTokenBit)
    return fail(MS_ERR_TOKEN_RANGE, "a dataset or instrument id was outside its table (status 0x%x)", w);
  if (w & ms::kErrShapeBit) return fail(MS_ERR_SHAPE, "a device-side size check failed (status 0x%x)", w);
  return MS_OK;
}

}  // extern "C"
