"""CPU oracle for the MuScriptor KV-cached INT4 decoder step.

TEST INFRASTRUCTURE ONLY.  This is the slow, plain reference that the CUDA
library is checked against.  Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import it; the library never does, and the two share no
code (the seeded input draws in ``synth`` are the only common module, and they
hold none of the arithmetic below).

Floating point: every activation, normalisation, softmax and dot product is
computed in float64 (numpy; BLAS matmul as the one library primitive).  Two
things are integer or fp32 decisions and are taken in fp32 on purpose, because
the method fixes them there: the RTN INT4 quantiser (scale = absmax/7 and
q = rint(w/scale), both IEEE fp32) and the dequantised weight value q*scale
(one fp32 product).  The argmax is taken on the float64 logits, lowest index on
ties.

Sources (page title, section):
  [W4A32]  "MuScriptor Medium — optimized W4A32 ONNX Runtime", sections
           "Model variant" (INT4 g32 symmetric RTN backbone, fp32 activations,
           cache, embeddings and LM head; 96 MatMulNBits, 24 GroupQueryAttention,
           48 SkipLayerNormalization for 24 layers; fixed-capacity shared cache),
           "Quick smoke test" (default cache length 2504, 469.5 MiB).
  [ONNX-S] "MuScriptor small — ONNX conversion", section "muscriptor-small-lm.onnx"
           (tokens i64 [1,S], prefix f32 [1,P,d] with P = 0 after the first
           step, past_k/past_v [L,1,T,Hk,64], logits f32 [1,1393] last position
           only, positions implicit from the cache length, one branch-free graph
           for prefill and decode; greedy decoding).
  [CARD]   "MuScriptor — small (≈100M)" model card, sections "Model description"
           (decoder-only Transformer, spectrogram projected to d_model and used as
           a prefix condition, greedy argmax decoding) and "Model variants".

Readings where the pages are silent (each one is listed with its reason in the
design notes of the repository):
  * four backbone MatMuls per layer (96 / 24): fused QKV, O, FC1, FC2;
  * pre-LayerNorm blocks, a final LayerNorm, eps 1e-5, biased variance;
  * non-gated FFN of width d_ff with exact (erf) GELU;
  * no biases on any MatMul or on the LM head;
  * RoPE, base 1e4, on q and k at every position, pairs (i, i + 32) of each
    64-wide head, angle pos * base^(-2i/64), rotation
    (a, b) -> (a cos - b sin, a sin + b cos); the cache holds post-RoPE keys;
  * fully causal attention over [prefix ; tokens], scale 1/sqrt(64), query head
    h reads kv head h // (H / Hk);
  * INT4 storage: u = q + 8 in a nibble, element 2i in the low nibble of byte i,
    row-major [N][K/2] with row n = output feature n; scales fp32 [N][K/32];
  * ``accuracy_level=4`` (optional, ``act_int8``): activations quantised to INT8 per
    row in blocks of 32 with the weight quantiser's rule at 127 levels a side, integer
    block sums scaled by both scales.  The CUDA library has no such path: it keeps
    fp32 activations.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence

import numpy as np
from scipy.special import erf as _erf

GROUP = 32
QMAX = 7
A8MAX = 127


# ---------------------------------------------------------------------------
# INT4 weight format  [W4A32, "Model variant": symmetric RTN INT4, group size 32]
# ---------------------------------------------------------------------------

def _symmetric_rtn_g32(a: np.ndarray, qmax: int):
    """Symmetric round-to-nearest with one scale per 32 consecutive elements of a row.

    ``a`` is rounded to fp32 [R, K].  For each group: scale = absmax / qmax (fp32
    division), q = clamp(rint(a / scale), -qmax, qmax) (fp32 division, round half to
    even).  An all-zero group has scale 0 and q 0.  Returns (q int8 [R, K], scale fp32
    [R, K/32]).
    """
    a = np.ascontiguousarray(a, dtype=np.float32)
    n, k = a.shape
    if k % GROUP:
        raise ValueError("K must be a multiple of 32")
    g = a.reshape(n, k // GROUP, GROUP)
    absmax = np.max(np.abs(g), axis=2)                                    # fp32
    scale = (absmax / np.float32(qmax)).astype(np.float32)                # fp32 IEEE division
    safe = np.where(scale == 0, np.float32(1), scale).astype(np.float32)
    ratio = (g / safe[:, :, None]).astype(np.float32)                     # fp32 IEEE division
    q = np.clip(np.rint(ratio), -qmax, qmax)
    q = np.where(scale[:, :, None] == 0, 0, q).astype(np.int8)
    return q.reshape(n, k), scale


def quantize_int4_g32(w: np.ndarray):
    """Symmetric round-to-nearest INT4 with one scale per 32 consecutive K elements.

    ``w`` is fp32 [N, K] (row n = output feature n, K = input features).  For each
    group: scale = absmax / 7 (fp32 division), q = clamp(rint(w / scale), -7, 7)
    (fp32 division, round half to even).  An all-zero group has scale 0 and q 0.
    Returns (q int8 [N, K], scale fp32 [N, K/32]).
    """
    return _symmetric_rtn_g32(w, QMAX)


def pack_int4(q: np.ndarray) -> np.ndarray:
    """Pack int8 q in [-8, 7] into bytes: u = q + 8, element 2i low nibble, 2i+1 high nibble."""
    q = np.asarray(q)
    n, k = q.shape
    u = (q.astype(np.int16) + 8).astype(np.uint8)
    lo = u[:, 0::2]
    hi = u[:, 1::2]
    return (lo | (hi << 4)).astype(np.uint8).reshape(n, k // 2)


def unpack_int4(packed: np.ndarray) -> np.ndarray:
    """Inverse of :func:`pack_int4`: bytes [N, K/2] -> int8 q [N, K]."""
    packed = np.asarray(packed, dtype=np.uint8)
    n, kh = packed.shape
    q = np.empty((n, kh * 2), dtype=np.int8)
    q[:, 0::2] = (packed & 0x0F).astype(np.int8) - 8
    q[:, 1::2] = (packed >> 4).astype(np.int8) - 8
    return q


def dequantize(q: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """W[n, k] = q[n, k] * scale[n, k // 32], one fp32 product per element."""
    n, k = q.shape
    s = np.repeat(scale.astype(np.float32), GROUP, axis=1)
    return (q.astype(np.float32) * s).astype(np.float32)


# ---------------------------------------------------------------------------
# INT8 activations, INT32 accumulation  [W4A32, "Model variant": accuracy_level=4]
# ---------------------------------------------------------------------------

def quantize_act_int8_g32(x: np.ndarray):
    """Dynamic symmetric INT8 quantisation of activation rows, one scale per 32 elements.

    [W4A32, "Model variant"]: with ``accuracy_level=4`` the CPU kernels quantise the
    MatMul activations to INT8 at run time and accumulate in INT32.  The page gives
    neither the block length nor the scale or rounding rule.  The reading used: blocks
    of 32 consecutive K elements of a row (the weight group, so every block meets one
    weight scale), with the weight quantiser's rule at 127 levels a side: scale =
    absmax / 127, q = clamp(rint(x / scale), -127, 127), fp32 IEEE divisions, ties to
    even; an all-zero block has scale 0 and q 0.  The graph's activations are fp32, so
    ``x`` [M, K] is rounded to fp32 first.  Returns (q int8 [M, K], scale fp32 [M, K/32]).
    """
    return _symmetric_rtn_g32(x, A8MAX)


def matmul_w4a8(x: np.ndarray, q: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """y[m, n] = sum over blocks b of sa[m, b] * sw[n, b] * (sum_{k in b} qa[m, k] * q[n, k]).

    ``x`` [M, K] activations (quantised here by :func:`quantize_act_int8_g32`), ``q``
    INT4 codes [N, K] and ``scale`` fp32 [N, K/32] of the weight.  Each block's inner
    sum is an exact integer (|sum| <= 32 * 127 * 7 = 28448, which INT32 holds); the
    per-block products sa * sw are exact in float64 and the blocks are summed in
    float64.  Returns float64 [M, N].
    """
    qa, sa = quantize_act_int8_g32(x)
    m, k = qa.shape
    n = q.shape[0]
    y = np.zeros((m, n))
    for b in range(k // GROUP):
        cols = slice(b * GROUP, (b + 1) * GROUP)
        # integers well below 2^53: the float64 matmul is exact
        isum = qa[:, cols].astype(np.float64) @ q[:, cols].astype(np.float64).T
        y += isum * (sa[:, b].astype(np.float64)[:, None] * scale[:, b].astype(np.float64)[None, :])
    return y


# ---------------------------------------------------------------------------
# Layer primitives (float64)
# ---------------------------------------------------------------------------

def layer_norm(x: np.ndarray, gamma: np.ndarray, beta: np.ndarray, eps: float) -> np.ndarray:
    """LayerNorm over the last axis: (x - mean) / sqrt(var + eps) * gamma + beta, biased var.

    [W4A32, "Model variant"]: the SkipLayerNormalization nodes (residual add
    followed by this normalisation).
    """
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * np.asarray(gamma, np.float64) + np.asarray(beta, np.float64)


def gelu_erf(u: np.ndarray) -> np.ndarray:
    """Exact GELU: 0.5 u (1 + erf(u / sqrt 2))."""
    u = np.asarray(u, dtype=np.float64)
    return 0.5 * u * (1.0 + _erf(u / np.sqrt(2.0)))


def rope(x: np.ndarray, positions: np.ndarray, base: float) -> np.ndarray:
    """Rotary position embedding on [T, heads, 64], pairs (i, i + 32), angle pos * base^(-2i/64)."""
    x = np.asarray(x, dtype=np.float64)
    hd = x.shape[-1]
    half = hd // 2
    i = np.arange(half, dtype=np.float64)
    theta = base ** (-2.0 * i / hd)                                       # [32]
    ang = np.asarray(positions, dtype=np.float64)[:, None] * theta[None, :]   # [T, 32]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    a = x[..., :half]
    b = x[..., half:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray,
              q_pos: np.ndarray, k_pos: np.ndarray) -> np.ndarray:
    """Causal grouped-query attention.

    q [Tq, H, 64], k and v [Tk, Hk, 64]; query i sees key j iff k_pos[j] <= q_pos[i].
    Query head h reads kv head h // (H / Hk).  Scores scaled by 1/sqrt(64); softmax
    with the row maximum subtracted.  Returns [Tq, H, 64].
    [W4A32, "Model variant"]: GroupQueryAttention; [ONNX-S]: past_k/past_v heads.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    tq, h, hd = q.shape
    hk = k.shape[1]
    if h % hk:
        raise ValueError("heads must be a multiple of kv heads")
    rep = h // hk
    visible = np.asarray(k_pos)[None, :] <= np.asarray(q_pos)[:, None]   # [Tq, Tk]
    out = np.empty_like(q)
    scale = 1.0 / np.sqrt(hd)
    for hh in range(h):
        g = hh // rep
        s = (q[:, hh, :] @ k[:, g, :].T) * scale
        s = np.where(visible, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        p /= p.sum(axis=1, keepdims=True)
        out[:, hh, :] = p @ v[:, g, :]
    return out


def argmax_lowest(logits: np.ndarray) -> np.ndarray:
    """Greedy choice: index of the maximum, lowest index on ties (over the last axis)."""
    return np.argmax(np.asarray(logits), axis=-1)


def guided(logits_cond: np.ndarray, logits_uncond: np.ndarray, scale: float) -> np.ndarray:
    """Classifier-free guidance of one (conditional, unconditional) pair of logit vectors.

    "MuScriptor — small (≈100M)" model card, Model description: greedy decoding with optional
    classifier-free guidance.  The pages give no formula; the reading used is the usual
    u + scale * (k - u), k the conditional and u the unconditional logits (scale 1: the
    conditional stream alone; scale 0: the unconditional one).
    """
    u = np.asarray(logits_uncond, np.float64)
    return u + scale * (np.asarray(logits_cond, np.float64) - u)


def top2_margin(logits: np.ndarray) -> np.ndarray:
    """Largest minus second-largest logit (over the last axis)."""
    part = np.sort(np.asarray(logits, np.float64), axis=-1)
    return part[..., -1] - part[..., -2]


# ---------------------------------------------------------------------------
# Model
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class OracleLayer:
    ln1_g: np.ndarray
    ln1_b: np.ndarray
    ln2_g: np.ndarray
    ln2_b: np.ndarray
    w: List[np.ndarray]                 # dequantised weights [N, K]: QKV, O, FC1, FC2
    q: Optional[List[np.ndarray]] = None       # int8 codes (INT4 format only)
    s: Optional[List[np.ndarray]] = None       # fp32 scales (INT4 format only)
    packed: Optional[List[np.ndarray]] = None  # bytes (INT4 format only)


class OracleModel:
    """Decoder-only transformer of the pages, weights held dequantised.

    ``weight_format`` "int4": every backbone matrix goes through
    :func:`quantize_int4_g32` and :func:`dequantize` ([W4A32, "Model variant"]).
    "fp16": every backbone matrix is rounded to IEEE half (the half-precision
    weight variant of "MuScriptor for Core AI (.aimodel)", file table).  "fp32":
    the matrices as drawn.  Embeddings, LayerNorms and the LM head stay fp32.

    ``kv_store`` "fp16" (the half-precision cache option; the pages keep the cache in fp32):
    every post-RoPE key and every value is rounded to IEEE half, to nearest with ties to
    even, when it enters the cache, and attention reads the rounded values (the current
    position's included).  Everything else is unchanged.

    ``act_int8`` (INT4 format only): the four backbone MatMuls of every layer take
    their activations through :func:`matmul_w4a8` (the ``accuracy_level=4`` reading);
    attention and the LM head stay as they are, since only the backbone MatMuls are
    MatMulNBits nodes ([W4A32, "Model variant"]).
    """

    def __init__(self, draw, weight_format: str = "int4", store=np.float64, act_int8: bool = False,
                 kv_store: str = "fp32"):
        sh = draw.shape
        self.shape = sh
        self.weight_format = weight_format
        if kv_store not in ("fp32", "fp16"):
            raise ValueError(kv_store)
        self.kv_store = kv_store
        if act_int8 and weight_format != "int4":
            raise ValueError("int8 activations go with the INT4 weight format")
        self.act_int8 = act_int8
        self.L, self.d, self.H, self.Hk = sh.n_layers, sh.d_model, sh.n_heads, sh.n_kv_heads
        self.hd, self.F, self.V = sh.head_dim, sh.d_ff, sh.vocab
        self.base, self.eps = sh.rope_base, sh.ln_eps
        self.tok_emb = np.asarray(draw.tok_emb, np.float32)
        self.lm_head = np.asarray(draw.lm_head, np.float64)
        self.ln_f_g, self.ln_f_b = draw.ln_f_g, draw.ln_f_b
        self.layers: List[OracleLayer] = []
        for ld in draw.layers:
            ws, qs, ss, ps = [], [], [], []
            for w in ld.w:
                if weight_format == "int4":
                    q, s = quantize_int4_g32(w)
                    qs.append(q)
                    ss.append(s)
                    ps.append(pack_int4(q))
                    ws.append(dequantize(q, s).astype(store))
                elif weight_format == "fp16":
                    ws.append(np.asarray(w, np.float32).astype(np.float16).astype(store))
                elif weight_format == "fp32":
                    ws.append(np.asarray(w, np.float32).astype(store))
                else:
                    raise ValueError(weight_format)
            self.layers.append(OracleLayer(ld.ln1_g, ld.ln1_b, ld.ln2_g, ld.ln2_b, ws,
                                           qs or None, ss or None, ps or None))

    def _matmul(self, a: np.ndarray, ly: OracleLayer, i: int) -> np.ndarray:
        """a @ W_i^T for backbone matrix i (QKV, O, FC1, FC2) of layer ``ly``."""
        if self.act_int8:
            return matmul_w4a8(a, ly.q[i], ly.s[i])
        return a @ ly.w[i].T

    # -- one pass over new rows, attending to the cache plus themselves --------
    def _run(self, x: np.ndarray, cache: "OracleCache", all_logits: bool) -> np.ndarray:
        """Append the rows ``x`` [n, d] (in sequence order) to ``cache`` and return logits.

        Positions are implicit: the new rows take positions T..T+n-1 where T is the
        cache length ([ONNX-S]).  Returns logits of every new row if ``all_logits``
        else of the last row only.
        """
        n = x.shape[0]
        t0 = cache.length
        if t0 + n > cache.capacity:
            raise ValueError("cache capacity exceeded")
        pos = np.arange(t0, t0 + n)
        kpos = np.arange(t0 + n)
        H, Hk, hd = self.H, self.Hk, self.hd
        x = np.asarray(x, np.float64)
        for l, ly in enumerate(self.layers):
            h = layer_norm(x, ly.ln1_g, ly.ln1_b, self.eps)
            qkv = self._matmul(h, ly, 0)
            q = qkv[:, : H * hd].reshape(n, H, hd)
            k = qkv[:, H * hd: (H + Hk) * hd].reshape(n, Hk, hd)
            v = qkv[:, (H + Hk) * hd:].reshape(n, Hk, hd)
            q = rope(q, pos, self.base)
            k = rope(k, pos, self.base)
            if self.kv_store == "fp16":
                k = k.astype(np.float16).astype(np.float64)
                v = v.astype(np.float16).astype(np.float64)
            cache.k[l][t0: t0 + n] = k
            cache.v[l][t0: t0 + n] = v
            a = attention(q, cache.k[l][: t0 + n], cache.v[l][: t0 + n], pos, kpos)
            x = x + self._matmul(a.reshape(n, H * hd), ly, 1)
            h = layer_norm(x, ly.ln2_g, ly.ln2_b, self.eps)
            x = x + self._matmul(gelu_erf(self._matmul(h, ly, 2)), ly, 3)
        cache.length = t0 + n
        rows = x if all_logits else x[-1:]
        y = layer_norm(rows, self.ln_f_g, self.ln_f_b, self.eps)
        logits = y @ self.lm_head.T
        return logits if all_logits else logits[0]

    def embed(self, tokens: Sequence[int]) -> np.ndarray:
        tokens = np.asarray(tokens, dtype=np.int64).reshape(-1)
        if tokens.size and (tokens.min() < 0 or tokens.max() >= self.V):
            raise ValueError("token id out of range")
        return self.tok_emb[tokens].astype(np.float64)

    def sequence(self, prefix: Optional[np.ndarray], tokens: Sequence[int]) -> np.ndarray:
        """[prefix ; E[tokens]]: the prefix rows come first ([ONNX-S]; [CARD] prefix condition)."""
        e = self.embed(tokens)
        if prefix is None or len(prefix) == 0:
            return e
        return np.concatenate([np.asarray(prefix, np.float64), e], axis=0)

    def new_cache(self, capacity: int) -> "OracleCache":
        return OracleCache(self.L, self.Hk, self.hd, capacity)

    # -- mode (i): full recompute ------------------------------------------------
    def forward_full(self, prefix: Optional[np.ndarray], tokens: Sequence[int]):
        """Logits at every position of [prefix ; tokens] with no prior cache: [P+S, V]."""
        x = self.sequence(prefix, tokens)
        cache = self.new_cache(x.shape[0])
        return self._run(x, cache, all_logits=True), cache

    # -- mode (ii): incremental with a cache --------------------------------------
    def prefill(self, cache: "OracleCache", prefix: Optional[np.ndarray], tokens: Sequence[int]) -> np.ndarray:
        """Append [prefix ; tokens] to the cache; return last-position logits [V]."""
        return self._run(self.sequence(prefix, tokens), cache, all_logits=False)

    def decode_step(self, cache: "OracleCache", token: int) -> np.ndarray:
        """Append one token; return its logits [V]."""
        return self._run(self.embed([token]), cache, all_logits=False)

    def greedy(self, prefix, start_token: int, n_steps: int, capacity: int):
        """Prefill [prefix ; start], then ``n_steps`` greedy steps feeding the argmax back.

        Returns (tokens int64 [n_steps + 1], logits float64 [n_steps + 1, V]): row 0
        is the prefill's last-position output, row i the output of decode step i.
        """
        cache = self.new_cache(capacity)
        logits = [self.prefill(cache, prefix, [start_token])]
        toks = [int(argmax_lowest(logits[-1]))]
        for _ in range(n_steps):
            logits.append(self.decode_step(cache, toks[-1]))
            toks.append(int(argmax_lowest(logits[-1])))
        return np.array(toks, np.int64), np.stack(logits)

    def greedy_guided(self, prefix_cond, prefix_uncond, start_cond: int, start_uncond: int, n_steps: int,
                      scale: float, capacity: int):
        """Greedy decoding of a (conditional, unconditional) pair with classifier-free
        guidance: both streams are prefilled with their own prefix and start token, then every
        step both receive the argmax of ``guided(k, u, scale)``.

        Returns (tokens int64 [n_steps + 1], logits_cond [n_steps + 1, V], logits_uncond
        [n_steps + 1, V]); row 0 is the prefills' output.
        """
        cc, cu = self.new_cache(capacity), self.new_cache(capacity)
        lc = [self.prefill(cc, prefix_cond, [start_cond])]
        lu = [self.prefill(cu, prefix_uncond, [start_uncond])]
        toks = [int(argmax_lowest(guided(lc[-1], lu[-1], scale)))]
        for _ in range(n_steps):
            lc.append(self.decode_step(cc, toks[-1]))
            lu.append(self.decode_step(cu, toks[-1]))
            toks.append(int(argmax_lowest(guided(lc[-1], lu[-1], scale))))
        return np.array(toks, np.int64), np.stack(lc), np.stack(lu)

    def teacher_forced(self, prefix, tokens: Sequence[int]) -> np.ndarray:
        """Logits after the prefill and after every forced token: [len(tokens), V].

        Row 0 is the output at the first token's position, row i the output at
        token i's position; the same rows a prefill of (prefix, tokens[0]) followed
        by decode steps over tokens[1:] returns.
        """
        logits, _ = self.forward_full(prefix, tokens)
        p = 0 if prefix is None else len(prefix)
        return logits[p:]

    def param_count(self) -> int:
        n = 2 * self.V * self.d + self.d * 2
        for ly in self.layers:
            n += sum(w.size for w in ly.w) + 4 * self.d
        return n


class OracleCache:
    """Post-RoPE keys and values, [L][capacity, Hk, 64] each, plus the current length."""

    def __init__(self, n_layers: int, n_kv_heads: int, head_dim: int, capacity: int):
        self.capacity = capacity
        self.length = 0
        self.k = [np.zeros((capacity, n_kv_heads, head_dim)) for _ in range(n_layers)]
        self.v = [np.zeros((capacity, n_kv_heads, head_dim)) for _ in range(n_layers)]

    def load(self, k: np.ndarray, v: np.ndarray):
        """Set the cache to T given positions of one stream, k and v [L, T, Hk, 64] (the
        pages' past_k / past_v layout without the batch axis); the length becomes T."""
        t = k.shape[1]
        if t > self.capacity:
            raise ValueError("cache capacity exceeded")
        for l in range(len(self.k)):
            self.k[l][:t] = k[l]
            self.v[l][:t] = v[l]
        self.length = t

    def export(self):
        """The pages' cache layout [L, 1, T, Hk, 64] ([ONNX-S] past_k / past_v)."""
        t = self.length
        k = np.stack([kk[:t] for kk in self.k])[:, None]
        v = np.stack([vv[:t] for vv in self.v])[:, None]
        return k, v


# ---------------------------------------------------------------------------
# Conditioner front-end  ([ONNX-S] muscriptor-small-cond.onnx: audio f32 [1, 80000] at
# 16 kHz, instrument ids [1, K], dataset id [1, 1] -> prefix [1, 501 + 1 + K, d], the
# spectrogram inside the graph with the checkpoint's stored window and mel filterbank;
# [CARD] Model description: STFT n_fft 2048, hop 160, 512 mel bins, projected to d_model)
# ---------------------------------------------------------------------------

LOG_FLOOR = 1e-6

# Readings where the pages are silent: centred frames (the signal padded by n_fft / 2 on both
# sides by reflection without repeating the edge sample, so 1 + N // hop frames: 501 for
# 80000 samples, the pages' figure); the magnitude |X| (the pages speak of log-magnitude
# features); the natural logarithm of the mel energies clamped below at 1e-6 (the pages' log
# floor); the prefix rows in the order of the pages' shape 501 + 1 + K: the projected frames,
# then the dataset row, then the K instrument rows.


def stft_magnitude(audio: np.ndarray, window: np.ndarray, hop: int) -> np.ndarray:
    """|STFT| of one signal ``audio`` [N]: [frames, n_fft/2 + 1], frames = 1 + N // hop.

    Frame t covers padded samples [t*hop, t*hop + n_fft) of the signal padded by n_fft/2 on
    each side by reflection (sample -i is sample i), is multiplied by ``window`` and goes
    through the real DFT (numpy's FFT as the library primitive)."""
    x = np.asarray(audio, np.float64)
    w = np.asarray(window, np.float64)
    n_fft = w.shape[0]
    xp = np.pad(x, n_fft // 2, mode="reflect")
    frames = 1 + x.shape[0] // hop
    idx = np.arange(frames)[:, None] * hop + np.arange(n_fft)[None, :]
    return np.abs(np.fft.rfft(xp[idx] * w[None, :], axis=1))


def log_mel(mag: np.ndarray, mel_fb: np.ndarray) -> np.ndarray:
    """ln(max(mag @ fb^T, 1e-6)): [frames, n_mels] from [frames, n_freq] and fb [n_mels, n_freq]."""
    return np.log(np.maximum(mag @ np.asarray(mel_fb, np.float64).T, LOG_FLOOR))


def conditioner(audio: np.ndarray, dataset: Sequence[int], instruments: np.ndarray, cond, hop: int) -> np.ndarray:
    """The conditioner's prefix [B, frames + 1 + K, d] for audio [B, N], dataset ids [B] and
    instrument ids [B, K]; ``cond`` holds window, mel_fb, proj_w [d, n_mels], proj_b [d],
    inst_emb, ds_emb (synth.CondDraw)."""
    audio = np.asarray(audio)
    instruments = np.asarray(instruments, np.int64).reshape(audio.shape[0], -1)
    W = np.asarray(cond.proj_w, np.float64)
    out = []
    for b in range(audio.shape[0]):
        rows = log_mel(stft_magnitude(audio[b], cond.window, hop), cond.mel_fb) @ W.T + np.asarray(cond.proj_b,
                                                                                                    np.float64)
        ds = np.asarray(cond.ds_emb, np.float64)[[int(dataset[b])]]
        inst = np.asarray(cond.inst_emb, np.float64)[instruments[b]]
        out.append(np.concatenate([rows, ds, inst], axis=0))
    return np.stack(out)
