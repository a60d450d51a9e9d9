"""Pins for the CPU oracle: checks against what the pages and the mathematics fix.

None of these compares the oracle with itself.  Each test ties one part of it to
a hand-worked example, a figure the pages print, a closed form, an invariant,
brute force on tiny inputs, or a special case that reduces to a library routine
(torch's layer_norm, gelu and scaled_dot_product_attention).  The last test
plants mistakes in the oracle (on the CPU) and checks that the pins catch them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import synth
from oracle import ms_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------------------
# INT4 g32
# ----------------------------------------------------------------------------

def test_int4_hand_example():
    g = _gold("int4_g32_hand.json")
    w = np.zeros((1, 32 * len(g["groups"])), np.float32)
    for i, grp in enumerate(g["groups"]):
        w[0, 32 * i: 32 * i + len(grp["w_head"])] = grp["w_head"]
    q, s = O.quantize_int4_g32(w)
    packed = O.pack_int4(q)
    for i, grp in enumerate(g["groups"]):
        assert s[0, i] == np.float32(grp["scale"])
        assert list(q[0, 32 * i: 32 * i + 8]) == grp["q_head"]
        assert np.all(q[0, 32 * i + 8: 32 * i + 32] == 0)
        assert list(packed[0, 16 * i: 16 * i + 16]) == grp["bytes"]


def test_pack_unpack_roundtrip_all_bytes():
    b = np.arange(256, dtype=np.uint8).reshape(1, 256)
    q = O.unpack_int4(b)
    assert q.min() == -8 and q.max() == 7
    assert np.array_equal(O.pack_int4(q), b)
    allq = np.array([[a, c] for a in range(-8, 8) for c in range(-8, 8)], np.int8).reshape(1, -1)
    assert np.array_equal(O.unpack_int4(O.pack_int4(allq)), allq)


def test_pack_nibble_order_bruteforce():
    rng = np.random.default_rng(5)
    q = rng.integers(-7, 8, size=(3, 64)).astype(np.int8)
    p = O.pack_int4(q)
    for n in range(3):
        for i in range(32):
            byte = int(p[n, i])
            assert (byte & 15) - 8 == q[n, 2 * i]
            assert (byte >> 4) - 8 == q[n, 2 * i + 1]


def test_quantize_error_bound_and_extremes():
    w = synth.make_matrix(48, 256, seed=11)
    q, s = O.quantize_int4_g32(w)
    assert q.min() >= -7 and q.max() <= 7
    deq = O.dequantize(q, s).astype(np.float64)
    sfull = np.repeat(s, 32, axis=1).astype(np.float64)
    # |w - q s| <= s / 2 up to the fp32 rounding of the division and of the product
    assert np.all(np.abs(w - deq) <= sfull * (0.5 + 1e-5) + 1e-12)
    # the largest magnitude of every group maps to +-7
    g = np.abs(w.reshape(48, 8, 32))
    idx = g.argmax(axis=2)
    qg = q.reshape(48, 8, 32)
    picked = np.take_along_axis(qg, idx[..., None], axis=2)[..., 0]
    assert np.all(np.abs(picked) == 7)
    # no exact ties in continuous random draws (tie rule is then immaterial)
    r = (w.reshape(48, 8, 32) / s[..., None]).astype(np.float32)
    assert not np.any(np.abs(r - np.floor(r)) == 0.5)


def test_quantize_sign_flip_invariance():
    w = synth.make_matrix(8, 128, seed=12)
    q1, s1 = O.quantize_int4_g32(w)
    q2, s2 = O.quantize_int4_g32(-w)
    assert np.array_equal(s1, s2)
    assert np.array_equal(q1, -q2)
    # scaling a group by a power of two scales its scale and keeps its codes
    q3, s3 = O.quantize_int4_g32(w * np.float32(4.0))
    assert np.array_equal(q1, q3) and np.array_equal(s1 * 4, s3)


def test_dequant_matmul_bruteforce():
    w = synth.make_matrix(3, 64, seed=13)
    x = synth.make_activations(2, 64, seed=14)
    q, s = O.quantize_int4_g32(w)
    packed = O.pack_int4(q)
    got = x.astype(np.float64) @ O.dequantize(q, s).astype(np.float64).T
    for m in range(2):
        for n in range(3):
            acc = 0.0
            for k in range(64):
                byte = int(packed[n, k // 2])
                u = (byte >> 4) if (k & 1) else (byte & 15)
                wk = float(np.float32(np.float32(u - 8) * s[n, k // 32]))
                acc += float(x[m, k]) * wk
            assert abs(acc - got[m, n]) <= 1e-12 * (1 + abs(acc))


# ----------------------------------------------------------------------------
# Layer primitives
# ----------------------------------------------------------------------------

def test_layer_norm_closed_form_and_library():
    x = np.array([[1.0, 2.0, 3.0, 4.0]])
    eps = 1e-5
    want = (x - 2.5) / math.sqrt(1.25 + eps)
    assert np.allclose(O.layer_norm(x, np.ones(4), np.zeros(4), eps), want, rtol=0, atol=1e-15)
    c = np.full((1, 16), 3.25)
    beta = np.linspace(-1, 1, 16)
    assert np.allclose(O.layer_norm(c, np.ones(16) * 2.0, beta, eps), beta, atol=1e-15)
    xr = synth.make_activations(5, 96, seed=15).astype(np.float64) * 3 + 1
    gm = 1 + 0.1 * synth.make_activations(1, 96, seed=16)[0].astype(np.float64)
    bt = 0.1 * synth.make_activations(1, 96, seed=17)[0].astype(np.float64)
    lib = F.layer_norm(torch.from_numpy(xr), (96,), torch.from_numpy(gm), torch.from_numpy(bt), eps).numpy()
    assert np.allclose(O.layer_norm(xr, gm, bt, eps), lib, rtol=0, atol=1e-13)
    h = O.layer_norm(xr, np.ones(96), np.zeros(96), eps)
    assert np.allclose(h.mean(axis=1), 0, atol=1e-14)
    assert np.allclose(h.var(axis=1), 1.0, atol=1e-4)


def test_gelu_closed_forms_and_library():
    assert O.gelu_erf(np.array([0.0]))[0] == 0.0
    # Phi(1) = 0.841344746068542948585232545632...
    assert abs(O.gelu_erf(np.array([1.0]))[0] - 0.8413447460685429) < 1e-15
    u = np.linspace(-6, 6, 97)
    assert np.allclose(O.gelu_erf(u) - O.gelu_erf(-u), u, atol=1e-14)
    lib = F.gelu(torch.from_numpy(u), approximate="none").numpy()
    assert np.allclose(O.gelu_erf(u), lib, atol=1e-14)


def test_rope_identity_norm_and_unit_vectors():
    x = synth.make_activations(4, 3 * 64, seed=18).astype(np.float64).reshape(4, 3, 64)
    assert np.array_equal(O.rope(x, np.zeros(4), 1e4), x)
    pos = np.array([1, 7, 100, 2503])
    y = O.rope(x, pos, 1e4)
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    # unit vector e_i at position p lands on (cos p*theta_i, sin p*theta_i) at (i, i+32)
    for i in (0, 1, 13, 31):
        e = np.zeros((1, 1, 64))
        e[0, 0, i] = 1.0
        p = 37
        th = 1e4 ** (-2.0 * i / 64)
        r = O.rope(e, np.array([p]), 1e4)[0, 0]
        assert abs(r[i] - math.cos(p * th)) < 1e-14 and abs(r[i + 32] - math.sin(p * th)) < 1e-14
        assert np.count_nonzero(np.abs(r) > 1e-15) <= 2
        e2 = np.zeros((1, 1, 64))
        e2[0, 0, i + 32] = 1.0
        r2 = O.rope(e2, np.array([p]), 1e4)[0, 0]
        assert abs(r2[i] + math.sin(p * th)) < 1e-14 and abs(r2[i + 32] - math.cos(p * th)) < 1e-14


def test_rope_relative_position():
    q = synth.make_activations(1, 64, seed=19).astype(np.float64).reshape(1, 1, 64)
    k = synth.make_activations(1, 64, seed=20).astype(np.float64).reshape(1, 1, 64)
    dots = []
    for p0 in (0, 5, 123, 1999):
        rq = O.rope(q, np.array([p0 + 9]), 1e4)
        rk = O.rope(k, np.array([p0]), 1e4)
        dots.append(float((rq * rk).sum()))
    assert np.allclose(dots, dots[0], rtol=1e-10)


def _attention_bruteforce(q, k, v, qpos, kpos):
    tq, h, hd = q.shape
    hk = k.shape[1]
    out = np.zeros_like(q)
    for i in range(tq):
        for hh in range(h):
            g = hh // (h // hk)
            sc = []
            for j in range(k.shape[0]):
                if kpos[j] <= qpos[i]:
                    sc.append((j, sum(q[i, hh, c] * k[j, g, c] for c in range(hd)) / 8.0))
            m = max(s for _, s in sc)
            w = [(j, math.exp(s - m)) for j, s in sc]
            z = sum(e for _, e in w)
            for j, e in w:
                out[i, hh] += (e / z) * v[j, g]
    return out


@pytest.mark.parametrize("h,hk", [(1, 1), (2, 1), (4, 2), (4, 1), (2, 2)])
def test_attention_bruteforce(h, hk):
    tq, tk = 3, 6
    q = synth.make_activations(tq, h * 64, seed=21).astype(np.float64).reshape(tq, h, 64)
    k = synth.make_activations(tk, hk * 64, seed=22).astype(np.float64).reshape(tk, hk, 64)
    v = synth.make_activations(tk, hk * 64, seed=23).astype(np.float64).reshape(tk, hk, 64)
    qpos = np.array([3, 4, 5])
    kpos = np.arange(tk)
    got = O.attention(q, k, v, qpos, kpos)
    want = _attention_bruteforce(q, k, v, qpos, kpos)
    assert np.allclose(got, want, rtol=0, atol=1e-13)


def test_attention_special_cases():
    # one visible key: the output is that value exactly
    q = synth.make_activations(1, 128, seed=24).astype(np.float64).reshape(1, 2, 64)
    k = synth.make_activations(4, 64, seed=25).astype(np.float64).reshape(4, 1, 64)
    v = synth.make_activations(4, 64, seed=26).astype(np.float64).reshape(4, 1, 64)
    out = O.attention(q, k, v, np.array([0]), np.arange(4))
    assert np.array_equal(out[0, 0], v[0, 0]) and np.array_equal(out[0, 1], v[0, 0])
    # kv heads = heads, and GQA: torch's scaled_dot_product_attention (causal)
    for h, hk in ((3, 3), (4, 2), (6, 1)):
        t = 9
        q = synth.make_activations(t, h * 64, seed=27).astype(np.float64).reshape(t, h, 64)
        k = synth.make_activations(t, hk * 64, seed=28).astype(np.float64).reshape(t, hk, 64)
        v = synth.make_activations(t, hk * 64, seed=29).astype(np.float64).reshape(t, hk, 64)
        lib = F.scaled_dot_product_attention(
            torch.from_numpy(q).permute(1, 0, 2)[None], torch.from_numpy(k).permute(1, 0, 2)[None],
            torch.from_numpy(v).permute(1, 0, 2)[None], is_causal=True, enable_gqa=(h != hk))
        lib = lib[0].permute(1, 0, 2).numpy()
        assert np.allclose(O.attention(q, k, v, np.arange(t), np.arange(t)), lib, atol=1e-13)


# ----------------------------------------------------------------------------
# Whole model
# ----------------------------------------------------------------------------

def _tiny_model(L=2, h=2, hk=1, ln_random=True, fmt="int4", vocab=37):
    sh = synth.tiny_shape(n_layers=L, n_heads=h, n_kv_heads=hk, vocab=vocab)
    draw = synth.make_weights(sh, seed=31, std=0.08, ln_random=ln_random)
    return O.OracleModel(draw, fmt)


def _torch_library_forward(m, prefix, tokens):
    """The same decoder assembled from torch library routines in float64.

    RoPE is written as a complex rotation (a + ib) * exp(i p theta) of each
    (i, i + 32) pair, attention is torch's causal scaled_dot_product_attention
    with grouped KV heads, LayerNorm and GELU are torch's.
    """
    x = torch.from_numpy(m.sequence(prefix, tokens))
    n = x.shape[0]
    H, Hk, hd = m.H, m.Hk, m.hd
    pos = torch.arange(n, dtype=torch.float64)
    theta = m.base ** (-torch.arange(0, hd, 2, dtype=torch.float64) / hd)
    rot = torch.polar(torch.ones(n, hd // 2, dtype=torch.float64), pos[:, None] * theta[None])

    def rope_c(t):  # t [n, heads, 64]
        z = torch.complex(t[..., : hd // 2], t[..., hd // 2:]) * rot[:, None, :]
        return torch.cat([z.real, z.imag], dim=-1)

    def ln(t, g, b):
        return F.layer_norm(t, (m.d,), torch.from_numpy(np.asarray(g, np.float64)),
                            torch.from_numpy(np.asarray(b, np.float64)), m.eps)

    for ly in m.layers:
        W = [torch.from_numpy(w.astype(np.float64)) for w in ly.w]
        h = ln(x, ly.ln1_g, ly.ln1_b)
        qkv = F.linear(h, W[0])
        q = rope_c(qkv[:, : H * hd].reshape(n, H, hd))
        k = rope_c(qkv[:, H * hd: (H + Hk) * hd].reshape(n, Hk, hd))
        v = qkv[:, (H + Hk) * hd:].reshape(n, Hk, hd)
        a = F.scaled_dot_product_attention(q.permute(1, 0, 2)[None], k.permute(1, 0, 2)[None],
                                           v.permute(1, 0, 2)[None], is_causal=True,
                                           enable_gqa=(H != Hk))[0].permute(1, 0, 2)
        x = x + F.linear(a.reshape(n, H * hd), W[1])
        h = ln(x, ly.ln2_g, ly.ln2_b)
        x = x + F.linear(F.gelu(F.linear(h, W[2]), approximate="none"), W[3])
    y = ln(x, m.ln_f_g, m.ln_f_b)
    return F.linear(y, torch.from_numpy(m.lm_head)).numpy()


@pytest.mark.parametrize("h,hk,fmt", [(2, 1, "int4"), (2, 2, "int4"), (4, 2, "fp16")])
def test_model_matches_torch_library_assembly(h, hk, fmt):
    m = _tiny_model(L=2, h=h, hk=hk, fmt=fmt)
    prefix = synth.make_prefix(m.shape, 1, prefix_len=5, seed=32)[0]
    toks = synth.make_token_sequence(4, 1, vocab=m.V, seed=33)[0]
    got, _ = m.forward_full(prefix, toks)
    want = _torch_library_forward(m, prefix, toks)
    assert got.shape == (9, m.V)
    assert np.allclose(got, want, rtol=0, atol=1e-11)


def test_incremental_equals_full_recompute():
    m = _tiny_model(L=2, h=4, hk=2)
    prefix = synth.make_prefix(m.shape, 1, prefix_len=6, seed=34)[0]
    toks = synth.make_token_sequence(7, 1, vocab=m.V, seed=35)[0]
    full, full_cache = m.forward_full(prefix, toks)
    cache = m.new_cache(32)
    rows = [m.prefill(cache, prefix, toks[:1])]
    for t in toks[1:]:
        rows.append(m.decode_step(cache, int(t)))
    inc = np.stack(rows)
    assert np.allclose(inc, full[6:], rtol=0, atol=1e-12)
    ki, vi = cache.export()
    kf, vf = full_cache.export()
    assert np.allclose(ki, kf, atol=1e-12) and np.allclose(vi, vf, atol=1e-12)
    # prefill in two calls (prefix first, then tokens with no prefix) is the same sequence
    c2 = m.new_cache(32)
    m.prefill(c2, prefix, [])
    last = m.prefill(c2, None, toks)
    assert np.allclose(last, full[-1], atol=1e-12)


def test_causality():
    m = _tiny_model(L=2, h=2, hk=1)
    prefix = synth.make_prefix(m.shape, 1, prefix_len=4, seed=36)[0]
    toks = synth.make_token_sequence(6, 1, vocab=m.V, seed=37)[0]
    a, _ = m.forward_full(prefix, toks)
    toks2 = toks.copy()
    toks2[4] = (toks2[4] + 5) % m.V
    b, _ = m.forward_full(prefix, toks2)
    assert np.array_equal(a[: 4 + 4], b[: 4 + 4])
    assert not np.allclose(a[8], b[8])


def _sequence_mismatches(m, draw):
    """Where [prefix ; E[tokens]] differs from its definition, checked row by row against
    the drawn prefix and embedding table (muscriptor-small-lm.onnx of "MuScriptor small —
    ONNX conversion": the prefix rows come first, then one embedding row per token)."""
    prefix = synth.make_prefix(m.shape, 1, prefix_len=4, seed=45)[0]
    toks = [3, 0, m.V - 1, 3]
    seq = m.sequence(prefix, toks)
    bad = []
    if seq.shape != (4 + len(toks), m.d):
        return ["shape"]
    for i in range(4):
        if not np.array_equal(seq[i], prefix[i].astype(np.float64)):
            bad.append(("prefix row", i))
    for i, t in enumerate(toks):
        if not np.array_equal(seq[4 + i], draw.tok_emb[t].astype(np.float64)):
            bad.append(("token row", i))
    return bad


def test_sequence_is_prefix_then_token_embeddings():
    sh = synth.tiny_shape(n_layers=1, n_heads=2, n_kv_heads=1, vocab=37)
    draw = synth.make_weights(sh, seed=31, std=0.08)
    m = O.OracleModel(draw, "int4")
    assert _sequence_mismatches(m, draw) == []
    # the prefix conditions what follows it, and nothing after it reaches back
    prefix = synth.make_prefix(sh, 1, prefix_len=4, seed=46)[0]
    toks = synth.make_token_sequence(3, 1, vocab=m.V, seed=47)[0]
    a, _ = m.forward_full(prefix, toks)
    other = prefix.copy()
    other[1] = -other[1]            # (a constant shift would vanish in the LayerNorm)
    b, _ = m.forward_full(other, toks)
    assert np.array_equal(a[:1], b[:1]) and not np.allclose(a[4], b[4])
    toks2 = toks.copy()
    toks2[0] = (toks2[0] + 1) % m.V
    c, _ = m.forward_full(prefix, toks2)
    assert np.array_equal(a[:4], c[:4])


def test_fp16_weights_are_the_ieee_half_of_the_draw():
    """The fp16 variant ("MuScriptor for Core AI (.aimodel)", file table: weights cast to
    half) against torch's own float32 -> float16 cast (round to nearest even)."""
    sh = synth.tiny_shape(n_layers=2, n_heads=2, n_kv_heads=1, vocab=37)
    draw = synth.make_weights(sh, seed=31, std=0.08)
    m = O.OracleModel(draw, "fp16")
    for ly, ld in zip(m.layers, draw.layers):
        for w_oracle, w_drawn in zip(ly.w, ld.w):
            want = torch.from_numpy(np.asarray(w_drawn, np.float32)).half().double().numpy()
            assert np.array_equal(w_oracle, want)
    assert np.array_equal(m.lm_head, np.asarray(draw.lm_head, np.float32).astype(np.float64))


def test_sequence_order_mistake_is_caught(monkeypatch):
    sh = synth.tiny_shape(n_layers=1, n_heads=2, n_kv_heads=1, vocab=37)
    draw = synth.make_weights(sh, seed=31, std=0.08)
    m = O.OracleModel(draw, "int4")

    def tokens_first(prefix, tokens):
        return np.concatenate([m.embed(tokens), np.asarray(prefix, np.float64)], axis=0)

    monkeypatch.setattr(m, "sequence", tokens_first)
    assert _sequence_mismatches(m, draw)


def test_shapes_per_step_follow_the_pages():
    figs = _gold("pages_figures.json")
    m = _tiny_model(L=3, h=2, hk=1, vocab=figs["vocab"]["value"])
    prefix = synth.make_prefix(m.shape, 1, prefix_len=7, seed=38)[0]
    cache = m.new_cache(16)
    logits = m.prefill(cache, prefix, [5])
    assert logits.shape == (figs["vocab"]["value"],)
    k, v = cache.export()
    assert k.shape == (3, 1, 8, 1, 64) and v.shape == k.shape          # [L, 1, T, Hk, 64]
    m.decode_step(cache, int(O.argmax_lowest(logits)))
    assert cache.export()[0].shape == (3, 1, 9, 1, 64)
    with pytest.raises(ValueError):
        m.prefill(cache, prefix, [1])                                   # 9 + 8 > 16: no room


def test_zero_layers_is_embedding_then_head():
    sh = synth.tiny_shape(n_layers=0, vocab=29)
    draw = synth.make_weights(sh, seed=39, std=0.1, ln_random=True)
    m = O.OracleModel(draw, "int4")
    logits = m.prefill(m.new_cache(4), None, [17])
    e = [float(t) for t in draw.tok_emb[17]]
    mu = sum(e) / len(e)
    var = sum((t - mu) ** 2 for t in e) / len(e)
    y = [(t - mu) / math.sqrt(var + 1e-5) * float(g) + float(b) for t, g, b in zip(e, draw.ln_f_g, draw.ln_f_b)]
    want = [sum(yy * float(w) for yy, w in zip(y, row)) for row in draw.lm_head]
    assert np.allclose(logits, want, atol=1e-12)


def test_residual_passthrough_when_block_outputs_vanish():
    sh = synth.tiny_shape(n_layers=2, vocab=23)
    draw = synth.make_weights(sh, seed=40, std=0.1, ln_random=True)
    for ly in draw.layers:
        ly.w[1][:] = 0.0      # W_o
        ly.w[3][:] = 0.0      # W_2
    m = O.OracleModel(draw, "int4")
    prefix = synth.make_prefix(sh, 1, prefix_len=3, seed=41)[0]
    logits = m.prefill(m.new_cache(8), prefix, [4, 9])
    y = O.layer_norm(draw.tok_emb[9].astype(np.float64), draw.ln_f_g, draw.ln_f_b, 1e-5)
    assert np.allclose(logits, y @ draw.lm_head.astype(np.float64).T, atol=1e-12)


def test_param_counts_and_cache_size_match_the_pages():
    figs = _gold("pages_figures.json")
    for name, (d, h, L) in figs["variants"]["value"].items():
        # page-faithful attention: kv heads = heads (small page: past_k has 12 heads)
        sh = synth.Shape(name, L, d, h, h, 4 * d)
        n = 2 * sh.vocab * d + sum(nn * kk for nn, kk in sh.matmul_shapes()) * L + (4 * L + 2) * d
        lo, hi = figs["params"]["value"][name]
        assert 0.97 * lo <= n <= 1.03 * hi, (name, n)
    assert figs["medium_ops"]["value"]["MatMulNBits"] == 4 * figs["medium_ops"]["value"]["layers"]
    # the medium cache at 2504 positions with 16 kv heads of 64, K and V, fp32
    nbytes = 2 * 24 * 2504 * 16 * 64 * 4
    assert round(nbytes / 2 ** 20, 1) == figs["medium_cache_mib_at_2504"]["value"]
    c = O.OracleCache(24, 16, 64, 2504)
    assert 2 * sum(k.size for k in c.k) * 4 == nbytes
    assert list(figs["small_past_k"]["value"][:2]) == [synth.SMALL.n_layers, 1]
    assert figs["small_past_k"]["value"][3:] == [synth.SMALL.n_kv_heads, synth.HEAD_DIM]
    assert figs["prefix_rows"]["value"] == synth.PREFIX_LEN


def test_greedy_feeds_argmax_back():
    m = _tiny_model(L=1, h=2, hk=1)
    prefix = synth.make_prefix(m.shape, 1, prefix_len=3, seed=42)[0]
    toks, logits = m.greedy(prefix, 3, 5, capacity=16)
    assert toks.shape == (6,) and logits.shape == (6, m.V)
    forced = m.teacher_forced(prefix, [3] + list(toks[:-1]))
    assert np.allclose(forced, logits, atol=1e-12)
    assert np.array_equal(O.argmax_lowest(forced), toks)
    tie = np.array([0.5, 2.0, 2.0, -1.0])
    assert O.argmax_lowest(tie) == 1


def _top2_margin_mismatches(fn):
    """The checks top2_margin must pass (it decides where the greedy comparisons stop):
    a hand-worked batch of rows, ties, a single row, and a brute-force scan on random rows.
    Returns the names of the checks that fail."""
    bad = []
    # rows: max 3.5 over 3.0; a tie at the top (margin 0); max 5 over a tied 4.25
    hand = np.array([[1.0, 3.5, 2.0, 3.0], [0.0, -1.0, -1.0, 0.0], [5.0, 4.25, -3.0, 4.25]])
    try:
        if not np.array_equal(np.asarray(fn(hand)), np.array([0.5, 0.0, 0.75])):
            bad.append("hand rows")
        if float(fn(np.array([2.0, -7.0, 1.5]))) != 0.5:
            bad.append("single row")
        rng = np.random.default_rng(7)
        x = rng.standard_normal((5, 11))
        want = []
        for row in x:
            i = max(range(len(row)), key=lambda j: row[j])
            second = max(row[j] for j in range(len(row)) if j != i)
            want.append(row[i] - second)
        if not np.allclose(np.asarray(fn(x)), want, rtol=0, atol=0):
            bad.append("brute force")
    except Exception:            # a planted mistake may not even run
        bad.append("raised")
    return bad


def test_top2_margin_pins():
    assert _top2_margin_mismatches(O.top2_margin) == []


def test_top2_margin_wrong_axis_is_caught():
    def wrong_axis(logits):
        part = np.sort(np.asarray(logits, np.float64), axis=0)
        return part[..., -1] - part[..., -2]

    def abs_gap_of_ends(logits):
        part = np.sort(np.asarray(logits, np.float64), axis=-1)
        return part[..., -1] - part[..., 0]

    assert _top2_margin_mismatches(wrong_axis)
    assert _top2_margin_mismatches(abs_gap_of_ends)


# ----------------------------------------------------------------------------
# Planted mistakes: each must be caught by at least one pin above
# ----------------------------------------------------------------------------

_ORIG_ROPE = O.rope


def _rope_wrong_sign(x, positions, base):
    return _ORIG_ROPE(x, -np.asarray(positions), base)


def _rope_interleaved(x, positions, base):
    y = np.asarray(x, np.float64).copy()
    a, b = y[..., 0::2].copy(), y[..., 1::2].copy()
    ang = np.asarray(positions, np.float64)[:, None] * base ** (-2.0 * np.arange(32) / 64)
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    y[..., 0::2], y[..., 1::2] = a * c - b * s, a * s + b * c
    return y


def _ln_unbiased(x, g, b, eps):
    x = np.asarray(x, np.float64)
    mu = x.mean(-1, keepdims=True)
    return (x - mu) / np.sqrt(x.var(-1, ddof=1, keepdims=True) + eps) * g + b


def _gelu_tanh(u):
    u = np.asarray(u, np.float64)
    return 0.5 * u * (1 + np.tanh(np.sqrt(2 / np.pi) * (u + 0.044715 * u ** 3)))


def _attention_interleaved_groups(q, k, v, qp, kp):
    h, hk = q.shape[1], k.shape[1]
    perm = np.array([hh % hk for hh in range(h)])     # h -> h mod Hk instead of h // (H/Hk)
    kk = k[:, perm, :]
    vv = v[:, perm, :]
    return _ORIG_ATT(q, kk, vv, qp, kp)


_ORIG_ATT = O.attention


@pytest.mark.parametrize("name,patch", [
    ("rope sign", ("rope", _rope_wrong_sign)),
    ("rope pairing", ("rope", _rope_interleaved)),
    ("layernorm variance", ("layer_norm", _ln_unbiased)),
    ("gelu variant", ("gelu_erf", _gelu_tanh)),
    ("kv head mapping", ("attention", _attention_interleaved_groups)),
])
def test_planted_mistakes_are_caught(monkeypatch, name, patch):
    attr, fn = patch
    m = _tiny_model(L=2, h=4, hk=2, fmt="int4")
    prefix = synth.make_prefix(m.shape, 1, prefix_len=5, seed=43)[0]
    toks = synth.make_token_sequence(4, 1, vocab=m.V, seed=44)[0]
    want = _torch_library_forward(m, prefix, toks)
    monkeypatch.setattr(O, attr, fn)
    got, _ = m.forward_full(prefix, toks)
    assert not np.allclose(got, want, rtol=0, atol=1e-6), name


# ---------------------------------------------------------------------------
# Classifier-free guidance ("MuScriptor — small (≈100M)" model card, Model description;
# reading u + scale (k - u))
# ---------------------------------------------------------------------------

def test_guidance_combination_by_hand():
    # u = [0, 1], k = [2, 0]: scale 3 gives [6, -2] (picks 0, where u alone picks 1)
    g = O.guided(np.array([2.0, 0.0]), np.array([0.0, 1.0]), 3.0)
    assert np.array_equal(g, np.array([6.0, -2.0]))
    assert int(O.argmax_lowest(g)) == 0 and int(O.argmax_lowest(np.array([0.0, 1.0]))) == 1


def test_guided_greedy_reduces_to_each_stream():
    """Scale 1 follows the conditional stream alone, scale 0 the unconditional one: the
    guided driver then equals the plain greedy driver on that stream."""
    sh = synth.tiny_shape()
    om = O.OracleModel(synth.make_weights(sh, seed=0, std=0.05), "int4")
    pc = synth.make_prefix(sh, 1, prefix_len=6, seed=11)[0]
    pu = synth.make_prefix(sh, 1, prefix_len=6, seed=12)[0]
    for scale, (prefix, start) in ((1.0, (pc, 5)), (0.0, (pu, 9))):
        toks, lc, lu = om.greedy_guided(pc, pu, 5, 9, 6, scale, capacity=16)
        ref_toks, ref_lg = om.greedy(prefix, start, 6, capacity=16)
        assert np.array_equal(toks, ref_toks)
        assert np.array_equal(lc if scale == 1.0 else lu, ref_lg)


def test_guided_greedy_feeds_both_streams_the_same_token():
    sh = synth.tiny_shape()
    om = O.OracleModel(synth.make_weights(sh, seed=0, std=0.05), "int4")
    pc = synth.make_prefix(sh, 1, prefix_len=6, seed=11)[0]
    pu = synth.make_prefix(sh, 1, prefix_len=6, seed=12)[0]
    toks, lc, lu = om.greedy_guided(pc, pu, 5, 9, 5, 2.0, capacity=16)
    # each stream's logits are its own teacher-forced outputs on the shared tokens
    tf_c = om.teacher_forced(pc, [5] + list(toks[:-1]))
    tf_u = om.teacher_forced(pu, [9] + list(toks[:-1]))
    assert np.abs(lc - tf_c).max() < 1e-9 and np.abs(lu - tf_u).max() < 1e-9
    for i in range(len(toks)):
        assert toks[i] == int(np.argmax(lu[i] + 2.0 * (lc[i] - lu[i])))


# ---------------------------------------------------------------------------
# INT8 activations with INT32 accumulation ("MuScriptor Medium — optimized W4A32 ONNX
# Runtime", Model variant: accuracy_level=4; reading: blocks of 32, absmax / 127, ties to
# even, integer block sums scaled by both scales)
# ---------------------------------------------------------------------------

def _a8_hand_row(g):
    x = np.zeros((1, g["K"]), np.float32)
    for b, blk in enumerate(g["blocks"]):
        x[0, 32 * b: 32 * b + len(blk["x_head"])] = blk["x_head"]
    return x


def _a8_hand_mismatches(g):
    """What of the hand example the oracle's quantiser gets wrong (empty when right)."""
    bad = []
    try:
        qa, sa = O.quantize_act_int8_g32(_a8_hand_row(g))
    except Exception as e:          # a planted mistake may not even run
        return [repr(e)]
    if qa.shape != (1, g["K"]) or sa.shape != (1, len(g["blocks"])):
        return ["shapes"]
    for b, blk in enumerate(g["blocks"]):
        if float(sa[0, b]) != blk["scale"]:
            bad.append(("scale", b, float(sa[0, b])))
        head = [int(v) for v in qa[0, 32 * b: 32 * b + len(blk["q_head"])]]
        if head != blk["q_head"]:
            bad.append(("codes", b, head))
        if np.any(qa[0, 32 * b + len(blk["q_head"]): 32 * (b + 1)] != 0):
            bad.append(("tail", b))
    return bad


def _w4a8_bruteforce_err(seed):
    """Largest gap between matmul_w4a8 and scalar loops over bytes and Python integers."""
    x = synth.make_activations(2, 64, seed=seed)
    x[1, 32:] = 0.0                                    # an all-zero block
    w = synth.make_matrix(3, 64, seed=seed + 1)
    q, s = O.quantize_int4_g32(w)
    packed = O.pack_int4(q)
    got = O.matmul_w4a8(x, q, s)
    worst = 0.0
    for m in range(2):
        for n in range(3):
            acc = 0.0
            for b in range(2):
                blk = [np.float32(v) for v in x[m, 32 * b: 32 * b + 32]]
                amax = max(abs(v) for v in blk)
                sa = np.float32(amax / np.float32(127))
                isum = 0
                for j, v in enumerate(blk):
                    code = 0 if sa == 0 else max(-127, min(127, round(float(np.float32(v / sa)))))
                    byte = int(packed[n, (32 * b + j) // 2])
                    wq = ((byte >> 4) if (j & 1) else (byte & 15)) - 8
                    isum += code * wq
                acc += isum * (float(sa) * float(s[n, b]))
            worst = max(worst, abs(acc - got[m, n]) / (1 + abs(acc)))
    return worst


def test_a8_hand_example():
    g = _gold("a8_block_hand.json")
    assert _a8_hand_mismatches(g) == []
    mm = g["matmul"]
    q = np.zeros((1, g["K"]), np.int8)
    for b, (head, fill) in enumerate(zip(mm["w_q_head"], mm["w_q_fill"])):
        q[0, 32 * b: 32 * (b + 1)] = fill
        q[0, 32 * b: 32 * b + len(head)] = head
    s = np.array([mm["w_scale"]], np.float32)
    x = _a8_hand_row(g)
    assert O.matmul_w4a8(x, q, s)[0, 0] == mm["y"]
    # the same weights with fp32 activations, through the pinned dequantised path
    assert (x.astype(np.float64) @ O.dequantize(q, s).astype(np.float64).T)[0, 0] == mm["y_fp32_activations"]


def test_a8_error_bound_and_extremes():
    x = synth.make_activations(5, 256, seed=51) * np.float32(3.0)
    qa, sa = O.quantize_act_int8_g32(x)
    assert qa.dtype == np.int8 and np.abs(qa.astype(np.int32)).max() <= 127
    back = qa.astype(np.float64).reshape(5, 8, 32) * sa.astype(np.float64)[:, :, None]
    err = np.abs(back - x.astype(np.float64).reshape(5, 8, 32))
    assert np.all(err <= sa.astype(np.float64)[:, :, None] * (0.5 + 1e-6))
    # each block's largest magnitude lands on +-127, with its sign
    blocks = x.reshape(5, 8, 32)
    arg = np.abs(blocks).argmax(axis=2)
    top = np.take_along_axis(qa.reshape(5, 8, 32), arg[:, :, None], axis=2)[:, :, 0]
    sign = np.sign(np.take_along_axis(blocks, arg[:, :, None], axis=2)[:, :, 0])
    assert np.array_equal(top.astype(np.int32), (127 * sign).astype(np.int32))


def test_a8_power_of_two_and_sign_invariance():
    x = synth.make_activations(3, 128, seed=52)
    w = synth.make_matrix(4, 128, seed=53)
    q, s = O.quantize_int4_g32(w)
    qa, sa = O.quantize_act_int8_g32(x)
    y = O.matmul_w4a8(x, q, s)
    for j in (-12, 5):
        f = np.float32(2.0 ** j)
        qa2, sa2 = O.quantize_act_int8_g32(x * f)
        assert np.array_equal(qa2, qa) and np.array_equal(sa2, sa * f)
        assert np.array_equal(O.matmul_w4a8(x * f, q, s), y * float(f))
    qn, sn = O.quantize_act_int8_g32(-x)
    assert np.array_equal(qn, -qa) and np.array_equal(sn, sa)


def test_w4a8_matmul_bruteforce():
    assert _w4a8_bruteforce_err(54) <= 1e-12


def test_w4a8_reduces_to_w4a32_on_exact_activations():
    """Blocks of integers whose largest magnitude is 127 have scale 1 and codes equal to the
    values, so the INT8 path must give the plain product x W^T with W = q * s.  (W is formed
    in float64 here: the INT8 path scales exact integer sums and never rounds q * s to fp32
    the way the W4A32 dequantiser does.)"""
    g = np.random.default_rng(55)
    x = g.integers(-127, 128, size=(3, 96)).astype(np.float32)
    x[:, ::32] = np.float32(127) * np.where(g.random((3, 3)) < 0.5, -1, 1)
    qa, sa = O.quantize_act_int8_g32(x)
    assert np.all(sa == 1) and np.array_equal(qa.astype(np.float32), x)
    w = synth.make_matrix(5, 96, seed=56)
    q, s = O.quantize_int4_g32(w)
    wd = q.astype(np.float64) * np.repeat(s.astype(np.float64), 32, axis=1)
    want = x.astype(np.float64) @ wd.T
    assert np.allclose(O.matmul_w4a8(x, q, s), want, rtol=1e-13, atol=1e-13)


def test_w4a8_model_is_causal_and_incremental():
    sh = synth.tiny_shape()
    m = O.OracleModel(synth.make_weights(sh, seed=0, std=0.05), "int4", act_int8=True)
    plain = O.OracleModel(synth.make_weights(sh, seed=0, std=0.05), "int4")
    prefix = synth.make_prefix(sh, 1, prefix_len=6, seed=57)[0]
    toks = synth.make_token_sequence(5, 1, vocab=m.V, seed=58)[0]
    full, _ = m.forward_full(prefix, toks)
    cache = m.new_cache(16)
    rows = [m.prefill(cache, prefix, toks[:1])] + [m.decode_step(cache, int(t)) for t in toks[1:]]
    assert np.allclose(np.stack(rows), full[6:], rtol=0, atol=1e-12)
    toks2 = toks.copy()
    toks2[3] = (toks2[3] + 1) % m.V
    full2, _ = m.forward_full(prefix, toks2)
    assert np.array_equal(full[: 6 + 3], full2[: 6 + 3])
    # the INT8 activations change the logits, but only by quantisation noise
    ref, _ = plain.forward_full(prefix, toks)
    rel = np.linalg.norm(full - ref) / np.linalg.norm(ref)
    assert 0 < rel < 0.05, rel
    with pytest.raises(ValueError):
        O.OracleModel(synth.make_weights(sh, seed=0, std=0.05), "fp16", act_int8=True)


_ORIG_A8 = O.quantize_act_int8_g32
_ORIG_W4A8 = O.matmul_w4a8


def _a8_divisor_128(x):
    return O._symmetric_rtn_g32(x * np.float32(127.0 / 128.0), 127)


def _a8_one_scale_per_row(x):
    x = np.asarray(x, np.float32)
    sa = (np.abs(x).max(axis=1) / np.float32(127)).astype(np.float32)
    safe = np.where(sa == 0, np.float32(1), sa)
    qa = np.clip(np.rint(x / safe[:, None]), -127, 127).astype(np.int8)
    return qa, np.repeat(sa[:, None], x.shape[1] // 32, axis=1)


def _a8_half_away_from_zero(x):
    x = np.asarray(x, np.float32)
    b = x.reshape(x.shape[0], -1, 32)
    sa = (np.abs(b).max(axis=2) / np.float32(127)).astype(np.float32)
    safe = np.where(sa == 0, np.float32(1), sa)
    r = (b / safe[:, :, None]).astype(np.float32)
    qa = (np.sign(r) * np.floor(np.abs(r) + 0.5)).astype(np.int8)
    return qa.reshape(x.shape), sa


def _w4a8_first_block_scale(x, q, s):
    qa, sa = _ORIG_A8(x)
    sa = np.repeat(sa[:, :1], sa.shape[1], axis=1)
    y = np.zeros((qa.shape[0], q.shape[0]))
    for b in range(qa.shape[1] // 32):
        c = slice(32 * b, 32 * b + 32)
        y += (qa[:, c].astype(np.float64) @ q[:, c].astype(np.float64).T) * (sa[:, b, None] * s[None, :, b])
    return y


def _w4a8_weight_transposed_blocks(x, q, s):
    return _ORIG_W4A8(x, q, s[:, ::-1].copy())


@pytest.mark.parametrize("name,attr,fn", [
    ("activation divisor 128", "quantize_act_int8_g32", _a8_divisor_128),
    ("one activation scale per row", "quantize_act_int8_g32", _a8_one_scale_per_row),
    ("round half away from zero", "quantize_act_int8_g32", _a8_half_away_from_zero),
    ("activation scale of the wrong block", "matmul_w4a8", _w4a8_first_block_scale),
    ("weight scales in the wrong order", "matmul_w4a8", _w4a8_weight_transposed_blocks),
])
def test_w4a8_planted_mistakes_are_caught(monkeypatch, name, attr, fn):
    monkeypatch.setattr(O, attr, fn)
    g = _gold("a8_block_hand.json")
    caught = bool(_a8_hand_mismatches(g)) or _w4a8_bruteforce_err(54) > 1e-12
    assert caught, name


# ---------------------------------------------------------------------------
# Half-precision KV cache option (kv_store="fp16"): keys and values rounded to IEEE half,
# to nearest with ties to even, when they enter the cache
# ---------------------------------------------------------------------------

def _f16_rne_bits(x: float) -> int:
    """IEEE binary16 bits of x by the definition: sign, exponent and the 10-bit fraction
    rounded to nearest, ties to the even fraction, subnormals below 2^-14 (no library
    conversion involved)."""
    import fractions
    sign = 0x8000 if math.copysign(1.0, x) < 0 else 0
    a = fractions.Fraction(abs(x))
    if a == 0:
        return sign
    e = math.floor(math.log2(a)) if a >= fractions.Fraction(1, 2 ** 14) else -14
    while a >= 2 ** (e + 1):
        e += 1
    while e > -14 and a < 2 ** e:
        e -= 1
    ulp = fractions.Fraction(2) ** (e - 10)
    m = a / ulp                                  # in [1024, 2048) for normals, [0, 1024) below
    mi = math.floor(m)
    rem = m - mi
    if rem > fractions.Fraction(1, 2) or (rem == fractions.Fraction(1, 2) and mi % 2 == 1):
        mi += 1
    if e > -14 or mi >= 1024:
        if mi == 2048:
            mi, e = 1024, e + 1
        if e > 15:
            return sign | 0x7C00
        return sign | ((e + 15) << 10) | (mi - 1024)
    return sign | mi


def test_f16_reference_rounding_by_hand():
    assert _f16_rne_bits(1.0 + 2.0 ** -11) == 0x3C00          # tie -> even (1.0)
    assert _f16_rne_bits(1.0 + 3 * 2.0 ** -11) == 0x3C02      # tie -> even (1 + 2^-9)
    assert _f16_rne_bits(-2.5) == 0xC100
    assert _f16_rne_bits(2.0 ** -24) == 0x0001                # smallest subnormal
    assert _f16_rne_bits(65504.0) == 0x7BFF


def test_fp16_cache_holds_the_rounded_keys_and_values():
    """Layer 0's cache rows depend only on the inputs, so with kv_store="fp16" they must be
    the round-to-nearest-even halves of the fp32-cache model's rows, element by element."""
    m32 = _tiny_model(L=2, h=2, hk=1)
    draw = synth.make_weights(m32.shape, seed=0, std=0.05, ln_random=True)
    m16 = O.OracleModel(draw, "int4", kv_store="fp16")
    m32 = O.OracleModel(draw, "int4")
    prefix = synth.make_prefix(m32.shape, 1, prefix_len=6, seed=61)[0]
    c32, c16 = m32.new_cache(16), m16.new_cache(16)
    m32.prefill(c32, prefix, [3, 4])
    m16.prefill(c16, prefix, [3, 4])
    for which in ("k", "v"):
        a32 = getattr(c32, which)[0][:8].ravel()
        a16 = getattr(c16, which)[0][:8].ravel()
        want = np.array([_f16_rne_bits(float(x)) for x in a32], np.uint16).view(np.float16).astype(np.float64)
        assert np.array_equal(a16, want), which


def test_fp16_cache_incremental_equals_full_and_stays_close_to_fp32():
    draw = synth.make_weights(synth.tiny_shape(2, 64, 2, 1, 128, 37), seed=0, std=0.05, ln_random=True)
    m16 = O.OracleModel(draw, "int4", kv_store="fp16")
    m32 = O.OracleModel(draw, "int4")
    prefix = synth.make_prefix(m16.shape, 1, prefix_len=5, seed=62)[0]
    toks = [1, 5, 9, 2, 7]
    full = m16.teacher_forced(prefix, toks)
    c = m16.new_cache(16)
    inc = [m16.prefill(c, prefix, toks[:1])] + [m16.decode_step(c, t) for t in toks[1:]]
    assert np.allclose(np.stack(inc), full, rtol=0, atol=1e-12)
    # the stated distance of the half cache from the fp32 one on this model: below 1e-2
    d = np.abs(full - m32.teacher_forced(prefix, toks)).max()
    assert 0 < d < 1e-2


def test_fp16_cache_truncation_mistake_is_caught(monkeypatch):
    """Planted mistake: rounding toward zero instead of to nearest."""
    draw = synth.make_weights(synth.tiny_shape(1, 64, 2, 1, 128, 37), seed=0, std=0.05, ln_random=True)
    m16 = O.OracleModel(draw, "int4", kv_store="fp16")
    m32 = O.OracleModel(draw, "int4")
    prefix = synth.make_prefix(m16.shape, 1, prefix_len=6, seed=63)[0]

    def trunc16(a):
        h = np.asarray(a, np.float64).astype(np.float16)
        back = h.astype(np.float64)
        over = np.abs(back) > np.abs(np.asarray(a, np.float64))
        h = h.view(np.uint16) - over.astype(np.uint16)
        return h.view(np.float16)

    c32, c16 = m32.new_cache(8), m16.new_cache(8)
    m32.prefill(c32, prefix, [3])
    m16.prefill(c16, prefix, [3])
    a32 = c32.k[0][:7].ravel()
    good = np.array([_f16_rne_bits(float(x)) for x in a32], np.uint16).view(np.float16).astype(np.float64)
    bad = trunc16(a32).astype(np.float64)
    assert np.array_equal(c16.k[0][:7].ravel(), good)
    assert not np.array_equal(bad, good)


# ---------------------------------------------------------------------------
# Conditioner front-end ([ONNX-S] muscriptor-small-cond.onnx; [CARD] Model description)
# ---------------------------------------------------------------------------

def test_conditioner_shape_follows_the_pages():
    cond = synth.make_cond_weights(64)
    audio = synth.make_noise_audio(1, seed=171)
    p = O.conditioner(audio, [1], np.array([[1]]), cond, synth.HOP)
    figs = _gold("pages_figures.json")
    assert p.shape == (1, 501 + 1 + 1, 64)                      # 501 frames + dataset + K = 1
    assert p.shape[1] == figs["prefix_rows"]["value"]            # the decoder's 503 prefix rows


def test_stft_magnitude_matches_torch_stft():
    cond = synth.make_cond_weights(8)
    x = synth.make_noise_audio(1, seed=172)[0]
    ours = O.stft_magnitude(x, cond.window, synth.HOP)
    ref = torch.stft(torch.from_numpy(x.astype(np.float64)), synth.N_FFT, synth.HOP,
                     window=torch.from_numpy(cond.window.astype(np.float64)), center=True, pad_mode="reflect",
                     return_complex=True).abs().numpy().T
    assert ours.shape == ref.shape == (501, 1025)
    assert np.allclose(ours, ref, rtol=1e-9, atol=1e-9)


def test_stft_of_a_bin_frequency_tone_closed_form():
    """x = A cos(2 pi k0 n / N): an interior frame's bin k0 holds A/2 sum(w) plus the
    negative-frequency image A/2 sum(w e^{-2 pi i 2 k0 m / N}).  The exact periodic Hann window
    has no DFT weight at bin 2 k0 = 112, so the image comes only from the stored window's
    rounding to half: at most A/2 sum|w - w_exact|."""
    cond = synth.make_cond_weights(8)
    k0, A = 56, 0.5
    n = np.arange(synth.N_SAMPLES)
    x = A * np.cos(2 * np.pi * k0 * n / synth.N_FFT)
    mag = O.stft_magnitude(x, cond.window, synth.HOP)
    w = cond.window.astype(np.float64)
    want = A / 2 * w.sum()
    image = A / 2 * np.abs(w - (0.5 - 0.5 * np.cos(2 * np.pi * np.arange(2048) / 2048))).sum()
    assert 0 < image < 1e-3 * want
    assert np.all(np.abs(mag[20:480, k0] - want) <= image * (1 + 1e-9) + 1e-9)
    assert np.all(mag[20:480].argmax(axis=1) == k0)


def test_stft_parseval_with_a_rectangular_window():
    x = synth.make_noise_audio(1, seed=173, n_samples=4000)[0].astype(np.float64)
    N = 256
    mag = O.stft_magnitude(x, np.ones(N), 64)
    xp = np.pad(x, N // 2, mode="reflect")
    for t in (0, 3, 40, mag.shape[0] - 1):
        fr = xp[t * 64: t * 64 + N]
        e = (mag[t, 0] ** 2 + 2 * (mag[t, 1:-1] ** 2).sum() + mag[t, -1] ** 2) / N
        assert math.isclose(e, (fr ** 2).sum(), rel_tol=1e-10)


def test_log_mel_floor_and_empty_bands():
    cond = synth.make_cond_weights(8)
    empty = np.where(cond.mel_fb.sum(axis=1) == 0)[0]
    assert empty.size > 0                                           # 512 htk bands over 1025 bins
    lm = O.log_mel(np.ones((3, 1025)), cond.mel_fb)
    assert np.all(lm[:, empty] == np.log(1e-6))
    full = np.where(cond.mel_fb.sum(axis=1) > 0)[0]
    assert np.allclose(lm[:, full], np.log(cond.mel_fb[full].astype(np.float64).sum(axis=1)))


def test_mel_filterbank_is_the_htk_triangles():
    """The stored filterbank against the htk definition restated here in float64 (half-ulp
    apart: the checkpoint's buffer is an fp32 computation rounded to half)."""
    cond = synth.make_cond_weights(8)
    freqs = np.linspace(0, 8000, 1025)
    mel = lambda f: 2595 * np.log10(1 + f / 700)
    pts = 700 * (10 ** (np.linspace(0, mel(8000.0), 514) / 2595) - 1)
    fb = np.maximum(0, np.minimum((freqs[None] - pts[:-2, None]) / (pts[1:-1] - pts[:-2])[:, None],
                                  (pts[2:, None] - freqs[None]) / (pts[2:] - pts[1:-1])[:, None]))
    assert np.abs(cond.mel_fb - fb).max() <= 2.0 ** -11 + 1e-6
    hann = 0.5 - 0.5 * np.cos(2 * np.pi * np.arange(2048) / 2048)
    assert np.abs(cond.window - hann).max() <= 2.0 ** -11


def test_conditioner_rows_by_hand_and_the_tone():
    """Rows: projected log-mel frames, the dataset row, the instrument rows (in that order);
    the 440 Hz tone of the W4A32 page's validation puts its energy in the mel band whose
    centre is nearest 440 Hz."""
    cond = synth.make_cond_weights(16)
    tone = synth.make_tone(1)
    p = O.conditioner(tone, [1], np.array([[5, 7]]), cond, synth.HOP)
    assert np.array_equal(p[0, 501], cond.ds_emb[1].astype(np.float64))
    assert np.array_equal(p[0, 502], cond.inst_emb[5].astype(np.float64))
    assert np.array_equal(p[0, 503], cond.inst_emb[7].astype(np.float64))
    lm = O.log_mel(O.stft_magnitude(tone[0], cond.window, synth.HOP), cond.mel_fb)
    rows = lm @ cond.proj_w.astype(np.float64).T + cond.proj_b
    assert np.allclose(p[0, :501], rows, rtol=0, atol=1e-12)
    centres = (np.arange(1025) * 8000 / 1024) @ np.where(cond.mel_fb > 0, cond.mel_fb, 0).T / \
        np.maximum(cond.mel_fb.sum(axis=1), 1e-30)
    band = int(np.argmax(lm[250]))
    assert abs(centres[band] - 440.0) < 20.0


@pytest.mark.parametrize("mistake", ["power", "zero-pad", "log10"])
def test_conditioner_planted_mistakes_are_caught(monkeypatch, mistake):
    cond = synth.make_cond_weights(8)
    x = synth.make_noise_audio(1, seed=174)[0]
    ref = torch.stft(torch.from_numpy(x.astype(np.float64)), synth.N_FFT, synth.HOP,
                     window=torch.from_numpy(cond.window.astype(np.float64)), center=True, pad_mode="reflect",
                     return_complex=True).abs().numpy().T
    orig_stft, orig_log = O.stft_magnitude, O.log_mel
    if mistake == "power":
        monkeypatch.setattr(O, "stft_magnitude", lambda a, w, h: orig_stft(a, w, h) ** 2)
    elif mistake == "zero-pad":
        def zp(a, w, h):
            xp = np.pad(np.asarray(a, np.float64), len(w) // 2)
            idx = np.arange(1 + len(a) // h)[:, None] * h + np.arange(len(w))[None, :]
            return np.abs(np.fft.rfft(xp[idx] * np.asarray(w, np.float64)[None], axis=1))
        monkeypatch.setattr(O, "stft_magnitude", zp)
    else:
        monkeypatch.setattr(O, "log_mel", lambda m, fb: np.log10(np.maximum(m @ np.asarray(fb, np.float64).T, 1e-6)))
    caught = not np.allclose(O.stft_magnitude(x, cond.window, synth.HOP), ref, rtol=1e-9, atol=1e-9)
    lm = O.log_mel(np.ones((2, 1025)), cond.mel_fb)
    empty = np.where(cond.mel_fb.sum(axis=1) == 0)[0]
    caught = caught or not np.all(lm[:, empty] == np.log(1e-6))
    assert caught, mistake


def test_stored_buffers_match_the_pages_figures():
    """The page puts the stored window and filterbank about 2.4e-4 from the textbook ones (the
    half rounding of values in [0.5, 1) moves them by up to 2^-12 = 2.44e-4), and says that with
    them the bins the textbook buffers leave at the log(1e-6) floor sit near -4.  For the
    440 Hz tone (amplitude 0.5; the page's amplitude is not given) those bands land between -7
    and -3, and they are at the floor with the textbook buffers."""
    figs = _gold("pages_figures.json")
    cond = synth.make_cond_weights(8)
    hann = 0.5 - 0.5 * np.cos(2 * np.pi * np.arange(2048) / 2048)
    freqs = np.linspace(0, 8000, 1025)
    mel = lambda f: 2595 * np.log10(1 + f / 700)
    pts = 700 * (10 ** (np.linspace(0, mel(8000.0), 514) / 2595) - 1)
    fb = np.maximum(0, np.minimum((freqs[None] - pts[:-2, None]) / (pts[1:-1] - pts[:-2])[:, None],
                                  (pts[2:, None] - freqs[None]) / (pts[2:] - pts[1:-1])[:, None]))
    dev = figs["cond_buffer_deviation"]["value"]
    assert abs(np.abs(cond.window - hann).max() - dev) < 0.05e-4
    # the filterbank's fresh computation is fp32 arithmetic (up to ~3e-5 from these fp64 triangles)
    assert abs(np.abs(cond.mel_fb - fb).max() - dev) < 0.4e-4
    tone = synth.make_tone(1)[0].astype(np.float64)
    lm_text = O.log_mel(O.stft_magnitude(tone, hann, synth.HOP), fb)[250]
    lm_stored = O.log_mel(O.stft_magnitude(tone, cond.window, synth.HOP), cond.mel_fb)[250]
    floor = np.log(figs["cond_floor_bins_stored"]["floor"])
    at_floor = (lm_text <= floor + 1e-9) & (fb.sum(axis=1) > 0)
    assert at_floor.sum() >= 20
    near = figs["cond_floor_bins_stored"]["value"]
    assert np.all(np.abs(lm_stored[at_floor] - near) <= 3.0)
