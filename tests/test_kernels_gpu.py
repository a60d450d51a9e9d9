"""Kernel-level parity: each single-operation entry point of the C ABI against the oracle.

Integer and byte work (INT4 codes, packing, scales, argmax decisions) must match bit for
bit.  Floating-point results are held to the fp32 rounding bound of a K-term dot product,
|err| <= K * 2^-24 * sum_k |x_k w_k|, which any correct fp32 summation order meets.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import ms_oracle as O

pytestmark = pytest.mark.gpu
ms = pytest.importorskip("decoder_only_transformer_int4_b200")

U32 = 2.0 ** -24
SHAPES = sorted({nk for sh in (synth.SMALL, synth.MEDIUM, synth.LARGE) for nk in sh.matmul_shapes()})


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _dot_bound(x, W):
    K = x.shape[1]
    return K * U32 * (np.abs(x.astype(np.float64)) @ np.abs(W.astype(np.float64)).T) + 1e-30


@pytest.mark.parametrize("N,K", SHAPES)
def test_quantizer_bit_exact(N, K):
    w = synth.make_matrix(N, K, seed=100 + N + K)
    q, s = O.quantize_int4_g32(w)
    pg, sg = ms.quantize_int4_g32(_dev(w))
    assert np.array_equal(pg.cpu().numpy(), O.pack_int4(q))
    assert np.array_equal(sg.cpu().numpy().view(np.uint32), s.view(np.uint32))


def test_quantizer_edge_groups():
    w = np.zeros((4, 128), np.float32)
    w[0, :8] = [7.0, 3.5, 2.5, -0.5, 1.49, -6.51, 0.0, -7.0]     # ties to even, exact scale 1
    w[1, 32:64] = np.float32(1e-30) * np.arange(32)                # subnormal-scale group
    w[2, 64:96] = -0.0                                             # negative zeros
    w[3, :] = np.float32(3.0e38) * np.sign(np.sin(np.arange(128)))  # near the fp32 maximum
    q, s = O.quantize_int4_g32(w)
    pg, sg = ms.quantize_int4_g32(_dev(w))
    assert np.array_equal(pg.cpu().numpy(), O.pack_int4(q))
    assert np.array_equal(sg.cpu().numpy().view(np.uint32), s.view(np.uint32))
    assert list(pg.cpu().numpy()[0, :4]) == [207, 138, 25, 24]


@pytest.mark.parametrize("M", [1, 2, 4, 8, 3, 16, 64, 130, 504])
@pytest.mark.parametrize("N,K", [(2304, 768), (768, 3072), (1536, 1024), (1024, 4096), (1536, 6144), (200, 512)])
def test_matmul_w4(M, N, K):
    w = synth.make_matrix(N, K, seed=200 + K)
    x = synth.make_activations(M, K, seed=300 + M)
    pg, sg = ms.quantize_int4_g32(_dev(w))
    q, s = O.quantize_int4_g32(w)
    W = O.dequantize(q, s)
    y = ms.matmul_w4(_dev(x), pg, sg).cpu().numpy().astype(np.float64)
    ref = x.astype(np.float64) @ W.astype(np.float64).T
    assert np.all(np.abs(y - ref) <= _dot_bound(x, W))


@pytest.mark.parametrize("M", [1, 8, 40])
@pytest.mark.parametrize("N,K", [(2560, 1536), (6144, 1536), (1536, 6144)])
def test_matmul_f16(M, N, K):
    w = synth.make_matrix(N, K, seed=400 + K).astype(np.float16)
    x = synth.make_activations(M, K, seed=500 + M)
    y = ms.matmul_f16(_dev(x), _dev(w.view(np.int16))).cpu().numpy().astype(np.float64)
    ref = x.astype(np.float64) @ w.astype(np.float64).T
    assert np.all(np.abs(y - ref) <= _dot_bound(x, w.astype(np.float32)))


def test_matmul_all_config_shapes_gemv():
    for (N, K) in SHAPES:
        w = synth.make_matrix(N, K, seed=600 + N)
        x = synth.make_activations(1, K, seed=601)
        pg, sg = ms.quantize_int4_g32(_dev(w))
        q, s = O.quantize_int4_g32(w)
        W = O.dequantize(q, s)
        y = ms.matmul_w4(_dev(x), pg, sg).cpu().numpy().astype(np.float64)
        ref = x.astype(np.float64) @ W.astype(np.float64).T
        assert np.all(np.abs(y - ref) <= _dot_bound(x, W)), (N, K)


@pytest.mark.parametrize("d", [768, 1024, 1536])
@pytest.mark.parametrize("with_y", [True, False])
def test_skip_layernorm(d, with_y):
    R = 37
    x = synth.make_activations(R, d, seed=700) * 3 + 0.5
    y = synth.make_activations(R, d, seed=701)
    g = 1 + 0.1 * synth.make_activations(1, d, seed=702)[0]
    b = 0.1 * synth.make_activations(1, d, seed=703)[0]
    xd = _dev(x)
    h = ms.skip_layernorm(xd, _dev(y) if with_y else None, _dev(g), _dev(b), 1e-5).cpu().numpy()
    s = (x + y).astype(np.float32) if with_y else x
    assert np.array_equal(xd.cpu().numpy(), s)            # fp32 add, bit-exact
    ref = O.layer_norm(s, g, b, 1e-5)
    assert np.max(np.abs(h - ref)) < 2e-5


@pytest.mark.parametrize("M", [1, 2, 3, 8, 13, 64])
@pytest.mark.parametrize("with_ln", [True, False])
def test_lm_head_argmax(M, with_ln):
    d, V = 1024, 1393
    x = synth.make_activations(M, d, seed=800 + M)
    W = synth.make_matrix(V, d, seed=801)
    g = 1 + 0.1 * synth.make_activations(1, d, seed=802)[0]
    b = 0.1 * synth.make_activations(1, d, seed=803)[0]
    if with_ln:
        lg, am = ms.lm_head_argmax(_dev(x), _dev(W), _dev(g), _dev(b), 1e-5)
        h = O.layer_norm(x, g, b, 1e-5)
    else:
        lg, am = ms.lm_head_argmax(_dev(x), _dev(W))
        h = x.astype(np.float64)
    lg = lg.cpu().numpy().astype(np.float64)
    am = am.cpu().numpy()
    ref = h @ W.astype(np.float64).T
    tol = _dot_bound(h, W) + (1e-5 * np.abs(W).astype(np.float64).sum(1)[None, :] if with_ln else 0)
    assert np.all(np.abs(lg - ref) <= tol)
    # the kernel's argmax is the lowest index of the maximum of its own logits
    assert np.array_equal(am, np.argmax(lg, axis=1))
    # and the oracle's wherever the top-2 margin exceeds the logit tolerance
    margin = O.top2_margin(ref)
    sure = margin > 2 * tol.max()
    assert np.array_equal(am[sure], O.argmax_lowest(ref)[sure])


def test_lm_head_argmax_ties_pick_the_lowest_index_across_ctas():
    d, V = 256, 1393
    W = synth.make_matrix(V, d, seed=900)
    x = np.abs(synth.make_activations(2, d, seed=901))
    top = np.full(d, 0.5, np.float32)
    for v in (1300, 700, 5):           # identical rows in different CTAs, same logit
        W[v] = top
    lg, am = ms.lm_head_argmax(_dev(x), _dev(W))
    lg = lg.cpu().numpy()
    assert lg[0, 5] == lg[0, 700] == lg[0, 1300]
    assert list(am.cpu().numpy()) == [5, 5]


# ---- the tcgen05 GEMM's operand planes and the model's own MatMuls ---------------------------

def test_split_f16_planes_bit_exact():
    """hi = fp16(x), lo = fp16(x - hi) with round-to-nearest-even, over magnitudes from
    subnormal halves to near the half maximum, signed zeros and a ragged row stride."""
    rng = np.random.default_rng(5)
    M, K = 37, 520
    x = (rng.standard_normal((M, K)) * np.exp2(rng.integers(-30, 15, (M, K)))).astype(np.float32)
    x[0, :4] = [0.0, -0.0, 65000.0, -6.0e-8]
    hi, lo = ms.split_f16(_dev(x))
    want_hi = x.astype(np.float16)
    want_lo = (x - want_hi.astype(np.float32)).astype(np.float16)
    assert np.array_equal(hi.cpu().numpy().view(np.uint16), want_hi.view(np.uint16))
    assert np.array_equal(lo.cpu().numpy().view(np.uint16), want_lo.view(np.uint16))


@pytest.mark.parametrize("fmt", ["int4", "fp16"])
@pytest.mark.parametrize("M", [1, 3, 64, 200, 504])
def test_model_matmul_against_the_oracle_weights(fmt, M):
    """ms_model_matmul (the GEMM prefill and batched decode run, on the model's tile-packed
    weights) against the oracle's dequantised matrices, on split activation planes, every
    matrix of a 2-layer shape; M from one row to several 256-row tiles with a ragged tail.
    (Ragged N is covered through ms_op_matmul_w4 with N = 200.)"""
    sh = synth.Shape("gemm", 2, 768, 12, 4, 1280, vocab=64)
    draw = synth.make_weights(sh, seed=7, std=0.05)
    om = O.OracleModel(draw, fmt)
    gm = ms.Model.from_draw(draw, fmt)
    for l in range(sh.n_layers):
        for i, (N, K) in enumerate(sh.matmul_shapes()):
            x = synth.make_activations(M, K, seed=900 + 10 * l + i)
            hi, lo = ms.split_f16(_dev(x))
            xs = hi.cpu().numpy().astype(np.float64) + lo.cpu().numpy().astype(np.float64)
            assert np.all(np.abs(xs - x) <= 2.0 ** -22 * np.abs(x) + 2.0 ** -25)
            y = gm.matmul(l, i, hi, lo).cpu().numpy().astype(np.float64)
            W = om.layers[l].w[i]
            ref = xs @ W.T
            assert np.all(np.abs(y - ref) <= _dot_bound(x, W.astype(np.float32))), (l, i)
