"""Parity late in a run, where each attention split holds more than one staged run of keys.

The decode kernels split each (stream, kv head) over several CTAs and stage a split's keys
and values in runs of 64 positions, with an online-softmax rescale between runs.  At the
benchmark lengths (the medium model decoding to 2504 positions, the large one to 2504) a
split holds more than one run only near the end of the cache.  These tests resume decoding
there: a seeded cache state of T positions (``synth.make_kv_cache``) is imported into both
the library (``ms_cache_import``) and the oracle, then the same tokens are decoded on both.

Acceptance as in the other decoder tests: teacher-forced logits within max-abs 2e-3 of the
fp64 oracle at every step; greedy tokens equal wherever the oracle's top-2 margin is above
1e-2 (the comparison stops at the first step below it).

"MuScriptor Medium — optimized W4A32 ONNX Runtime", Quick smoke test: the default cache of
2504 positions; "MuScriptor small — ONNX conversion", muscriptor-small-lm.onnx: the cache
layout past_k / past_v [L, 1, T, Hk, 64] that the import takes.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import ms_oracle as O

pytestmark = pytest.mark.gpu
ms = pytest.importorskip("decoder_only_transformer_int4_b200")

TOL = 2e-3
MARGIN = 1e-2

_MODELS = {}


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _models(sh, fmt, **kw):
    """(oracle, library model) of a shape; only the last one is kept (the large model's
    oracle holds ~10 GB of float64 weights)."""
    key = (sh, fmt, tuple(sorted(kw.items())))
    if key not in _MODELS:
        _MODELS.clear()
        draw = synth.make_weights(sh, **kw)
        _MODELS[key] = (O.OracleModel(draw, fmt), ms.Model.from_draw(draw, fmt))
    return _MODELS[key]


def _host_room(nbytes):
    try:
        import psutil
        return psutil.virtual_memory().available > 3 * nbytes
    except Exception:
        return True


def _greedy_agree(gpu_tokens, ora_tokens, ora_logits):
    margins = O.top2_margin(ora_logits)
    for i, (a, b) in enumerate(zip(gpu_tokens, ora_tokens)):
        if margins[i] <= MARGIN:
            return i
        assert a == b, f"step {i}: gpu {a} oracle {b} (margin {margins[i]:.4f})"
    return len(ora_tokens)


def _late_window(sh, fmt, batch, cap, T, steps, streams, path, greedy=True, seed=4, **kw):
    """Import a seeded T-position cache, teacher-force `steps` seeded tokens through
    ms_decode_step (logits compared at every step), then, from a second import, one forced
    step followed by ms_generate for the rest (tokens compared under the margin rule).
    Returns the teacher-forced logits [steps, B, V]."""
    om, gm = _models(sh, fmt, **kw)
    k, v = synth.make_kv_cache(sh, batch, T, seed=seed)
    forced = synth.make_token_sequence(steps, batch, vocab=sh.vocab, seed=seed + 1)
    cache = ms.Cache(gm, batch, cap)
    cache.set_decode_path(path)
    assert cache.decode_path == path
    cache.import_(k, v)
    assert cache.length == T
    rows = []
    for i in range(steps):
        lg, _ = cache.decode_step(_dev(forced[:, i].astype(np.int32)))
        rows.append(lg.cpu().numpy())
    assert cache.device_status() == ms.MS_OK
    got = np.stack(rows)
    for b in streams:
        oc = om.new_cache(cap)
        oc.load(k[:, b], v[:, b])
        ref = np.stack([om.decode_step(oc, int(t)) for t in forced[b]])
        err = np.abs(got[:, b] - ref).max()
        assert err <= TOL, (sh.name, fmt, T, b, err)
    if greedy:
        cache.close()
        c2 = ms.Cache(gm, batch, cap)
        c2.set_decode_path(path)
        c2.import_(k, v)
        _, am = c2.decode_step(_dev(forced[:, 0].astype(np.int32)))
        toks, _ = c2.generate(steps - 1)
        assert c2.device_status() == ms.MS_OK
        gpu = np.concatenate([am.cpu().numpy()[None], toks.cpu().numpy()], 0)     # [steps, B]
        for b in streams:
            oc = om.new_cache(cap)
            oc.load(k[:, b], v[:, b])
            lgs = [om.decode_step(oc, int(forced[b, 0]))]
            toks_o = [int(O.argmax_lowest(lgs[-1]))]
            for _ in range(steps - 1):
                lgs.append(om.decode_step(oc, toks_o[-1]))
                toks_o.append(int(O.argmax_lowest(lgs[-1])))
            _greedy_agree(list(gpu[:, b]), toks_o, np.stack(lgs))
        assert c2.length == T + steps
    return got


# ---- a small model with a long cache: every split holds 2 to 6 runs of 64 positions --------

LONG = synth.Shape("long-cache", 2, 512, 8, 4, 1024, vocab=300)


@pytest.mark.parametrize("path", [1, 2])
@pytest.mark.parametrize("T", [2400, 4760, 7140, 11900])
def test_long_cache_multi_run_splits(T, path):
    """Batch 1 with 4 kv heads: the persistent kernel splits each kv head over 148 / 4 = 37
    CTAs, so a split holds ceil(T / 37) positions: 65, 129, 193 and 322 positions here, i.e.
    2, 3, 4 and 6 staged runs, with the new position in the last run of the last split."""
    got = _late_window(LONG, "int4", 1, 12000, T, 6, [0], path, greedy=(T == 11900), std=0.05, ln_random=True)
    assert got.shape == (6, 1, LONG.vocab)


def test_long_cache_paths_agree():
    a = _late_window(LONG, "int4", 2, 12000, 11900, 4, [0, 1], 1, greedy=False, std=0.05, ln_random=True)
    b = _late_window(LONG, "int4", 2, 12000, 11900, 4, [], 2, greedy=False, std=0.05, ln_random=True)
    assert np.abs(a - b).max() < 1e-4


# ---- the benchmark workloads, resumed 64 steps before a full cache --------------------------

@pytest.mark.slow
@pytest.mark.parametrize("path", [1, 2])
def test_late_c3_medium(path):
    """The medium model at batch 1 (the benchmark's workload) from T = 2440 to the 2504
    capacity: the persistent kernel's splits hold 66 to 68 positions (two runs)."""
    wl = synth.WORKLOADS["c3"]
    _late_window(wl.shape, "int4", 1, wl.capacity, wl.capacity - 64, 64, [0], path)


@pytest.mark.slow
def test_late_c3pages_medium_mha():
    wl = synth.WORKLOADS["c3pages"]
    _late_window(wl.shape, "int4", 1, wl.capacity, wl.capacity - 64, 64, [0], 1)


@pytest.mark.slow
def test_late_c5_large():
    wl = synth.WORKLOADS["c5"]
    _late_window(wl.shape, "int4", 1, wl.capacity, wl.capacity - 64, 64, [0], 1)


@pytest.mark.slow
def test_late_c5_large_fp16():
    wl = synth.WORKLOADS["c5fp16"]
    _late_window(wl.shape, "fp16", 1, wl.capacity, wl.capacity - 64, 64, [0], 1)


@pytest.mark.slow
def test_late_c5_large_16_streams():
    wl = synth.WORKLOADS["c5b16"]
    T = wl.capacity - 16
    sh = wl.shape
    nbytes = 2 * sh.n_layers * wl.batch * T * sh.n_kv_heads * 64 * 4
    if not _host_room(nbytes):
        pytest.skip("not enough host memory for the 16-stream cache draw")
    _late_window(sh, "int4", wl.batch, wl.capacity, T, 16, [0, 7, 15], 2)


@pytest.mark.slow
def test_late_c4_medium_64_streams():
    wl = synth.WORKLOADS["c4"]
    _late_window(wl.shape, "int4", wl.batch, wl.capacity, wl.capacity - 32, 32, [0, 21, 42, 63], 2)


@pytest.mark.parametrize("dims,kv_format", [
    ((2, 512, 8, 2, 1024), ms.MS_KV_F32),   # 4 query heads per kv head: 32 new rows per tile
    ((2, 768, 12, 4, 1024), ms.MS_KV_F16),  # 3 per kv head (42 rows per tile), half-precision cache
    ((1, 256, 4, 4, 512), ms.MS_KV_F32),    # 1 per kv head: 128 rows per tile
])
def test_prefill_onto_a_long_cache(dims, kv_format):
    """Prefill of 200 token rows onto an imported cache of 2000 positions (two streams): each
    new row attends over 2000+ keys, i.e. 32 and more key tiles of the tensor-core prefill
    attention, with the causal offset of its position and a ragged last tile.  Last-position
    logits within 2e-3 of the oracle given the same cache; the rows the prefill appended
    (post-RoPE k, v) against the oracle's.  With the half cache the imported state is rounded
    to halves on both sides first, and the oracle stores each new key and value as its half."""
    L, d, H, Hk, F = dims
    sh = synth.Shape("late-prefill", L, d, H, Hk, F, vocab=300)
    half = kv_format == ms.MS_KV_F16
    draw = synth.make_weights(sh, seed=0, std=0.05, ln_random=True)
    om = O.OracleModel(draw, "int4", kv_store="fp16" if half else "fp32")
    gm = ms.Model.from_draw(draw, "int4")
    T, S, cap, B = 2000, 200, 2304, 2
    k, v = synth.make_kv_cache(sh, B, T, seed=4)
    if half:
        k, v = k.astype(np.float16).astype(np.float32), v.astype(np.float16).astype(np.float32)
    g = torch.Generator().manual_seed(3)
    toks = torch.randint(0, sh.vocab, (B, S), generator=g, dtype=torch.int64).numpy()
    cache = ms.Cache(gm, B, cap, kv_format=kv_format)
    cache.import_(k, v)
    lg, _ = cache.prefill(_dev(toks), None)
    assert cache.device_status() == ms.MS_OK
    assert cache.length == T + S
    ke, ve = cache.export()
    got = lg.cpu().numpy()
    for b in range(B):
        oc = om.new_cache(cap)
        oc.load(k[:, b], v[:, b])
        ref = om.prefill(oc, None, [int(t) for t in toks[b]])
        assert np.abs(got[b] - ref).max() <= TOL, (dims, b, float(np.abs(got[b] - ref).max()))
        ok_, ov_ = oc.export()
        # appended rows.  fp32: the two sides' rounding.  Halves: layer 0's keys and values agree
        # before rounding up to the prefill GEMM's absolute error (22-bit operands: about
        # 2^-22 sum |x w|, a few 1e-6 here, which matters where cancellation leaves a key near
        # zero), so the two roundings to half differ by one half ulp plus that; deeper layers'
        # inputs already carry the previous layers' half-cache rounding differences (attention
        # over 2000 + 200 rounded keys: a few 1e-4 on a layer-1 key), bounded by half the
        # decoder's 2e-3 logits bar.  A wrong position, head or rotation moves values by O(1).
        for name, got_kv, ref_kv in (("k", ke[:, b, T:], ok_[:, 0, T:]), ("v", ve[:, b, T:], ov_[:, 0, T:])):
            mag = np.maximum(np.abs(got_kv), np.abs(ref_kv))
            for l in range(L):
                if half:
                    bound = 2.0 ** -10 * mag[l] + 1e-5 if l == 0 else 2.0 ** -8 * mag[l] + 1e-3
                else:
                    bound = 1e-5 * mag[l] + 1e-4
                err = np.abs(got_kv[l] - ref_kv[l])
                w = np.unravel_index(np.argmax(err - bound), err.shape)
                assert np.all(err <= bound), (dims, b, name, l, w, float(got_kv[l][w]), float(ref_kv[l][w]),
                                              float(bound[w]), int((err > bound).sum()))
