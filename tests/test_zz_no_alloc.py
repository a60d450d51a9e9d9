"""The allocation-free LM head + argmax entry point (ms_op_lm_head_argmax_static).

Some callers cannot allocate device memory at the point where they need the LM head:
code running while a stream is captured into a CUDA graph, code whose device memory
belongs to another allocator, latency-critical loops where an allocation could
synchronise the device.  This entry point serves them from a fixed scratch array inside
the library.  The test calls it through the C ABI three times in a row and compares each result
with the allocating entry point's on the same inputs, within the fp32 dot-product bound the
kernel tests use.  The array keeps the previous call's contents: the second call has a
smaller vocabulary, so it launches fewer CTAs than the first and the first call's extra
per-CTA slots stay behind in the array (the result must not pick them up); a third call
follows a call the library rejected, on the same stream.  It lives in its own file,
collected last, and works both alone in a fresh process and after the other tests.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import ms_oracle as O

pytestmark = pytest.mark.gpu
ms = pytest.importorskip("decoder_only_transformer_int4_b200")

U32 = 2.0 ** -24


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _rejected_call():
    x = torch.zeros((65, 256), dtype=torch.float32, device="cuda")
    W = torch.zeros((50, 256), dtype=torch.float32, device="cuda")
    st = ms._lib.ms_op_lm_head_argmax_static(ms._ptr(x), 256, 65, 256, None, None, 1e-5, ms._ptr(W), 50, None, None,
                                             ms._stream())
    assert st == ms.MS_ERR_SHAPE


def test_static_lm_head_matches_the_allocating_entry_point_on_calls_in_a_row():
    d = 1024
    W_all = synth.make_matrix(1393, d, seed=1801)
    g = 1 + 0.1 * synth.make_activations(1, d, seed=1802)[0]
    b = 0.1 * synth.make_activations(1, d, seed=1803)[0]
    gd, bd = _dev(g), _dev(b)
    # the vocabulary shrinks from call to call (fewer CTAs, stale slots left behind); the
    # third call comes right after a rejected call
    for call, (M, V) in enumerate(((3, 1393), (8, 300), (5, 97))):
        if call == 2:
            _rejected_call()
        W = W_all[:V]
        Wd = _dev(W)
        x = synth.make_activations(M, d, seed=1810 + call)
        xd = _dev(x)
        ref_lg, ref_am = ms.lm_head_argmax(xd, Wd, gd, bd, 1e-5)
        logits = torch.full((M, V), float("nan"), dtype=torch.float32, device="cuda")
        am = torch.full((M,), -1, dtype=torch.int32, device="cuda")
        st = ms._lib.ms_op_lm_head_argmax_static(ms._ptr(xd), d, M, d, ms._ptr(gd), ms._ptr(bd), 1e-5, ms._ptr(Wd), V,
                                                 ms._ptr(logits), ms._ptr(am), ms._stream())
        assert st == ms.MS_OK, ms.last_error()
        lg = logits.cpu().numpy().astype(np.float64)
        ref = ref_lg.cpu().numpy().astype(np.float64)
        h = O.layer_norm(x, g, b, 1e-5)
        tol = d * U32 * (np.abs(h) @ np.abs(W).astype(np.float64).T) + 1e-5 * np.abs(W).astype(np.float64).sum(1)
        assert np.all(np.abs(lg - ref) <= tol)
        assert np.array_equal(am.cpu().numpy(), ref_am.cpu().numpy())
        assert np.array_equal(am.cpu().numpy(), np.argmax(lg, axis=1))


def test_static_lm_head_rejects_sizes_beyond_its_scratch():
    d, V = 256, 50
    x = torch.zeros((65, d), dtype=torch.float32, device="cuda")
    W = torch.zeros((V, d), dtype=torch.float32, device="cuda")
    out = torch.empty((65, V), dtype=torch.float32, device="cuda")
    am = torch.empty((65,), dtype=torch.int32, device="cuda")
    st = ms._lib.ms_op_lm_head_argmax_static(ms._ptr(x), d, 65, d, None, None, 1e-5, ms._ptr(W), V, ms._ptr(out),
                                             ms._ptr(am), ms._stream())
    assert st == ms.MS_ERR_SHAPE and "M must be in [1, 64]" in ms.last_error()
