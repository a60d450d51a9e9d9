"""The persistent decode kernel's bounded waits, made to run out on purpose.

Every wait of that kernel gives up after a limit: the wait for another CTA's stamped
activation words and the grid barrier between decode steps.  A test-only setter on the cache
shortens the limit to a few hundred polls and injects a wait that nothing will satisfy (an
attention unit waiting for an epoch no phase writes, or a grid barrier one arrival short).  The
kernel must then return on its own, the status word must report MS_ERR_TIMEOUT, and the next
calls must be correct again: on a fresh cache, and on the same cache after a reset.  No fault,
trap or hang is involved: the waits end by their own limits.
"""
import time

import numpy as np
import pytest
import torch

import synth
from oracle import ms_oracle as O

pytestmark = pytest.mark.gpu
ms = pytest.importorskip("decoder_only_transformer_int4_b200")

TOL = 2e-3
MARGIN = 1e-2


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _check_greedy_run(gm, om, prefix, start, steps, cap, cache=None):
    if cache is None:
        cache = ms.Cache(gm, 1, cap)
        cache.set_decode_path(1)
    lg0, am = cache.prefill(_dev(start.reshape(1, 1)), _dev(prefix))
    toks, lg = cache.generate(steps)
    assert cache.device_status() == ms.MS_OK
    gpu = [int(am.item())] + [int(t) for t in toks.cpu().numpy()[:, 0]]
    ref_tok, ref_lg = om.greedy(prefix[0], int(start[0]), steps, capacity=cap)
    assert np.abs(lg0.cpu().numpy()[0] - ref_lg[0]).max() <= TOL
    margins = O.top2_margin(ref_lg)
    for i in range(steps + 1):
        if margins[i] <= MARGIN:
            break
        assert gpu[i] == int(ref_tok[i]), (i, gpu[i], int(ref_tok[i]))
    if margins[:steps + 1].min() > MARGIN:
        assert np.abs(lg.cpu().numpy()[0] - ref_lg[-1]).max() <= TOL
    return cache


@pytest.mark.parametrize("stall", [1, 2])
def test_persistent_wait_runs_out_and_reports_a_timeout(stall):
    """stall 1: the attention units wait for a stamped word that no phase writes; stall 2: the
    grid barrier between steps waits for one CTA more than the grid has."""
    sh = synth.Shape("tiny-timeout", 2, 256, 4, 2, 512, vocab=300)
    draw = synth.make_weights(sh, seed=0, std=0.05, ln_random=True)
    om, gm = O.OracleModel(draw, "int4"), ms.Model.from_draw(draw, "int4")
    prefix = synth.make_prefix(sh, 1, prefix_len=30, seed=131)
    start = synth.make_start_tokens(1, vocab=300, seed=132)
    cap, steps = 64, 6
    cache = ms.Cache(gm, 1, cap)
    cache.set_decode_path(1)
    assert cache.decode_path == 1
    cache.prefill(_dev(start.reshape(1, 1)), _dev(prefix))
    assert cache.device_status() == ms.MS_OK
    cache.set_wait_limits(300, stall)
    t0 = time.perf_counter()
    cache.generate(steps)
    status = cache.device_status()          # synchronises: the launch has returned by itself
    elapsed = time.perf_counter() - t0
    assert status == ms.MS_ERR_TIMEOUT, status
    assert "wait ran out" in ms.last_error()
    assert elapsed < 5.0, elapsed
    assert cache.device_status() == ms.MS_OK   # reading cleared the word
    # a fresh cache decodes correctly
    _check_greedy_run(gm, om, prefix, start, steps, cap)
    # and so does the cache that timed out, once reset with the default limits restored
    cache.set_wait_limits(0, 0)
    cache.reset()
    _check_greedy_run(gm, om, prefix, start, steps, cap, cache=cache)


def test_wait_limit_arguments_are_checked():
    sh = synth.Shape("tiny-timeout2", 1, 256, 4, 4, 512, vocab=50)
    gm = ms.Model.from_draw(synth.make_weights(sh, seed=0), "int4")
    c = ms.Cache(gm, 1, 16)
    with pytest.raises(ms.MsError) as e:
        c.set_wait_limits(-1, 0)
    assert e.value.status == ms.MS_ERR_INVALID_ARG
    with pytest.raises(ms.MsError):
        c.set_wait_limits(100, 3)
    c.set_wait_limits(0, 0)
