"""One stamped hand-off between CTAs, measured in isolation (the unit the persistent decode
kernel's phase boundaries are made of; see tests/probes/handoff_probe.cu).  The probe is built
with nvcc for sm_100a into a temporary directory and run once per mode; the numbers are printed
(run with -s) and checked only for being measured."""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

SRC = os.path.join(os.path.dirname(__file__), "probes", "handoff_probe.cu")


def _nvcc():
    return shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"


@pytest.fixture(scope="module")
def probe(tmp_path_factory):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    so = str(tmp_path_factory.mktemp("probe") / "libhandoff.so")
    subprocess.run([_nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-shared", "-Xcompiler", "-fPIC",
                    "-o", so, SRC], check=True)
    lib = ctypes.CDLL(so)
    lib.handoff_probe.restype = ctypes.c_int
    lib.handoff_probe.argtypes = [ctypes.c_int] * 4 + [ctypes.c_void_p, ctypes.c_void_p]
    return lib


def _run(lib, mode, ctas, rounds, width):
    out = np.zeros(ctas, np.float64)
    sm = np.zeros(ctas, np.int32)
    rc = lib.handoff_probe(mode, ctas, rounds, width, out.ctypes.data, sm.ctypes.data)
    assert rc == 0, rc
    return out, sm


def test_ping_pong_round_trip(probe):
    out, sm = _run(probe, 0, 148, 200, 1)
    rt = out[1:]
    assert np.all(rt > 0)
    print(f"\nstamped ping-pong, CTA 0 (SM {sm[0]}) with each of 147 CTAs, 200 round trips each: "
          f"round trip min {rt.min():.0f} ns, median {np.median(rt):.0f} ns, max {rt.max():.0f} ns")
    assert np.median(rt) < 50_000


@pytest.mark.parametrize("mode", [1, 2])
@pytest.mark.parametrize("width", [8, 28])
def test_all_to_all_handoff(probe, mode, width):
    """148 CTAs publish `width` words each and every CTA reads all of them per round: 9.2 KiB
    (width 8: a 1024-long vector's stamped words, as the LN1 and LN2 inputs) or 32 KiB (the
    largest per-CTA read of the decode kernel, four K-split slices).  Mode 1 is the whole
    hand-off (publish, then wait for every CTA's words); mode 2 the reads alone."""
    out, _ = _run(probe, mode, 148, 200, width)
    assert np.all(out > 0)
    what = "hand-off" if mode == 1 else "read of published words"
    print(f"\nall-to-all stamped {what}, 148 CTAs x {width} words ({148 * width * 8 / 1024:.1f} KiB read by "
          f"every CTA): {out.max():.0f} ns per round (max over CTAs), median {np.median(out):.0f} ns")
    assert out.max() < 200_000
