"""Host-side checks of the C ABI: the library loads, exports what include/ms.h declares, and
rejects bad arguments before any device work.  No GPU needed."""
import ctypes
import json
import os
import subprocess

import pytest

import synth

ms = pytest.importorskip("decoder_only_transformer_int4_b200")
GOLD = os.path.join(os.path.dirname(__file__), "golden")


def test_library_exports_every_declared_function():
    declared = ms.header_functions()
    assert "ms_prefill" in declared and "ms_decode_step" in declared and "ms_model_create" in declared
    out = subprocess.run(["nm", "-D", "--defined-only", ms.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [f for f in declared if f not in exported]
    assert not missing, missing
    for f in declared:
        assert hasattr(ms._lib, f)


def test_cache_kv_bytes_matches_the_page_figure():
    with open(os.path.join(GOLD, "pages_figures.json")) as f:
        figs = json.load(f)
    cfg = ms.make_config(synth.MEDIUM_MHA)
    nbytes = ms.cache_kv_bytes(cfg, 1, 2504)
    assert round(nbytes / 2 ** 20, 1) == figs["medium_cache_mib_at_2504"]["value"]
    # the medium shape as configured for the benchmark (4 kv heads) is a quarter of that
    assert ms.cache_kv_bytes(ms.make_config(synth.MEDIUM), 1, 2504) * 4 == nbytes
    assert ms.cache_kv_bytes(cfg, 0, 2504) == 0
    assert ms._lib.ms_cache_kv_bytes(None, 1, 2504) == 0


def _weights_stub():
    return ms.Weights()


def test_model_create_rejects_bad_shapes_on_the_host():
    out = ctypes.c_void_p()
    bad = [
        dict(head_dim=32),
        dict(d_model=700),
        dict(n_kv_heads=5),
        dict(d_ff=1000),
        dict(vocab=0),
        dict(n_heads=20, n_kv_heads=2),   # 10 query heads per kv head: unsupported group size
    ]
    for change in bad:
        cfg = ms.make_config(synth.SMALL)
        for k, v in change.items():
            setattr(cfg, k, v)
        st = ms._lib.ms_model_create(ctypes.byref(cfg), ctypes.byref(_weights_stub()), 0, ctypes.byref(out))
        assert st == ms.MS_ERR_SHAPE, (change, ms.last_error())
        assert out.value is None
    cfg = ms.make_config(synth.SMALL)
    st = ms._lib.ms_model_create(ctypes.byref(cfg), ctypes.byref(_weights_stub()), 0, ctypes.byref(out))
    assert st == ms.MS_ERR_INVALID_ARG and "null weight" in ms.last_error()
    assert ms._lib.ms_model_create(None, None, 0, None) == ms.MS_ERR_INVALID_ARG


def test_calls_reject_null_handles_and_bad_sizes_on_the_host():
    L = ms._lib
    assert L.ms_prefill(None, None, None, 1, None, 0, None, None, None) == ms.MS_ERR_INVALID_ARG
    assert L.ms_decode_step(None, None, None, None, None, None) == ms.MS_ERR_INVALID_ARG
    assert L.ms_generate(None, None, 4, None, None, None) == ms.MS_ERR_INVALID_ARG
    assert L.ms_cache_create(None, 1, 16, None) == ms.MS_ERR_INVALID_ARG
    assert L.ms_cache_export(None, None, None) == ms.MS_ERR_INVALID_ARG
    assert L.ms_device_status(None, None) == ms.MS_ERR_INVALID_ARG
    assert L.ms_cache_length(None) == -1
    assert L.ms_quantize_int4_g32(None, 4, 64, None, None, None) == ms.MS_ERR_INVALID_ARG
    p = ctypes.c_void_p(16)
    assert L.ms_quantize_int4_g32(p, 4, 48, p, p, None) == ms.MS_ERR_SHAPE
    assert L.ms_op_matmul_w4(p, 1, 100, p, p, 8, p, None) == ms.MS_ERR_SHAPE
    assert L.ms_op_skip_layernorm(p, None, p, p, 1e-5, 4, 100, p, None) == ms.MS_ERR_SHAPE
    assert L.ms_op_lm_head_argmax(p, 256, 65, 256, None, None, 1e-5, p, 10, p, p, None) == ms.MS_ERR_SHAPE
    assert ms.last_error()


def test_every_handle_call_rejects_null_on_the_host():
    """The documented answer of each call to a NULL handle, before any device work."""
    L = ms._lib
    bad = ms.MS_ERR_INVALID_ARG
    assert L.ms_model_destroy(None) == bad
    assert L.ms_cache_destroy(None) == bad
    assert L.ms_cache_reset(None) == bad
    assert L.ms_cache_set_decode_path(None, 1) == bad
    assert L.ms_cache_import(None, None, None, 0) == bad
    assert L.ms_cache_capacity(None) == -1 and L.ms_cache_batch(None) == -1
    assert L.ms_cache_decode_path(None) == -1
    assert L.ms_model_weight_bytes(None) == 0 and L.ms_cache_kernel_launches(None) == 0
    assert L.ms_cache_kv_bytes(None, 1, 16) == 0
    cfg = ms.make_config(synth.SMALL)
    assert L.ms_cache_kv_bytes(ctypes.byref(cfg), 0, 16) == 0
    assert L.ms_cache_kv_bytes(ctypes.byref(cfg), 1, 0) == 0
    p = ctypes.c_void_p(16)
    assert L.ms_op_matmul_f16(None, 1, 64, p, 8, p, None) == bad
    assert L.ms_op_lm_head_argmax(None, 256, 1, 256, None, None, 1e-5, p, 10, p, p, None) == bad
    # gamma without beta is refused before the scratch is touched
    assert L.ms_op_lm_head_argmax_static(p, 256, 1, 256, p, None, 1e-5, p, 10, p, p, None) == bad
    assert L.ms_op_lm_head_argmax_static(p, 256, 65, 256, None, None, 1e-5, p, 10, p, p, None) == ms.MS_ERR_SHAPE
    assert "ms_op_lm_head_argmax_static" in ms.last_error()


def test_guidance_rejects_null_cache():
    import ctypes
    assert ms._lib.ms_cache_set_guidance(None, ctypes.c_float(2.0)) == ms.MS_ERR_INVALID_ARG
    assert ms._lib.ms_cache_guidance(None) == 0.0


def _cond_cfg(**change):
    c = ms.CondConfig(80000, 2048, 160, 512, 1024, 130, 2, 1)
    for k, v in change.items():
        setattr(c, k, v)
    return c


def test_cond_create_rejects_bad_configs_on_the_host():
    buf = (ctypes.c_float * 16)()
    p = ctypes.cast(buf, ctypes.c_void_p).value
    W = ms.CondWeights(p, p, p, p, p, p)
    out = ctypes.c_void_p()
    bad = [dict(n_fft=2000), dict(n_fft=8), dict(n_fft=8192), dict(hop=0), dict(n_samples=1024),
           dict(n_mels=0), dict(n_mels=5000), dict(d_model=1022), dict(n_instruments=0), dict(n_datasets=0),
           dict(max_batch=0)]
    for change in bad:
        st = ms._lib.ms_cond_create(ctypes.byref(_cond_cfg(**change)), ctypes.byref(W), 0, ctypes.byref(out))
        assert st == ms.MS_ERR_INVALID_ARG, (change, ms.last_error())
        assert out.value is None
    W0 = ms.CondWeights(p, None, p, p, p, p)
    assert ms._lib.ms_cond_create(ctypes.byref(_cond_cfg()), ctypes.byref(W0), 0, ctypes.byref(out)) == \
        ms.MS_ERR_INVALID_ARG
    assert ms._lib.ms_cond_create(None, ctypes.byref(W), 0, ctypes.byref(out)) == ms.MS_ERR_INVALID_ARG
    assert ms._lib.ms_cond_frames(None) == 0
    assert ms._lib.ms_cond_destroy(None) == ms.MS_OK
    assert ms._lib.ms_condition(None, None, 1, None, None, 0, None, None) == ms.MS_ERR_INVALID_ARG
    assert ms._lib.ms_cond_log_mel(None, None, 1, None, None) == ms.MS_ERR_INVALID_ARG
    assert ms._lib.ms_cond_device_status(None, None) == ms.MS_ERR_INVALID_ARG
