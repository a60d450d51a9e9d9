"""Python binding of libms_b200.so, the MuScriptor KV-cached INT4 decoder step on B200.

Argument marshalling only: every step of the decoder runs in the library's CUDA kernels.
PyTorch is used for device memory and streams (tensors are passed by data_ptr(), the
stream is torch's current stream).  Importing this module loads the compiled library
and raises ImportError if it has not been built (python
decoder_only_transformer_int4_b200/build.py); there is no other implementation to fall
back to.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libms_b200.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "ms.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python decoder_only_transformer_int4_b200/build.py`")
_lib = ctypes.CDLL(LIB_PATH)

MS_OK, MS_ERR_INVALID_ARG, MS_ERR_SHAPE, MS_ERR_CACHE_FULL, MS_ERR_TOKEN_RANGE = 0, 1, 2, 3, 4
MS_ERR_OOM, MS_ERR_CUDA, MS_ERR_TIMEOUT, MS_ERR_UNSUPPORTED = 5, 6, 7, 8
STATUS_NAMES = {0: "MS_OK", 1: "MS_ERR_INVALID_ARG", 2: "MS_ERR_SHAPE", 3: "MS_ERR_CACHE_FULL",
                4: "MS_ERR_TOKEN_RANGE", 5: "MS_ERR_OOM", 6: "MS_ERR_CUDA", 7: "MS_ERR_TIMEOUT",
                8: "MS_ERR_UNSUPPORTED"}
MS_W_INT4_G32, MS_W_FP16 = 0, 1
MS_KV_F32, MS_KV_F16 = 0, 1


class MsError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class Config(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int), ("d_model", ctypes.c_int), ("n_heads", ctypes.c_int),
                ("n_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("d_ff", ctypes.c_int),
                ("vocab", ctypes.c_int), ("rope_base", ctypes.c_float), ("ln_eps", ctypes.c_float),
                ("weight_format", ctypes.c_int)]


class LayerWeights(ctypes.Structure):
    _fields_ = [("ln1_g", ctypes.c_void_p), ("ln1_b", ctypes.c_void_p), ("ln2_g", ctypes.c_void_p),
                ("ln2_b", ctypes.c_void_p), ("w", ctypes.c_void_p * 4), ("s", ctypes.c_void_p * 4),
                ("w16", ctypes.c_void_p * 4)]


class Weights(ctypes.Structure):
    _fields_ = [("tok_emb", ctypes.c_void_p), ("lm_head", ctypes.c_void_p), ("ln_f_g", ctypes.c_void_p),
                ("ln_f_b", ctypes.c_void_p), ("layers", ctypes.POINTER(LayerWeights))]


class CondConfig(ctypes.Structure):
    _fields_ = [("n_samples", ctypes.c_int), ("n_fft", ctypes.c_int), ("hop", ctypes.c_int),
                ("n_mels", ctypes.c_int), ("d_model", ctypes.c_int), ("n_instruments", ctypes.c_int),
                ("n_datasets", ctypes.c_int), ("max_batch", ctypes.c_int)]


class CondWeights(ctypes.Structure):
    _fields_ = [("window", ctypes.c_void_p), ("mel_fb", ctypes.c_void_p), ("proj_w", ctypes.c_void_p),
                ("proj_b", ctypes.c_void_p), ("inst_emb", ctypes.c_void_p), ("ds_emb", ctypes.c_void_p)]


_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_PROTOS = {
    "ms_last_error": (ctypes.c_char_p, []),
    "ms_quantize_int4_g32": (_I, [_P, _I, _I, _P, _P, _P]),
    "ms_model_create": (_I, [ctypes.POINTER(Config), ctypes.POINTER(Weights), _I, ctypes.POINTER(_P)]),
    "ms_model_destroy": (_I, [_P]),
    "ms_model_weight_bytes": (ctypes.c_size_t, [_P]),
    "ms_cache_create": (_I, [_P, _I, _I, ctypes.POINTER(_P)]),
    "ms_cache_create_ex": (_I, [_P, _I, _I, _I, ctypes.POINTER(_P)]),
    "ms_cache_kv_format": (_I, [_P]),
    "ms_cache_kv_bytes_ex": (ctypes.c_size_t, [ctypes.POINTER(Config), _I, _I, _I]),
    "ms_cache_reset": (_I, [_P]),
    "ms_cache_length": (_I, [_P]),
    "ms_cache_capacity": (_I, [_P]),
    "ms_cache_batch": (_I, [_P]),
    "ms_cache_kernel_launches": (ctypes.c_uint64, [_P]),
    "ms_cache_set_decode_path": (_I, [_P, _I]),
    "ms_cache_decode_path": (_I, [_P]),
    "ms_cache_set_guidance": (_I, [_P, ctypes.c_float]),
    "ms_cache_guidance": (ctypes.c_float, [_P]),
    "ms_cache_set_wait_limits": (_I, [_P, ctypes.c_longlong, _I]),
    "ms_cache_set_act_int8": (_I, [_P, _I]),
    "ms_cache_act_int8": (_I, [_P]),
    "ms_op_quantize_act_int8": (_I, [_P, _I, _I, _I, _P, _P, _P]),
    "ms_op_matmul_w4a8": (_I, [_P, _P, _I, _I, _P, _P, _I, _P, _P]),
    "ms_cache_destroy": (_I, [_P]),
    "ms_cache_kv_bytes": (ctypes.c_size_t, [ctypes.POINTER(Config), _I, _I]),
    "ms_prefill": (_I, [_P, _P, _P, _I, _P, _I, _P, _P, _P]),
    "ms_decode_step": (_I, [_P, _P, _P, _P, _P, _P]),
    "ms_generate": (_I, [_P, _P, _I, _P, _P, _P]),
    "ms_cache_export": (_I, [_P, _P, _P]),
    "ms_cache_import": (_I, [_P, _P, _P, _I]),
    "ms_device_status": (_I, [_P, _P]),
    "ms_op_matmul_w4": (_I, [_P, _I, _I, _P, _P, _I, _P, _P]),
    "ms_op_matmul_f16": (_I, [_P, _I, _I, _P, _I, _P, _P]),
    "ms_op_skip_layernorm": (_I, [_P, _P, _P, _P, _F, _I, _I, _P, _P]),
    "ms_op_split_f16": (_I, [_P, _I, _I, _I, _P, _P, _I, _P]),
    "ms_model_matmul": (_I, [_P, _I, _I, _P, _P, _I, _I, _P, _I, _P]),
    "ms_op_lm_head_argmax": (_I, [_P, _I, _I, _I, _P, _P, _F, _P, _I, _P, _P, _P]),
    "ms_op_lm_head_argmax_static": (_I, [_P, _I, _I, _I, _P, _P, _F, _P, _I, _P, _P, _P]),
    "ms_cond_create": (_I, [ctypes.POINTER(CondConfig), ctypes.POINTER(CondWeights), _I, ctypes.POINTER(_P)]),
    "ms_cond_destroy": (_I, [_P]),
    "ms_cond_frames": (_I, [_P]),
    "ms_condition": (_I, [_P, _P, _I, _P, _P, _I, _P, _P]),
    "ms_cond_log_mel": (_I, [_P, _P, _I, _P, _P]),
    "ms_cond_device_status": (_I, [_P, _P]),
}
for _name, (_res, _args) in _PROTOS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


def header_functions() -> List[str]:
    """Names of the functions include/ms.h declares."""
    with open(HEADER_PATH) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ms_[a-z0-9_]+)\s*\(", text)))


def last_error() -> str:
    return (_lib.ms_last_error() or b"").decode()


def _check(status: int, what: str):
    if status != MS_OK:
        raise MsError(status, f"{what}: {last_error()}")


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def make_config(shape, weight_format: int = MS_W_INT4_G32) -> Config:
    return Config(shape.n_layers, shape.d_model, shape.n_heads, shape.n_kv_heads, shape.head_dim, shape.d_ff,
                  shape.vocab, shape.rope_base, shape.ln_eps, weight_format)


def cache_kv_bytes(cfg: Config, batch: int, capacity: int, kv_format: int = MS_KV_F32) -> int:
    return int(_lib.ms_cache_kv_bytes_ex(ctypes.byref(cfg), batch, capacity, kv_format))


# ---- single operations --------------------------------------------------------------

def quantize_int4_g32(w: torch.Tensor) -> Tuple[torch.Tensor, torch.Tensor]:
    """RTN INT4 g32 of an fp32 [N, K] CUDA tensor -> (packed uint8 [N, K/2], scales fp32 [N, K/32])."""
    n, k = w.shape
    packed = torch.empty((n, k // 2), dtype=torch.uint8, device=w.device)
    scales = torch.empty((n, k // 32), dtype=torch.float32, device=w.device)
    _check(_lib.ms_quantize_int4_g32(_ptr(w), n, k, _ptr(packed), _ptr(scales), _stream()), "ms_quantize_int4_g32")
    return packed, scales


def matmul_w4(x: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor,
              out: Optional[torch.Tensor] = None) -> torch.Tensor:
    m, k = x.shape
    n = packed.shape[0]
    y = torch.empty((m, n), dtype=torch.float32, device=x.device) if out is None else out
    _check(_lib.ms_op_matmul_w4(_ptr(x), m, k, _ptr(packed), _ptr(scales), n, _ptr(y), _stream()), "ms_op_matmul_w4")
    return y


def matmul_f16(x: torch.Tensor, w16: torch.Tensor) -> torch.Tensor:
    m, k = x.shape
    n = w16.shape[0]
    y = torch.empty((m, n), dtype=torch.float32, device=x.device)
    _check(_lib.ms_op_matmul_f16(_ptr(x), m, k, _ptr(w16), n, _ptr(y), _stream()), "ms_op_matmul_f16")
    return y


def split_f16(x: torch.Tensor) -> Tuple[torch.Tensor, torch.Tensor]:
    """fp32 [M, K] -> (hi, lo) fp16 [M, K] with hi + lo carrying x to a 22-bit significand
    (the tcgen05 GEMM's operand form)."""
    m, k = x.shape
    hi = torch.empty((m, k), dtype=torch.float16, device=x.device)
    lo = torch.empty((m, k), dtype=torch.float16, device=x.device)
    _check(_lib.ms_op_split_f16(_ptr(x), k, m, k, _ptr(hi), _ptr(lo), k, _stream()), "ms_op_split_f16")
    return hi, lo


def quantize_act_int8(x: torch.Tensor) -> Tuple[torch.Tensor, torch.Tensor]:
    """fp32 [M, K] -> (codes int8 [M, K], scales fp32 [M, K/32]) (ms_op_quantize_act_int8)."""
    m, k = x.shape
    q = torch.empty((m, k), dtype=torch.int8, device=x.device)
    s = torch.empty((m, k // 32), dtype=torch.float32, device=x.device)
    _check(_lib.ms_op_quantize_act_int8(_ptr(x), k, m, k, _ptr(q), _ptr(s), _stream()), "ms_op_quantize_act_int8")
    return q, s


def matmul_w4a8(qa: torch.Tensor, sa: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor) -> torch.Tensor:
    m, k = qa.shape
    n = packed.shape[0]
    y = torch.empty((m, n), dtype=torch.float32, device=qa.device)
    _check(_lib.ms_op_matmul_w4a8(_ptr(qa), _ptr(sa), m, k, _ptr(packed), _ptr(scales), n, _ptr(y), _stream()),
           "ms_op_matmul_w4a8")
    return y


def skip_layernorm(x: torch.Tensor, y: Optional[torch.Tensor], gamma: torch.Tensor, beta: torch.Tensor,
                   eps: float = 1e-5) -> torch.Tensor:
    """x <- x + y in place (y may be None), returns LN(x) * gamma + beta."""
    r, d = x.shape
    h = torch.empty_like(x)
    _check(_lib.ms_op_skip_layernorm(_ptr(x), _ptr(y), _ptr(gamma), _ptr(beta), eps, r, d, _ptr(h), _stream()),
           "ms_op_skip_layernorm")
    return h


def lm_head_argmax(x: torch.Tensor, W: torch.Tensor, gamma: Optional[torch.Tensor] = None,
                   beta: Optional[torch.Tensor] = None, eps: float = 1e-5):
    m, d = x.shape
    v = W.shape[0]
    logits = torch.empty((m, v), dtype=torch.float32, device=x.device)
    am = torch.empty((m,), dtype=torch.int32, device=x.device)
    _check(_lib.ms_op_lm_head_argmax(_ptr(x), d, m, d, _ptr(gamma), _ptr(beta), eps, _ptr(W), v, _ptr(logits),
                                     _ptr(am), _stream()), "ms_op_lm_head_argmax")
    return logits, am


def lm_head_argmax_static(x: torch.Tensor, W: torch.Tensor, gamma: Optional[torch.Tensor] = None,
                          beta: Optional[torch.Tensor] = None, eps: float = 1e-5, logits: Optional[torch.Tensor] = None,
                          argmax: Optional[torch.Tensor] = None):
    """ms_op_lm_head_argmax_static: the LM head + argmax without any device allocation by
    the library (its scratch is a fixed array inside the library).  Output tensors may be
    passed in so that the call allocates nothing on the Python side either."""
    m, d = x.shape
    v = W.shape[0]
    if logits is None:
        logits = torch.empty((m, v), dtype=torch.float32, device=x.device)
    if argmax is None:
        argmax = torch.empty((m,), dtype=torch.int32, device=x.device)
    _check(_lib.ms_op_lm_head_argmax_static(_ptr(x), d, m, d, _ptr(gamma), _ptr(beta), eps, _ptr(W), v,
                                            _ptr(logits), _ptr(argmax), _stream()), "ms_op_lm_head_argmax_static")
    return logits, argmax


# ---- model and cache -------------------------------------------------------------------

class Model:
    """Device copy of a decoder's weights (ms_model_create)."""

    def __init__(self, cfg: Config, weights: Weights, device: int = 0, _keep=None):
        self.cfg = cfg
        self.device = device
        h = ctypes.c_void_p()
        _check(_lib.ms_model_create(ctypes.byref(cfg), ctypes.byref(weights), device, ctypes.byref(h)),
               "ms_model_create")
        self._h = h
        del _keep

    @classmethod
    def from_draw(cls, draw, weight_format: str = "int4", device: int = 0) -> "Model":
        """Build from fp32 host draws (synth.WeightDraw).  INT4 weights are quantised by the
        library's own kernel; fp16 weights are the draws rounded to IEEE half on the host."""
        sh = draw.shape
        fmt = MS_W_INT4_G32 if weight_format == "int4" else MS_W_FP16
        cfg = make_config(sh, fmt)
        dev = torch.device("cuda", device)
        keep = []

        def up(a, dtype=torch.float32):
            t = torch.from_numpy(np.ascontiguousarray(a)).to(dev, dtype=dtype)
            keep.append(t)
            return t.data_ptr()

        layers = (LayerWeights * max(1, sh.n_layers))()
        for l, ld in enumerate(draw.layers):
            L = layers[l]
            L.ln1_g, L.ln1_b, L.ln2_g, L.ln2_b = up(ld.ln1_g), up(ld.ln1_b), up(ld.ln2_g), up(ld.ln2_b)
            for i, w in enumerate(ld.w):
                if fmt == MS_W_INT4_G32:
                    wd = torch.from_numpy(np.ascontiguousarray(w)).to(dev)
                    p, s = quantize_int4_g32(wd)
                    keep += [p, s]
                    L.w[i], L.s[i] = p.data_ptr(), s.data_ptr()
                else:
                    h16 = np.ascontiguousarray(w, dtype=np.float32).astype(np.float16).view(np.uint16)
                    t = torch.from_numpy(h16.view(np.int16)).to(dev)
                    keep.append(t)
                    L.w16[i] = t.data_ptr()
        W = Weights(up(draw.tok_emb), up(draw.lm_head), up(draw.ln_f_g), up(draw.ln_f_b), layers)
        torch.cuda.current_stream(dev).synchronize()
        return cls(cfg, W, device, _keep=keep)

    def matmul(self, layer: int, which: int, x_hi: torch.Tensor, x_lo: torch.Tensor,
               out: Optional[torch.Tensor] = None) -> torch.Tensor:
        """Backbone MatMul `which` (0 QKV, 1 O, 2 FC1, 3 FC2) of `layer` on split activation
        planes [M, K] (see split_f16) -> fp32 [M, N] (ms_model_matmul)."""
        m, k = x_hi.shape
        c = self.cfg
        n = [(c.n_heads + 2 * c.n_kv_heads) * 64, c.d_model, c.d_ff, c.d_model][which]
        y = torch.empty((m, n), dtype=torch.float32, device=x_hi.device) if out is None else out
        _check(_lib.ms_model_matmul(self._h, layer, which, _ptr(x_hi), _ptr(x_lo), k, m, _ptr(y), n, _stream()),
               "ms_model_matmul")
        return y

    @property
    def weight_bytes(self) -> int:
        return int(_lib.ms_model_weight_bytes(self._h))

    def close(self):
        if getattr(self, "_h", None):
            _lib.ms_model_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class Cache:
    """A fixed-capacity KV cache for `batch` streams (ms_cache_create) and the calls on it."""

    def __init__(self, model: Model, batch: int, capacity: int, kv_format: int = MS_KV_F32):
        self.model = model
        h = ctypes.c_void_p()
        _check(_lib.ms_cache_create_ex(model._h, batch, capacity, kv_format, ctypes.byref(h)), "ms_cache_create_ex")
        self._h = h
        self.batch = batch
        self.capacity = capacity
        self.vocab = model.cfg.vocab
        self._dev = torch.device("cuda", model.device)

    @property
    def length(self) -> int:
        return int(_lib.ms_cache_length(self._h))

    @property
    def kv_format(self) -> int:
        return int(_lib.ms_cache_kv_format(self._h))

    @property
    def kernel_launches(self) -> int:
        return int(_lib.ms_cache_kernel_launches(self._h))

    PATH_AUTO, PATH_PERSISTENT, PATH_PER_OP = 0, 1, 2

    def set_guidance(self, scale: float):
        """Classifier-free guidance over stream pairs (2p, 2p+1) = (conditional,
        unconditional): both take the argmax of u + scale (k - u); 0 turns it off."""
        _check(_lib.ms_cache_set_guidance(self._h, ctypes.c_float(scale)), "ms_cache_set_guidance")

    def set_act_int8(self, on: bool):
        """W4A8: the backbone MatMuls on INT8 activation codes (ms_cache_set_act_int8)."""
        _check(_lib.ms_cache_set_act_int8(self._h, 1 if on else 0), "ms_cache_set_act_int8")

    @property
    def act_int8(self) -> bool:
        return bool(_lib.ms_cache_act_int8(self._h))

    def set_wait_limits(self, polls: int, stall: int = 0):
        """Persistent kernel's wait limits (0 = defaults); stall 1 or 2 injects a wait that
        nothing satisfies (tests of the timeout path only)."""
        _check(_lib.ms_cache_set_wait_limits(self._h, polls, stall), "ms_cache_set_wait_limits")

    @property
    def guidance(self) -> float:
        return float(_lib.ms_cache_guidance(self._h))

    def set_decode_path(self, path: int):
        """0 automatic, 1 persistent decode kernel, 2 one kernel per operation."""
        _check(_lib.ms_cache_set_decode_path(self._h, path), "ms_cache_set_decode_path")

    @property
    def decode_path(self) -> int:
        return int(_lib.ms_cache_decode_path(self._h))

    def reset(self):
        _check(_lib.ms_cache_reset(self._h), "ms_cache_reset")

    def prefill(self, tokens: Optional[torch.Tensor], prefix: Optional[torch.Tensor],
                logits: Optional[torch.Tensor] = None, argmax: Optional[torch.Tensor] = None):
        """tokens int64 [B, S] (or None), prefix fp32 [B, P, d] (or None) -> (logits [B, V], argmax [B])."""
        S = 0 if tokens is None else tokens.shape[1]
        P = 0 if prefix is None else prefix.shape[1]
        if logits is None:
            logits = torch.empty((self.batch, self.vocab), dtype=torch.float32, device=self._dev)
        if argmax is None:
            argmax = torch.empty((self.batch,), dtype=torch.int32, device=self._dev)
        _check(_lib.ms_prefill(self.model._h, self._h, _ptr(tokens), S, _ptr(prefix), P, _ptr(logits), _ptr(argmax),
                               _stream()), "ms_prefill")
        return logits, argmax

    def decode_step(self, tokens: torch.Tensor, logits: Optional[torch.Tensor] = None,
                    argmax: Optional[torch.Tensor] = None):
        """tokens int32 [B] -> (logits [B, V], argmax [B]); appends one position."""
        if logits is None:
            logits = torch.empty((self.batch, self.vocab), dtype=torch.float32, device=self._dev)
        if argmax is None:
            argmax = torch.empty((self.batch,), dtype=torch.int32, device=self._dev)
        _check(_lib.ms_decode_step(self.model._h, self._h, _ptr(tokens), _ptr(logits), _ptr(argmax), _stream()),
               "ms_decode_step")
        return logits, argmax

    def generate(self, n_steps: int, out_tokens: Optional[torch.Tensor] = None, logits: bool = True):
        """Greedy loop of n_steps -> (tokens int32 [n, B], last logits [B, V] or None)."""
        if out_tokens is None:
            out_tokens = torch.empty((n_steps, self.batch), dtype=torch.int32, device=self._dev)
        lg = torch.empty((self.batch, self.vocab), dtype=torch.float32, device=self._dev) if logits else None
        _check(_lib.ms_generate(self.model._h, self._h, n_steps, _ptr(out_tokens), _ptr(lg), _stream()), "ms_generate")
        return out_tokens, lg

    def export(self):
        """Cache contents in the pages' layout: (k, v) fp32 numpy [L, B, T, Hk, 64]."""
        c = self.model.cfg
        shape = (c.n_layers, self.batch, self.length, c.n_kv_heads, 64)
        k = np.empty(shape, np.float32)
        v = np.empty(shape, np.float32)
        _check(_lib.ms_cache_export(self._h, k.ctypes.data_as(_P), v.ctypes.data_as(_P)), "ms_cache_export")
        return k, v

    def import_(self, k: np.ndarray, v: np.ndarray):
        k = np.ascontiguousarray(k, np.float32)
        v = np.ascontiguousarray(v, np.float32)
        _check(_lib.ms_cache_import(self._h, k.ctypes.data_as(_P), v.ctypes.data_as(_P), k.shape[2]),
               "ms_cache_import")

    def device_status(self) -> int:
        """Synchronise and return the device-side status (0 = MS_OK); clears it."""
        return int(_lib.ms_device_status(self._h, _stream()))

    def close(self):
        if getattr(self, "_h", None):
            _lib.ms_cache_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class Conditioner:
    """The conditioner front-end (ms_cond_create): audio [B, n_samples] -> the decoder's prefix
    [B, frames + 1 + K, d_model] (log-mel frames projected, then the dataset row and the K
    instrument rows)."""

    def __init__(self, window, mel_fb, proj_w, proj_b, inst_emb, ds_emb, n_samples: int, hop: int,
                 max_batch: int = 1, device: int = 0):
        mel_fb = np.ascontiguousarray(mel_fb, dtype=np.float32)
        proj_w = np.ascontiguousarray(proj_w, dtype=np.float32)
        inst_emb = np.ascontiguousarray(inst_emb, dtype=np.float32)
        ds_emb = np.ascontiguousarray(ds_emb, dtype=np.float32)
        window = np.ascontiguousarray(window, dtype=np.float32)
        proj_b = np.ascontiguousarray(proj_b, dtype=np.float32)
        self.cfg = CondConfig(int(n_samples), int(window.shape[0]), int(hop), int(mel_fb.shape[0]),
                              int(proj_w.shape[0]), int(inst_emb.shape[0]), int(ds_emb.shape[0]), int(max_batch))
        self.device = device
        W = CondWeights(*(a.ctypes.data for a in (window, mel_fb, proj_w, proj_b, inst_emb, ds_emb)))
        h = ctypes.c_void_p()
        _check(_lib.ms_cond_create(ctypes.byref(self.cfg), ctypes.byref(W), device, ctypes.byref(h)),
               "ms_cond_create")
        self._h = h

    @classmethod
    def from_draw(cls, draw, n_samples: int, hop: int, max_batch: int = 1, device: int = 0) -> "Conditioner":
        """From host arrays (synth.CondDraw)."""
        return cls(draw.window, draw.mel_fb, draw.proj_w, draw.proj_b, draw.inst_emb, draw.ds_emb, n_samples, hop,
                   max_batch, device)

    @property
    def frames(self) -> int:
        return int(_lib.ms_cond_frames(self._h))

    def rows(self, K: int) -> int:
        return self.frames + 1 + K

    def __call__(self, audio: torch.Tensor, dataset: torch.Tensor, instruments: Optional[torch.Tensor],
                 out: Optional[torch.Tensor] = None) -> torch.Tensor:
        """audio fp32 [B, n_samples], dataset int32 [B], instruments int32 [B, K] (or None for
        K = 0) -> prefix fp32 [B, frames + 1 + K, d_model] (ms_condition)."""
        B = audio.shape[0]
        K = 0 if instruments is None else instruments.shape[1]
        y = out if out is not None else torch.empty((B, self.rows(K), self.cfg.d_model), dtype=torch.float32,
                                                   device=audio.device)
        _check(_lib.ms_condition(self._h, _ptr(audio), B, _ptr(dataset), _ptr(instruments), K, _ptr(y), _stream()),
               "ms_condition")
        return y

    def log_mel(self, audio: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
        """audio fp32 [B, n_samples] -> fp32 [B, frames, n_mels] (ms_cond_log_mel)."""
        B = audio.shape[0]
        y = out if out is not None else torch.empty((B, self.frames, self.cfg.n_mels), dtype=torch.float32,
                                                   device=audio.device)
        _check(_lib.ms_cond_log_mel(self._h, _ptr(audio), B, _ptr(y), _stream()), "ms_cond_log_mel")
        return y

    def device_status(self) -> int:
        """ms_cond_device_status: synchronises and returns (and clears) the status."""
        return int(_lib.ms_cond_device_status(self._h, _stream()))

    def close(self):
        if getattr(self, "_h", None):
            _lib.ms_cond_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
