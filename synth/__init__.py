"""Seeded synthetic inputs for the MuScriptor decoder step.

This module only draws random numbers and states shapes.  It holds none of the
decoder's arithmetic (no quantisation, no normalisation, no attention): both the
CUDA library's tests/benchmarks and the CPU oracle take their inputs from here,
and each side then does its own work on them.

Shapes follow the model descriptions on the pages:
  * MuScriptor small model card, "Model variants" table: small d=768, 12 heads,
    14 layers; medium d=1024, 16 heads, 24 layers; large d=1536, 24 heads,
    48 layers.
  * muscriptor-small-onnx, "muscriptor-small-lm.onnx" signature: tokens
    i64 [1, S], prefix f32 [1, P, d] with P = 501 + 1 + K (503 unconditional),
    logits over the 1393-token MT3 vocabulary.
  * muscriptor-medium-onnx README, "Model variant" and "Quick smoke test":
    fixed-capacity shared fp32 KV cache (2504 positions by default).

Draw recipe (fixed order, torch CPU generator so that every machine with the
same torch build sees the same numbers):
  * weights, seed 0: token embedding [V, d]; then per layer W_qkv [(H+2Hk)*64, d],
    W_o [d, H*64], W_1 [F, d], W_2 [d, F]; then the LM head [V, d].  Every matrix
    is N(0, 0.02) in fp32.  LayerNorm gains are 1 and biases 0 unless
    ``ln_random`` is set, in which case gamma ~ 1 + N(0, 0.1) and beta ~ N(0, 0.1)
    are drawn from a second generator (seed + 1000) so the matrices stay the same.
  * prefixes, seed 1: N(0, 1) fp32 [B, 503, d].
  * start tokens, seed 2: uniform integers in [0, 1393).
  * teacher-forcing token sequences, seed 3: uniform integers in [0, 1393).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List

import numpy as np
import torch

VOCAB = 1393          # MT3 vocabulary (muscriptor-small-onnx, lm.onnx logits shape)
PREFIX_LEN = 503      # 501 frames + 1 dataset + 1 instrument token (cond.onnx output, K = 1)
HEAD_DIM = 64         # past_k [14, 1, T, 12, 64] on the small-onnx page


@dataclasses.dataclass(frozen=True)
class Shape:
    """Model shape.  ``n_kv_heads`` < ``n_heads`` selects grouped-query attention."""
    name: str
    n_layers: int
    d_model: int
    n_heads: int
    n_kv_heads: int
    d_ff: int
    vocab: int = VOCAB
    head_dim: int = HEAD_DIM
    rope_base: float = 1.0e4
    ln_eps: float = 1.0e-5

    @property
    def qkv_dim(self) -> int:
        return (self.n_heads + 2 * self.n_kv_heads) * self.head_dim

    def matmul_shapes(self):
        """(N, K) of the four backbone MatMuls of one layer: QKV, O, FC1, FC2."""
        d, f, hd = self.d_model, self.d_ff, self.head_dim
        return [(self.qkv_dim, d), (d, self.n_heads * hd), (f, d), (d, f)]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One run: shape, streams, prefix rows, greedy decode steps, cache capacity."""
    name: str
    shape: Shape
    batch: int
    prefix_len: int
    decode_steps: int
    capacity: int
    weight_format: str = "int4"   # "int4" or "fp16"


SMALL_SLICE = Shape("small-2layer", 2, 768, 12, 12, 3072)
SMALL = Shape("small", 14, 768, 12, 12, 3072)
MEDIUM = Shape("medium-gqa4", 24, 1024, 16, 4, 4096)
MEDIUM_MHA = Shape("medium-mha", 24, 1024, 16, 16, 4096)
LARGE = Shape("large-gqa8", 48, 1536, 24, 8, 6144)

WORKLOADS: Dict[str, Workload] = {
    "c1": Workload("c1 small 2-layer b1", SMALL_SLICE, 1, PREFIX_LEN, 8, 576),
    "c2": Workload("c2 small b1", SMALL, 1, PREFIX_LEN, 64, 576),
    "c3": Workload("c3 medium b1", MEDIUM, 1, PREFIX_LEN, 2000, 2504),
    "c4": Workload("c4 medium b64", MEDIUM, 64, PREFIX_LEN, 512, 1024),
    "c5": Workload("c5 large b1 int4", LARGE, 1, PREFIX_LEN, 1500, 2504),
    "c5b16": Workload("c5 large b16 int4", LARGE, 16, PREFIX_LEN, 1500, 2504),
    "c5fp16": Workload("c5 large b1 fp16", LARGE, 1, PREFIX_LEN, 1500, 2504, "fp16"),
    "c3pages": Workload("c3 medium b1, kv heads = heads", MEDIUM_MHA, 1, PREFIX_LEN, 2000, 2504),
}


def tiny_shape(n_layers=1, d_model=64, n_heads=2, n_kv_heads=1, d_ff=128, vocab=37) -> Shape:
    """A shape small enough for brute-force checks (head_dim stays 64)."""
    return Shape(f"tiny-L{n_layers}-d{d_model}-h{n_heads}-kv{n_kv_heads}", n_layers, d_model,
                 n_heads, n_kv_heads, d_ff, vocab=vocab)


@dataclasses.dataclass
class LayerDraw:
    ln1_g: np.ndarray
    ln1_b: np.ndarray
    ln2_g: np.ndarray
    ln2_b: np.ndarray
    w: List[np.ndarray]      # fp32 [N, K] for QKV, O, FC1, FC2 (row = output feature)


@dataclasses.dataclass
class WeightDraw:
    shape: Shape
    tok_emb: np.ndarray      # fp32 [V, d]
    lm_head: np.ndarray      # fp32 [V, d]
    ln_f_g: np.ndarray
    ln_f_b: np.ndarray
    layers: List[LayerDraw]


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _normal(g: torch.Generator, shape, std: float) -> np.ndarray:
    return (torch.randn(*shape, generator=g, dtype=torch.float32) * std).numpy()


def make_weights(shape: Shape, seed: int = 0, std: float = 0.02, ln_random: bool = False) -> WeightDraw:
    """fp32 weights of ``shape`` in the fixed draw order stated in the module docstring."""
    g = _gen(seed)
    d, v = shape.d_model, shape.vocab
    tok_emb = _normal(g, (v, d), std)
    mats = []
    for _ in range(shape.n_layers):
        mats.append([_normal(g, (n, k), std) for (n, k) in shape.matmul_shapes()])
    lm_head = _normal(g, (v, d), std)

    gl = _gen(seed + 1000)

    def ln_pair():
        if ln_random:
            return (1.0 + _normal(gl, (d,), 0.1)).astype(np.float32), _normal(gl, (d,), 0.1)
        return np.ones(d, np.float32), np.zeros(d, np.float32)

    layers = []
    for l in range(shape.n_layers):
        g1, b1 = ln_pair()
        g2, b2 = ln_pair()
        layers.append(LayerDraw(g1, b1, g2, b2, mats[l]))
    gf, bf = ln_pair()
    return WeightDraw(shape, tok_emb, lm_head, gf, bf, layers)


def make_prefix(shape: Shape, batch: int = 1, prefix_len: int = PREFIX_LEN, seed: int = 1) -> np.ndarray:
    """Stand-in for the conditioner output: fp32 [B, P, d] ~ N(0, 1)."""
    g = _gen(seed)
    return torch.randn(batch, prefix_len, shape.d_model, generator=g, dtype=torch.float32).numpy()


def make_start_tokens(batch: int = 1, vocab: int = VOCAB, seed: int = 2) -> np.ndarray:
    """One start token per stream, uniform in [0, vocab): int64 [B]."""
    g = _gen(seed)
    return torch.randint(0, vocab, (batch,), generator=g, dtype=torch.int64).numpy()


def make_token_sequence(n: int, batch: int = 1, vocab: int = VOCAB, seed: int = 3) -> np.ndarray:
    """A fixed token sequence for teacher forcing: int64 [B, n], uniform in [0, vocab)."""
    g = _gen(seed)
    return torch.randint(0, vocab, (batch, n), generator=g, dtype=torch.int64).numpy()


def make_matrix(n: int, k: int, seed: int, std: float = 0.02) -> np.ndarray:
    """A single fp32 [n, k] N(0, std) matrix (kernel-level tests)."""
    return _normal(_gen(seed), (n, k), std)


def make_activations(m: int, k: int, seed: int, std: float = 1.0) -> np.ndarray:
    """fp32 [m, k] N(0, std) activations (kernel-level tests)."""
    return _normal(_gen(seed), (m, k), std)


def make_kv_cache(shape: Shape, batch: int, T: int, seed: int = 4, std: float = 1.0):
    """A cache state of T positions for resuming decode late in a run, in the pages' layout
    (past_k / past_v [L, B, T, Hk, 64]): keys and values N(0, std) fp32, drawn layer by layer
    (all of layer l's keys, then its values).  Any contents are a valid state for the decoder
    step (it reads the cache, it does not check how the cache was made), so parity tests
    import the same draws into both sides."""
    g = _gen(seed)
    sz = (batch, T, shape.n_kv_heads, shape.head_dim)
    k = np.empty((shape.n_layers,) + sz, np.float32)
    v = np.empty_like(k)
    for l in range(shape.n_layers):
        k[l] = torch.randn(*sz, generator=g, dtype=torch.float32).numpy() * std
        v[l] = torch.randn(*sz, generator=g, dtype=torch.float32).numpy() * std
    return k, v


# ---- conditioner front-end inputs --------------------------------------------------------
# "MuScriptor small — ONNX conversion", muscriptor-small-cond.onnx: audio f32 [1, 80000] (one
# 5-second chunk at 16 kHz), instrument ids [1, K] (1 = unconditional), dataset id [1, 1]
# (always 1); the checkpoint stores its STFT window and mel filterbank as half-precision
# buffers.  "MuScriptor — small (≈100M)" model card: STFT n_fft 2048, hop 160, 512 mel bins,
# the spectrogram projected to d_model.  The validation input of the W4A32 page is a 5-second
# 440 Hz tone.

SAMPLE_RATE = 16000
N_SAMPLES = 80000
N_FFT = 2048
HOP = 160
N_MELS = 512
N_INSTRUMENTS = 130
N_DATASETS = 2


@dataclasses.dataclass
class CondDraw:
    window: np.ndarray      # fp32 [n_fft]: the half rounding of the periodic Hann window
    mel_fb: np.ndarray      # fp32 [n_mels, n_fft/2 + 1]: the half rounding of the htk filterbank
    proj_w: np.ndarray      # fp32 [d, n_mels]  (stand-in for the trained projection)
    proj_b: np.ndarray      # fp32 [d]
    inst_emb: np.ndarray    # fp32 [n_instruments, d]
    ds_emb: np.ndarray      # fp32 [n_datasets, d]


def make_tone(batch: int = 1, freq: float = 440.0, amplitude: float = 0.5, n_samples: int = N_SAMPLES,
              sample_rate: int = SAMPLE_RATE) -> np.ndarray:
    """A sine tone, fp32 [B, n_samples]: amplitude * sin(2 pi freq t), t = n / sample_rate."""
    n = np.arange(n_samples, dtype=np.float64)
    x = amplitude * np.sin(2.0 * np.pi * freq * n / sample_rate)
    return np.repeat(x[None].astype(np.float32), batch, axis=0)


def make_noise_audio(batch: int, seed: int = 6, n_samples: int = N_SAMPLES, std: float = 0.1) -> np.ndarray:
    """Seeded N(0, std) audio, fp32 [B, n_samples]."""
    return _normal(_gen(seed), (batch, n_samples), std)


def make_cond_weights(d_model: int, seed: int = 7, n_fft: int = N_FFT, n_mels: int = N_MELS,
                      sample_rate: int = SAMPLE_RATE) -> CondDraw:
    """The conditioner's buffers, as the checkpoint stores them: the half rounding of
    torch.hann_window(n_fft) (periodic, fp32) and the half rounding of the htk mel
    filterbank (no normalisation, 0 .. sample_rate / 2; torchaudio's melscale_fbanks, fp32).
    Projection and embeddings: seeded N(0, 0.02) stand-ins for the trained ones."""
    import warnings
    import torchaudio
    window = torch.hann_window(n_fft, periodic=True, dtype=torch.float32).half().float().numpy()
    with warnings.catch_warnings():
        warnings.simplefilter("ignore")    # 512 htk bands over 1025 bins leave some bands empty
        fb = torchaudio.functional.melscale_fbanks(n_fft // 2 + 1, 0.0, sample_rate / 2.0, n_mels, sample_rate,
                                                   norm=None, mel_scale="htk")
    fb = fb.T.contiguous().half().float().numpy()
    g = _gen(seed)
    proj_w = _normal(g, (d_model, n_mels), 0.02)
    proj_b = _normal(g, (d_model,), 0.02)
    inst_emb = _normal(g, (N_INSTRUMENTS, d_model), 0.02)
    ds_emb = _normal(g, (N_DATASETS, d_model), 0.02)
    return CondDraw(window, fb, proj_w, proj_b, inst_emb, ds_emb)
