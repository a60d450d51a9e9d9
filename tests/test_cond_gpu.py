"""The conditioner front-end on the GPU against the oracle's conditioner.

MuScriptor small — ONNX conversion, the conditioner graph (audio [1, 80000] at 16 kHz,
instrument ids, dataset id -> prefix [1, 501 + 1 + K, d]); MuScriptor model card, Model
description (STFT 2048 / 160, 512 mel bands, log, projection).

Bars:
- log-mel features: the GPU computes them in double and rounds to fp32, so each is within one
  fp32 rounding of the oracle's double value (2^-23 relative covers the rounding of a value
  that differs from the oracle's in its last double bits), plus 1e-9.
- projected rows: the features and the weights enter the tensor cores as fp16 hi + lo pairs
  (22-bit significands) and the K = n_mels products are summed in fp32 in chunks; the bar is
  4e-6 of sum_k |x_k w_k| (about 64 fp32 roundings of the largest partial sum) plus 1e-6 and
  the bias's own rounding.  Dropping the weights' lo halves would leave errors of ~2^-12 of the
  products, several times this bar.
- dataset and instrument rows: copies, bit-exact.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import ms_oracle as O

pytestmark = pytest.mark.gpu
ms = pytest.importorskip("decoder_only_transformer_int4_b200")


def _dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t if dtype is None else t.to(dtype)


def _check_log_mel(gpu, audio, cond, hop):
    for b in range(audio.shape[0]):
        ref = O.log_mel(O.stft_magnitude(audio[b], cond.window, hop), cond.mel_fb)
        g = gpu[b].astype(np.float64)
        err = np.abs(g - ref)
        bound = 2.0 ** -23 * np.abs(ref) + 1e-9
        assert np.all(err <= bound), (b, float((err / bound).max()))


def _check_prefix(gpu, audio, dataset, inst, cond, hop):
    ref = O.conditioner(audio, dataset, inst, cond, hop)
    assert gpu.shape == ref.shape
    frames = 1 + audio.shape[1] // hop
    W = cond.proj_w.astype(np.float64)
    for b in range(audio.shape[0]):
        x = O.log_mel(O.stft_magnitude(audio[b], cond.window, hop), cond.mel_fb)
        mass = np.abs(x) @ np.abs(W).T
        err = np.abs(gpu[b, :frames].astype(np.float64) - ref[b, :frames])
        bound = 4e-6 * mass + 1e-6 + 2.0 ** -23 * np.abs(cond.proj_b)[None, :]
        assert np.all(err <= bound), (b, float((err / bound).max()))
        # the rows after the frames are copies of table rows
        assert np.array_equal(gpu[b, frames], cond.ds_emb[dataset[b]])
        for k in range(inst.shape[1]):
            assert np.array_equal(gpu[b, frames + 1 + k], cond.inst_emb[inst[b, k]])


def test_log_mel_full_size_noise_and_tone():
    """5 s at 16 kHz, n_fft 2048, hop 160, 512 bands: 501 frames; noise and the 440 Hz tone."""
    cond = synth.make_cond_weights(256)
    audio = np.concatenate([synth.make_noise_audio(1, seed=181), synth.make_tone(1)], axis=0)
    c = ms.Conditioner.from_draw(cond, synth.N_SAMPLES, synth.HOP, max_batch=2)
    assert c.frames == 501
    lm = c.log_mel(_dev(audio)).cpu().numpy()
    assert c.device_status() == ms.MS_OK
    _check_log_mel(lm, audio, cond, synth.HOP)


def test_prefix_full_size_matches_the_oracle():
    """The decoder's 503 prefix rows: 501 projected frames, the dataset row, one instrument."""
    d = 1024
    cond = synth.make_cond_weights(d)
    audio = np.concatenate([synth.make_tone(1), synth.make_noise_audio(1, seed=182)], axis=0)
    dataset = np.array([1, 0], dtype=np.int32)
    inst = np.array([[0], [129]], dtype=np.int32)
    c = ms.Conditioner.from_draw(cond, synth.N_SAMPLES, synth.HOP, max_batch=2)
    p = c(_dev(audio), _dev(dataset), _dev(inst)).cpu().numpy()
    assert c.device_status() == ms.MS_OK
    assert p.shape == (2, 503, d)
    _check_prefix(p, audio, dataset, inst, cond, synth.HOP)


@pytest.mark.parametrize("n_fft,hop,n_samples,n_mels,d,B,K", [
    (256, 64, 4001, 40, 128, 3, 2),      # ragged: 4001 = 62 * 64 + 33; 40 bands pad to 64 columns
    (16, 3, 50, 5, 4, 2, 0),             # the smallest transform, no instrument rows
    (4096, 512, 9000, 100, 200, 1, 3),   # the largest transform (shared memory above 48 KiB)
    (512, 160, 257, 64, 256, 2, 1),      # a signal barely longer than half a frame
])
def test_prefix_small_and_edge_configs(n_fft, hop, n_samples, n_mels, d, B, K):
    cond = synth.make_cond_weights(d, seed=11, n_fft=n_fft, n_mels=n_mels)
    audio = synth.make_noise_audio(B, seed=183, n_samples=n_samples)
    rng = np.random.default_rng(5)
    dataset = rng.integers(0, synth.N_DATASETS, size=B).astype(np.int32)
    inst = rng.integers(0, synth.N_INSTRUMENTS, size=(B, K)).astype(np.int32)
    c = ms.Conditioner.from_draw(cond, n_samples, hop, max_batch=B)
    frames = 1 + n_samples // hop
    assert c.frames == frames
    p = c(_dev(audio), _dev(dataset), _dev(inst) if K else None).cpu().numpy()
    lm = c.log_mel(_dev(audio)).cpu().numpy()
    assert c.device_status() == ms.MS_OK
    assert p.shape == (B, frames + 1 + K, d)
    _check_log_mel(lm, audio, cond, hop)
    _check_prefix(p, audio, dataset, inst, cond, hop)


def test_ids_out_of_range_are_clamped_and_reported():
    d = 128
    cond = synth.make_cond_weights(d, n_fft=256, n_mels=40)
    audio = synth.make_noise_audio(1, seed=184, n_samples=2000)
    c = ms.Conditioner.from_draw(cond, 2000, 64)
    p = c(_dev(audio), _dev(np.array([7], np.int32)), _dev(np.array([[-3, 130]], np.int32))).cpu().numpy()
    assert c.device_status() == ms.MS_ERR_TOKEN_RANGE
    f = c.frames
    assert np.array_equal(p[0, f], cond.ds_emb[1])
    assert np.array_equal(p[0, f + 1], cond.inst_emb[0])
    assert np.array_equal(p[0, f + 2], cond.inst_emb[129])
    assert c.device_status() == ms.MS_OK
    with pytest.raises(ms.MsError) as e:
        c(_dev(np.concatenate([audio, audio])), _dev(np.array([0, 0], np.int32)), None)
    assert e.value.status == ms.MS_ERR_SHAPE


def test_audio_to_first_token_matches_the_oracle_pipeline():
    """Tone -> conditioner -> 503-row prefix -> prefill on a two-layer decoder: last-position
    logits within the decoder's 2e-3 bar of the oracle's conditioner + decoder."""
    sh = synth.Shape("cond-pipeline", 2, 256, 4, 2, 1024)
    draw = synth.make_weights(sh, seed=0)
    om, gm = O.OracleModel(draw, "int4"), ms.Model.from_draw(draw, "int4")
    cond = synth.make_cond_weights(sh.d_model)
    audio = synth.make_tone(1)
    dataset, inst = np.array([1], np.int32), np.array([[0]], np.int32)
    c = ms.Conditioner.from_draw(cond, synth.N_SAMPLES, synth.HOP)
    prefix = c(_dev(audio), _dev(dataset), _dev(inst))
    assert prefix.shape == (1, 503, sh.d_model)
    start = synth.make_start_tokens(1, vocab=sh.vocab, seed=185)
    cache = ms.Cache(gm, 1, 520)
    lg, am = cache.prefill(_dev(start.reshape(1, 1)), prefix)
    assert cache.device_status() == ms.MS_OK and c.device_status() == ms.MS_OK
    ref_prefix = O.conditioner(audio, dataset, inst, cond, synth.HOP)[0]
    ref = om.prefill(om.new_cache(520), ref_prefix, [int(start[0])])
    assert np.abs(lg.cpu().numpy()[0] - ref).max() <= 2e-3
