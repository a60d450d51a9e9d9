"""The roofline numerator of bench.py, the algorithmic bytes of a decode step, against figures
worked out by hand from each workload's shapes: per weight row K/2 bytes of INT4 codes and
K/8 bytes of fp32 scales (or 2K bytes of fp16), the fp32 LM head, one fp32 embedding row per
stream, and fp32 K and V over every position a step attends (the cached ones and its own)."""
import pytest

import bench
import synth


def _per_step(key):
    wl = synth.WORKLOADS[key]
    w, kv = bench._decode_bytes_per_token(wl)
    return w, sum(kv) / len(kv)


def test_medium_batch1_to_the_byte():
    # medium model, per layer: N*K = 1536*1024 + 1024*1024 + 4096*1024 + 1024*4096 = 11,010,048
    codes = 24 * 11_010_048 // 2                 # 132,120,576
    scales = 24 * (11_010_048 // 32) * 4         # 33,030,144
    head = 1393 * 1024 * 4                       # 5,705,728
    emb = 1024 * 4
    # decode step i = 0..1999 attends 503 + 1 + i + 1 positions: mean 1504.5;
    # K and V x 24 layers x 4 kv heads x 64 fp32
    kv = 2 * 24 * 4 * 64 * 4 * 1504.5            # 73,949,184
    w, kvm = _per_step("c3")
    assert w == codes + scales + head + emb
    assert kvm == kv
    assert w + kvm == 244_809_728
    # the per-launch figure the recorded DRAM traffic is compared with: 128 steps at T = 1401..1528
    wl = synth.WORKLOADS["c3"]
    launch = sum(bench._decode_bytes_at(wl, t) for t in range(1401, 1529))
    assert launch == 128 * (codes + scales + head + emb) + 2 * 24 * 4 * 64 * 4 * sum(range(1401, 1529))


# (workload, weights + scales + LM head + embedding rows in MB, mean K/V read per step in MB),
# each from the hand-worked per-workload table (MB = 1e6 bytes, rounded as printed there)
HAND = [
    ("c1", 7.08 + 1.77 + 4.28, 6.24),
    ("c2", 49.5 + 12.4 + 4.28, 46.1),
    ("c3pages", 151.0 + 37.7 + 5.7, 295.6),
    ("c4", 170.9, 2389.0),
    ("c5", 604.0 + 151.0 + 8.6, 246.5),
    ("c5b16", 763.5, 3943.0),
    ("c5fp16", 2415.9 + 8.6, 246.5),
]


@pytest.mark.parametrize("key,weights_mb,kv_mb", HAND)
def test_every_workload_matches_its_hand_figures(key, weights_mb, kv_mb):
    w, kvm = _per_step(key)
    # the printed figures carry rounding of a few parts in a thousand at most
    assert abs(w / 1e6 - weights_mb) <= 2e-3 * weights_mb + 0.05, (key, w / 1e6)
    assert abs(kvm / 1e6 - kv_mb) <= 2e-3 * kv_mb + 0.05, (key, kvm / 1e6)
