"""Host-side check of the persistent decode kernel's work split, on CPU.

The kernel (decoder_only_transformer_int4_b200/csrc/k_decode_persistent.cu) cuts each
matrix's 16-row tiles along K into S = 1, 2 or 4 units, spreads the units over the CTAs,
streams each CTA's records through 16 KiB ring slots, splits every slot's records into eight
contiguous warp runs and walks each run unit segment by unit segment, kUnroll records at a
time (records past a segment's end are read but not added).  This test restates that
arithmetic and checks, for every workload shape and for shapes whose warp runs cross tile
boundaries: every record of a CTA's range is added exactly once, with its own group index
and unit; units per CTA stay within the kernel's 4; the per-step slice table fits its
capacity; the shared memory fits a CTA.  (An earlier version of the walk skipped records
whenever a run crossed a tile boundary; this is the check that would have caught it.)
"""
import pytest

import synth

kSlot, kTile, kMaxUnits, kWarps = 16384, 16, 4, 8
OPTIN, STATIC = 232448, 5120   # shared memory: opt-in limit per CTA, the kernel's static part


def align16(x):
    return (x + 15) & ~15


def choose_split(nt, KG, G):
    best, best_cost = 1, -1
    for S in (1, 2, 4):
        if KG % S:
            continue
        units = (nt * S + G - 1) // G
        if units > kMaxUnits:
            continue
        cost = units * (KG // S) * (10 + S - 1)
        if best_cost < 0 or cost < best_cost:
            best, best_cost = S, cost
    return best


def unit_rec(u, S, KG):
    return (u // S) * KG + (KG * (u % S)) // S


def persist_main(M, d, H, F):
    kmax = max(d, H * 64, F)
    mv = align16(2 * M * (2 * kmax + 64)) + align16(kmax * 4) + align16(d * 8) + kMaxUnits * kWarps * M * kTile * 4
    return max(mv, align16(4 * 9892), align16(M * d * 4))


def check_shape(M, L, d, H, Hk, F, V, fmt="int4", G=148):
    rb = 320 if fmt == "int4" else 1024
    per = kSlot // rb
    U = 4 if M <= 4 else 2
    Ns = [(H + 2 * Hk) * 64, d, F, d]
    Ks = [d, H * 64, d, F]
    splits, cap_pl = [], 0
    for s in range(4):
        nt, KG = Ns[s] // kTile, Ks[s] // 32
        S = 1 if s == 0 else choose_split(nt, KG, G)
        assert (nt * S + G - 1) // G <= kMaxUnits
        splits.append(S)
        cap_pl += (((nt * S + G - 1) // G) * (KG // S) + per - 1) // per
    rpp = kSlot // (d * 4)
    cap = L * cap_pl + ((V + G - 1) // G + rpp - 1) // rpp
    kmax = max(d, H * 64, F)
    region = persist_main(M, d, H, F) + align16(kmax * 2 + 64) + align16(M * d * 4)
    fixed = 1024 + ((cap * 16 + 1023) & ~1023) + region
    nslot = min(16, (OPTIN - STATIC - 256 - fixed) // kSlot)
    for c in range(G):
        slices = 0
        for s in range(4):
            nt, KG, S = Ns[s] // kTile, Ks[s] // 32, splits[s]
            u0, u1 = nt * S * c // G, nt * S * (c + 1) // G
            rbeg, rend = unit_rec(u0, S, KG), unit_rec(u1, S, KG)
            seen = {}
            for p in range(rbeg, rend, per):
                n = min(per, rend - p)
                slices += 1
                for w in range(kWarps):
                    c0, c1 = (n * w) >> 3, (n * (w + 1)) >> 3
                    i = c0
                    while i < c1:
                        r = p + i
                        t, g = divmod(r, KG)
                        h = ((g + 1) * S - 1) // KG
                        end_u = t * KG + (KG * (h + 1)) // S
                        assert unit_rec(t * S + h, S, KG) <= r < end_u
                        assert 0 <= t * S + h - u0 < u1 - u0
                        s1 = min(c1, i + (end_u - r))
                        gi = g
                        while i < s1:
                            for j in range(U):
                                ij = min(i + j, s1 - 1)
                                assert 0 <= ij < n and 0 <= gi + (ij - i) < KG
                                if i + j < s1:
                                    rec = p + i + j
                                    assert gi + j == rec % KG
                                    seen[rec] = seen.get(rec, 0) + 1
                            i += U
                            gi += U
                        i = s1   # the next segment starts exactly where this one ends
            assert sorted(seen) == list(range(rbeg, rend)) and set(seen.values()) <= {1}
        rows = V * (c + 1) // G - V * c // G
        assert slices * L + (rows + rpp - 1) // rpp <= cap
    return splits, nslot


SHAPES = {
    "c1/c2 small": (14, 768, 12, 12, 3072, 1393),
    "c3 medium": (24, 1024, 16, 4, 4096, 1393),
    "c3 pages": (24, 1024, 16, 16, 4096, 1393),
    "c5 large": (48, 1536, 24, 8, 6144, 1393),
    "tiles crossing warp runs": (2, 256, 4, 4, 4096, 300),
    "tiny gqa": (3, 512, 8, 2, 1024, 700),
}


@pytest.mark.parametrize("name", list(SHAPES))
@pytest.mark.parametrize("M", [1, 2, 4])
def test_every_record_exactly_once(name, M):
    L, d, H, Hk, F, V = SHAPES[name]
    splits, nslot = check_shape(M, L, d, H, Hk, F, V)
    # fewer than 4 ring slots: the runtime takes the per-operation path instead (the large
    # model at 4 streams); one stream always fits
    if M == 1:
        assert nslot >= 4


def test_fp16_large_model_fits():
    splits, nslot = check_shape(1, 48, 1536, 24, 8, 6144, 1393, fmt="fp16")
    assert nslot >= 4


def test_medium_model_splits():
    """The medium model splits O and FC2 in two (64 tiles would leave 84 CTAs idle) and keeps
    QKV and FC1 whole."""
    assert check_shape(1, 24, 1024, 16, 4, 4096, 1393)[0] == [1, 2, 1, 2]


def test_workloads_are_covered():
    for key in ("c1", "c2", "c3", "c3pages", "c5"):
        sh = synth.WORKLOADS[key].shape
        assert (sh.n_layers, sh.d_model, sh.n_heads, sh.n_kv_heads, sh.d_ff) in {v[:5] for v in SHAPES.values()} or \
            key == "c1"
