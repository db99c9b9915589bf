"""The seeded input generator: counter-based, deterministic, right distributions."""
import math

import numpy as np

from combine_moe_pw_b200 import synth

M64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15


def _mix(z):
    """SplitMix64 output function (Steele, Lea & Flood 2014), pure Python."""
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
    return z ^ (z >> 31)


def test_splitmix_stream_definition():
    for seed, stream in [(0, 1), (0, 3), (12345, 5)]:
        key = _mix((_mix((seed + GAMMA) & M64) + (stream + 1) * GAMMA) & M64)
        for i in [0, 1, 2, 1000, 10**9]:
            assert synth.raw_u64(seed, stream, i) == _mix((key + (i + 1) * GAMMA) & M64)


def test_box_muller_definition():
    for n in [0, 5, 777]:
        u1 = (synth.raw_u64(0, 3, 2 * n) >> 11) * 2.0 ** -53
        u2 = (synth.raw_u64(0, 3, 2 * n + 1) >> 11) * 2.0 ** -53
        z = math.sqrt(-2.0 * math.log(1.0 - u1)) * math.cos(2 * math.pi * u2)
        assert abs(synth.raw_normal(0, 3, n) - z) <= 1e-15 * max(1.0, abs(z))


def test_deterministic_and_sliceable():
    w = synth.WORKLOADS["tiny"]
    a, b = synth.logits(w), synth.logits(w)
    np.testing.assert_array_equal(a, b)
    # a prefix of a longer batch is the shorter batch (counter-based)
    short = synth.x_bf16(w.with_(T=100))
    np.testing.assert_array_equal(short, synth.x_bf16(w)[:100])
    assert not np.array_equal(synth.x_bf16(w.with_(seed=1))[:10], short[:10])


def test_distributions():
    w = synth.WORKLOADS["tiny"]
    lg = synth.logits(w).astype(np.float64)
    assert abs(lg.mean()) < 0.02 and abs(lg.std() - 1.0) < 0.02
    x = synth.bf16_bits_to_f32(synth.x_bf16(w)).astype(np.float64)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    s = synth.scales(w)
    assert s.min() >= 0.5 and s.max() < 1.5
    # sequence bias: tokens of one sequence share a per-expert offset
    wl = w.with_(logit_kind=synth.LOGIT_SEQBIAS, T=4096, seq_len=2048)
    l2 = synth.logits(wl).astype(np.float64)
    b0 = l2[:2048].mean(axis=0)
    b1 = l2[2048:].mean(axis=0)
    assert 0.35 < b0.std() < 0.65 and np.corrcoef(b0, b1)[0, 1] < 0.5
    # Zipf popularity: experts' mean logits are -ln(rank) for a permutation of ranks
    wz = w.with_(logit_kind=synth.LOGIT_ZIPF, T=4096)
    m = synth.logits(wz).astype(np.float64).mean(axis=0)
    keys = np.array([synth.raw_u64(0, 5, e) for e in range(w.E)], dtype=np.uint64)
    ranks = 1 + np.argsort(np.argsort(keys, kind="stable"), kind="stable")
    assert sorted(ranks) == list(range(1, w.E + 1))
    assert np.abs(m + np.log(ranks)).max() < 0.08  # 5 sigma of a 4096-token mean


def test_workloads_match_recipes():
    W = synth.WORKLOADS
    assert (W["tiny"].E, W["tiny"].T, W["tiny"].D) == (48, 2048, 128)
    assert W["tiny"].T // W["tiny"].seq_len == 8
    assert W["layer"].T // W["layer"].seq_len == 16
    assert W["rack"].T // W["rack"].seq_len == 64
    assert W["long"].T // W["long"].seq_len == 4
    assert W["ragged"].T // W["ragged"].seq_len == 32 and W["ragged"].mode == synth.MODE_RAGGED
    for name in ["layer", "rack", "long", "ragged"]:
        w = W[name]
        assert (w.E, w.k, w.D, w.R, w.L, w.W, w.P) == (384, 8, 3072, 64, 6, 3, 2)


def test_row_slices_equal_the_whole():
    """One GPU's share of a batch is generated on its own: rows [t0, t0+n)
    equal the same rows of the whole batch, for every logit kind."""
    for kind in (synth.LOGIT_IID, synth.LOGIT_SEQBIAS, synth.LOGIT_ZIPF):
        w = synth.WORKLOADS["tiny"].with_(logit_kind=kind, seq_len=100)
        lg, x = synth.logits(w), synth.x_bf16(w)
        for t0, n in [(0, 5), (37, 300), (w.T - 9, 9)]:
            np.testing.assert_array_equal(synth.logits_rows(w, t0, n), lg[t0:t0 + n])
            np.testing.assert_array_equal(synth.x_bf16_rows(w, t0, n), x[t0:t0 + n])
