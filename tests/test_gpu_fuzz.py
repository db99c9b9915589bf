"""Seeded random small configurations: the whole GPU path against the whole
oracle, with the same bar as tests/test_gpu_parity.py (bit-exact integer and
byte outputs, gates within 1e-6 relative, combine within 1e-6 of its scale).

Each case draws its geometry (ranks, experts per rank, waves, top-k, width,
tokens per source, capacity factors, pooled or dropless mode, logit
distribution) from a fixed seed, so a failure names a case that reproduces.
The draws cover shapes the named workloads do not: one-token sources, widths
that are not a multiple of 128 bytes, P up to 6, k up to 12, factors below
the mean load (heavy drops) and far above it.
"""
import numpy as np
import pytest

from combine_moe_pw_b200 import synth
from test_gpu_parity import _inputs, check_full, run_gpu

N_CASES = 24


def random_workload(i: int) -> synth.Workload:
    rng = np.random.default_rng(7000 + i)
    while True:
        R = int(rng.choice([1, 2, 3, 4, 5, 8, 16]))
        W = int(rng.choice([1, 2, 3]))
        P = int(rng.choice([1, 2, 3, 4, 6]))
        L = W * P
        E = R * L
        if E % 4 != 0 or E > 2048:  # the router reads logits 16 bytes at a time
            continue
        k = int(rng.integers(1, min(E, 12) + 1))
        D = int(rng.choice([8, 16, 40, 64, 136, 264]))
        T_s = int(rng.choice([1, 2, 7, 33, 100, 257]))
        mode = synth.MODE_RAGGED if rng.random() < 0.25 else synth.MODE_POOLED
        cf_send = int(rng.choice([0, 40, 100, 110, 250]))
        cf_recv = int(rng.choice([0, 50, 115, 300]))
        if mode == synth.MODE_RAGGED:
            cf_send = cf_recv = 0
        kind = int(rng.choice([synth.LOGIT_IID, synth.LOGIT_SEQBIAS, synth.LOGIT_ZIPF]))
        seq_len = int(rng.choice([1, 5, 64, 1000]))
        return synth.Workload(f"fuzz{i}", T=R * T_s, R=R, L=L, W=W, P=P, k=k, D=D,
                              seq_len=seq_len, logit_kind=kind, cf_send_pct=cf_send,
                              cf_recv_pct=cf_recv, mode=mode, seed=i)


def test_draws_are_varied():
    ws = [random_workload(i) for i in range(N_CASES)]
    assert len({(w.R, w.L, w.W, w.P, w.k, w.D) for w in ws}) > N_CASES // 2
    assert any(w.mode == synth.MODE_RAGGED for w in ws)
    assert any(w.cf_send_pct and w.cf_send_pct < 100 for w in ws)


@pytest.mark.gpu
@pytest.mark.parametrize("i", range(N_CASES))
def test_random_config_full_parity(i):
    w = random_workload(i)
    lg, x, s = _inputs(w)
    b, st = run_gpu(w, lg, x, s)
    check_full(w, lg, x, s, b, st)
