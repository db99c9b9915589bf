"""Seeded random batch geometries shared by the GPU fuzz tests and the
oracle's CPU self-consistency tests.  Each draw depends only on its index, so a
failing case reproduces from its name.  No arithmetic of the method lives here.
"""
import numpy as np

from combine_moe_pw_b200 import synth


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


def random_wide_workload(i: int) -> synth.Workload:
    """Draws at the widths the method uses (1024 to 6144 bf16), where the row
    copies run through the shared-memory rings with few stages per block."""
    rng = np.random.default_rng(8000 + i)
    R = int(rng.choice([2, 4, 8, 16]))
    W = int(rng.choice([1, 3]))
    P = int(rng.choice([1, 2, 4]))
    L = W * P
    k = int(rng.integers(1, min(R * L, 8) + 1))
    D = int(rng.choice([1024, 3072, 6144]))
    T_s = int(rng.choice([3, 64, 129]))
    mode = synth.MODE_RAGGED if rng.random() < 0.25 else synth.MODE_POOLED
    cf_send, cf_recv = (0, 0) if mode == synth.MODE_RAGGED else (
        int(rng.choice([60, 110])), int(rng.choice([80, 115])))
    kind = int(rng.choice([synth.LOGIT_IID, synth.LOGIT_SEQBIAS, synth.LOGIT_ZIPF]))
    return synth.Workload(f"wide{i}", T=R * T_s, R=R, L=L, W=W, P=P, k=k, D=D,
                          seq_len=T_s, logit_kind=kind, cf_send_pct=cf_send,
                          cf_recv_pct=cf_recv, mode=mode, seed=100 + i)
