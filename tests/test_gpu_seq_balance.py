"""Sequence-level balancing on the GPU (moe_pw_seq_balance) against the
oracle's definition (orc_seq_balance), through the C ABI.

Bounds (derived from the fp32 arithmetic; u = 2^-24):
- f: an integer count times E/(kL): two roundings, 2u relative.
- P: each probability (expf, a reciprocal and a product) within 5u; a lane adds at most
  32 of them per chunk (of 128 tokens: 16 per warp), the block 8 warps, then
  the chunks in order: within (32 + 8 + chunks + 8) u of the positive sum,
  doubled for margin.
- loss: P's bound plus the fixed-order sum over E positive terms,
  (E/256 + 8) u.
- dlogits = alpha/L * p (f - dot): dot is a sum of E positive products
  (E/32 per lane, then a 5-level tree), so |err| <= alpha/L * p * (f + dot)
  * (E/32 + 24) u.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_moe_pw_b200 import moe_pw as mp
from combine_moe_pw_b200 import synth

pytestmark = pytest.mark.gpu

U = 2.0 ** -24
ALPHA = 0.01


def run(w, L, accumulate_on=None):
    cfg = mp.Config.from_workload(w)
    lg = synth.logits(w)
    g = oracle.geom_for(w)
    idx, _ = oracle.route(g, lg)
    dev = torch.device("cuda")
    t_lg = torch.from_numpy(lg).to(dev)
    t_idx = torch.from_numpy(idx).to(dev)
    n_seq = w.T // L
    f = torch.full((n_seq, w.E), -1.0, device=dev)
    P = torch.full((n_seq, w.E), -1.0, device=dev)
    loss = torch.full((n_seq,), -1.0, device=dev)
    dl = (torch.full((w.T, w.E), 7.0, device=dev) if accumulate_on is None
          else torch.from_numpy(accumulate_on).to(dev))
    ws = torch.empty((max(mp.moe_pw_seq_balance_plan(cfg, L), 256),), dtype=torch.uint8, device=dev)
    mp.moe_pw_seq_balance(cfg, L, ALPHA, t_lg, t_idx, f, P, loss, ws, dlogits=dl,
                          accumulate=accumulate_on is not None)
    torch.cuda.synchronize()
    return (g, lg, idx, f.cpu().numpy().astype(np.float64), P.cpu().numpy().astype(np.float64),
            loss.cpu().numpy().astype(np.float64), dl.cpu().numpy().astype(np.float64))


def check(w, L, g, lg, idx, f, P, loss, dl, base=None):
    fr, Pr, lr, dr = oracle.seq_balance(g, L, ALPHA, lg, idx)
    chunks = (L + 127) // 128
    np.testing.assert_allclose(f, fr, rtol=2 * U, atol=0)
    rp = 2 * (32 + 8 + chunks + 8) * U
    assert np.all(np.abs(P - Pr) <= rp * Pr + 1e-30)
    rl = rp + (w.E / 256 + 8) * U + 2 * U
    assert np.all(np.abs(loss - lr) <= rl * lr)
    # the gradient: every token of small batches, a sample of large ones
    rows = (np.arange(w.T) if w.T <= 65536 else
            np.unique(np.random.default_rng(2).integers(0, w.T, 4096)))
    fseq = fr[rows // L]
    x = lg[rows].astype(np.float64)
    probs = np.exp(x - x.max(axis=1, keepdims=True))
    probs /= probs.sum(axis=1, keepdims=True)
    dot = (fseq * probs).sum(axis=1, keepdims=True)
    bound = ALPHA / L * probs * (fseq + dot) * (w.E / 32 + 24) * U + 1e-30
    ref = dr[rows] if base is None else dr[rows] + base[rows]
    if base is not None:
        bound = bound + np.abs(base[rows]) * U
    assert np.all(np.abs(dl[rows] - ref) <= bound)


CASES = {
    "tiny": (synth.WORKLOADS["tiny"], 256),
    "tiny_one_sequence": (synth.WORKLOADS["tiny"].with_(logit_kind=synth.LOGIT_SEQBIAS), 2048),
    "tiny_short_sequences": (synth.WORKLOADS["tiny"].with_(logit_kind=synth.LOGIT_ZIPF), 32),
    "pages_shapes": (synth.Workload("ps", T=64 * 64, R=64, L=6, W=3, P=2, k=8, D=8,
                                    seq_len=1024, logit_kind=synth.LOGIT_SEQBIAS), 1024),
    "E1024_partial_lanes": (synth.Workload("e1k", T=512, R=128, L=8, W=4, P=2, k=6, D=8,
                                           seq_len=128, logit_kind=synth.LOGIT_IID), 128),
    "E200_ragged_tail": (synth.Workload("e200", T=3 * 100, R=50, L=4, W=2, P=2, k=3, D=8,
                                        seq_len=100, logit_kind=synth.LOGIT_SEQBIAS), 100),
}


@pytest.mark.parametrize("name", list(CASES))
def test_seq_balance_matches_oracle(name):
    w, L = CASES[name]
    out = run(w, L)
    check(w, L, *out)


def test_seq_balance_accumulates_onto_existing_gradient():
    w, L = CASES["tiny"]
    base = synth.logits(w.with_(seed=9)).astype(np.float32)
    out = run(w, L, accumulate_on=base)
    check(w, L, *out, base=base.astype(np.float64))


def test_seq_balance_rack_full_size():
    """The rack batch (262,144 tokens, 384 experts, 64 sequences of 4096)."""
    w = synth.WORKLOADS["rack"]
    out = run(w, w.seq_len)
    check(w, w.seq_len, *out)
    torch.cuda.empty_cache()
