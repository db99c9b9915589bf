"""Pins for the oracle's sequence-level balance term (orc_seq_balance).

"Marin 开始公开训练 535B 参数 MoE 模型", section 四, names sequence-level
balancing as a remedy for drops without a formula; the reading implemented is
a per-sequence balance term of the training loss, alpha * sum_e f_e * P_e,
with f_e the expert's share of the sequence's assignments (scaled so that
perfect balance is 1) and P_e its mean router probability over the sequence.

Pins: f against a library histogram, P against a library softmax, the closed
forms of perfect balance (loss = alpha for any logits) and of equal logits,
the gradient against torch.autograd, and the softmax-gradient invariant (each
token's gradient row sums to zero).
"""
import numpy as np
import pytest
import scipy.special
import torch

import oracle
from combine_moe_pw_b200 import synth

W = synth.WORKLOADS["tiny"]
ALPHA = 0.01


def _geom(w):
    return oracle.geom_for(w)


def test_f_and_P_against_library_routines():
    w = W.with_(logit_kind=synth.LOGIT_SEQBIAS)
    g = _geom(w)
    lg = synth.logits(w)
    idx, _ = oracle.route(g, lg)
    L = 256
    f, P, loss, _ = oracle.seq_balance(g, L, ALPHA, lg, idx)
    for s in range(w.T // L):
        counts = np.bincount(idx[s * L:(s + 1) * L].reshape(-1), minlength=w.E)
        np.testing.assert_allclose(f[s] * (w.k * L / w.E), counts, rtol=0, atol=1e-9)
        p = scipy.special.softmax(lg[s * L:(s + 1) * L].astype(np.float64), axis=1)
        np.testing.assert_allclose(P[s], p.mean(axis=0), rtol=1e-12, atol=1e-15)
        np.testing.assert_allclose(loss[s], ALPHA * np.dot(f[s], P[s]), rtol=1e-12)
    # skewed routing inside a sequence costs more than balance
    assert loss.min() > ALPHA


def test_perfect_balance_gives_alpha_for_any_logits():
    """Token t of a sequence picks experts (k t + j) mod E: every expert gets
    the same share, f = 1, and the probabilities sum to one per token, so the
    term is exactly alpha whatever the logits."""
    g = _geom(W)
    lg = synth.logits(W.with_(logit_kind=synth.LOGIT_ZIPF))
    t = np.arange(W.T)[:, None]
    idx = ((W.k * t + np.arange(W.k)[None, :]) % W.E).astype(np.int32)
    L = 48  # a multiple of E / gcd(E, k): whole rounds of the round robin
    f, P, loss, dl = oracle.seq_balance(g.__class__(**{**g.__dict__, "T": 2016}), L, ALPHA,
                                        lg[:2016], idx[:2016])
    np.testing.assert_allclose(f, 1.0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(loss, ALPHA, rtol=1e-12)


def test_equal_logits_closed_form():
    """All logits equal: top-k takes experts 0..k-1 (ties to the lower id),
    p = 1/E; f = E/k on those experts and 0 elsewhere, so the term is alpha,
    and the gradient is alpha/L * (1/E) * (f_e - 1)."""
    g = _geom(W)
    lg = np.full((W.T, W.E), 0.5, np.float32)
    idx, _ = oracle.route(g, lg)
    L = 512
    f, P, loss, dl = oracle.seq_balance(g, L, ALPHA, lg, idx)
    expect_f = np.where(np.arange(W.E) < W.k, W.E / W.k, 0.0)
    np.testing.assert_allclose(f, np.tile(expect_f, (W.T // L, 1)), rtol=1e-12)
    np.testing.assert_allclose(P, 1.0 / W.E, rtol=1e-12)
    np.testing.assert_allclose(loss, ALPHA, rtol=1e-12)
    np.testing.assert_allclose(dl, np.tile(ALPHA / L / W.E * (expect_f - 1.0), (W.T, 1)),
                               rtol=1e-12, atol=1e-18)


def test_gradient_matches_autograd_and_rows_sum_to_zero():
    w = W.with_(logit_kind=synth.LOGIT_SEQBIAS, T=1024)
    g = _geom(w)
    lg = synth.logits(w)
    idx, _ = oracle.route(g, lg)
    L = 128
    f, P, loss, dl = oracle.seq_balance(g, L, ALPHA, lg, idx)
    x = torch.from_numpy(lg.astype(np.float64)).requires_grad_(True)
    p = torch.softmax(x, dim=1).reshape(w.T // L, L, w.E)
    ft = torch.from_numpy(f)  # the routing is held fixed
    total = (ALPHA * (ft * p.mean(dim=1)).sum(dim=1)).sum()
    total.backward()
    np.testing.assert_allclose(dl, x.grad.numpy(), rtol=1e-9, atol=1e-20)
    np.testing.assert_allclose(dl.sum(axis=1), 0.0, atol=1e-18)
