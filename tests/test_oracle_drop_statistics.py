"""Statistical sanity of the oracle's sender drops (not a parity test).

With i.i.d. logits every token's top-k is a uniformly random k-subset of the
E experts (the logits are exchangeable).  A pool (s, d, w) holds P experts, so
one token adds X in {0, ..., min(k, P)} arrivals to it, with the
hypergeometric law P(X = x) = C(P, x) C(E - P, k - x) / C(E, k).  A pool's
count N is the sum of X over the T_s tokens of its source (independent
tokens), so its exact law is a T_s-fold convolution, and its expected sender
drops are E[max(N - C_s, 0)].  Expectation is linear, so the expected drop
rate of the whole batch is n_pools * E[max(N - C_s, 0)] / (T k), whatever the
dependence between the pools of one token.

The oracle's measured rate, averaged over 48 seeded batches, must match that
exact expectation within 4 standard errors (estimated from the seeds); with
the same data, the expectations for a capacity one slot smaller or larger lie
outside that band (about 7 standard errors away), which the test checks too.
"""
from math import comb

import numpy as np

import oracle
from combine_moe_pw_b200 import synth


def exact_expected_drop_rate(w: synth.Workload, C_s: int) -> float:
    E, k, P = w.E, w.k, w.P
    T_s = w.T // w.R
    px = np.array([comb(P, x) * comb(E - P, k - x) for x in range(min(k, P) + 1)], dtype=float)
    px /= comb(E, k)
    law = np.array([1.0])
    for _ in range(T_s):
        law = np.convolve(law, px)
    n = np.arange(law.size)
    per_pool = float((law * np.maximum(n - C_s, 0)).sum())
    n_pools = w.R * w.R * w.W
    return n_pools * per_pool / (w.T * w.k)


def test_law_of_one_token_sums_to_one_and_has_the_right_mean():
    w = synth.WORKLOADS["tiny"]
    E, k, P = w.E, w.k, w.P
    px = [comb(P, x) * comb(E - P, k - x) / comb(E, k) for x in range(min(k, P) + 1)]
    assert abs(sum(px) - 1.0) < 1e-12
    assert abs(sum(x * p for x, p in enumerate(px)) - k * P / E) < 1e-12


def test_sender_drop_rate_matches_the_exact_expectation():
    base = synth.WORKLOADS["tiny"]  # 8 ranks x 6 experts, top-8, 2048 tokens, iid logits
    assert base.logit_kind == synth.LOGIT_IID
    C_s, _ = oracle.capacity(base.T, base.T // base.R, base.E, base.k, base.P,
                             base.cf_send_pct, base.cf_recv_pct)
    expected = exact_expected_drop_rate(base, C_s)
    rates = []
    for seed in range(48):
        w = base.with_(seed=100 + seed)
        r = oracle.run_headers(w, synth.logits(w))
        rates.append(r["sender_dropped"] / (w.T * w.k))
    rates = np.array(rates)
    mean, se = rates.mean(), rates.std(ddof=1) / np.sqrt(rates.size)
    assert 0.003 < expected < 0.02  # a regime where drops happen but are rare
    tol = 4 * se + 1e-4
    assert abs(mean - expected) <= tol, (mean, se, expected)
    # the same data tell a capacity one slot off apart
    for off in (-1, 1):
        assert abs(mean - exact_expected_drop_rate(base, C_s + off)) > tol, off


def test_tighter_factor_drops_more_in_expectation_and_in_the_oracle():
    base = synth.WORKLOADS["tiny"].with_(cf_send_pct=100, cf_recv_pct=0)
    C_s, _ = oracle.capacity(base.T, base.T // base.R, base.E, base.k, base.P, 100, 0)
    expected = exact_expected_drop_rate(base, C_s)
    rates = []
    for seed in range(24):
        w = base.with_(seed=200 + seed)
        r = oracle.run_headers(w, synth.logits(w))
        rates.append(r["sender_dropped"] / (w.T * w.k))
    rates = np.array(rates)
    mean, se = rates.mean(), rates.std(ddof=1) / np.sqrt(rates.size)
    assert expected > exact_expected_drop_rate(synth.WORKLOADS["tiny"], C_s + 9)
    assert abs(mean - expected) <= 4 * se + 1e-4, (mean, se, expected)
