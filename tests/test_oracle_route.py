"""Pins for the oracle's route stage (top-k selection + softmax gates).

The router picks k of E experts per token ("Marin 开始公开训练 535B 参数 MoE 模型",
section 二); ties go to the lower expert index and gates are the softmax over
the chosen logits (readings).  The oracle's selection is held against a full
sort (numpy lexsort), its gates against torch.softmax, and both against closed
forms.
"""
import numpy as np
import pytest
import torch

import oracle


def _geom(T, E, k, R=None):
    R = R or 1
    return oracle.Geom(T=T, T_s=T, R=R, L=E // R, W=1, P=E // R, k=k, D=8, C_s=1, C_r=1)


def _sort_topk(lg, k):
    """Brute force: full stable sort by (value desc, index asc)."""
    T, E = lg.shape
    out = np.empty((T, k), np.int32)
    for t in range(T):
        # lexsort sorts by last key first: primary = -value, secondary = index
        order = np.lexsort((np.arange(E), -lg[t].astype(np.float64)))
        out[t] = order[:k]
    return out


@pytest.mark.parametrize("E,k", [(48, 8), (384, 8), (64, 1), (16, 16), (40, 5)])
def test_topk_matches_full_sort(E, k):
    rng = np.random.default_rng(E * 100 + k)
    T = 300
    lg = rng.standard_normal((T, E)).astype(np.float32)
    # plant many ties: quantise half the rows to a coarse grid
    lg[::2] = np.round(lg[::2] * 2) / 2
    idx, gates = oracle.route(_geom(T, E, k), lg)
    np.testing.assert_array_equal(idx, _sort_topk(lg, k))


def test_signed_zero_ties_to_lower_index():
    E, k = 16, 8
    lg = np.full((1, E), -1.0, np.float32)
    lg[0, 3] = -0.0
    lg[0, 1] = 0.0
    lg[0, 9] = -0.0
    idx, _ = oracle.route(_geom(1, E, k), lg)
    # -0.0 == +0.0: the three zeros tie and come out in index order
    assert list(idx[0, :3]) == [1, 3, 9]
    assert list(idx[0, 3:]) == [0, 2, 4, 5, 6]


def test_all_equal_logits_closed_form():
    """All-equal logits: indices 0..k-1, every gate exp(0)/k = 1/8 exactly."""
    E, k, T = 384, 8, 5
    lg = np.full((T, E), 0.37, np.float32)
    idx, gates = oracle.route(_geom(T, E, k), lg)
    np.testing.assert_array_equal(idx, np.tile(np.arange(k, dtype=np.int32), (T, 1)))
    assert np.all(gates == 0.125)


def test_k1_gate_is_one():
    rng = np.random.default_rng(7)
    lg = rng.standard_normal((50, 48)).astype(np.float32)
    idx, gates = oracle.route(_geom(50, 48, 1), lg)
    np.testing.assert_array_equal(idx[:, 0], np.argmax(lg, axis=1))
    assert np.all(gates == 1.0)


def test_gates_match_library_softmax(tiny_inputs):
    w, lg, _, _ = tiny_inputs
    g = oracle.geom_for(w)
    idx, gates = oracle.route(g, lg)
    sel = np.take_along_axis(lg, idx, axis=1).astype(np.float64)
    ref = torch.softmax(torch.from_numpy(sel), dim=1).numpy()
    np.testing.assert_allclose(gates, ref, rtol=1e-14, atol=0)
    np.testing.assert_allclose(gates.sum(axis=1), 1.0, rtol=0, atol=1e-14)
    # gates follow the descending order of the logits
    assert np.all(np.diff(gates, axis=1) <= 0)


def test_extreme_spread_gates():
    """A logit far below the top gives a gate of exp(-delta)/sum, not NaN."""
    lg = np.zeros((1, 16), np.float32)
    lg[0, :8] = [30.0, 0.0, -5.0, -10.0, -20.0, -40.0, -80.0, -100.0]
    lg[0, 8:] = -1000.0
    idx, gates = oracle.route(_geom(1, 16, 8), lg)
    np.testing.assert_array_equal(idx[0], np.arange(8))
    ex = np.exp(np.array([0.0, -30.0, -35.0, -40.0, -50.0, -70.0, -110.0, -130.0]))
    np.testing.assert_allclose(gates[0], ex / ex.sum(), rtol=1e-14)
