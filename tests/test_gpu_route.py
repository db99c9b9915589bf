"""The route kernel alone against the oracle's route, on shapes the
end-to-end parity cases do not reach: 128, 256, 320 and 384 experts, odd
token counts, a single token, k = 6 with 384 experts, many exact ties (ranked
among the candidates, or, with more than 32 logits at or above the
threshold, by the exact rounds), all-equal logits, signed zeros and masked
(-inf) experts.  Ids bit for bit,
gates within the gate tolerance of the parity tests.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_moe_pw_b200 import moe_pw as mp
from combine_moe_pw_b200 import synth
from test_gpu_parity import _np, check_gates

pytestmark = pytest.mark.gpu

SHAPES = {
    # E = R * L; T = R * seq_len, odd where R is odd
    "E384_odd_T": synth.Workload("E384", T=3 * 333, R=3, L=128, W=4, P=32, k=8, D=8,
                                 seq_len=333, logit_kind=synth.LOGIT_SEQBIAS),
    "E384_zipf": synth.Workload("E384z", T=64 * 40, R=64, L=6, W=3, P=2, k=8, D=8,
                                seq_len=40, logit_kind=synth.LOGIT_ZIPF),
    "E256_odd_T": synth.Workload("E256", T=777, R=1, L=256, W=8, P=32, k=8, D=8, seq_len=777,
                                 logit_kind=synth.LOGIT_IID),
    "E128_odd_T": synth.Workload("E128", T=301, R=1, L=128, W=4, P=32, k=8, D=8, seq_len=301,
                                 logit_kind=synth.LOGIT_ZIPF),
    "one_token": synth.Workload("one", T=1, R=1, L=384, W=12, P=32, k=8, D=8, seq_len=1,
                                logit_kind=synth.LOGIT_IID),
    "E320": synth.Workload("E320", T=5 * 101, R=5, L=64, W=2, P=32, k=8, D=8, seq_len=101,
                           logit_kind=synth.LOGIT_IID),
    "E384_k6": synth.Workload("E384k6", T=3 * 111, R=3, L=128, W=4, P=32, k=6, D=8,
                              seq_len=111, logit_kind=synth.LOGIT_SEQBIAS),
}


def _route(w, lg):
    b = mp.Buffers(mp.Config.from_workload(w))
    b.logits.copy_(torch.from_numpy(lg))
    b.idx.fill_(-5)
    b.gates.fill_(float("nan"))
    b.route()
    torch.cuda.synchronize()
    idx, gates = oracle.route(oracle.geom_for(w), lg)
    np.testing.assert_array_equal(_np(b.idx), idx)
    check_gates(_np(b.gates), gates)
    return _np(b.idx), _np(b.gates)


@pytest.mark.parametrize("name", list(SHAPES))
def test_route_against_oracle(name):
    w = SHAPES[name]
    _route(w, synth.logits(w))


@pytest.mark.parametrize("grid", [0.5, 2.0])
@pytest.mark.parametrize("name", ["E384_odd_T", "E128_odd_T", "E320"])
def test_route_ties(name, grid):
    """Logits rounded to a grid, so many tie exactly.  On the 0.5 grid the
    ties fall among the ranked candidates (at most 32 logits at or above the
    threshold); on the 2.0 grid every such token of the 320- and 384-expert
    shapes, and about a third of the 128-expert one, has more than 32 and
    takes the exact rounds.  Every third token keeps its fine values, so a
    launch mixes both paths."""
    w = SHAPES[name]
    lg = synth.logits(w)
    q = (np.round(lg / grid) * grid).astype(np.float32)
    q[::3] = lg[::3]
    q[::7, 5] = -0.0
    q[::7, 9] = 0.0
    _route(w, q)


@pytest.mark.parametrize("name", ["E384_odd_T", "E256_odd_T"])
def test_route_all_equal_closed_form(name):
    w = SHAPES[name]
    lg = np.full((w.T, w.E), 0.25, np.float32)
    idx, gates = _route(w, lg)
    np.testing.assert_array_equal(idx, np.tile(np.arange(8, dtype=np.int32), (w.T, 1)))
    assert np.all(gates == np.float32(0.125))  # exp(0)/8 exactly


def test_route_masked_experts():
    """A third of the experts masked with -inf in every row: none is chosen."""
    w = SHAPES["E384_odd_T"]
    lg = synth.logits(w)
    rng = np.random.default_rng(5)
    for t in range(w.T):
        lg[t, rng.choice(w.E, w.E // 3, replace=False)] = -np.inf
    idx, _ = _route(w, lg)
    assert np.isfinite(np.take_along_axis(lg, idx.astype(np.int64), axis=1)).all()
