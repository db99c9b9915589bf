"""Drop-rate study on the GPU: counts equal the oracle's on a sampled grid
point, drops never increase with the capacity factor, and longer sequences
(fewer per batch) drop more."""
import numpy as np
import pytest

import oracle
from combine_moe_pw_b200 import drop_study, synth

pytestmark = pytest.mark.gpu


def test_drop_study_trends_and_oracle_point():
    T = 65536
    rows = list(drop_study.study(T, [1024, 16384], [100, 110, 150, 0]))
    by = {(r["seq_len"], r["cf_send"]): r for r in rows}
    for L in (1024, 16384):
        totals = [by[(L, cf)]["drop_total"] for cf in (1.0, 1.1, 1.5)]
        assert totals[0] >= totals[1] >= totals[2]
        assert by[(L, 0.0)]["drop_total"] == 0.0  # unbounded factors drop nothing
        for cf in (1.0, 1.1, 1.5):
            r = by[(L, cf)]
            assert r["kept"] + r["sender_dropped"] + r["receiver_dropped"] == r["assignments"]
    assert by[(16384, 1.1)]["drop_total"] > by[(1024, 1.1)]["drop_total"]
    # the balance term is above 1 (skewed sequences) and the same for every factor
    for L in (1024, 16384):
        vals = {by[(L, cf)]["sequence_balance"] for cf in (1.0, 1.1, 1.5, 0.0)}
        assert len(vals) == 1 and vals.pop() > 1.0
    # one grid point against the oracle, bit for bit
    w = synth.WORKLOADS["rack"].with_(T=T, D=8, seq_len=16384, cf_send_pct=110, cf_recv_pct=115)
    r = oracle.run_headers(w, synth.logits(w))
    got = by[(16384, 1.1)]
    assert (got["sender_dropped"], got["receiver_dropped"], got["kept"]) == (
        r["sender_dropped"], r["receiver_dropped"], r["kept"])
