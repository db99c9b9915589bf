"""Pins for the oracle's header-only path and its dropless receiver.

The full-size GPU parity tests take their expected headers, receiver rows,
buckets and drop counts from ``oracle.run_headers``, which builds the pool
headers with ``orc_pack_headers`` instead of the full ``orc_pack`` (the pools
of a full batch are too large for the host).  These tests tie the two
together on every small geometry the GPU tests use, so the header path cannot
drift from the pinned full path.

Dropless mode ("Marin 开始公开训练 535B 参数 MoE 模型", section 四: a dropless
ragged all-to-all is the listed alternative): every row reaches its expert,
and the receiver numbers the arrivals of each expert in the order the rows
arrive.  ``orc_bucket_ragged`` is pinned here by an O(n^2) count written from
that definition and by the grouped layout's closed form (row id minus the
expert's first row).
"""
import numpy as np
import pytest

import oracle
from combine_moe_pw_b200 import synth
from fuzz_cases import random_workload

N_FUZZ = 24

CASES = {
    "tiny": synth.WORKLOADS["tiny"],
    "tiny_ragged": synth.WORKLOADS["tiny"].with_(mode=synth.MODE_RAGGED, cf_send_pct=0,
                                                 cf_recv_pct=0),
    "tiny_tight": synth.WORKLOADS["tiny"].with_(cf_send_pct=60, cf_recv_pct=70),
    **{f"fuzz{i}": random_workload(i) for i in range(N_FUZZ)},
}

INTEGER_KEYS = ["idx", "slot_map", "slot_tok", "pool_hdr", "recv_row", "arrivals", "bucket_cnt"]


def check_headers_equal_full(w):
    lg, x, s = synth.logits(w), synth.x_bf16(w), synth.scales(w)
    full = oracle.run(w, lg, x, s)
    hdr = oracle.run_headers(w, lg)
    keys = INTEGER_KEYS + (["occ", "bucket_slot"] if w.mode == synth.MODE_POOLED
                           else ["row_off", "row_cnt"])
    for key in keys:
        np.testing.assert_array_equal(hdr[key], full[key], err_msg=key)
    np.testing.assert_array_equal(hdr["gates"], full["gates"])
    for key in ["sender_dropped", "receiver_dropped", "kept"]:
        assert hdr[key] == full[key], key
    assert hdr["kept"] + hdr["sender_dropped"] + hdr["receiver_dropped"] == w.T * w.k


@pytest.mark.parametrize("name", list(CASES))
def test_run_headers_equals_run(name):
    check_headers_equal_full(CASES[name])


def _brute_ragged_rows(row_hdr):
    """Row of arrival q in its expert's bucket = earlier arrivals with the
    same header (O(n^2)); -1 for a row without a header."""
    out = np.full(row_hdr.size, -1, np.int64)
    for q in range(row_hdr.size):
        if row_hdr[q] >= 0:
            out[q] = int((row_hdr[:q] == row_hdr[q]).sum())
    return out


def _ragged_geom(T, R, L, W, P, k):
    return oracle.Geom(T=T, T_s=T // R, R=R, L=L, W=W, P=P, k=k, D=8, C_s=T // R * min(k, P),
                       C_r=T)


def test_ragged_receiver_rows_brute_force():
    rng = np.random.default_rng(21)
    g = _ragged_geom(T=160, R=4, L=6, W=3, P=2, k=6)
    pref = rng.standard_normal((g.T, g.E)) - 1.2 * np.log1p(np.arange(g.E))
    idx = np.argsort(-pref, axis=1, kind="stable")[:, :g.k].astype(np.int32)
    slot_map, row_off, row_cnt, _ = oracle.assign_ragged(g, idx)
    hdr = oracle.pack_headers(g, g.T * g.k, idx, slot_map)
    recv_row, arrivals, bucket_cnt = oracle.bucket_ragged(g, hdr)
    np.testing.assert_array_equal(recv_row, _brute_ragged_rows(hdr))
    # rows are grouped by expert, so a row's place is its distance from the
    # expert's first row
    q = np.arange(g.T * g.k)
    np.testing.assert_array_equal(recv_row, q - row_off[hdr])
    np.testing.assert_array_equal(arrivals, np.bincount(idx.reshape(-1), minlength=g.E))
    np.testing.assert_array_equal(bucket_cnt, arrivals)
    assert oracle.kept(g, bucket_cnt) == g.T * g.k


def test_ragged_receiver_rows_any_order():
    """The receiver's numbering is defined for rows in any arrival order, not
    only the grouped one: shuffled headers (with a few empty rows) against
    the brute force."""
    rng = np.random.default_rng(4)
    g = _ragged_geom(T=64, R=2, L=4, W=2, P=2, k=3)
    hdr = rng.integers(-1, g.E, 200).astype(np.int32)
    recv_row, arrivals, _ = oracle.bucket_ragged(g, hdr)
    np.testing.assert_array_equal(recv_row, _brute_ragged_rows(hdr))
    np.testing.assert_array_equal(arrivals, np.bincount(hdr[hdr >= 0], minlength=g.E))
