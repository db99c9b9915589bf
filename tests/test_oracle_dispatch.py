"""Pins for the oracle's sender assignment, pack and receiver bucketing.

Method ("Marin 开始公开训练 535B 参数 MoE 模型", section 二): one fixed pool per
(source, destination) and wave, the expert id packed with the row, sender cap
1.10 per source->destination pool, receiver cap 1.15 per local expert, drops
counted apart.  Readings: contiguous expert placement, wave w = local experts
{2w, 2w+1}, first-come order (token, rank-in-top-k) at the sender and
(source, slot) at the receiver.

Pins: capacities worked by hand (golden fixture), O(n^2) brute-force ranks
written from the definition, closed-form routing patterns, invariants and the
R=1/W=1 special case (plain first-come capacity routing).
"""
import json
import os

import numpy as np
import pytest

import oracle
from combine_moe_pw_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_pages_constants_fixture():
    c = json.load(open(os.path.join(GOLDEN, "pages_constants.json")))
    w = synth.WORKLOADS["rack"]
    assert w.E == c["routed_experts"] == c["ep_ranks"] * c["experts_per_rank"]
    assert w.k == c["experts_per_token"]
    assert w.D == c["latent_width"] == c["model_width"] // 2
    assert w.R == c["ep_ranks"] and w.L == c["experts_per_rank"] and w.W == c["waves"]
    assert w.P * w.W == w.L
    assert w.cf_send_pct == round(100 * c["cf_send"]) and w.cf_recv_pct == round(100 * c["cf_recv"])


@pytest.mark.parametrize("case", json.load(open(os.path.join(GOLDEN, "capacities.json")))["cases"],
                         ids=lambda c: c["name"])
def test_capacity_golden(case):
    T_s = case["T"] // case["R"]
    cs, cr = oracle.capacity(case["T"], T_s, case["E"], case["k"], case["P"],
                             case["cf_send_pct"], case["cf_recv_pct"])
    assert (cs, cr) == (case["C_s"], case["C_r"])


def _geom(T, R, L, W, P, k, D, cf_s=110, cf_r=115):
    E = R * L
    T_s = T // R
    cs, cr = oracle.capacity(T, T_s, E, k, P, cf_s, cf_r)
    return oracle.Geom(T=T, T_s=T_s, R=R, L=L, W=W, P=P, k=k, D=D, C_s=cs, C_r=cr)


def _random_idx(rng, T, E, k, skew=0.0):
    """k distinct experts per token; ``skew`` > 0 concentrates on low ids."""
    pref = rng.standard_normal((T, E)) - skew * np.log1p(np.arange(E))
    return np.argsort(-pref, axis=1, kind="stable")[:, :k].astype(np.int32)


def _brute_sender(g, idx):
    """Slot of (t, j) = number of earlier (t', j') of the same source in the
    same pool (O(n^2)); kept iff below C_s."""
    T, k = idx.shape
    pool_of = lambda e: (e // g.L, (e % g.L) // g.P)
    slot_map = np.full((T, k), -1, np.int64)
    flat = [(t, j) for t in range(T) for j in range(k)]
    for a, (t, j) in enumerate(flat):
        s = t // g.T_s
        d, w = pool_of(int(idx[t, j]))
        rank = sum(1 for (t2, j2) in flat[:a]
                   if t2 // g.T_s == s and pool_of(int(idx[t2, j2])) == (d, w))
        if rank < g.C_s:
            slot_map[t, j] = ((s * g.R + d) * g.W + w) * g.C_s + rank
    return slot_map


@pytest.mark.parametrize("skew", [0.0, 1.5])
def test_sender_assignment_brute_force(skew):
    rng = np.random.default_rng(11)
    g = _geom(T=96, R=4, L=6, W=3, P=2, k=4, D=8)
    idx = _random_idx(rng, g.T, g.E, g.k, skew)
    slot_map, occ, slot_tok, dropped = oracle.assign_pooled(g, idx)
    ref = _brute_sender(g, idx)
    np.testing.assert_array_equal(slot_map, ref)
    assert dropped == int((ref < 0).sum())
    if skew > 0:
        assert dropped > 0  # the case exercises the cap
    # occupancy = kept rows per pool, slot_tok its inverse
    for p in range(g.n_pools):
        kept = ref[(ref >= p * g.C_s) & (ref < (p + 1) * g.C_s)]
        assert occ.reshape(-1)[p] == kept.size
    for t in range(g.T):
        for j in range(g.k):
            if slot_map[t, j] >= 0:
                assert slot_tok[slot_map[t, j]] == t


def test_closed_form_every_token_picks_experts_0_to_7(tiny_inputs):
    """Every token picks experts 0..7: experts 0..5 live on destination 0 (waves
    0,1,2 with two experts each) and 6,7 on destination 1 wave 0.  Each of those
    four pools per source receives 2*T_s rows in (t, j) order; the first C_s are
    kept, so slots hold tokens 0..ceil(C_s/2)-1 of the shard."""
    w = synth.WORKLOADS["tiny"]
    g = oracle.geom_for(w)
    lg = np.full((w.T, w.E), -1.0, np.float32)
    lg[:, :8] = np.linspace(8.0, 1.0, 8, dtype=np.float32)
    idx, _ = oracle.route(g, lg)
    np.testing.assert_array_equal(idx, np.tile(np.arange(8), (w.T, 1)))
    slot_map, occ, slot_tok, dropped = oracle.assign_pooled(g, idx)
    per_pool = min(2 * g.T_s, g.C_s)
    assert dropped == w.R * 4 * (2 * g.T_s - per_pool)
    occ = occ.reshape(w.R, w.R, w.W)
    for s in range(w.R):
        assert occ[s, 0, 0] == occ[s, 0, 1] == occ[s, 0, 2] == occ[s, 1, 0] == per_pool
        assert occ[s].sum() == 4 * per_pool
        for (d, ww) in [(0, 0), (0, 1), (0, 2), (1, 0)]:
            base = ((s * w.R + d) * w.W + ww) * g.C_s
            toks = slot_tok[base:base + per_pool]
            np.testing.assert_array_equal(toks, s * g.T_s + np.arange(per_pool) // 2)
    # receiver: each expert gets per_pool/2 rows from every source
    pool_x, pool_hdr = oracle.pack(g, g.n_slots, synth.x_bf16(w), idx, slot_map)
    recv_row, bucket_slot, arrivals, bucket_cnt, rdrop = oracle.bucket(g, pool_hdr, occ)
    expect = np.zeros(w.E, np.int64)
    expect[:8] = w.R * ((per_pool + 1) // 2)  # even c -> first expert of the wave
    expect[1:6:2] = expect[7] = w.R * (per_pool // 2)
    np.testing.assert_array_equal(arrivals, expect)
    np.testing.assert_array_equal(bucket_cnt, np.minimum(expect, g.C_r))
    assert rdrop == int(np.maximum(expect - g.C_r, 0).sum())


def test_round_robin_has_no_drops():
    """Token t picks experts (8t + i) mod E: every pool and expert gets exactly
    its mean load, so capacities >= mean drop nothing."""
    g = _geom(T=2304, R=8, L=6, W=3, P=2, k=8, D=8, cf_s=100, cf_r=100)
    t = np.arange(g.T)[:, None]
    idx = ((8 * t + np.arange(8)[None, :]) % g.E).astype(np.int32)
    slot_map, occ, _, dropped = oracle.assign_pooled(g, idx)
    assert dropped == 0 and np.all(slot_map >= 0)
    pool_x, pool_hdr = oracle.pack(g, g.n_slots, np.zeros((g.T, 8), np.uint16), idx, slot_map)
    _, _, arrivals, bucket_cnt, rdrop = oracle.bucket(g, pool_hdr, occ)
    assert rdrop == 0 and np.all(arrivals == g.T * g.k // g.E)


def test_single_pool_reduces_to_first_come():
    """R = 1, W = 1, P = L: one pool per source; the kept assignments are the
    first C_s in (t, j) order and the rest are dropped."""
    rng = np.random.default_rng(3)
    g = _geom(T=200, R=1, L=16, W=1, P=16, k=4, D=8, cf_s=50, cf_r=0)
    idx = _random_idx(rng, g.T, g.E, g.k)
    slot_map, occ, _, dropped = oracle.assign_pooled(g, idx)
    flat = slot_map.reshape(-1)
    assert g.C_s == 400  # ceil(0.5 * 200*4*16/16)
    np.testing.assert_array_equal(flat[:g.C_s], np.arange(g.C_s))
    assert np.all(flat[g.C_s:] == -1) and dropped == g.T * g.k - g.C_s


def _brute_receiver(g, pool_hdr, occ):
    """Row of a slot in its expert's bucket = number of earlier slots in the
    (source, position) walk of the same (d, w) with the same expert (O(n^2))."""
    occ = occ.reshape(g.n_src, g.R, g.W)
    recv = np.full(g.n_slots, -1, np.int64)
    for d in range(g.R):
        for w in range(g.W):
            walk = [((s * g.R + d) * g.W + w) * g.C_s + c
                    for s in range(g.n_src) for c in range(occ[s, d, w])]
            for a, slot in enumerate(walk):
                r = sum(1 for q in walk[:a] if pool_hdr[q] == pool_hdr[slot])
                if r < g.C_r:
                    recv[slot] = r
    return recv


def test_receiver_bucketing_brute_force():
    rng = np.random.default_rng(5)
    g = _geom(T=192, R=4, L=6, W=3, P=2, k=4, D=8, cf_s=200, cf_r=90)
    idx = _random_idx(rng, g.T, g.E, g.k, skew=0.8)
    slot_map, occ, _, _ = oracle.assign_pooled(g, idx)
    x = rng.integers(0, 1 << 16, (g.T, g.D), dtype=np.uint16)
    pool_x, pool_hdr = oracle.pack(g, g.n_slots, x, idx, slot_map)
    recv_row, bucket_slot, arrivals, bucket_cnt, rdrop = oracle.bucket(g, pool_hdr, occ)
    ref = _brute_receiver(g, pool_hdr, occ)
    np.testing.assert_array_equal(recv_row, ref)
    assert rdrop > 0
    assert rdrop == int(((pool_hdr >= 0) & (ref < 0)).sum())


def test_invariants_tiny(tiny_inputs, tiny_oracle):
    w, lg, x, _ = tiny_inputs
    r = tiny_oracle
    g = r["geom"]
    T, k = w.T, w.k
    # kept + sender drops + receiver drops = T*k
    assert r["kept"] + r["sender_dropped"] + r["receiver_dropped"] == T * k
    assert int((r["slot_map"] < 0).sum()) == r["sender_dropped"]
    # occupancy never above C_s = ceil(cf * expected); buckets never above C_r
    assert r["occ"].max() <= g.C_s and r["bucket_cnt"].max() <= g.C_r
    # each kept pool row is x[t] bit for bit; empty slots are zero with header -1
    for t in range(T):
        for j in range(k):
            s = r["slot_map"][t, j]
            if s >= 0:
                np.testing.assert_array_equal(r["pool_x"][s], x[t])
                assert r["pool_hdr"][s] == r["idx"][t, j]
    empty = r["slot_tok"] < 0
    assert np.all(r["pool_hdr"][empty] == -1) and not r["pool_x"][empty].any()
    # header multiset = expert ids of the kept (t, j)
    kept_e = r["idx"][r["slot_map"] >= 0]
    np.testing.assert_array_equal(np.bincount(r["pool_hdr"][~empty], minlength=w.E),
                                  np.bincount(kept_e, minlength=w.E))
    # recv_row and bucket_slot are inverse maps
    bs = r["bucket_slot"]
    for e in range(w.E):
        for q in range(g.C_r):
            slot = bs[e, q]
            if q < r["bucket_cnt"][e]:
                assert slot >= 0 and r["recv_row"][slot] == q and r["pool_hdr"][slot] == e
            else:
                assert slot == -1
    assert int((r["recv_row"] >= 0).sum()) == r["kept"]
    # a pool's header only names experts of its (destination, wave)
    hdr = r["pool_hdr"].reshape(g.n_src, w.R, w.W, g.C_s)
    for d in range(w.R):
        for ww in range(w.W):
            h = hdr[:, d, ww][hdr[:, d, ww] >= 0]
            assert set(np.unique(h)) <= {d * w.L + ww * w.P + p for p in range(w.P)}


def test_drops_monotone_in_capacity_factor(tiny_inputs):
    w, lg, _, _ = tiny_inputs
    prev = None
    for cf in [80, 95, 110, 125, 150, 200, 0]:
        g = oracle.geom_for(w.with_(cf_send_pct=cf, cf_recv_pct=cf))
        idx, _ = oracle.route(g, lg)
        slot_map, occ, _, sd = oracle.assign_pooled(g, idx)
        pool_x, hdr = oracle.pack(g, g.n_slots, np.zeros((w.T, 8), np.uint16), idx, slot_map)
        *_, rd = oracle.bucket(g, hdr, occ)
        total = sd + rd
        if prev is not None:
            assert total <= prev
        prev = total
    assert prev == 0  # unbounded capacity drops nothing


def test_ragged_assignment():
    """Dropless mode: rows grouped by expert in ascending expert order, token
    order inside an expert, nothing dropped."""
    rng = np.random.default_rng(9)
    g = _geom(T=300, R=4, L=6, W=3, P=2, k=8, D=8, cf_s=0, cf_r=0)
    idx = _random_idx(rng, g.T, g.E, g.k, skew=1.0)
    slot_map, row_off, row_cnt, slot_tok = oracle.assign_ragged(g, idx)
    np.testing.assert_array_equal(row_cnt, np.bincount(idx.reshape(-1), minlength=g.E))
    np.testing.assert_array_equal(row_off, np.concatenate([[0], np.cumsum(row_cnt)]))
    # rows sorted by (expert, token): compare with a library stable sort
    a = np.arange(g.T * g.k)
    order = np.lexsort((a // g.k, idx.reshape(-1)))
    expect = np.empty_like(a)
    expect[order] = np.arange(a.size)
    np.testing.assert_array_equal(slot_map.reshape(-1), expect)
    np.testing.assert_array_equal(slot_tok, (a // g.k)[order])
