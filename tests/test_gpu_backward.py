"""GPU backward (combine backward, expert-op backward, pack backward) against
the CPU oracle, through the C ABI.

Tolerances (derived from the arithmetic):
- dgates: each lane accumulates D/32 products with fmaf, then a 5-level xor
  tree: |err| <= (D/32 + 5) * 2^-24 * sum_i |dout_i y_i|  -> 1e-5 of that sum
  covers D <= 3072.
- dlogits: g_j (dgate_j - sum_i g_i dgate_i) with fp32 gates (1e-6) and the
  dgate bound -> 2e-5 * g_j * (M_j + sum_i g_i M_i), M = sum_i |dout_i y_i|.
- gradient rows (bf16): the fp32 product g_j * dout uses the GPU's gate, which
  can differ from the oracle's by a few fp32 ulp, so a row element may round
  to the neighbouring bf16 value: |err| <= 1 bf16 ulp, on at most 0.1% of the
  elements or 2 of them, whichever is more (each element flips independently
  with a tiny probability, so a small case may show one or two).
- dx: a sum of those bf16 rows (scaled once more): |err| <= 2^-7 * sum of
  |terms|, and all but a tiny fraction within 1e-6 of that sum.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_moe_pw_b200 import moe_pw as mp
from combine_moe_pw_b200 import synth

pytestmark = pytest.mark.gpu


def _f32(u16):
    return (u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _ulp_bf16(v):
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, 2.0 ** (e - 7), 2.0 ** -133)


def run_both(w):
    lg, x, s, dout = synth.logits(w), synth.x_bf16(w), synth.scales(w), synth.dout(w)
    b = mp.Buffers(mp.Config.from_workload(w))
    b.logits.copy_(torch.from_numpy(lg))
    b.x.copy_(torch.from_numpy(x.view(np.int16)))
    b.scale.copy_(torch.from_numpy(s))
    b.run_step()
    b.alloc_backward()
    b.dout.copy_(torch.from_numpy(dout))
    b.run_backward()
    st = b.stats(raise_on_device_error=False)
    torch.cuda.synchronize()
    r = oracle.run(w, lg, x, s)
    ob = oracle.run_backward(w, r, dout, s)
    return b, st, r, ob, dout


def check_backward(w, b, st, r, ob, dout):
    assert st.error == 0
    g = r["gates"]
    sm = r["slot_map"]
    keep = sm >= 0
    keep &= r["ret_hdr"][np.where(keep, sm, 0)] >= 0
    rows = np.where(keep[:, :, None], _f32(r["ret_x"][np.where(keep, sm, 0)]), 0.0)
    M = (np.abs(dout.astype(np.float64))[:, None, :] * np.abs(rows)).sum(axis=2)
    # dgates
    dg = b.dgates.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(dg - ob["dgate"]) <= 1e-5 * M + 1e-30)
    # dlogits (dense rows: zeros off the chosen experts)
    dl = b.dlogits.cpu().numpy().astype(np.float64)
    idx = r["idx"].astype(np.int64)
    tol = 2e-5 * g * (M + (g * M).sum(axis=1, keepdims=True)) + 1e-30
    assert np.all(np.abs(np.take_along_axis(dl, idx, 1)
                         - np.take_along_axis(ob["dlogits"], idx, 1)) <= tol)
    off = np.ones_like(dl, bool)
    np.put_along_axis(off, idx, False, axis=1)
    assert not dl[off].any()
    # gradient pool: zero where nothing survived, else within one bf16 ulp
    d_ret = b.d_ret.cpu().numpy().view(np.uint16)
    live = r["ret_hdr"] >= 0
    assert not d_ret[~live].any()
    got, ref = _f32(d_ret[live]), _f32(ob["d_ret"][live])
    assert np.all(np.abs(got - ref) <= _ulp_bf16(ref))
    assert (got != ref).sum() <= max(1e-3 * got.size, 2)
    # expert backward rows
    d_pool = b.d_pool.cpu().numpy().view(np.uint16)
    assert not d_pool[~live].any()
    gp, rp = _f32(d_pool[live]), _f32(ob["d_pool"][live])
    assert np.all(np.abs(gp - rp) <= 2 * _ulp_bf16(rp))
    # dx
    dx = b.dx.cpu().numpy().astype(np.float64)
    terms = np.where(keep[:, :, None], np.abs(_f32(ob["d_pool"][np.where(keep, sm, 0)])), 0.0)
    mag = terms.sum(axis=1)
    err = np.abs(dx - ob["dx"])
    assert np.all(err <= 2.0 ** -7 * mag + 1e-30)
    assert (err > 1e-6 * mag + 1e-30).sum() <= max(1e-3 * err.size, 2)


CASES = {
    "tiny": synth.WORKLOADS["tiny"],
    "tiny_tight": synth.WORKLOADS["tiny"].with_(cf_send_pct=60, cf_recv_pct=70),
    "tiny_ragged": synth.WORKLOADS["tiny"].with_(mode=1, cf_send_pct=0, cf_recv_pct=0,
                                                 logit_kind=synth.LOGIT_ZIPF),
    "k1": synth.WORKLOADS["tiny"].with_(k=1),
    "k16": synth.WORKLOADS["tiny"].with_(k=16),
    "k32": synth.WORKLOADS["tiny"].with_(k=32),
    "E8_ragged_tail": synth.Workload("E8", T=6 * 37, R=1, L=8, W=4, P=2, k=2, D=24, seq_len=37,
                                     logit_kind=synth.LOGIT_IID),
    "pages_ranks_small": synth.Workload("pages_ranks_small", T=64 * 64, R=64, L=6, W=3, P=2, k=8,
                                        D=512, seq_len=1024, logit_kind=synth.LOGIT_SEQBIAS),
}


@pytest.mark.parametrize("name", list(CASES))
def test_backward_parity(name):
    w = CASES[name]
    b, st, r, ob, dout = run_both(w)
    check_backward(w, b, st, r, ob, dout)


def test_backward_deterministic():
    w = CASES["pages_ranks_small"]
    b1, *_ = run_both(w)
    b2, *_ = run_both(w)
    for n in ["d_ret", "dgates", "dlogits", "d_pool", "dx"]:
        assert torch.equal(getattr(b1, n), getattr(b2, n)), n


@pytest.mark.parametrize("name", ["rack", "ragged"])
def test_backward_full_size_sampled(name):
    """The pages' shapes in the bench's launch configuration; the oracle's
    integer path in full, the backward on sampled tokens."""
    w = synth.WORKLOADS[name]
    lg, x, s, dout = synth.logits(w), synth.x_bf16(w), synth.scales(w), synth.dout(w)
    b = mp.Buffers(mp.Config.from_workload(w))
    b.logits.copy_(torch.from_numpy(lg))
    b.x.copy_(torch.from_numpy(x.view(np.int16)))
    b.scale.copy_(torch.from_numpy(s))
    b.run_step()
    b.alloc_backward()
    b.dout.copy_(torch.from_numpy(dout))
    b.run_backward()
    assert b.stats(raise_on_device_error=False).error == 0
    r = oracle.run_headers(w, lg)
    rng = np.random.default_rng(3)
    toks = np.unique(np.concatenate([rng.integers(0, w.T, 512), [0, w.T - 1]]))
    d_ret, dgate, dlog, dx = oracle.backward_tokens(r["geom"], x, r["idx"], r["gates"],
                                                    r["slot_map"], r["recv_row"], s, dout, toks)
    tt = torch.from_numpy(toks).cuda()
    sm = r["slot_map"][toks]
    live = (sm >= 0) & (r["recv_row"][np.where(sm >= 0, sm, 0)] >= 0)
    # y rows and magnitudes for the tolerances
    e = r["idx"][toks]
    y = _f32(oracle.expert_product(np.repeat(s[e].reshape(-1, 1), w.D, axis=1),
                                   np.repeat(x[toks], w.k, axis=0))).reshape(toks.size, w.k, w.D)
    M = (np.abs(dout[toks].astype(np.float64))[:, None, :] * np.abs(y)).sum(axis=2) * live
    g = r["gates"][toks]
    dg = b.dgates[tt].cpu().numpy().astype(np.float64)
    assert np.all(np.abs(dg - dgate) <= 1e-5 * M + 1e-30)
    dl = b.dlogits[tt].cpu().numpy().astype(np.float64)
    ii = e.astype(np.int64)
    tol = 2e-5 * g * (M + (g * M).sum(axis=1, keepdims=True)) + 1e-30
    assert np.all(np.abs(np.take_along_axis(dl, ii, 1) - np.take_along_axis(dlog, ii, 1)) <= tol)
    off = np.ones_like(dl, bool)
    np.put_along_axis(off, ii, False, axis=1)
    assert not dl[off].any()
    slots = torch.from_numpy(np.where(live, sm, 0).reshape(-1).astype(np.int64)).cuda()
    got = _f32(b.d_ret.index_select(0, slots).cpu().numpy().view(np.uint16)).reshape(
        toks.size, w.k, w.D)
    ref = _f32(d_ret)
    assert np.all(np.abs(got - ref)[live] <= _ulp_bf16(ref)[live])
    gdx = b.dx[tt].cpu().numpy().astype(np.float64)
    mag = (np.abs(ref) * s[e][:, :, None] * live[:, :, None]).sum(axis=1) * (1 + 2.0 ** -7)
    err = np.abs(gdx - dx)
    assert np.all(err <= 2.0 ** -7 * mag + 1e-30)
    assert (err > 1e-6 * mag + 1e-30).sum() <= max(1e-3 * err.size, 2)
    del b
    torch.cuda.empty_cache()
