"""Pins for the oracle's backward (combine backward, expert-op backward, pack
transpose).

The forward is re-expressed in fp64 torch ops with the oracle's routing and
keep masks held fixed (top-k and the capacity drops are piecewise constant),
and torch.autograd differentiates it.  The oracle must agree: dlogits and the
gate gradients to double rounding, the bf16 gradient rows to bf16 rounding.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_moe_pw_b200 import synth


def _bf16_to_f64(a):
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@pytest.fixture(scope="module")
def case():
    w = synth.WORKLOADS["tiny"]
    lg, x, s = synth.logits(w), synth.x_bf16(w), synth.scales(w)
    r = oracle.run(w, lg, x, s)
    dout = synth.dout(w)
    b = oracle.run_backward(w, r, dout, s)
    return w, lg, x, s, r, dout, b


def _autograd(w, lg, x, s, r, dout):
    T, k, D, E = w.T, w.k, w.D, w.E
    idx = torch.from_numpy(r["idx"].astype(np.int64))
    sm = r["slot_map"]
    keep = (sm >= 0)
    keep &= r["ret_hdr"][np.where(keep, sm, 0)] >= 0
    keep_t = torch.from_numpy(keep.astype(np.float64))
    logits = torch.from_numpy(lg.astype(np.float64)).requires_grad_(True)
    xt = torch.from_numpy(_bf16_to_f64(x)).requires_grad_(True)
    sc = torch.from_numpy(s.astype(np.float64))
    sel = torch.gather(logits, 1, idx)
    g = torch.softmax(sel, dim=1)
    g.retain_grad()
    # returned rows: y_j = s_e * x_t for kept (t, j) (the stand-in op, unrounded)
    y = sc[idx][:, :, None] * xt[:, None, :]
    y.retain_grad()
    out = (keep_t[:, :, None] * g[:, :, None] * y).sum(dim=1)
    loss = (out * torch.from_numpy(dout.astype(np.float64))).sum()
    loss.backward()
    return logits.grad.numpy(), g.grad.numpy(), y.grad.numpy(), xt.grad.numpy(), keep


def test_backward_matches_autograd(case):
    w, lg, x, s, r, dout, b = case
    dlog_ref, dg_ref, dy_ref, dx_ref, keep = _autograd(w, lg, x, s, r, dout)
    # gate gradients: <dout, y_j>, the oracle's y_j being s_e*x rounded to bf16
    # (each term within 2^-9 relative of autograd's unrounded product)
    g = r["gates"]
    mag = np.abs(dout.astype(np.float64))[:, None, :] * np.abs(
        s[r["idx"]][:, :, None].astype(np.float64) * _bf16_to_f64(x)[:, None, :])
    dg_bound = 2.0 ** -8 * mag.sum(axis=2) * keep + 1e-30
    assert np.all(np.abs(b["dgate"] - np.where(keep, dg_ref, 0)) <= dg_bound)
    # dlogits: exact softmax backward given the oracle's own dgate ...
    dl = g * (b["dgate"] - (g * b["dgate"]).sum(axis=1, keepdims=True))
    expect = np.zeros_like(b["dlogits"])
    np.put_along_axis(expect, r["idx"].astype(np.int64), dl, axis=1)
    np.testing.assert_allclose(b["dlogits"], expect, rtol=1e-12, atol=1e-15)
    # ... and within the propagated dgate bound of autograd's
    dl_bound = g * (dg_bound + (g * dg_bound).sum(axis=1, keepdims=True))
    got_sel = np.take_along_axis(b["dlogits"], r["idx"].astype(np.int64), axis=1)
    ref_sel = np.take_along_axis(dlog_ref, r["idx"].astype(np.int64), axis=1)
    assert np.all(np.abs(got_sel - ref_sel) <= dl_bound * (1 + 1e-9) + 1e-15)
    off = np.ones_like(dlog_ref, bool)
    np.put_along_axis(off, r["idx"].astype(np.int64), False, axis=1)
    assert not b["dlogits"][off].any() and not dlog_ref[off].any()
    # gradient rows: bf16(g_j * dout) at the surviving slots
    sm = r["slot_map"]
    for t, j in zip(*np.nonzero(keep)):
        got = _bf16_to_f64(b["d_ret"][sm[t, j]])
        ref = dy_ref[t, j]
        assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-30)
    # dx: sum_j s_e g_j dout over surviving j, two bf16 roundings per term
    bound = 2.0 ** -7 * (np.abs(keep[:, :, None] * s[r["idx"]][:, :, None] * g[:, :, None]
                               * dout[:, None, :].astype(np.float64)).sum(axis=1)) + 1e-30
    assert np.all(np.abs(b["dx"] - dx_ref) <= bound)


def test_backward_with_exact_rows(case):
    """With autograd's y replaced by the oracle's returned bf16 rows, the gate
    gradients and dlogits agree to double rounding."""
    w, lg, x, s, r, dout, b = case
    idx = torch.from_numpy(r["idx"].astype(np.int64))
    sm = r["slot_map"]
    keep = (sm >= 0)
    keep &= r["ret_hdr"][np.where(keep, sm, 0)] >= 0
    rows = np.where(keep[:, :, None], _bf16_to_f64(r["ret_x"][np.where(keep, sm, 0)]), 0.0)
    logits = torch.from_numpy(lg.astype(np.float64)).requires_grad_(True)
    g = torch.softmax(torch.gather(logits, 1, idx), dim=1)
    g.retain_grad()
    out = (g[:, :, None] * torch.from_numpy(rows)).sum(dim=1)
    (out * torch.from_numpy(dout.astype(np.float64))).sum().backward()
    np.testing.assert_allclose(b["dgate"], g.grad.numpy(), rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(b["dlogits"], logits.grad.numpy(), rtol=1e-9, atol=1e-12)


def test_unsurviving_slots_are_zero(case):
    w, lg, x, s, r, dout, b = case
    dead = r["ret_hdr"] < 0
    assert dead.any() and not b["d_ret"][dead].any() and not b["d_pool"][dead].any()


def test_ragged_backward_equals_unbounded_pooled():
    w = synth.WORKLOADS["tiny"].with_(cf_send_pct=0, cf_recv_pct=0)
    lg, x, s = synth.logits(w), synth.x_bf16(w), synth.scales(w)
    dout = synth.dout(w)
    rp = oracle.run(w, lg, x, s)
    rr = oracle.run(w.with_(mode=1), lg, x, s)
    bp = oracle.run_backward(w, rp, dout, s)
    br = oracle.run_backward(w.with_(mode=1), rr, dout, s)
    np.testing.assert_array_equal(bp["dx"], br["dx"])
    np.testing.assert_array_equal(bp["dlogits"], br["dlogits"])
    np.testing.assert_array_equal(bp["dgate"], br["dgate"])


def test_backward_tokens_equals_full_backward(case):
    w, lg, x, s, r, dout, b = case
    toks = np.array([0, 3, 255, 256, 1500, 2047])
    d_ret, dgate, dlogits, dx = oracle.backward_tokens(r["geom"], x, r["idx"], r["gates"],
                                                       r["slot_map"], r["recv_row"], s, dout, toks)
    np.testing.assert_array_equal(dgate, b["dgate"][toks])
    np.testing.assert_array_equal(dlogits, b["dlogits"][toks])
    np.testing.assert_array_equal(dx, b["dx"][toks])
    sm = r["slot_map"][toks]
    for n in range(toks.size):
        for j in range(w.k):
            if sm[n, j] >= 0 and r["recv_row"][sm[n, j]] >= 0:
                np.testing.assert_array_equal(d_ret[n, j], b["d_ret"][sm[n, j]])
            else:
                assert not d_ret[n, j].any()
