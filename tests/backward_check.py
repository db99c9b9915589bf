"""Checks of a backward result (combine backward, expert-op backward, pack
backward) against the oracle, on host arrays.

Two comparisons, both without any allowance for a number of mismatches:

1. Stage by stage.  The gradient rows are bf16 codes decided by the fp32
   product g_j * dout, so the decision depends on the gate the device used.
   The oracle's backward is run again with the device's own fp32 gates (the
   route stage's output, itself checked within 1e-6 by the forward tests):
   given the same gate, the oracle decides every bf16 code in the same
   precision, so d_ret and d_pool must match it bit for bit.  dx is an fp32
   sum of those identical bf16 rows, j ascending, one rounding per add after
   the first: |dx - exact| <= (n - 1) * 2^-24 * sum |terms| for n live terms.
2. Against the plain oracle (its own double gates): d_ret within one bf16 ulp
   everywhere (the two gates differ by a few fp32 ulp), dgates and dlogits
   within the derived bounds.

Bounds:
- dgates: each lane accumulates D/32 products with fmaf, then a 5-level xor
  tree: |err| <= (D/32 + 5) * 2^-24 * sum_i |dout_i y_i| -> 1e-5 of that sum
  covers D <= 3072.
- dlogits: g_j (dgate_j - sum_i g_i dgate_i) with fp32 gates (1e-6) and the
  dgate bound -> 2e-5 * g_j * (M_j + sum_i g_i M_i), M = sum_i |dout_i y_i|.
"""
import numpy as np

import oracle


def f32(u16):
    return (np.asarray(u16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def ulp_bf16(v):
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, 2.0 ** (e - 7), 2.0 ** -133)


def live_mask(r):
    sm = r["slot_map"]
    keep = sm >= 0
    keep &= r["ret_hdr"][np.where(keep, sm, 0)] >= 0
    return keep


def check_backward_arrays(w, got, r, ob, dout, scale):
    """got: host arrays of the device result: gates f32 [T, k], d_ret / d_pool
    bf16 bits [n_slots, D], dgates f32 [T, k], dlogits f32 [T, E], dx f32
    [T, D].  r / ob: the oracle's forward and backward."""
    k = w.k
    g_dev = np.asarray(got["gates"], np.float32).astype(np.float64)
    r_dev = dict(r)
    r_dev["gates"] = g_dev
    obs = oracle.run_backward(w, r_dev, dout, scale)

    keep = live_mask(r)
    sm = r["slot_map"]
    live_slot = r["ret_hdr"] >= 0

    # 1. stage by stage, bit for bit
    np.testing.assert_array_equal(got["d_ret"], obs["d_ret"], err_msg="d_ret")
    np.testing.assert_array_equal(got["d_pool"][live_slot], obs["d_pool"][live_slot],
                                  err_msg="d_pool")
    assert not got["d_pool"][~live_slot].any()
    terms = np.where(keep[:, :, None], np.abs(f32(obs["d_pool"][np.where(keep, sm, 0)])), 0.0)
    mag = terms.sum(axis=1)
    n_live = keep.sum(axis=1)[:, None]
    dx = np.asarray(got["dx"], np.float64)
    assert np.all(np.abs(dx - obs["dx"]) <= np.maximum(n_live - 1, 0) * 2.0 ** -24 * 1.001 * mag
                  + 1e-30), "dx"

    # 2. against the plain oracle
    rows = np.where(keep[:, :, None], f32(r["ret_x"][np.where(keep, sm, 0)]), 0.0)
    M = (np.abs(dout.astype(np.float64))[:, None, :] * np.abs(rows)).sum(axis=2)
    dg = np.asarray(got["dgates"], np.float64)
    assert np.all(np.abs(dg - ob["dgate"]) <= 1e-5 * M + 1e-30), "dgates"
    g = r["gates"]
    dl = np.asarray(got["dlogits"], np.float64)
    idx = r["idx"].astype(np.int64)
    tol = 2e-5 * g * (M + (g * M).sum(axis=1, keepdims=True)) + 1e-30
    assert np.all(np.abs(np.take_along_axis(dl, idx, 1)
                         - np.take_along_axis(ob["dlogits"], idx, 1)) <= tol), "dlogits"
    off = np.ones_like(dl, bool)
    np.put_along_axis(off, idx, False, axis=1)
    assert not dl[off].any(), "dlogits off the chosen experts"
    assert not got["d_ret"][~live_slot].any()
    a, b = f32(got["d_ret"][live_slot]), f32(ob["d_ret"][live_slot])
    assert np.all(np.abs(a - b) <= ulp_bf16(b)), "d_ret within one bf16 ulp of the oracle"
    return obs
