"""Pins for the oracle's per-expert op and combine.

Readings: the expert op stand-in is y = s_e * x with the product in fp32 and a
round-to-nearest-even to bf16; the combine is out[t] = sum_j g_j * y_j over the
surviving assignments, no renormalisation (a dropped assignment leaves the
token to the shared experts, "Marin 开始公开训练 535B 参数 MoE 模型", section 四).

Pins: bf16 rounding against torch's conversion, the combine against a numpy
einsum, identity experts with unbounded capacity give x back (gates sum to 1),
power-of-two scales, k = 1, and the dropless mode equal to the unbounded
pooled result.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_moe_pw_b200 import synth


def _bf16_to_f32(a):
    return (a.astype(np.uint32) << 16).view(np.float32)


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(1)
    a = rng.standard_normal(100000).astype(np.float32) * np.float32(3.0)
    # exact ties at the bf16 boundary, both parities, and signed zeros
    base = rng.integers(0, 1 << 15, 2000).astype(np.uint32) << 16
    ties = np.concatenate([(base | 0x8000), (base | 0x18000), (base | 0x7FFF), (base | 0x8001)])
    a = np.concatenate([a, ties.view(np.float32), np.array([0.0, -0.0, 1e-40, -1e-40], np.float32)])
    a = a[np.isfinite(a)]
    ours = oracle.bf16_round(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)


def test_expert_product_matches_torch():
    rng = np.random.default_rng(2)
    n = 200000
    s = rng.uniform(0.5, 1.5, n).astype(np.float32)
    x = torch.from_numpy(rng.standard_normal(n).astype(np.float32)).to(torch.bfloat16)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    ours = oracle.expert_product(s, xb)
    ref = (torch.from_numpy(s) * x.float()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)


def test_combine_matches_einsum(tiny_oracle):
    r = tiny_oracle
    g = r["geom"]
    keep = (r["slot_map"] >= 0)
    sm = np.where(keep, r["slot_map"], 0)
    keep &= r["ret_hdr"][sm] >= 0
    y = _bf16_to_f32(r["ret_x"][sm]).astype(np.float64)          # [T, k, D]
    ref = np.einsum("tk,tkd->td", r["gates"] * keep, y)
    np.testing.assert_allclose(r["out"], ref, rtol=1e-13, atol=1e-13)
    mag = np.einsum("tk,tkd->td", r["gates"] * keep, np.abs(y))
    np.testing.assert_allclose(r["mag"], mag, rtol=1e-13, atol=1e-13)


def test_combine_tokens_equals_full_combine(tiny_inputs, tiny_oracle):
    w, lg, x, s = tiny_inputs
    r = tiny_oracle
    toks = np.array([0, 1, 2, 255, 256, 1000, 2047])
    out, mag = oracle.combine_tokens(r["geom"], x, r["idx"], r["gates"], r["slot_map"],
                                     r["recv_row"], s, toks)
    np.testing.assert_array_equal(out, r["out"][toks])
    np.testing.assert_array_equal(mag, r["mag"][toks])


def test_identity_experts_unbounded_capacity_return_x(tiny_inputs):
    """No drops and s_e = 1: combine(x) = x * sum_j g_j = x up to the double
    rounding of eight products and sums (bound 16 * 2^-53 < 2e-15)."""
    w, lg, x, _ = tiny_inputs
    wu = w.with_(cf_send_pct=0, cf_recv_pct=0)
    r = oracle.run(wu, lg, x, np.ones(w.E, np.float32))
    assert r["sender_dropped"] == r["receiver_dropped"] == 0
    xf = _bf16_to_f32(x).astype(np.float64)
    np.testing.assert_allclose(r["out"], xf, rtol=2e-15, atol=0)


def test_power_of_two_scale(tiny_inputs):
    """s_e = 2 for all e: bf16(2x) = 2x exactly, so out = 2 x sum_j(kept) g_j."""
    w, lg, x, _ = tiny_inputs
    r = oracle.run(w, lg, x, np.full(w.E, 2.0, np.float32))
    keep = r["slot_map"] >= 0
    keep &= r["recv_row"][np.where(keep, r["slot_map"], 0)] >= 0
    gsum = (r["gates"] * keep).sum(axis=1, keepdims=True)
    np.testing.assert_allclose(r["out"], 2.0 * _bf16_to_f32(x) * gsum, rtol=1e-14, atol=0)
    assert r["sender_dropped"] > 0  # the tiny case does drop at cf 1.10


def test_k1_output_is_the_expert_row():
    w = synth.WORKLOADS["tiny"].with_(k=1, cf_send_pct=0, cf_recv_pct=0)
    lg, x, s = synth.logits(w), synth.x_bf16(w), synth.scales(w)
    r = oracle.run(w, lg, x, s)
    e = r["idx"][:, 0]
    y = oracle.expert_product(np.repeat(s[e][:, None], w.D, axis=1), x)
    np.testing.assert_array_equal(r["out"], _bf16_to_f32(y).astype(np.float64))


def test_ragged_equals_unbounded_pooled(tiny_inputs):
    """Both modes keep every assignment; the same j-order sum over the same bf16
    rows gives the same double result bit for bit."""
    w, lg, x, s = tiny_inputs
    pooled = oracle.run(w.with_(cf_send_pct=0, cf_recv_pct=0), lg, x, s)
    ragged = oracle.run(w.with_(cf_send_pct=0, cf_recv_pct=0, mode=1), lg, x, s)
    assert ragged["kept"] == w.T * w.k
    np.testing.assert_array_equal(pooled["out"], ragged["out"])
    np.testing.assert_array_equal(ragged["row_cnt"],
                                  np.bincount(ragged["idx"].reshape(-1), minlength=w.E))


def test_dropped_terms_are_not_renormalised(tiny_inputs):
    """With cf 1.10 some assignments drop; their gates are left out, so the
    surviving gate mass of such a token is below one."""
    w, lg, x, _ = tiny_inputs
    r = oracle.run(w, lg, x, np.ones(w.E, np.float32))
    dropped_tok = np.unique(np.nonzero(r["slot_map"] < 0)[0])
    assert dropped_tok.size > 0
    t = dropped_tok[0]
    keep = r["slot_map"][t] >= 0
    xf = _bf16_to_f32(x[t]).astype(np.float64)
    np.testing.assert_allclose(r["out"][t], xf * r["gates"][t][keep].sum(), rtol=1e-14)
