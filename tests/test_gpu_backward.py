"""GPU backward (combine backward, expert-op backward, pack backward) against
the CPU oracle, through the C ABI.  The checks and their bounds are in
tests/backward_check.py: the gradient rows bit for bit against the oracle run
with the device's own fp32 gates, dx within the fp32 summation bound of those
rows, and dgates / dlogits within bounds derived from the arithmetic.
"""
import numpy as np
import pytest
import torch

import oracle
from backward_check import check_backward_arrays, f32, ulp_bf16
from combine_moe_pw_b200 import moe_pw as mp
from combine_moe_pw_b200 import synth

pytestmark = pytest.mark.gpu


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
    got = {"gates": b.gates.cpu().numpy(),
           "d_ret": b.d_ret.cpu().numpy().view(np.uint16),
           "d_pool": b.d_pool.cpu().numpy().view(np.uint16),
           "dgates": b.dgates.cpu().numpy(),
           "dlogits": b.dlogits.cpu().numpy(),
           "dx": b.dx.cpu().numpy()}
    check_backward_arrays(w, got, r, ob, dout, synth.scales(w))


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
    # the same tokens with the device's own fp32 gates: every bf16 code of the
    # gradient rows is then decided from the same product, bit for bit
    g_dev = b.gates.cpu().numpy().astype(np.float64)
    d_ret_s, _, _, dx_s = oracle.backward_tokens(r["geom"], x, r["idx"], g_dev, r["slot_map"],
                                                 r["recv_row"], s, dout, toks)
    tt = torch.from_numpy(toks).cuda()
    sm = r["slot_map"][toks]
    live = (sm >= 0) & (r["recv_row"][np.where(sm >= 0, sm, 0)] >= 0)
    # y rows and magnitudes for the tolerances
    e = r["idx"][toks]
    y = f32(oracle.expert_product(np.repeat(s[e].reshape(-1, 1), w.D, axis=1),
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
    got = f32(b.d_ret.index_select(0, slots).cpu().numpy().view(np.uint16)).reshape(
        toks.size, w.k, w.D)
    ref = f32(d_ret)
    assert np.all(np.abs(got - ref)[live] <= ulp_bf16(ref)[live])
    np.testing.assert_array_equal(got[live], f32(d_ret_s)[live])
    gdx = b.dx[tt].cpu().numpy().astype(np.float64)
    # dx against the stage-wise oracle: an fp32 sum of the same bf16 rows
    ys = f32(oracle.expert_product(np.repeat(s[e].reshape(-1, 1), w.D, axis=1),
                                   d_ret_s.reshape(-1, w.D))).reshape(toks.size, w.k, w.D)
    mag = (np.abs(ys) * live[:, :, None]).sum(axis=1)
    n_live = live.sum(axis=1)[:, None]
    assert np.all(np.abs(gdx - dx_s) <= np.maximum(n_live - 1, 0) * 2.0 ** -24 * 1.001 * mag + 1e-30)
    del b
    torch.cuda.empty_cache()
