"""The backward checker (tests/backward_check.py) on the CPU: a result that
follows the method exactly passes it, and one bf16 ulp planted in a single
gradient element, or a dx element off by more than its fp32 summation bound,
fails it.  The "device" result here is the oracle's own backward run with
fp32-rounded gates, the precision the device holds its gates in.
"""
import numpy as np
import pytest

import oracle
from backward_check import check_backward_arrays, live_mask
from combine_moe_pw_b200 import synth


def _case(w):
    lg, x, s, dout = synth.logits(w), synth.x_bf16(w), synth.scales(w), synth.dout(w)
    r = oracle.run(w, lg, x, s)
    ob = oracle.run_backward(w, r, dout, s)
    g32 = r["gates"].astype(np.float32)
    r32 = dict(r)
    r32["gates"] = g32.astype(np.float64)
    dev = oracle.run_backward(w, r32, dout, s)
    got = {"gates": g32, "d_ret": dev["d_ret"].copy(), "d_pool": dev["d_pool"].copy(),
           "dgates": dev["dgate"].astype(np.float32), "dlogits": dev["dlogits"].astype(np.float32),
           "dx": dev["dx"].astype(np.float32)}
    return w, got, r, ob, dout, s


CASES = {"tiny": synth.WORKLOADS["tiny"],
         "tiny_tight": synth.WORKLOADS["tiny"].with_(cf_send_pct=60, cf_recv_pct=70)}


@pytest.mark.parametrize("name", list(CASES))
def test_exact_result_passes(name):
    w, got, r, ob, dout, s = _case(CASES[name])
    check_backward_arrays(w, got, r, ob, dout, s)


def test_one_ulp_in_one_gradient_element_fails():
    w, got, r, ob, dout, s = _case(CASES["tiny"])
    slot = int(np.flatnonzero(r["ret_hdr"] >= 0)[7])
    i = int(np.flatnonzero(got["d_ret"][slot])[0])
    got["d_ret"][slot, i] += 1  # the neighbouring bf16 code
    with pytest.raises(AssertionError):
        check_backward_arrays(w, got, r, ob, dout, s)


def test_dx_beyond_its_summation_bound_fails():
    w, got, r, ob, dout, s = _case(CASES["tiny"])
    t = int(np.flatnonzero(live_mask(r).sum(axis=1) >= 3)[0])
    i = int(np.flatnonzero(got["dx"][t])[0])
    got["dx"][t, i] = np.nextafter(np.nextafter(np.float32(got["dx"][t, i]), np.float32(np.inf)),
                                   np.float32(np.inf)) * np.float32(1 + 2 ** -10)
    with pytest.raises(AssertionError):
        check_backward_arrays(w, got, r, ob, dout, s)
