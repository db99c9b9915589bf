"""The fused dispatch against the separate launches and the oracle: route and
assignment in one clustered launch (moe_pw_route_assign), the assignment with
headers (moe_pw_assign_headers), and pack and bucketing in one launch
(moe_pw_pack_bucket).

Every output buffer is poisoned before each path runs, so a word the fused
launch fails to write shows up.  The cases cover bucket items of one and of
several tiles (positions per (destination, wave) item above the fused
launch's tile of 4096), more items than blocks (each block then takes
several), one wave with 16 experts per rank, one expert per wave, heavy
sender and receiver drops, and the pages' rank count.
"""
import numpy as np
import pytest
import torch

from combine_moe_pw_b200 import moe_pw as mp
from combine_moe_pw_b200 import synth
from test_gpu_parity import SMALL_CASES, TINY, _inputs, check_full

pytestmark = pytest.mark.gpu

OUTPUTS = ["slot_map", "occ", "pool_x", "pool_hdr", "recv_row", "bucket_slot", "expert_counts"]

CASES = {
    "tiny": TINY,
    "tiny_tight": SMALL_CASES["tiny_tight"],
    "single_pool": SMALL_CASES["single_pool"],
    "one_expert_per_wave": TINY.with_(W=6, P=1),
    "wide_E": SMALL_CASES["wide_E"],
    "E2048": SMALL_CASES["E2048"],              # 1024 items: several per block
    "pages_ranks_small": SMALL_CASES["pages_ranks_small"],
    "max_P": SMALL_CASES["max_P"],                # 32 experts per bucket item
    # 2 sources of 10,000 tokens: ~29,000 positions per item, 8 tiles
    "long_sources": SMALL_CASES["long_sources"],
    "multi_tile_ragged_tail": synth.Workload("multi_tile", T=8 * 5001, R=8, L=6, W=3, P=2, k=8,
                                             D=24, seq_len=5001,
                                             logit_kind=synth.LOGIT_SEQBIAS),
}


def _fresh(w, lg, x, s):
    b = mp.Buffers(mp.Config.from_workload(w))
    b.logits.copy_(torch.from_numpy(lg))
    b.x.copy_(torch.from_numpy(x.view(np.int16)))
    b.scale.copy_(torch.from_numpy(s))
    return b


def _poison(b):
    b.slot_map.fill_(-77)
    b.occ.fill_(-77)
    b.pool_x.fill_(0x2A2A)
    b.pool_hdr.fill_(-55)
    b.recv_row.fill_(-66)
    b.bucket_slot.fill_(-88)
    b.expert_counts.fill_(99)


@pytest.mark.parametrize("name", list(CASES))
def test_fused_equals_separate_launches(name):
    w = CASES[name]
    lg, x, s = _inputs(w)
    ref = _fresh(w, lg, x, s)
    ref.route()
    _poison(ref)
    ref.assign()
    ref.pack()
    ref.bucket()
    st_ref = ref.stats()

    b = _fresh(w, lg, x, s)
    b.route()
    _poison(b)
    b.assign_headers()
    b.pack_bucket()
    st = b.stats()
    torch.cuda.synchronize()
    for n in OUTPUTS:
        assert torch.equal(getattr(b, n), getattr(ref, n)), n
    assert (st.kept, st.sender_dropped, st.receiver_dropped, st.error, st.max_fill) == (
        st_ref.kept, st_ref.sender_dropped, st_ref.receiver_dropped, st_ref.error,
        st_ref.max_fill)
    np.testing.assert_array_equal(b.host_expert_counts, ref.host_expert_counts)


@pytest.mark.parametrize("name", ["multi_tile_ragged_tail", "one_expert_per_wave"])
def test_fused_step_full_parity(name):
    """The whole step through moe_pw_dispatch (the fused path) against the
    whole oracle, on buffers poisoned first."""
    w = CASES[name]
    lg, x, s = _inputs(w)
    b = _fresh(w, lg, x, s)
    _poison(b)
    b.run_step()
    st = b.stats(raise_on_device_error=False)
    torch.cuda.synchronize()
    check_full(w, lg, x, s, b, st)


def test_fused_repeat_rebuilds_every_word():
    """A second fused launch on poisoned pools (same assignment) rebuilds the
    same bytes: headers of empty slots come from the bucketing, rows from the
    pack's zero fill."""
    w = TINY.with_(T=8 * 1024, seq_len=1024, D=256, logit_kind=synth.LOGIT_SEQBIAS)
    lg, x, s = _inputs(w)
    b = _fresh(w, lg, x, s)
    b.run_step()
    torch.cuda.synchronize()
    keep = {n: getattr(b, n).clone() for n in OUTPUTS}
    assert (keep["pool_hdr"] < 0).any()
    for _ in range(2):
        b.assign_headers()
        b.pool_x.fill_(0x1357)
        # the kept slots' headers stay (the assignment wrote them); the rest is poisoned
        b.pool_hdr.masked_fill_(keep["pool_hdr"] < 0, -9)
        b.recv_row.fill_(-66)
        b.bucket_slot.fill_(-88)
        b.pack_bucket()
        torch.cuda.synchronize()
        for n in OUTPUTS:
            assert torch.equal(getattr(b, n), keep[n]), n
    assert b.stats().error == 0


RA_OUTPUTS = ["idx", "gates", "slot_map", "occ", "pool_hdr"]

RA_CASES = {
    **{n: CASES[n] for n in ["tiny", "tiny_tight", "single_pool", "one_expert_per_wave",
                             "wide_E", "E2048", "pages_ranks_small", "long_sources",
                             "multi_tile_ragged_tail"]},
    "k1": SMALL_CASES["k1"],
    "k16": SMALL_CASES["k16"],
    "k32": SMALL_CASES["k32"],
    "odd_E": synth.Workload("odd_E", T=4 * 300, R=4, L=5, W=1, P=5, k=6, D=8, seq_len=300,
                            logit_kind=synth.LOGIT_ZIPF),   # E = 20: NV = 1, not full
    "one_token_sources": synth.Workload("one_token", T=16, R=16, L=4, W=2, P=2, k=3, D=8,
                                       seq_len=1, logit_kind=synth.LOGIT_IID),
    # 48,000 tokens per source: the one-launch form's shared memory would pass
    # its limit, so the call runs route + assignment instead (same outputs)
    "fallback_long_sources": synth.Workload("fallback", T=2 * 48000, R=2, L=6, W=3, P=2, k=8,
                                            D=8, seq_len=48000,
                                            logit_kind=synth.LOGIT_SEQBIAS),
}


# cases the clustered launch does not fit (its call then refuses with
# MOE_PW_EUNSUPPORTED): its shared memory per block would pass the launch's
# limit with 48,000 tokens per source, and with 1,024 pools per source
# (E2048: the per-warp pool counts alone take 32 KB)
NOT_CLUSTER = {"fallback_long_sources", "E2048"}


def _poison_route(b):
    b.idx.fill_(-5)
    b.gates.fill_(float("nan"))
    b.slot_map.fill_(-77)
    b.occ.fill_(-77)
    b.pool_hdr.fill_(-55)


@pytest.mark.parametrize("name", list(RA_CASES))
def test_route_assign_equals_separate_launches(name):
    """The clustered launch of moe_pw_route_assign against moe_pw_route +
    moe_pw_assign_headers: ids, gates (bit for bit: the same selection code),
    slots, occupancies, the kept slots' headers and the sender counters."""
    w = RA_CASES[name]
    lg, x, s = _inputs(w)
    ref = _fresh(w, lg, x, s)
    _poison_route(ref)
    ref.route()
    ref.assign_headers()
    st_ref = ref.stats()

    b = _fresh(w, lg, x, s)
    _poison_route(b)
    b.counters.fill_(-1)  # the call zeroes the counters itself
    if name in NOT_CLUSTER:
        with pytest.raises(mp.MoePwError) as ei:
            b.route_assign(form=mp.RA_CLUSTER)
        assert ei.value.code == mp.MOE_PW_EUNSUPPORTED
        return
    b.route_assign(form=mp.RA_CLUSTER)
    st = b.stats()
    torch.cuda.synchronize()
    for n in RA_OUTPUTS:
        assert torch.equal(getattr(b, n), getattr(ref, n)), n
    assert (st.assignments, st.sender_dropped, st.max_occ, st.error) == (
        st_ref.assignments, st_ref.sender_dropped, st_ref.max_occ, st_ref.error)


@pytest.mark.parametrize("name", list(RA_CASES))
def test_route_assign_default_form(name):
    """The default form: the clustered launch up to 256 tokens per SM where
    it fits, else the two calls; same outputs either way."""
    w = RA_CASES[name]
    cfg = mp.Config.from_workload(w)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    small = w.T <= 256 * sms
    expect = mp.RA_CLUSTER if small and name not in NOT_CLUSTER else mp.RA_SEPARATE
    assert mp.moe_pw_route_assign_plan(cfg) == expect
    lg, x, s = _inputs(w)
    ref = _fresh(w, lg, x, s)
    _poison_route(ref)
    ref.route()
    ref.assign_headers()
    st_ref = ref.stats()
    b = _fresh(w, lg, x, s)
    _poison_route(b)
    b.counters.fill_(-1)  # zeroed by the call, whichever form runs
    b.route_assign()
    st = b.stats()
    torch.cuda.synchronize()
    for n in RA_OUTPUTS:
        assert torch.equal(getattr(b, n), getattr(ref, n)), n
    assert (st.sender_dropped, st.max_occ, st.error, st.kept) == (
        st_ref.sender_dropped, st_ref.max_occ, st_ref.error, st_ref.kept)


@pytest.mark.parametrize("name", ["k16", "E2048", "fallback_long_sources"])
def test_route_assign_step_full_parity(name):
    """The whole step (run_step: route + assignment, pack + bucketing, expert
    op, combine) against the whole oracle."""
    w = RA_CASES[name]
    lg, x, s = _inputs(w)
    b = _fresh(w, lg, x, s)
    _poison(b)
    b.run_step()
    st = b.stats(raise_on_device_error=False)
    torch.cuda.synchronize()
    check_full(w, lg, x, s, b, st)


def test_route_assign_plan_follows_tokens_per_sm():
    """The clustered launch up to 256 tokens per SM: a 16,384-token batch of
    the layer shapes takes it; the 65,536-token layer and 262,144-token rack
    batches (above 148 * 256) take the separate kernels."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    cases = [synth.WORKLOADS["layer"].with_(T=16384)] + [synth.WORKLOADS[n] for n in
                                                         ["layer", "rack", "long"]]
    for w in cases:
        expect = mp.RA_CLUSTER if w.T <= 256 * sms else mp.RA_SEPARATE
        assert mp.moe_pw_route_assign_plan(mp.Config.from_workload(w)) == expect, w.T
