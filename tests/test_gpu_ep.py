"""Expert parallelism over several GPUs, emulated on one GPU, against the
oracle through the C ABI.

Every GPU of an n-GPU run is a share of buffers on this one device; the
shares' peer tables hold the other shares' plain addresses, so the pack and
the expert op store across shares exactly as they store across GPUs.  Each
phase of the step runs for every share before the next phase (which stands in
for the barrier); no kernel waits on another.  The shares are reassembled into
the single-batch layout and held to the same bar as the single-GPU path:
bit-exact integer and byte outputs, gates within 1e-6, combine within 1e-6 of
its scale.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_moe_pw_b200 import ep
from combine_moe_pw_b200 import moe_pw as mp
from combine_moe_pw_b200 import synth
from ep_check import assemble
from test_gpu_parity import _inputs, check_full, check_sampled

pytestmark = pytest.mark.gpu

TINY = synth.WORKLOADS["tiny"]


def run_ep(w, n_gpus, overlap=True, lg=None):
    lg, x, s = _inputs(w, lg)
    cfg = mp.Config.from_workload(w)
    shares = [ep.EpBuffers(cfg, n_gpus, g) for g in range(n_gpus)]
    for b in shares:
        t = b.share.token_range
        b.logits.copy_(torch.from_numpy(lg[t.start:t.stop]))
        b.x.copy_(torch.from_numpy(x[t.start:t.stop].view(np.int16)))
        b.scale.copy_(torch.from_numpy(s))
        # stale contents must not survive: every pool entry is rewritten
        for name in ("recv_x", "recv_hdr", "recv_row", "ret_x", "ret_hdr", "bucket_slot"):
            getattr(b, name).fill_(0x3C3C)
    ep.emulate_step(shares, overlap)
    stats = [b.stats(raise_on_device_error=False) for b in shares]
    torch.cuda.synchronize()
    return lg, x, s, shares, stats


CASES = {
    "tiny_n1": (TINY, 1), "tiny_n2": (TINY, 2), "tiny_n4": (TINY, 4), "tiny_n8": (TINY, 8),
    "tiny_tight_n2": (TINY.with_(cf_send_pct=60, cf_recv_pct=70), 2),
    "tiny_seqbias_n4": (TINY.with_(logit_kind=synth.LOGIT_SEQBIAS), 4),
    "one_wave_n2": (synth.Workload("w1", T=4 * 50, R=4, L=3, W=1, P=3, k=2, D=24, seq_len=50,
                                   logit_kind=synth.LOGIT_IID), 2),
    "k16_n2": (TINY.with_(k=16), 2),
    "odd_width_n4": (TINY.with_(D=136), 4),
    "pages_ranks_small_n8": (synth.Workload("prs", T=64 * 64, R=64, L=6, W=3, P=2, k=8, D=256,
                                            seq_len=1024, logit_kind=synth.LOGIT_SEQBIAS), 8),
}


@pytest.mark.parametrize("overlap", [True, False], ids=["waves_overlapped", "one_pack"])
@pytest.mark.parametrize("name", list(CASES))
def test_ep_emulated_full_parity(name, overlap):
    w, n = CASES[name]
    lg, x, s, shares, stats = run_ep(w, n, overlap)
    b, st = assemble(mp.Config.from_workload(w), shares, stats)
    check_full(w, lg, x, s, b, st)


def test_ep_shares_partition_the_batch():
    """Each share's own statistics: its sources' sender drops, its experts'
    arrivals; together they are the whole batch's."""
    w = TINY.with_(logit_kind=synth.LOGIT_SEQBIAS)
    lg, x, s, shares, stats = run_ep(w, 4)
    r = oracle.run_headers(w, lg)
    g = r["geom"]
    n_src = w.R // 4
    for h, (b, st) in enumerate(zip(shares, stats)):
        assert st.assignments == b.share.tokens * w.k
        occ = r["occ"].reshape(w.R, w.R, w.W)[h * n_src:(h + 1) * n_src]
        tr = b.share.token_range
        assert st.sender_dropped == int((r["slot_map"][tr.start:tr.stop] < 0).sum())
        np.testing.assert_array_equal(b.occ.cpu().numpy(), occ.reshape(-1))
        er = b.share.expert_range
        np.testing.assert_array_equal(b.host_expert_counts[0], r["arrivals"][er.start:er.stop])
        assert st.kept == int(r["bucket_cnt"][er.start:er.stop].sum())
    assert sum(st.kept for st in stats) == r["kept"]
    assert g.n_slots == sum(b.share.n_slots for b in shares)


@pytest.mark.parametrize("n_gpus", [2, 4])
def test_ep_layer_sampled(n_gpus):
    """The one-layer batch (65,536 tokens, 3072 wide) split over 2 and 4
    emulated GPUs: the integer path in full, rows and combine on samples."""
    w = synth.WORKLOADS["layer"]
    lg, x, s, shares, stats = run_ep(w, n_gpus)
    b, st = assemble(mp.Config.from_workload(w), shares, stats)
    del shares
    torch.cuda.empty_cache()
    check_sampled(w, lg, x, s, b, st, n_tok=512, n_slot=4096)


def test_ep_repeat_steps_are_identical():
    """A second step on the same shares (pools full of the first step's
    rows) gives the same bytes: no stale row, header or bucket survives."""
    w = TINY.with_(logit_kind=synth.LOGIT_SEQBIAS)
    lg, x, s, shares, stats = run_ep(w, 2)
    first = {n: [getattr(b, n).clone() for b in shares]
             for n in ("recv_x", "recv_hdr", "recv_row", "ret_x", "ret_hdr", "out", "bucket_slot")}
    ep.emulate_step(shares, overlap=True)
    torch.cuda.synchronize()
    for n, ts in first.items():
        for b, t in zip(shares, ts):
            assert torch.equal(getattr(b, n), t), n


def test_ep_rejects_bad_shares():
    cfg = mp.Config.from_workload(TINY)
    with pytest.raises(mp.MoePwError):
        mp.moe_pw_ep_plan(cfg, 3, 0)          # 8 ranks do not split over 3 GPUs
    with pytest.raises(mp.MoePwError):
        mp.moe_pw_ep_plan(cfg, 2, 2)          # no GPU 2 of 2
    with pytest.raises(mp.MoePwError):
        mp.moe_pw_ep_plan(mp.Config.from_workload(TINY.with_(mode=1, cf_send_pct=0,
                                                             cf_recv_pct=0)), 2, 0)
    b = ep.EpBuffers(cfg, 2, 0)
    with pytest.raises(mp.MoePwError):
        b.pack()                              # GPU 1's receive pool is not in the table


def test_ep_empty_batch():
    """No tokens: every share's step runs and reports nothing kept or dropped."""
    w = TINY.with_(T=0)
    cfg = mp.Config.from_workload(w)
    shares = [ep.EpBuffers(cfg, 2, g) for g in range(2)]
    for b in shares:
        b.expert_counts.fill_(7)
    ep.emulate_step(shares)
    for b in shares:
        st = b.stats()
        assert (st.assignments, st.kept, st.sender_dropped, st.receiver_dropped) == (0, 0, 0, 0)
        assert int(b.expert_counts.abs().sum()) == 0
