"""moe_pw_assign_noalloc: the sender/expert assignment without a caller-given
workspace.

This entry point exists for callers that cannot allocate device memory for the
ranking scratch: a plugin whose host process owns every device allocation and
offers it no allocator, or a latency-critical loop that may not call
cudaMalloc/cudaFree because they can synchronise the whole device.  It uses a
fixed scratch array built into the library instead.

The GPU test calls it through the C ABI twice in a row (the second call finds
the first call's leftovers in the shared array) and requires the same bytes as
moe_pw_assign with a workspace; the host test checks that a batch needing more
scratch than the built-in array is refused before any launch.  This file is
named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

from combine_moe_pw_b200 import moe_pw as mp
from combine_moe_pw_b200 import synth


def _with_workspace(cfg, idx):
    """Reference: the existing entry point with its own workspace."""
    s = mp.moe_pw_plan(cfg)
    dev = idx.device
    slot_map = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=dev)
    occ = torch.empty((s.occ_len,), dtype=torch.int32, device=dev)
    ctr = torch.zeros((mp.COUNTERS_BYTES // 8,), dtype=torch.int64, device=dev)
    ws = torch.empty((s.workspace_bytes,), dtype=torch.uint8, device=dev)
    mp.moe_pw_assign(cfg, idx, slot_map, occ, ctr, ws)
    return slot_map, occ, ctr


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["tiny", "rack", "ragged"])
def test_noalloc_assign_matches_workspace_assign(name):
    w = synth.WORKLOADS[name]
    cfg = mp.Config.from_workload(w)
    s = mp.moe_pw_plan(cfg)
    assert s.workspace_bytes <= mp.NOALLOC_SCRATCH_BYTES
    dev = torch.device("cuda")
    logits = torch.from_numpy(synth.logits(w)).to(dev)
    idx = torch.empty((w.T, w.k), dtype=torch.int32, device=dev)
    gates = torch.empty((w.T, w.k), dtype=torch.float32, device=dev)
    mp.moe_pw_route(cfg, logits, idx, gates)
    ref_slot, ref_occ, ref_ctr = _with_workspace(cfg, idx)
    ref_stats = mp.moe_pw_stats(cfg, ref_ctr)

    for call in range(2):
        slot_map = torch.full((w.T, w.k), -77, dtype=torch.int32, device=dev)
        occ = torch.full((s.occ_len,), -77, dtype=torch.int32, device=dev)
        ctr = torch.full((mp.COUNTERS_BYTES // 8,), 12345, dtype=torch.int64, device=dev)
        mp.moe_pw_assign_noalloc(cfg, idx, slot_map, occ, ctr)
        st = mp.moe_pw_stats(cfg, ctr)
        assert torch.equal(slot_map, ref_slot), f"slot_map differs on call {call}"
        assert torch.equal(occ, ref_occ), f"occ differs on call {call}"
        assert (st.sender_dropped, st.max_occ, st.error) == (
            ref_stats.sender_dropped, ref_stats.max_occ, ref_stats.error), f"call {call}"
    torch.cuda.synchronize()


def test_noalloc_refuses_batches_beyond_the_scratch_limit():
    """512 ranks x 4 waves = 2048 pools per source: the ranking would need
    8 MiB of scratch, more than the 4 MiB array, so the call returns
    MOE_PW_ENOMEM without touching the GPU."""
    cfg = mp.Config(T=512 * 256, E=2048, k=8, D=64, R=512, L=4, W=4, P=1)
    assert mp.moe_pw_plan(cfg).workspace_bytes > mp.NOALLOC_SCRATCH_BYTES
    fake = 1 << 20  # aligned placeholder addresses: the call must refuse before using them
    with pytest.raises(mp.MoePwError) as ei:
        mp.moe_pw_assign_noalloc(cfg, fake, fake, fake, fake, stream=0)
    assert ei.value.code == mp.MOE_PW_ENOMEM
