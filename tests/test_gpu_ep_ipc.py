"""Expert parallelism across processes, through CUDA IPC, on one GPU.

Two processes each own the share of one GPU of a 2-GPU run (both on this
device).  They exchange their pools' IPC descriptions over a gloo group
(moe_pw_ipc_export / moe_pw_ipc_open through ep.PeerLinks), so the pack and
the expert op of each process store into the other process's memory, as they
would into another GPU's.  The phases of the step are separated on the host:
each process synchronises its device and meets the other at a gloo barrier,
so no kernel ever waits on another.  The shares, reassembled, must match the
oracle exactly as the single-GPU path does.
"""
import os
import socket
from types import SimpleNamespace

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp_

from combine_moe_pw_b200 import moe_pw as mp
from combine_moe_pw_b200 import synth
from ep_check import assemble
from test_gpu_parity import _inputs, check_full

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
NAMES = ("idx", "gates", "slot_map", "occ", "recv_x", "recv_hdr", "recv_row", "bucket_slot",
         "expert_counts", "ret_x", "ret_hdr", "out")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, overlap, q):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from combine_moe_pw_b200 import ep
    from combine_moe_pw_b200 import moe_pw as mpw
    from combine_moe_pw_b200 import synth as sy
    from datetime import timedelta
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=timedelta(seconds=120))
    try:
        torch.cuda.set_device(0)
        w = sy.WORKLOADS["tiny"].with_(logit_kind=sy.LOGIT_SEQBIAS)
        cfg = mpw.Config.from_workload(w)
        b = ep.EpBuffers(cfg, world, rank)
        t = b.share.token_range
        b.logits.copy_(torch.from_numpy(sy.logits(w)[t.start:t.stop]))
        b.x.copy_(torch.from_numpy(sy.x_bf16(w)[t.start:t.stop].view(np.int16)))
        b.scale.copy_(torch.from_numpy(sy.scales(w)))
        for name in ("recv_x", "recv_hdr", "recv_row", "ret_x", "ret_hdr"):
            getattr(b, name).fill_(0x3C3C)
        torch.cuda.synchronize()
        links = ep.PeerLinks(b, dist.all_gather_object)
        for phase in ep.schedule(cfg.W, overlap):
            for _, name, mask in phase:
                b.run_op(name, mask)
            torch.cuda.synchronize()
            dist.barrier()
        st = b.stats(raise_on_device_error=False)
        res = {n: getattr(b, n).cpu().numpy() for n in NAMES}
        res["host_expert_counts"] = b.host_expert_counts.copy()
        res["stats"] = (st.assignments, st.kept, st.sender_dropped, st.receiver_dropped, st.error)
        dist.barrier()            # nobody writes into the other's pools any more
        links.close()
        dist.barrier()            # both unmapped before either frees its pools
        q.put((rank, res))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("overlap", [True, False], ids=["waves_overlapped", "one_pack"])
def test_two_processes_exchange_through_ipc(overlap):
    ctx = mp_.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, overlap, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=600) for _ in range(2))
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    w = synth.WORKLOADS["tiny"].with_(logit_kind=synth.LOGIT_SEQBIAS)
    cfg = mp.Config.from_workload(w)
    from combine_moe_pw_b200 import ep
    shares, stats = [], []
    for r in range(2):
        res = got[r]
        sh = SimpleNamespace(share=ep.share(cfg, 2, r), host_expert_counts=res["host_expert_counts"],
                             **{n: torch.from_numpy(res[n]) for n in NAMES})
        shares.append(sh)
        a, k, sd, rd, e = res["stats"]
        stats.append(SimpleNamespace(assignments=a, kept=k, sender_dropped=sd,
                                     receiver_dropped=rd, error=e))
    b, st = assemble(cfg, shares, stats)
    lg, x, s = _inputs(w)
    check_full(w, lg, x, s, b, st)
