"""Host logic of the expert-parallel path on the CPU: the step's schedule of
waves and barriers, the shares' partition of tokens, experts and pool slots
(from the host-only moe_pw_ep_plan), and the exchange of pool addresses
between two gloo ranks, with the CUDA IPC calls replaced by fakes.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp_

from combine_moe_pw_b200 import ep
from combine_moe_pw_b200 import moe_pw as mp
from combine_moe_pw_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("W", [1, 2, 3, 4])
def test_overlapped_schedule_sends_each_wave_before_its_receivers(W):
    phases = ep.schedule(W, overlap=True)
    where = {}
    for i, ph in enumerate(phases):
        for stream, name, mask in ph:
            where.setdefault((name, mask), []).append((i, stream))
    for w in range(W):
        (p_pack, s_pack), = where[("pack", 1 << w)]
        (p_bucket, s_bucket), = where[("bucket", 1 << w)]
        (p_expert, s_expert), = where[("expert", 1 << w)]
        # a barrier separates a wave's sends from every receiver's walk of it
        assert p_bucket > p_pack and p_expert == p_bucket and s_bucket == s_expert
        assert s_pack == "a"
        # wave w + 1 is sent while wave w is bucketed (the overlap)
        if w + 1 < W:
            assert where[("pack", 1 << (w + 1))][0][0] == p_bucket
    (p_route, _), = where[("route", 0)]
    (p_combine, _), = where[("combine", 0)]
    assert p_route == 0 and p_combine == len(phases) - 1
    # the combine comes after every expert op's return stores
    assert all(p_combine > where[("expert", 1 << w)][0][0] for w in range(W))
    assert len(phases) == W + 2


def test_schedule_without_overlap():
    names = [[op[1] for op in ph] for ph in ep.schedule(3, overlap=False)]
    assert names == [["route", "assign", "pack"], ["bucket", "expert"], ["combine"]]


@pytest.mark.parametrize("name", ["tiny", "layer", "rack"])
@pytest.mark.parametrize("n", [1, 2, 4, 8])
def test_shares_partition_the_batch(name, n):
    w = synth.WORKLOADS[name]
    cfg = mp.Config.from_workload(w)
    one = mp.moe_pw_plan(cfg)
    shares = [ep.share(cfg, n, g) for g in range(n)]
    assert [s.token_range.start for s in shares] == [g * w.T // n for g in range(n)]
    assert sum(s.tokens for s in shares) == w.T
    assert sum(s.local_experts for s in shares) == w.E
    assert sum(s.n_slots for s in shares) == one.n_slots
    assert sum(s.n_pools for s in shares) == one.n_pools
    assert all((s.C_s, s.C_r) == (one.C_s, one.C_r) for s in shares)
    assert [s.ranks for s in shares] == [range(g * w.R // n, (g + 1) * w.R // n) for g in range(n)]
    # memory per GPU: a share of the single-GPU total
    assert max(s.total_bytes for s in shares) <= one.total_bytes // n + one.total_bytes // 50


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch.distributed as dist
    import oracle
    from combine_moe_pw_b200 import ep as ep_
    from combine_moe_pw_b200 import moe_pw as mp_b
    from combine_moe_pw_b200 import synth as sy
    from ep_check import recv_to_global
    from datetime import timedelta
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=timedelta(seconds=120))
    try:
        w = sy.WORKLOADS["tiny"]
        cfg = mp_b.Config.from_workload(w)
        b = ep_.EpBuffers(cfg, world, rank, device="cpu")

        # fake IPC: a description names (exporting rank, array); "opening" it
        # gives a recognisable address
        def export(t):
            h = mp_b.moe_pw_ipc_handle()
            arr = [id(a) for a in (b.recv_x, b.recv_hdr, b.ret_x, b.ret_hdr)].index(id(t))
            h.handle[0], h.handle[1] = rank, arr
            h.offset = 64 * arr
            return h
        opened, closed = [], []

        def open_(h):
            ptr = 0x7F0000000000 + (h.handle[0] << 20) + (h.handle[1] << 12) + h.offset
            opened.append(ptr)
            return ptr

        def close(ptr, h):
            closed.append(ptr)

        links = ep_.PeerLinks(b, dist.all_gather_object, export, open_, close)
        table = [(b.peers.recv_x[h], b.peers.recv_hdr[h], b.peers.ret_x[h], b.peers.ret_hdr[h])
                 for h in range(world)]
        links.close()

        # this rank's slices of the oracle's single-batch arrays, by its share
        lg, x, s = sy.logits(w), sy.x_bf16(w), sy.scales(w)
        r = oracle.run(w, lg, x, s)
        sh = b.share
        Rn = cfg.R // world
        m = recv_to_global(cfg.R, Rn, cfg.W, sh.C_s, rank)
        tr, er = sh.token_range, sh.expert_range
        mine = {"out": r["out"][tr.start:tr.stop], "recv_hdr": r["pool_hdr"][m],
                "ret_hdr": r["ret_hdr"][rank * sh.n_slots:(rank + 1) * sh.n_slots],
                "arrivals": r["arrivals"][er.start:er.stop], "recv_slots": m}
        got = [None] * world
        dist.all_gather_object(got, mine)
        q.put((rank, table, b.addresses(), opened, closed, got if rank == 0 else None))
    finally:
        dist.destroy_process_group()


def test_two_rank_address_exchange_and_oracle_slices():
    ctx = mp_.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    # drain the queue before joining: a child blocks on a full pipe until read
    out = dict((o[0], o[1:]) for o in (q.get(timeout=300) for _ in range(2)))
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    for rank in (0, 1):
        table, own, opened, closed, _ = out[rank]
        other = 1 - rank
        assert table[rank] == own                      # own pools by their own address
        expect = tuple(0x7F0000000000 + (other << 20) + (a << 12) + 64 * a for a in range(4))
        assert table[other] == expect                  # the other rank's four pools, opened
        assert sorted(opened) == sorted(expect) and sorted(closed) == sorted(expect)
    # the two shares' slices reassemble the oracle's single-batch arrays
    import oracle
    w = synth.WORKLOADS["tiny"]
    r = oracle.run(w, synth.logits(w), synth.x_bf16(w), synth.scales(w))
    got = out[0][4]
    np.testing.assert_array_equal(np.concatenate([g["out"] for g in got]), r["out"])
    np.testing.assert_array_equal(np.concatenate([g["ret_hdr"] for g in got]), r["ret_hdr"])
    np.testing.assert_array_equal(np.concatenate([g["arrivals"] for g in got]), r["arrivals"])
    slots = np.concatenate([g["recv_slots"] for g in got])
    np.testing.assert_array_equal(np.sort(slots), np.arange(r["pool_hdr"].size))
    hdr = np.empty_like(r["pool_hdr"])
    hdr[slots] = np.concatenate([g["recv_hdr"] for g in got])
    np.testing.assert_array_equal(hdr, r["pool_hdr"])
