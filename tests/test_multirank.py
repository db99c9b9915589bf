"""Host logic of the multi-rank bench on CPU: 2 gloo ranks.

Every rank runs its own independent batch (no collective on the data path);
only the timings meet, as a max over ranks, and the whole-job rate divides
all ranks' units by the slowest rank's time.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp_

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    from combine_moe_pw_b200 import synth
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        w = bench.rank_workload(synth.WORKLOADS["rack"], rank)
        local = [10.0 + 5 * rank, 3.0 - rank]  # rank 1 is slower overall, faster in part
        got = bench.max_over_ranks(local, world)
        rate = bench.throughput(w.T * w.k, 20, world, got[0])
        q.put((rank, w.seed, got, rate))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_reduction():
    ctx = mp_.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    out = sorted(q.get() for _ in range(2))
    (r0, s0, g0, v0), (r1, s1, g1, v1) = out
    assert (s0, s1) == (0, 1)                  # independent batches
    assert g0 == g1 == [15.0, 3.0]             # element-wise max over ranks
    assert v0 == v1 == pytest.approx(262144 * 8 * 20 * 2 / 0.015)


def test_reference_arm_other_ranks_do_no_work(monkeypatch, capsys):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--gpus", "2",
                                      "--steps", "1", "--warmup", "0"])
    bench.main()
    assert capsys.readouterr().out == ""


def test_metric_bytes_match_the_definition_and_the_rack_upper_bound():
    """B_alg of the metric, written out term by term from its definition, and
    its value at K = T k for the rack batch (262,144 x 3072, C_s = 188):
    32,399,360,000 bytes, the 32.40 GB upper bound of the scope table."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from combine_moe_pw_b200 import synth

    class St:
        sender_dropped = 0
        kept = 0

    w = synth.WORKLOADS["rack"]
    T, E, k, D = w.T, w.E, w.k, w.D
    st = St()
    st.kept = T * k
    assert bench.metric_bytes(w, st, 188) == 32_399_360_000
    # with drops: every term that depends on K_s or K moves by its row bytes
    st.sender_dropped, st.kept = 1000, T * k - 1500
    assert bench.metric_bytes(w, st, 188) == 32_399_360_000 - 4 * 1000 - 2 * D * 1500
    # the per-kernel figures add only the pack's second read of ids and slot map
    ab = bench.alg_bytes(w, st, 188)
    dc = sum(ab[n] for n in ("route", "assign", "pack", "bucket", "combine"))
    assert dc - bench.metric_bytes(w, st, 188) == 8 * T * k
