"""GPU path against the CPU oracle, element by element, through the C ABI.

Bar: bit-exact for every integer/byte output (top-k ids, slot maps, pool
occupancy, pool rows and headers, receiver rows, buckets, per-expert counts,
returned rows and headers, drop counts); the fp32 gates within 1e-6 relative;
the fp32 combine within 1e-6 of sum_j g_j |y_j| (the combine's own scale, so
cancelling terms do not make the bound meaningless; where that scale is 0 the
output must be exactly 0).

Small cases run the whole oracle.  Full-size cases (the pages' shapes) run
the oracle's integer path completely and check rows on sampled slots and the
combine on sampled tokens, in the same launch configuration bench.py times.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_moe_pw_b200 import moe_pw as mp
from combine_moe_pw_b200 import synth

pytestmark = pytest.mark.gpu

GATE_RTOL = 1e-6
COMBINE_TOL = 1e-6


def _inputs(w, logits=None):
    lg = synth.logits(w) if logits is None else logits
    return lg, synth.x_bf16(w), synth.scales(w)


def run_gpu(w, lg, x, s, sub_steps=False):
    cfg = mp.Config.from_workload(w)
    b = mp.Buffers(cfg)
    b.logits.copy_(torch.from_numpy(lg))
    b.x.copy_(torch.from_numpy(x.view(np.int16)))
    b.scale.copy_(torch.from_numpy(s))
    if sub_steps:
        b.route()
        b.assign()
        b.pack()
        b.bucket()
        b.expert()
        b.combine()
    else:
        b.run_step()
    st = b.stats(raise_on_device_error=False)
    torch.cuda.synchronize()
    return b, st


def _np(t):
    return t.cpu().numpy()


def _u16(t):
    return t.cpu().numpy().view(np.uint16)


def check_gates(g_gpu, g_ref):
    rel = np.abs(g_gpu.astype(np.float64) - g_ref) / g_ref
    assert rel.max() <= GATE_RTOL, f"gate rel err {rel.max():.3e}"


def check_combine(out_gpu, ref, mag):
    diff = np.abs(out_gpu.astype(np.float64) - ref)
    zero = mag == 0
    assert not diff[zero].any(), "output must be exactly 0 where every term is 0"
    err = (diff[~zero] / mag[~zero]).max() if (~zero).any() else 0.0
    assert err <= COMBINE_TOL, f"combine err {err:.3e}"
    return err


def check_full(w, lg, x, s, b, st):
    """Every output against the whole oracle."""
    r = oracle.run(w, lg, x, s, with_mag=True)
    g = r["geom"]
    np.testing.assert_array_equal(_np(b.idx), r["idx"])
    check_gates(_np(b.gates), r["gates"])
    np.testing.assert_array_equal(_np(b.slot_map), r["slot_map"])
    if w.mode == synth.MODE_POOLED:
        np.testing.assert_array_equal(_np(b.occ)[: g.n_pools], r["occ"].reshape(-1))
        np.testing.assert_array_equal(_np(b.bucket_slot)[: w.E * g.C_r], r["bucket_slot"].reshape(-1))
    else:
        np.testing.assert_array_equal(_np(b.occ)[: w.E + 1], r["row_off"])
    np.testing.assert_array_equal(_u16(b.pool_x), r["pool_x"])
    np.testing.assert_array_equal(_np(b.pool_hdr), r["pool_hdr"])
    np.testing.assert_array_equal(_np(b.recv_row), r["recv_row"])
    ec = _np(b.expert_counts)
    np.testing.assert_array_equal(ec[0], r["arrivals"])
    np.testing.assert_array_equal(ec[1], r["bucket_cnt"])
    # the host copy moe_pw_stats made of the per-expert counts
    np.testing.assert_array_equal(b.host_expert_counts[0], r["arrivals"])
    np.testing.assert_array_equal(b.host_expert_counts[1], r["bucket_cnt"])
    np.testing.assert_array_equal(_u16(b.ret_x), r["ret_x"])
    np.testing.assert_array_equal(_np(b.ret_hdr), r["ret_hdr"])
    err = check_combine(_np(b.out), r["out"], r["mag"])
    assert st.error == 0
    assert (st.sender_dropped, st.receiver_dropped, st.kept) == (
        r["sender_dropped"], r["receiver_dropped"], r["kept"])
    assert st.assignments == w.T * w.k
    assert st.kept + st.sender_dropped + st.receiver_dropped == w.T * w.k
    return r, err


def check_sampled(w, lg, x, s, b, st, n_tok=1024, n_slot=8192, seed=0):
    """Integer path in full, rows and combine on samples (oracle per slot /
    per token)."""
    r = oracle.run_headers(w, lg)
    g = r["geom"]
    np.testing.assert_array_equal(_np(b.idx), r["idx"])
    check_gates(_np(b.gates), r["gates"])
    np.testing.assert_array_equal(_np(b.slot_map), r["slot_map"])
    if w.mode == synth.MODE_POOLED:
        np.testing.assert_array_equal(_np(b.occ)[: g.n_pools], r["occ"].reshape(-1))
        np.testing.assert_array_equal(_np(b.bucket_slot)[: w.E * g.C_r], r["bucket_slot"].reshape(-1))
    else:
        np.testing.assert_array_equal(_np(b.occ)[: w.E + 1], r["row_off"])
    np.testing.assert_array_equal(_np(b.pool_hdr), r["pool_hdr"])
    np.testing.assert_array_equal(_np(b.recv_row), r["recv_row"])
    ec = _np(b.expert_counts)
    np.testing.assert_array_equal(ec[0], r["arrivals"])
    np.testing.assert_array_equal(ec[1], r["bucket_cnt"])
    # the host copy moe_pw_stats made of the per-expert counts
    np.testing.assert_array_equal(b.host_expert_counts[0], r["arrivals"])
    np.testing.assert_array_equal(b.host_expert_counts[1], r["bucket_cnt"])
    assert (st.sender_dropped, st.receiver_dropped, st.kept, st.error) == (
        r["sender_dropped"], r["receiver_dropped"], r["kept"], 0)

    rng = np.random.default_rng(seed)
    n_slots = r["pool_hdr"].size
    slots = np.unique(np.concatenate([rng.integers(0, n_slots, n_slot), [0, n_slots - 1]]))
    st_idx = torch.from_numpy(slots).to(b.pool_x.device)
    pool_rows = _u16(b.pool_x.index_select(0, st_idx))
    ret_rows = _u16(b.ret_x.index_select(0, st_idx))
    tok = r["slot_tok"][slots]
    full = tok >= 0
    exp_pool = np.zeros_like(pool_rows)
    exp_pool[full] = x[tok[full]]
    np.testing.assert_array_equal(pool_rows, exp_pool)
    kept = r["recv_row"][slots] >= 0
    exp_ret = np.zeros_like(ret_rows)
    e = r["pool_hdr"][slots][kept]
    exp_ret[kept] = oracle.expert_product(np.repeat(s[e][:, None], w.D, axis=1), x[tok[kept]])
    np.testing.assert_array_equal(ret_rows, exp_ret)
    np.testing.assert_array_equal(_np(b.ret_hdr)[slots], np.where(kept, r["pool_hdr"][slots], -1))

    toks = np.unique(np.concatenate([rng.integers(0, w.T, n_tok), [0, w.T - 1]]))
    ref, mag = oracle.combine_tokens(g, x, r["idx"], r["gates"], r["slot_map"], r["recv_row"], s,
                                     toks)
    out = _np(b.out[torch.from_numpy(toks).to(b.out.device)])
    return r, check_combine(out, ref, mag)


# ---------------------------------------------------------------------------
# small cases, whole oracle
# ---------------------------------------------------------------------------

TINY = synth.WORKLOADS["tiny"]

SMALL_CASES = {
    "tiny": TINY,
    "tiny_ragged": TINY.with_(mode=synth.MODE_RAGGED, cf_send_pct=0, cf_recv_pct=0),
    "tiny_ragged_zipf": TINY.with_(mode=synth.MODE_RAGGED, cf_send_pct=0, cf_recv_pct=0,
                                   logit_kind=synth.LOGIT_ZIPF),
    "tiny_unbounded": TINY.with_(cf_send_pct=0, cf_recv_pct=0),
    "tiny_tight": TINY.with_(cf_send_pct=60, cf_recv_pct=70),
    "tiny_zipf": TINY.with_(logit_kind=synth.LOGIT_ZIPF),
    "tiny_seqbias": TINY.with_(logit_kind=synth.LOGIT_SEQBIAS),
    "k1": TINY.with_(k=1),
    "k4": TINY.with_(k=4),
    "k16": TINY.with_(k=16),
    "k32": TINY.with_(k=32),
    "min_width": TINY.with_(D=8),
    "odd_width": TINY.with_(D=136),
    # 8928: the widest row the expert op streams through its shared-memory
    # ring (13 row buffers in one block's 227 KB); 6144: one ring block per
    # SM (156 KB); 12288 takes its register-copy kernel
    "ring_max_width": TINY.with_(T=256, D=8928),
    "ring_one_block_per_sm": TINY.with_(T=256, D=6144),
    "max_width": TINY.with_(T=256, D=12288),
    "single_pool": TINY.with_(R=1, L=16, W=1, P=16, T=512, cf_send_pct=30),
    "ragged_tail": TINY.with_(T=8 * 37, seq_len=37),
    "ragged_tail_ragged": TINY.with_(T=8 * 37, seq_len=37, mode=synth.MODE_RAGGED,
                                     cf_send_pct=0, cf_recv_pct=0),
    "many_chunks": TINY.with_(T=8 * 1000 + 0, seq_len=1000, D=64),
    # 40 chunks per source: the assignment's separate scan pass (at most 32
    # chunks per source are summed inside the rank pass instead)
    "long_sources": synth.Workload("long_sources", T=2 * 10000, R=2, L=6, W=3, P=2, k=8, D=16,
                                   seq_len=10000, logit_kind=synth.LOGIT_SEQBIAS),
    "wide_E": synth.Workload("wide_E", T=64 * 24, R=64, L=16, W=4, P=4, k=8, D=64, seq_len=24,
                             logit_kind=synth.LOGIT_SEQBIAS),
    "E2048": synth.Workload("E2048", T=256 * 8, R=256, L=8, W=4, P=2, k=8, D=32, seq_len=64,
                            logit_kind=synth.LOGIT_IID),
    "pages_ranks_small": synth.Workload("pages_ranks_small", T=64 * 64, R=64, L=6, W=3, P=2, k=8,
                                        D=256, seq_len=1024, logit_kind=synth.LOGIT_SEQBIAS),
    # 32 experts per wave, the most a receiver bucket item takes
    "max_P": synth.Workload("max_P", T=2 * 512, R=2, L=64, W=2, P=32, k=8, D=64, seq_len=512,
                            logit_kind=synth.LOGIT_ZIPF, cf_send_pct=80, cf_recv_pct=90),
}


@pytest.mark.parametrize("name", list(SMALL_CASES))
def test_small_full_parity(name):
    w = SMALL_CASES[name]
    lg, x, s = _inputs(w)
    b, st = run_gpu(w, lg, x, s)
    check_full(w, lg, x, s, b, st)


def test_ties_quantised_logits():
    lg, x, s = _inputs(TINY)
    lg = (np.round(lg * 2) / 2).astype(np.float32)  # many exact ties
    lg[::7, 5] = -0.0
    lg[::7, 9] = 0.0
    b, st = run_gpu(TINY, lg, x, s)
    check_full(TINY, lg, x, s, b, st)


def test_all_equal_logits_closed_form():
    lg, x, s = _inputs(TINY)
    lg = np.full_like(lg, 0.25)
    b, st = run_gpu(TINY, lg, x, s)
    np.testing.assert_array_equal(_np(b.idx), np.tile(np.arange(8, dtype=np.int32), (TINY.T, 1)))
    assert np.all(_np(b.gates) == np.float32(0.125))  # exp(0)/8 exactly
    check_full(TINY, lg, x, s, b, st)


def test_identity_experts_return_x():
    """Unbounded capacity and s_e = 1: out = x * sum_j g_j, within a few fp32 ulp of x."""
    w = TINY.with_(cf_send_pct=0, cf_recv_pct=0)
    lg, x, _ = _inputs(w)
    s = np.ones(w.E, np.float32)
    b, st = run_gpu(w, lg, x, s)
    assert st.sender_dropped == st.receiver_dropped == 0
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    np.testing.assert_allclose(_np(b.out), xf, rtol=8 * 2.0 ** -23, atol=0)


def test_sub_steps_equal_dispatch():
    lg, x, s = _inputs(TINY)
    b1, st1 = run_gpu(TINY, lg, x, s)
    b2, st2 = run_gpu(TINY, lg, x, s, sub_steps=True)
    for name in ["idx", "gates", "slot_map", "occ", "pool_x", "pool_hdr", "recv_row",
                 "bucket_slot", "expert_counts", "ret_x", "ret_hdr", "out"]:
        assert torch.equal(getattr(b1, name), getattr(b2, name)), name


def test_deterministic_repeat():
    """Two runs, one on a side stream, give the same bytes everywhere."""
    w = synth.WORKLOADS["tiny"].with_(T=8 * 2048, seq_len=2048, D=256)
    lg, x, s = _inputs(w)
    b1, _ = run_gpu(w, lg, x, s)
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        b2, _ = run_gpu(w, lg, x, s)
    side.synchronize()
    for name in ["idx", "gates", "slot_map", "occ", "pool_x", "pool_hdr", "recv_row",
                 "bucket_slot", "expert_counts", "ret_x", "ret_hdr", "out"]:
        assert torch.equal(getattr(b1, name), getattr(b2, name)), name


def test_repeated_pack_refills_every_tail():
    """The pack's zero-fill phase hands pools out from a counter that the
    library resets before each launch: a second pack without a new assignment
    pass (pools poisoned in between) rebuilds the same pools byte for byte."""
    w = TINY.with_(T=8 * 1024, seq_len=1024, D=256, logit_kind=synth.LOGIT_SEQBIAS)
    lg, x, s = _inputs(w)
    b, _ = run_gpu(w, lg, x, s)
    ref_x, ref_hdr = b.pool_x.clone(), b.pool_hdr.clone()
    assert (ref_hdr < 0).any()  # there are empty tails to refill
    for _ in range(2):
        b.pool_x.fill_(0x1357)
        b.pool_hdr.fill_(-9)
        b.pack()
        torch.cuda.synchronize()
        assert torch.equal(b.pool_x, ref_x) and torch.equal(b.pool_hdr, ref_hdr)
    assert b.stats().error == 0


def test_empty_batch():
    for mode in (synth.MODE_POOLED, synth.MODE_RAGGED):
        w = TINY.with_(T=0, mode=mode)
        cfg = mp.Config.from_workload(w)
        b = mp.Buffers(cfg)
        b.expert_counts.fill_(7)
        b.run_step()
        st = b.stats()
        assert (st.assignments, st.kept, st.sender_dropped, st.receiver_dropped) == (0, 0, 0, 0)
        assert int(b.expert_counts.abs().sum()) == 0


def test_bad_expert_ids_are_flagged_not_faulted():
    """idx entries outside [0, E) are caught by the assignment kernels'
    bounds checks: the assignment gets no slot and the error bit is set."""
    lg, x, s = _inputs(TINY)
    cfg = mp.Config.from_workload(TINY)
    b = mp.Buffers(cfg)
    b.logits.copy_(torch.from_numpy(lg))
    b.x.copy_(torch.from_numpy(x.view(np.int16)))
    b.route()
    b.idx[5, 3] = -7
    b.idx[100, 0] = TINY.E + 3
    b.assign()
    b.pack()
    b.bucket()
    st = b.stats(raise_on_device_error=False)
    assert st.error & mp.DEVERR_EXPERT_ID
    assert int(b.slot_map[5, 3]) == -1 and int(b.slot_map[100, 0]) == -1
    with pytest.raises(mp.MoePwError) as ei:
        b.stats()
    assert ei.value.code == mp.MOE_PW_EDEVICE


def test_bad_slot_in_combine_is_flagged():
    lg, x, s = _inputs(TINY)
    b, st = run_gpu(TINY, lg, x, s)
    ref = b.out.clone()
    b.slot_map[3, 2] = int(b.pool_hdr.numel()) + 5
    b.combine()
    st = b.stats(raise_on_device_error=False)
    assert st.error & mp.DEVERR_SLOT
    assert torch.equal(b.out[:3], ref[:3]) and torch.equal(b.out[4:], ref[4:])


# ---------------------------------------------------------------------------
# the pages' shapes, bench launch configuration, sampled rows
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["layer", "rack", "long", "ragged"])
def test_full_size_sampled_parity(name):
    w = synth.WORKLOADS[name]
    lg, x, s = _inputs(w)
    b, st = run_gpu(w, lg, x, s)
    r, err = check_sampled(w, lg, x, s, b, st)
    if name == "long":  # fewer, longer sequences -> worse balance than the rack batch
        rr = oracle.run_headers(synth.WORKLOADS["rack"], synth.logits(synth.WORKLOADS["rack"]))
        assert r["sender_dropped"] + r["receiver_dropped"] > rr["sender_dropped"] + rr["receiver_dropped"]
    if name == "ragged":
        assert r["kept"] == w.T * w.k
    del b
    torch.cuda.empty_cache()


def test_combine_bf16_is_rounded_fp32_combine():
    """The bf16 combine is the fp32 combine rounded to nearest-even, bit for bit."""
    lg, x, s = _inputs(TINY)
    b, st = run_gpu(TINY, lg, x, s)
    out16 = torch.empty((TINY.T, TINY.D), dtype=torch.int16, device="cuda")
    mp.moe_pw_combine_bf16(b.cfg, b.ret_x, b.ret_hdr, b.slot_map, b.gates, out16, b.counters)
    torch.cuda.synchronize()
    ref = b.out.to(torch.bfloat16).view(torch.int16)
    assert torch.equal(out16, ref)


def test_bounded_wait_times_out_and_context_survives():
    """A wait nothing satisfies gives up after its bound and reports
    MOE_PW_DEVERR_TIMEOUT; the next real step on the same context is exact."""
    cfg = mp.Config.from_workload(TINY)
    ctr = torch.zeros((mp.COUNTERS_BYTES // 8,), dtype=torch.int64, device="cuda")
    mp.moe_pw_selftest_wait_timeout(ctr, polls=4096)
    st = mp.moe_pw_stats(cfg, ctr, raise_on_device_error=False)
    assert st.error & mp.DEVERR_TIMEOUT
    lg, x, s = _inputs(TINY)
    b, st = run_gpu(TINY, lg, x, s)
    check_full(TINY, lg, x, s, b, st)


def test_pipeline_matches_single_steps():
    """Batches streamed through the overlapped pipeline give the same bytes as
    one step at a time."""
    ws = [TINY.with_(seed=i) for i in range(5)]
    cfg = mp.Config.from_workload(TINY)
    pipe = mp.Pipeline(cfg, depth=2)
    outs, ctrs = [], []
    for w in ws:
        lg, x, s = _inputs(w)
        h_out = torch.empty((w.T, w.D), dtype=torch.float32).pin_memory()
        k = pipe.submit(torch.from_numpy(lg).pin_memory(),
                        torch.from_numpy(x.view(np.int16)).pin_memory(),
                        torch.from_numpy(s).pin_memory(), h_out)
        outs.append(h_out)
    pipe.synchronize()
    for w, h_out in zip(ws, outs):
        lg, x, s = _inputs(w)
        b, st = run_gpu(w, lg, x, s)
        assert torch.equal(h_out, b.out.cpu())
    last = pipe.stats((len(ws) - 1) % 2)
    assert last.error == 0 and last.kept > 0


def test_step_host_equals_device_step():
    """moe_pw_step_host (host buffers in and out, one C call): the same
    output and counters as the step on device buffers, on one stream and on
    three."""
    for name in ("tiny", "tiny_ragged"):
        w = SMALL_CASES[name]
        lg, x, s = _inputs(w)
        ref, st = run_gpu(w, lg, x, s)
        cfg = mp.Config.from_workload(w)
        b = mp.Buffers(cfg)
        h_lg = torch.from_numpy(lg).pin_memory()
        h_x = torch.from_numpy(x.view(np.int16)).pin_memory()
        h_s = torch.from_numpy(s).pin_memory()
        for streams in (1, 3):
            h_out = torch.full((w.T, w.D), 7.0, dtype=torch.float32).pin_memory()
            h_ctr = torch.zeros((mp.COUNTERS_BYTES // 8,), dtype=torch.int64).pin_memory()
            extra = [torch.cuda.Stream(), torch.cuda.Stream()] if streams == 3 else [None, None]
            mp.moe_pw_step_host(cfg, h_lg, h_x, h_s, h_out, h_ctr, b.device_buffers(),
                                torch.cuda.current_stream(), *extra)
            torch.cuda.synchronize()
            assert torch.equal(h_out, ref.out.cpu())
            c = mp.moe_pw_counters.from_buffer_copy(h_ctr.numpy().tobytes())
            assert (c.kept, c.sender_dropped, c.receiver_dropped, c.error) == (
                st.kept, st.sender_dropped, st.receiver_dropped, 0)


def test_captured_step_replays_bit_identical():
    """The forward step recorded as a CUDA graph: a replay equals an eager
    step byte for byte, and after new inputs are copied into the same
    buffers the replay equals an eager step on those inputs."""
    w = TINY.with_(T=8 * 1024, seq_len=1024, D=256, logit_kind=synth.LOGIT_SEQBIAS)
    names = ["idx", "gates", "slot_map", "occ", "pool_x", "pool_hdr", "recv_row",
             "bucket_slot", "expert_counts", "ret_x", "ret_hdr", "out"]
    lg, x, s = _inputs(w)
    ref, _ = run_gpu(w, lg, x, s)
    b, _ = run_gpu(w, lg, x, s)
    graph = b.capture_step()
    for n in names:
        getattr(b, n).fill_(0x55 if getattr(b, n).dtype != torch.float32 else 7.0)
    graph.replay()
    torch.cuda.synchronize()
    for n in names:
        assert torch.equal(getattr(b, n), getattr(ref, n)), n
    assert b.stats().error == 0
    w2 = w.with_(seed=5)
    lg2, x2, s2 = _inputs(w2)
    ref2, _ = run_gpu(w2, lg2, x2, s2)
    b.logits.copy_(torch.from_numpy(lg2))
    b.x.copy_(torch.from_numpy(x2.view(np.int16)))
    b.scale.copy_(torch.from_numpy(s2))
    graph.replay()
    torch.cuda.synchronize()
    for n in names:
        assert torch.equal(getattr(b, n), getattr(ref2, n)), n
    st, st2 = b.stats(), ref2.stats()
    assert (st.kept, st.sender_dropped, st.receiver_dropped) == (
        st2.kept, st2.sender_dropped, st2.receiver_dropped)
