"""Benchmark of the pooled-wave MoE dispatch/combine path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload rack]
    python bench.py --impl reference ...        # the CPU oracle as the reference arm
    torchrun --nproc-per-node N bench.py --gpus N ...

One step = route -> dispatch (assign, pack, bucket) -> per-expert op ->
combine -> drop statistics, on one synthetic batch already resident in HBM.
Pooled mode runs route + assignment as one launch and pack + bucketing as
one launch (--dispatch selects the split forms); dropless ragged mode runs
route, assign, pack, bucket.  The metric is routed assignments per second for
dispatch + combine: T*k divided by the device time of every stage but the
expert op, each timed with CUDA events on the launching stream inside the K
timed steps (the
per-expert op runs in every step but is timed apart, since it stands in for
the expert network).  HBM GB/s and the fraction of the measured copy peak use
the algorithmic bytes of those stages.

Multi-GPU: every rank runs its own batch (seed = rank); the path needs no
collective, so scaling is weak and the value is the sum over ranks of T*k
divided by the slowest rank's time.

Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "routed assignments/s and HBM GB/s (% of peak) for dispatch+combine; drop rate"
HBM_DATASHEET_GBS = 8000.0  # B200 HBM3e, vendor figure (context beside the measured peak)
UNIT = "assignments/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="rack")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--dispatch", default="fused", choices=["fused", "split-route", "separate"],
                    help="pooled mode: fused = route+assignment and pack+bucketing as two "
                         "launches; split-route = route, assignment, pack+bucketing; separate = "
                         "route, assignment, pack, bucketing")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=0, help="0: same as --steps")
    ap.add_argument("--cpu-sample-sources", type=int, default=16)
    ap.add_argument("--cpu-sample-reps", type=int, default=3)
    ap.add_argument("--no-graph", action="store_true",
                    help="skip the CUDA-graph timing of the whole forward step")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the backward timing (reported apart from the metric)")
    ap.add_argument("--no-projection", action="store_true",
                    help="skip the latent-projection timing (reported apart from the metric)")
    ap.add_argument("--projection-only", action="store_true",
                    help="time only the tensor-core projections (profiling)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override the batch's token count (profiling a smaller case)")
    ap.add_argument("--balance-only", action="store_true",
                    help="time only the sequence balance term and its gradient (profiling)")
    ap.add_argument("--ep", action="store_true",
                    help="expert parallelism over the GPUs even at one GPU (the default for "
                         "more than one): the R ranks split over the GPUs, the pools "
                         "exchanged by the kernels' peer stores")
    ap.add_argument("--replicas", action="store_true",
                    help="with several GPUs: an independent batch per GPU instead of one "
                         "expert-parallel batch")
    return ap.parse_args()


def measured_tflops():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        return float(json.load(open(p))["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


def time_projection(w, dev, stream, steps: int, b=None):
    """The latent projections on the tensor cores: down (model width 6144 ->
    latent), up (latent -> model width), and the down-projection fused with the
    pack against project-then-pack.  Inputs are seeded random activations and
    random-init weights already in HBM."""
    import torch
    from combine_moe_pw_b200 import moe_pw as mp
    from combine_moe_pw_b200 import synth
    T, D, Dm = w.T, w.D, synth.MODEL_WIDTH
    g = torch.Generator(device=dev).manual_seed(w.seed)
    h = torch.randn(T, Dm, device=dev, generator=g).to(torch.bfloat16).view(torch.int16)
    wd = (torch.randn(D, Dm, device=dev, generator=g) * Dm ** -0.5).to(torch.bfloat16).view(torch.int16)
    wu = (torch.randn(Dm, D, device=dev, generator=g) * D ** -0.5).to(torch.bfloat16).view(torch.int16)
    xl = torch.empty(T, D, dtype=torch.int16, device=dev)
    y = torch.empty(T, Dm, dtype=torch.int16, device=dev)
    ctr = torch.zeros(mp.COUNTERS_BYTES // 8, dtype=torch.int64, device=dev)

    def timed(fn):
        for _ in range(3):
            fn()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        torch.cuda.synchronize(dev)
        for e0, e1 in evs:
            e0.record(stream)
            fn()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        return statistics.median(e0.elapsed_time(e1) for e0, e1 in evs)

    flops = 2.0 * T * D * Dm
    peak, kind = measured_tflops()
    sustained = peak
    pth = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(pth):
        sustained = float(json.load(open(pth)).get("bf16_tflops_sustained", peak))
    out = {"model_width": Dm, "latent_width": D, "tokens": T, "flops_per_gemm": flops,
           "peak_tflops": peak, "peak_sustained_tflops": sustained, "peak_kind": kind}
    ms = timed(lambda: mp.moe_pw_project(h, wd, xl, T, D, Dm, ctr, stream))
    out["down_ms"] = ms
    out["down_tflops"] = flops / ms / 1e9
    ms = timed(lambda: mp.moe_pw_project(xl, wu, y, T, Dm, D, ctr, stream))
    out["up_ms"] = ms
    out["up_tflops"] = flops / ms / 1e9
    out["down_frac"] = out["down_tflops"] / peak
    out["up_frac"] = out["up_tflops"] / peak
    out["down_frac_sustained"] = out["down_tflops"] / sustained
    out["up_frac_sustained"] = out["up_tflops"] / sustained
    if b is not None:
        cfg = b.cfg
        out["project_pack_ms"] = timed(lambda: mp.moe_pw_project_pack(
            cfg, h, wd, Dm, b.idx, b.slot_map, b.occ, b.pool_x, b.pool_hdr, b.counters, stream))

        def two_step():
            mp.moe_pw_project(h, wd, b.x, T, D, Dm, b.counters, stream)
            b.pack(stream)
        out["project_then_pack_ms"] = timed(two_step)
        # the whole routed branch, model width to model width
        lat = torch.empty(T, D, dtype=torch.int16, device=dev)
        out["routed_layer_ms"] = timed(lambda: b.run_routed_layer(h, wd, wu, Dm, lat, y, stream,
                                                                  overlap=False))
        out["routed_layer_tokens_per_s"] = T / (out["routed_layer_ms"] / 1e3)
        # merged with a shared-path output, sequential and with the combine
        # and up-projection overlapped in 8192-token blocks
        sh = torch.randn(T, Dm, device=dev, generator=g).to(torch.bfloat16).view(torch.int16)
        out["routed_layer_merged_ms"] = timed(
            lambda: b.run_routed_layer(h, wd, wu, Dm, lat, y, stream, shared_out=sh,
                                       overlap=False))
        out["routed_layer_merged_overlap_ms"] = timed(
            lambda: b.run_routed_layer(h, wd, wu, Dm, lat, y, stream, shared_out=sh,
                                       overlap=True))
        for chunk in (4096, 8192, 16384):
            out[f"routed_layer_merged_pipelined_{chunk}_ms"] = timed(
                lambda: b.run_routed_layer_pipelined(h, wd, wu, Dm, y, shared_out=sh,
                                                     chunk_tokens=chunk, stream=stream))
        out["routed_layer_merged_pipelined_ms"] = min(
            out[f"routed_layer_merged_pipelined_{c}_ms"] for c in (4096, 8192, 16384))
        del lat, sh
    del h, wd, wu, xl, y
    torch.cuda.empty_cache()
    return out


def time_balance(w, cfg, b, dev, stream, steps: int, world: int):
    """The sequence-level balance term and its gradient on the routed batch
    in b: logits read twice (statistics, gradient), dlogits written once."""
    import torch
    from combine_moe_pw_b200 import moe_pw as mp
    if w.T % w.seq_len != 0:
        return None
    n_seq = w.T // w.seq_len
    bf = torch.empty((n_seq, w.E), dtype=torch.float32, device=dev)
    bP = torch.empty_like(bf)
    bl = torch.empty((n_seq,), dtype=torch.float32, device=dev)
    bd = torch.empty((w.T, w.E), dtype=torch.float32, device=dev)
    bws = torch.empty((max(mp.moe_pw_seq_balance_plan(cfg, w.seq_len), 256),),
                      dtype=torch.uint8, device=dev)

    def bal_step():
        mp.moe_pw_seq_balance(cfg, w.seq_len, 0.01, b.logits, b.idx, bf, bP, bl, bws,
                              dlogits=bd, stream=stream)
    for _ in range(3):
        bal_step()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        bal_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    (bms,) = max_over_ranks([e0.elapsed_time(e1) / steps], world, dev)
    # logits read once, dlogits written once, the ids read once (the counts
    # pass); the per-chunk sums and counts are small
    bbytes = 4 * w.T * w.E + 4 * w.T * w.k + 4 * w.T * w.E
    return {"ms_per_step": bms, "alg_bytes_per_step": bbytes,
            "hbm_gbs": bbytes / (bms / 1e3) / 1e9,
            "hbm_frac_of_peak": bbytes / (bms / 1e3) / 1e9 / measured_peaks()[0],
            "mean_term_alpha_1": float(bl.double().mean().item()) / 0.01,
            "scope": "balance term per sequence and its gradient (ids counted first; "
                     "logits read once, dlogits written)"}


def rank_workload(base, rank: int):
    """Each rank runs its own independent batch: same shape, seed offset by rank."""
    return base.with_(seed=base.seed + rank)


def max_over_ranks(values, world: int, device=None):
    """Element-wise max of per-rank timings (all ranks call it in the same order)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def throughput(units_per_rank_step: int, steps: int, world: int, ms: float) -> float:
    """Whole-job rate: units of all ranks over the slowest rank's time."""
    return units_per_rank_step * steps * world / (ms / 1e3)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def backward_bytes(w, stats, C_s):
    """Algorithmic bytes of the backward stages (K = rows the receiver kept)."""
    T, E, k, D = w.T, w.E, w.k, w.D
    S = w.R * w.R * w.W * C_s if w.mode == 0 else T * k
    K = stats.kept
    combine_bwd = (4 * T * D + 2 * D * K + 2 * D * K + 2 * D * (S - K) + 4 * S + 12 * T * k
                   + 4 * T * E + 4 * T * k)
    expert_bwd = 2 * D * K + 8 * S + S * (2 * D + 4)
    dispatch_bwd = 2 * D * K + 4 * T * D + 4 * T * k + 4 * K
    return {"combine_bwd": combine_bwd, "expert_bwd": expert_bwd, "dispatch_bwd": dispatch_bwd}


def alg_bytes(w, stats, C_s):
    """Algorithmic bytes of route + dispatch + combine (what the method must
    move; the exchange is an index relabel and moves nothing).  K_s = rows the
    sender kept, K = rows the receiver kept."""
    T, E, k, D = w.T, w.E, w.k, w.D
    S = w.R * w.R * w.W * C_s if w.mode == 0 else T * k
    K_s = T * k - stats.sender_dropped
    K = stats.kept
    route = 4 * T * E + 8 * T * k
    assign = 4 * T * k + 4 * T * k                      # read idx, write slot_map
    pack = 2 * T * D + 8 * T * k + S * (2 * D + 4)      # x rows, slot_map + idx, pool rows + headers
    bucket = 8 * S                                      # read headers, write receiver rows
    combine = 8 * T * k + 4 * K_s + 2 * D * K + 4 * T * D
    # fused dispatch: the assignment writes the kept slots' headers; the
    # pack + bucketing launch reads the slot map (not the ids), writes rows
    # and the empty slots' headers, and buckets
    assign_headers = assign + 4 * K_s
    pack_bucket = 2 * T * D + 4 * T * k + S * 2 * D + 4 * (S - K_s) + bucket
    # route + assignment in one launch: the ids stay on chip for the ranking
    route_assign = route + 4 * T * k + 4 * K_s
    return {"route": route, "assign": assign, "pack": pack, "bucket": bucket, "combine": combine,
            "assign_headers": assign_headers, "pack_bucket": pack_bucket,
            "route_assign": route_assign,
            "expert": 2 * D * K + 8 * S + S * (2 * D + 4)}


def metric_bytes(w, stats, C_s):
    """B_alg of the metric: route + dispatch + combine as the method defines
    them (what it must move; the exchange moves nothing):
      route     4TE + 8Tk                      logits in; ids and gates out
      dispatch  4Tk + 2TD + S(2D+4) + 4Tk + 8S ids in; x rows in; pool rows and
                                               headers out; slot map out;
                                               headers in, receiver rows out
      combine   8Tk + 4K_s + 2DK + 4TD         slot map and gates in; return
                                               headers of the sender-kept
                                               assignments in; kept rows in;
                                               fp32 out
    with S pool slots, K_s rows the sender kept and K rows the receiver kept.
    The per-kernel figures of alg_bytes add the metadata each separate kernel
    reads again (the pack's slot map and ids), which a fused dispatch would
    not; the metric leaves those out."""
    T, E, k, D = w.T, w.E, w.k, w.D
    S = w.R * w.R * w.W * C_s if w.mode == 0 else T * k
    K_s = T * k - stats.sender_dropped
    K = stats.kept
    route = 4 * T * E + 8 * T * k
    dispatch = 4 * T * k + 2 * T * D + S * (2 * D + 4) + 4 * T * k + 8 * S
    combine = 8 * T * k + 4 * K_s + 2 * D * K + 4 * T * D
    return route + dispatch + combine


class ClockSampler:
    """nvidia-smi clocks and throttle reasons during the timed region (reads only)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        self.proc.wait(timeout=10)
        rows = [r.split(", ") for r in open(self.path).read().strip().splitlines() if r.strip()]
        os.unlink(self.path)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def traffic_from_profiles(kernel: str, alg_bytes: float):
    """DRAM bytes per launch for ``kernel``, scaled from a committed small-case
    ncu summary: the capture's dram__bytes_read.sum + dram__bytes_write.sum
    over that launch's algorithmic bytes, times this launch's algorithmic
    bytes (the kernel streams its rows once, so its traffic grows in
    proportion).  None unless the kernel source is unchanged since the capture
    (the sha256 of every source file is recorded there)."""
    import hashlib
    import re
    prof = os.path.join(ROOT, "profiles", f"{kernel}_small_case_traffic.txt")
    if not os.path.exists(prof):
        return None
    text = open(prof).read()
    m_r = re.search(r"^traffic_per_algorithmic_byte:\s*([0-9.eE+]+)", text, re.M)
    files = re.findall(r"^source_file:\s*(\S+)", text, re.M)
    hashes = re.findall(r"^source_sha256:\s*([0-9a-f]+)", text, re.M)
    if not (m_r and files and len(files) == len(hashes)):
        return None
    for f, h in zip(files, hashes):  # every source of the kernel unchanged
        src = os.path.join(ROOT, f)
        if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest() != h:
            return None
    return float(m_r.group(1)) * alg_bytes


def host_cpu():
    """The host the oracle is timed on: logical cores and CPU model."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"host_cores": os.cpu_count(), "cpu_model": model}


def cpu_oracle_sample(w, n_src: int, reps: int = 1):
    """Time the CPU oracle (single thread) on the first n_src source shards of
    the batch: route, assignment, pack, bucketing, expert op and combine, run
    `reps` times on the same inputs.  Returns (assignments routed, seconds)."""
    import oracle
    from combine_moe_pw_b200 import synth
    T = n_src * (w.T // w.R)
    ws = w.with_(T=T)
    lg, x, s = synth.logits(ws), synth.x_bf16(ws), synth.scales(w)
    dt = 0.0
    for _ in range(reps):
        t0 = time.perf_counter()
        if w.mode == 0:
            oracle.run(w, lg, x, s, T=T)
        else:
            oracle.run(ws, lg, x, s)
        dt += time.perf_counter() - t0
    return reps * T * w.k, dt


def run_reference(a):
    """Reference arm: the CPU oracle on the host cores, as it stands."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from combine_moe_pw_b200 import synth
    w = synth.WORKLOADS[a.workload]
    n_src = 1
    for _ in range(a.warmup):
        cpu_oracle_sample(w, n_src)
    units, times = 0, []
    for _ in range(a.steps):
        u, dt = cpu_oracle_sample(w, n_src)
        units += u
        times.append(dt)
    total = sum(times)
    value = units / total
    sample = (f"first {n_src} of {w.R} source shards ({n_src * (w.T // w.R)} tokens) of the "
              f"{w.name} batch per step; whole oracle path (route..combine), one thread")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "impl": "reference",
            "n_gpus": a.gpus, "steps": a.steps, "warmup": a.warmup,
            "ms_per_step": 1e3 * total / a.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": sample, **host_cpu()},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_of(w):
    return {"workload": w.name, "tokens": w.T, "experts": w.E, "top_k": w.k, "width": w.D,
            "ranks": w.R, "experts_per_rank": w.L, "waves": w.W,
            "cf_send": w.cf_send_pct / 100 if w.cf_send_pct > 0 else None,
            "cf_recv": w.cf_recv_pct / 100 if w.cf_recv_pct > 0 else None,
            "mode": "pooled" if w.mode == 0 else "ragged",
            "sequences": w.T // w.seq_len, "seq_len": w.seq_len,
            "l2": "inputs larger than L2 (no flush)",
            "metric_scope": "route + assign + pack + bucket + combine; expert op timed apart"}


NVLINK_PEER_GBS = 770.0  # measured peer copy per direction on this machine (900 nominal)


def ep_link_bytes(share, D: int, n: int, kept_send: int, kept_recv: int) -> int:
    """Bytes one GPU sends to the other GPUs per step (and, by symmetry,
    receives): the rows it keeps for other GPUs' experts plus every slot's
    header, and the rows and headers it returns to other GPUs' sources; a
    slot with header -1 sends its header only.  (n - 1) / n of the traffic
    leaves the GPU (its own experts' pools stay local).  kept_send /
    kept_recv: this GPU's share of the rows the senders and receivers kept."""
    rows = (kept_send + kept_recv) * 2 * D + 2 * share.n_slots * 4
    return rows * (n - 1) // n


def run_ep_bench(a, world: int, rank: int, local: int):
    """Expert-parallel run: the rack-shaped batch is split over the GPUs by
    rank, weak scaling (every GPU holds the single-GPU batch's token count,
    so the whole batch has world x that many tokens over the same 64 ranks).
    One step = route, assign, pack and send (per wave, overlapped with the
    previous wave's bucketing and expert op, whose kernel returns the rows),
    combine; barriers are one-element NCCL all-reduces on the step's stream."""
    import torch
    import torch.distributed as dist
    from combine_moe_pw_b200 import ep
    from combine_moe_pw_b200 import moe_pw as mp
    from combine_moe_pw_b200 import synth

    dev = torch.device("cuda", local)
    base = synth.WORKLOADS[a.workload]
    w = base.with_(T=(a.tokens or base.T) * world)
    cfg = mp.Config.from_workload(w)
    b = ep.EpBuffers(cfg, world, rank, dev)
    t = b.share.token_range
    b.logits.copy_(torch.from_numpy(synth.logits_rows(w, t.start, len(t))))
    b.x.copy_(torch.from_numpy(synth.x_bf16_rows(w, t.start, len(t)).view(np.int16)))
    b.scale.copy_(torch.from_numpy(synth.scales(w)))
    torch.cuda.synchronize(dev)
    links = ep.PeerLinks(b, dist.all_gather_object) if world > 1 else None
    one = torch.zeros(1, dtype=torch.int32, device=dev)

    def barrier(stream):
        if world > 1:
            with torch.cuda.stream(stream):
                dist.all_reduce(one)

    sa = torch.cuda.current_stream(dev)
    sb = torch.cuda.Stream(dev)

    def timed(overlap: bool, steps: int):
        for _ in range(max(a.warmup, 3)):
            ep.run_step(b, barrier, sa, sb, overlap)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(sa)
        for _ in range(steps):
            ep.run_step(b, barrier, sa, sb, overlap)
        e1.record(sa)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / steps

    sampler = ClockSampler(local)
    sampler.start()
    ms = timed(True, a.steps)
    clocks = sampler.stop()
    ms_one = timed(False, a.steps)
    st = b.stats(sa)
    counts = torch.tensor([st.assignments, st.kept, st.sender_dropped, st.receiver_dropped,
                           st.error], dtype=torch.int64, device=dev)
    if world > 1:
        dist.all_reduce(counts)
    ms, ms_one = max_over_ranks([ms, ms_one], world, dev)
    TK, kept, sd, rd, err = [int(v) for v in counts.tolist()]
    # both schedules compute the same step; the line reports the faster
    schedule = "waves overlapped" if ms <= ms_one else "one pack for all waves"
    chunk_tokens = min(max(2048 // w.k, 1), w.T // w.R)
    assign_kernels = 2 if -(-(w.T // w.R) // chunk_tokens) <= 32 else 3
    ms_best = min(ms, ms_one)
    value = TK / (ms_best / 1e3)
    link = ep_link_bytes(b.share, w.D, world, (TK - sd) // world, kept // world)

    # end to end: this GPU's inputs from pinned host memory, its output back
    h_lg = b.logits.cpu().pin_memory()
    h_x = b.x.cpu().pin_memory()
    h_out = torch.empty(b.out.shape, dtype=b.out.dtype).pin_memory()

    def e2e_step():
        b.logits.copy_(h_lg, non_blocking=True)
        b.x.copy_(h_x, non_blocking=True)
        ep.run_step(b, barrier, sa, sb, True)
        h_out.copy_(b.out, non_blocking=True)
    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ke = min(a.e2e_steps or a.steps, 10)
    e0.record(sa)
    for _ in range(ke):
        e2e_step()
    e1.record(sa)
    torch.cuda.synchronize(dev)
    (e_ms,) = max_over_ranks([e0.elapsed_time(e1) / ke], world, dev)
    if links is not None:
        torch.cuda.synchronize(dev)
        dist.barrier()
        links.close()
        dist.barrier()
    if rank == 0:
        cfg_out = config_of(w)
        cfg_out.update({"parallelism": f"ep{world}", "tokens_per_gpu": len(t),
                        "schedule": schedule,
                        "metric_scope": "route + assign + pack/send + bucket + expert op/return "
                                        "+ combine: across GPUs the expert kernel carries the "
                                        "return exchange, so it is inside the step"})
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": a.steps, "warmup": max(a.warmup, 3), "ms_per_step": ms_best,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "payload_dtype": "bf16", "data": "synthetic", "config": cfg_out,
            "drop_rate": {"sender": sd / TK, "receiver": rd / TK, "total": (sd + rd) / TK},
            "roofline": {"bound": "nvlink", "achieved": 2 * link / (ms_best / 1e3) / 1e9,
                         "peak": 2 * NVLINK_PEER_GBS, "unit": "GB/s",
                         "frac": (2 * link / (ms_best / 1e3) / 1e9) / (2 * NVLINK_PEER_GBS),
                         "traffic": None,
                         "link_bytes_per_step_per_direction": link,
                         "peak_kind": "measured peer copy, both directions"},
            "ep": {"ms_per_step_waves_overlapped": ms, "ms_per_step_one_pack": ms_one,
                   "barriers_per_step": len(ep.schedule(w.W, True)) - 1},
            # per step of the reported schedule: route, the assignment kernels,
            # a pack, a bucketing and an expert kernel per wave (or one each),
            # the combine (NCCL's own all-reduce kernels not counted)
            "gpu_launches": (2 + assign_kernels + 3 * (w.W if ms <= ms_one else 1)) * a.steps,
            "clocks": clocks,
            "e2e": {"value": TK / (e_ms / 1e3), "unit": UNIT,
                    "h2d_bytes_per_step": h_lg.numel() * 4 + h_x.numel() * 2,
                    "d2h_bytes_per_step": h_out.numel() * 4, "ms_per_step": e_ms},
            "cpu_baseline": None,
            "kept": kept, "device_error": err,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    a = parse()
    if a.impl == "reference":
        run_reference(a)
        return
    import torch
    import torch.distributed as dist

    from combine_moe_pw_b200 import moe_pw as mp
    from combine_moe_pw_b200 import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", device_id=dev, timeout=timedelta(seconds=120))
    if a.ep or (world > 1 and not a.replicas):
        # the exchange stores into the other GPUs' memory: every pair of this
        # node's GPUs must reach each other (NVLink / NVSwitch peer access)
        peers_ok = all(torch.cuda.can_device_access_peer(local, j)
                       for j in range(world) if j != local)
        ok = torch.tensor([1 if peers_ok else 0], dtype=torch.int32, device=dev)
        if world > 1:
            dist.all_reduce(ok, op=dist.ReduceOp.MIN)
        if int(ok.item()) == 1:
            run_ep_bench(a, world, rank, local)
            return
        if rank == 0:
            print("expert-parallel mode needs peer access between every pair of GPUs; "
                  "running independent batches instead", file=sys.stderr, flush=True)

    base = synth.WORKLOADS[a.workload]
    if a.tokens:
        base = base.with_(T=a.tokens, seq_len=min(base.seq_len, a.tokens // base.R * base.R))
    w = rank_workload(base, rank)
    cfg = mp.Config.from_workload(w)
    if a.balance_only:
        # only what the balance term reads: logits and the routing
        from types import SimpleNamespace
        nb = SimpleNamespace(
            logits=torch.from_numpy(synth.logits(w)).to(dev),
            idx=torch.empty((w.T, w.k), dtype=torch.int32, device=dev),
            gates=torch.empty((w.T, w.k), dtype=torch.float32, device=dev))
        stream = torch.cuda.current_stream(dev)
        mp.moe_pw_route(cfg, nb.logits, nb.idx, nb.gates, stream)
        out = time_balance(w, cfg, nb, dev, stream, a.steps, world)
        if rank == 0:
            print(json.dumps({"seq_balance": out, "config": config_of(w)}), flush=True)
        return
    b = mp.Buffers(cfg, device=dev)
    sizes = b.sizes
    lg = synth.logits(w)
    x = synth.x_bf16(w)
    s = synth.scales(w)
    b.logits.copy_(torch.from_numpy(lg))
    b.x.copy_(torch.from_numpy(x.view(np.int16)))
    b.scale.copy_(torch.from_numpy(s))
    stream = torch.cuda.current_stream(dev)
    torch.cuda.synchronize(dev)
    if a.projection_only:
        b.route(stream)
        b.assign(stream)
        proj = time_projection(w, dev, stream, a.steps, b)
        if rank == 0:
            print(json.dumps({"projection": proj}), flush=True)
        return

    mode = a.dispatch if w.mode == 0 else "separate"
    if mode == "fused":
        stages = ["route_assign", "pack_bucket", "expert", "combine"]
        calls = [b.route_assign, b.pack_bucket, b.expert, b.combine]
    elif mode == "split-route":
        stages = ["route", "assign_headers", "pack_bucket", "expert", "combine"]
        calls = [b.route, b.assign_headers, b.pack_bucket, b.expert, b.combine]
    else:
        stages = ["route", "assign", "pack", "bucket", "expert", "combine"]
        calls = [b.route, b.assign, b.pack, b.bucket, b.expert, b.combine]
    fused = mode != "separate"

    def step(evs=None):
        for i, f in enumerate(calls):
            if evs is not None:
                evs[i].record(stream)
            f(stream)
        if evs is not None:
            evs[len(calls)].record(stream)

    # the counters are read after the loops, not per step: a per-step read
    # synchronises the host, and the GPU would then wait for the next step's
    # first launch inside the timed route stage (every step gives the same
    # counters: the path is deterministic)
    for _ in range(max(a.warmup, 3)):
        step()
    st = b.stats(stream)
    # kernels of ours per step.  fused: route + assignment (one clustered
    # launch up to 1,024 tokens per SM, else route and the assignment
    # passes), pack + bucketing, expert, combine.
    # split-route / separate: route; assignment count (+ scan when a source
    # has more than 32 chunks of 2048 assignments, + row offsets in ragged
    # mode) and rank; pack + bucketing, or pack and bucketing; expert; combine
    chunk_tokens = min(max(2048 // w.k, 1), w.T // w.R if w.mode == 0 else w.T)
    chunks_per_source = -(-(w.T // w.R) // chunk_tokens)
    assign_kernels = (2 if chunks_per_source <= 32 else 3) if w.mode == 0 else 4
    one_launch = mode == "fused" and mp.moe_pw_route_assign_plan(cfg) != mp.RA_SEPARATE
    launches_per_step = {"fused": 4 if one_launch else 4 + assign_kernels,
                         "split-route": 4 + assign_kernels,
                         "separate": 5 + assign_kernels}[mode]

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)]
           for _ in range(a.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    start.record(stream)
    for i in range(a.steps):
        step(evs[i])
    end.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    st = b.stats(stream)

    # the whole forward step (expert op included) as one CUDA graph, against
    # the same step launched call by call
    graph = None
    if not a.no_graph:
        g = b.capture_step()
        for _ in range(3):
            g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(a.steps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        g_ms = e0.elapsed_time(e1) / a.steps
        e0.record(stream)
        for _ in range(a.steps):
            b.run_step(stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        eager_ms = e0.elapsed_time(e1) / a.steps
        g_ms, eager_ms = max_over_ranks([g_ms, eager_ms], world, dev)
        graph = {"ms_per_step": g_ms, "eager_ms_per_step": eager_ms,
                 "scope": "route, dispatch, expert op, combine (whole forward step)",
                 "host_launches_per_step": 1}
        del g

    total_ms = start.elapsed_time(end)
    per_stage = {n: [evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(a.steps)]
                 for j, n in enumerate(stages)}
    dc_stages = [n for n in stages if n != "expert"]
    dc_ms = sum(sum(per_stage[n]) for n in dc_stages)  # over K steps
    total_ms, dc_ms = max_over_ranks([total_ms, dc_ms], world, dev)
    value = throughput(w.T * w.k, a.steps, world, dc_ms)
    ab = alg_bytes(w, st, sizes.C_s)
    b_alg = metric_bytes(w, st, sizes.C_s)
    peak, peak_kind = measured_peaks()
    gbs = b_alg * a.steps / (dc_ms / 1e3) / 1e9
    stage_ms = {n: statistics.mean(v) for n, v in per_stage.items()}
    pack_stage = "pack_bucket" if fused else "pack"
    dom = max([pack_stage, "combine"], key=lambda n: stage_ms[n])
    kname = {"pack": "pack_kernel", "pack_bucket": "pack_bucket_kernel",
             "combine": "combine_kernel"}[dom]
    achieved = ab[dom] / (stage_ms[dom] / 1e3) / 1e9
    traffic = traffic_from_profiles(kname, ab[dom])

    # backward (gradient of dispatch/combine), timed in its own loop
    bwd = None
    if not a.no_backward:
        b.alloc_backward()
        b.dout.copy_(torch.from_numpy(synth.dout(w)))  # host copy freed right away
        names = ["combine_bwd", "expert_bwd", "dispatch_bwd"]

        def bstep(ev=None):
            if ev is not None:
                ev[0].record(stream)
            mp.moe_pw_combine_backward(cfg, b.dout, b.ret_x, b.ret_hdr, b.slot_map, b.idx,
                                       b.gates, b.d_ret, b.dgates, b.dlogits, b.counters, stream)
            if ev is not None:
                ev[1].record(stream)
            mp.moe_pw_expert(cfg, b.d_ret, b.pool_hdr, b.recv_row, b.scale, b.d_pool,
                             b.d_pool_hdr, b.counters, stream)
            if ev is not None:
                ev[2].record(stream)
            mp.moe_pw_dispatch_backward(cfg, b.d_pool, b.recv_row, b.slot_map, b.dx, b.counters,
                                        stream)
            if ev is not None:
                ev[3].record(stream)

        for _ in range(3):
            bstep()
        bev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(a.steps)]
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        for i in range(a.steps):
            bstep(bev[i])
        torch.cuda.synchronize(dev)
        bms = {n: statistics.mean(bev[i][j].elapsed_time(bev[i][j + 1]) for i in range(a.steps))
               for j, n in enumerate(names)}
        bb = backward_bytes(w, st, sizes.C_s)
        tot_ms = max_over_ranks([sum(bms.values())], world, dev)[0]
        bwd = {"ms_per_step": tot_ms, "stage_ms": bms,
               "value": throughput(w.T * w.k, 1, world, tot_ms), "unit": UNIT,
               "hbm_gbs": sum(bb.values()) / (tot_ms / 1e3) / 1e9,
               "hbm_frac_of_peak": sum(bb.values()) / (tot_ms / 1e3) / 1e9 / measured_peaks()[0],
               "alg_bytes_per_step": sum(bb.values()),
               "stage_gbs": {n: bb[n] / (bms[n] / 1e3) / 1e9 for n in names}}
        del b.d_ret, b.d_pool, b.dout, b.dlogits, b.dx
        torch.cuda.empty_cache()

    # sequence-level balance term and its gradient (reported apart)
    bal = None
    if not a.no_backward:
        bal = time_balance(w, cfg, b, dev, stream, a.steps, world)

    proj = None
    if not a.no_projection:
        proj = time_projection(w, dev, stream, min(a.steps, 10), b)

    # end to end through the public API: pinned host inputs in, result out, every step.
    # The headline runs the batches through moe_pw.Pipeline (host copies of
    # neighbouring batches overlapped with compute); a short one-batch-at-a-time
    # run is reported beside it.
    e2e = None
    if not a.no_e2e:
        ke = a.e2e_steps or a.steps
        h_lg = torch.from_numpy(lg).pin_memory()
        h_x = torch.from_numpy(x.view(np.int16)).pin_memory()
        h_s = torch.from_numpy(s).pin_memory()
        h2d = h_lg.numel() * 4 + h_x.numel() * 2 + h_s.numel() * 4
        d2h = w.T * w.D * 4 + mp.COUNTERS_BYTES

        # one batch at a time on one buffer set
        h_out = torch.empty(b.out.shape, dtype=b.out.dtype).pin_memory()

        h_ctr = torch.empty_like(b.counters, device="cpu").pin_memory()
        dev_bufs = b.device_buffers()

        def e2e_step():
            # the C-ABI step with host buffers: upload, path, download, on one stream
            mp.moe_pw_step_host(cfg, h_lg, h_x, h_s, h_out, h_ctr, dev_bufs, stream)
            stream.synchronize()  # the step's result is on the host

        for _ in range(2):
            e2e_step()
        ks = min(ke, 5)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(ks):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        serial_ms = e0.elapsed_time(e1) / ks
        del b
        torch.cuda.empty_cache()

        # pipelined
        # one pinned result buffer: the downloads are ordered on the copy-out
        # stream, so consecutive batches never write it at the same time
        pipe = mp.Pipeline(cfg, device=dev, depth=2)
        h_outs = [h_out, h_out]
        for i in range(2):
            pipe.submit(h_lg, h_x, h_s, h_outs[i % 2])
        pipe.synchronize()
        if world > 1:
            dist.barrier()
        p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        p0.record(pipe.s_in)
        for i in range(ke):
            pipe.submit(h_lg, h_x, h_s, h_outs[i % 2])
        p1.record(pipe.s_out)
        pipe.synchronize()
        (e_ms,) = max_over_ranks([p0.elapsed_time(p1)], world, dev)
        e2e = {"value": throughput(w.T * w.k, ke, world, e_ms), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e_ms / ke, "pipeline_depth": 2,
               "api": "moe_pw_step_host (C ABI, host buffers in and out)",
               "serial_ms_per_step": serial_ms,
               "serial_value": throughput(w.T * w.k, 1, world, serial_ms)}
        del pipe

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        u, dt = cpu_oracle_sample(base, a.cpu_sample_sources, a.cpu_sample_reps)
        cpu = {"value": u / dt, "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": f"first {a.cpu_sample_sources} of {base.R} source shards "
                         f"({a.cpu_sample_sources * (base.T // base.R)} tokens) of the {base.name} "
                         f"batch, whole oracle path (route..combine), one thread, "
                         f"{a.cpu_sample_reps} runs on the same inputs, {dt:.1f} s in all",
               **host_cpu()}

    if rank == 0:
        TK = w.T * w.k
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": a.steps, "warmup": max(a.warmup, 3),
            "ms_per_step": total_ms / a.steps,
            "ms_dispatch_combine_per_step": dc_ms / a.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "payload_dtype": "bf16", "data": "synthetic",
            "config": config_of(w),
            "hbm_gbs": gbs, "hbm_frac_of_peak": gbs / peak, "hbm_peak_gbs": peak,
            "hbm_peak_kind": peak_kind,
            "hbm_datasheet_gbs": HBM_DATASHEET_GBS, "hbm_frac_of_datasheet": gbs / HBM_DATASHEET_GBS,
            "alg_bytes_per_step": b_alg,
            "drop_rate": {"sender": st.sender_dropped / TK, "receiver": st.receiver_dropped / TK,
                          "total": (st.sender_dropped + st.receiver_dropped) / TK},
            # the same time per assignment the receivers kept (dropped ones
            # move no combine bytes)
            "kept_assignments_per_s": throughput(st.kept, a.steps, world, dc_ms),
            "stage_ms": stage_ms,
            "roofline": {"bound": "hbm", "kernel": kname, "achieved": achieved, "peak": peak,
                         "unit": "GB/s", "frac": achieved / peak, "traffic": traffic,
                         "alg_bytes_per_launch": ab[dom], "peak_kind": peak_kind,
                         "traffic_source": "32,768-token capture of the same kernel, scaled by "
                                           "algorithmic bytes" if traffic else None},
            "gpu_launches": launches_per_step * a.steps,
            "graph": graph,
            "backward": bwd,
            "seq_balance": bal,
            "projection": proj,
            "clocks": clocks,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
