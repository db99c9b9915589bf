"""Expert parallelism over several GPUs: the pooled-wave exchange carried out
by the pack and expert kernels themselves, over peer memory.

"Marin 开始公开训练 535B 参数 MoE 模型", section 二: the 384 experts sit on a
64-GPU expert-parallel domain, 6 per GPU, and each sender ships fixed pools,
one per destination, in three waves of identical shape with the expert id in
the payload.  The huxiu article's JAX section adds that the exchange has to
overlap the expert compute.  Here the R logical ranks of a batch are spread
over ``n_gpus`` GPUs (include/moe_pw.h, "Expert parallelism over several
GPUs", gives the layouts): GPU g owns the token shards and the experts of the
ranks [g*Rn, (g+1)*Rn).  ``moe_pw_ep_pack`` stores each kept row straight into
the receive pool of the destination's GPU and ``moe_pw_ep_expert`` stores each
result into the return pool of the source's GPU, so no separate all-to-all
runs: the transfer is the kernels' own stores.

This module is plumbing around those calls: buffer allocation (torch), the
per-step schedule of waves and barriers, and the exchange of buffer addresses
between processes (CUDA IPC through ``moe_pw_ipc_*``).  Every step of the
path runs in the library's kernels.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from . import moe_pw as mp

ALL_WAVES = 0xFFFFFFFF


@dataclass(frozen=True)
class Share:
    """What GPU ``gpu`` of ``n_gpus`` holds (from ``moe_pw_ep_plan``)."""

    n_gpus: int
    gpu: int
    ranks_per_gpu: int
    tokens: int
    first_token: int
    C_s: int
    C_r: int
    n_pools: int
    n_slots: int
    local_experts: int
    bucket_len: int
    workspace_bytes: int
    total_bytes: int

    @property
    def ranks(self) -> range:
        return range(self.gpu * self.ranks_per_gpu, (self.gpu + 1) * self.ranks_per_gpu)

    @property
    def token_range(self) -> range:
        return range(self.first_token, self.first_token + self.tokens)

    @property
    def expert_range(self) -> range:
        return range(self.gpu * self.local_experts, (self.gpu + 1) * self.local_experts)


def share(cfg: mp.Config, n_gpus: int, gpu: int, budget_bytes: int = 0) -> Share:
    s = mp.moe_pw_ep_plan(cfg, n_gpus, gpu, budget_bytes)
    return Share(n_gpus=n_gpus, gpu=gpu, ranks_per_gpu=cfg.R // n_gpus, tokens=s.tokens,
                 first_token=s.first_token, C_s=s.C_s, C_r=s.C_r, n_pools=s.n_pools,
                 n_slots=s.n_slots, local_experts=s.local_experts, bucket_len=s.bucket_len,
                 workspace_bytes=s.workspace_bytes, total_bytes=s.total_bytes)


def schedule(W: int, overlap: bool = True) -> list[list[tuple]]:
    """One step as phases; consecutive phases are separated by a barrier that
    every GPU passes only when all GPUs have finished the previous phase (all
    streams).  Each op is (stream, name, wave mask).  Every GPU runs the same
    list, so the barriers (collectives) are taken in the same order everywhere.

    overlap: wave w is packed and sent (stream "a") while the receivers bucket
    and run the expert op on wave w - 1 (stream "b"): phase w sends wave w,
    the barrier after it makes wave w complete in every receive pool.
    Without overlap all waves go in one pack launch.
    """
    if not overlap:
        return [[("a", "route", 0), ("a", "assign", 0), ("a", "pack", ALL_WAVES)],
                [("a", "bucket", ALL_WAVES), ("a", "expert", ALL_WAVES)],
                [("a", "combine", 0)]]
    phases = [[("a", "route", 0), ("a", "assign", 0), ("a", "pack", 1)]]
    for w in range(1, W):
        phases.append([("a", "pack", 1 << w), ("b", "bucket", 1 << (w - 1)),
                       ("b", "expert", 1 << (w - 1))])
    phases.append([("b", "bucket", 1 << (W - 1)), ("b", "expert", 1 << (W - 1))])
    phases.append([("a", "combine", 0)])
    return phases


class EpBuffers:
    """Every device array of one GPU's share, allocated with torch.  bf16
    arrays hold raw bits in int16 tensors."""

    def __init__(self, cfg: mp.Config, n_gpus: int, gpu: int, device="cuda"):
        self.cfg, self.n_gpus, self.gpu = cfg, n_gpus, gpu
        self.share = sh = share(cfg, n_gpus, gpu)
        dev = torch.device(device)
        T, E, k, D = sh.tokens, cfg.E, cfg.k, cfg.D
        i32, f32, i16 = torch.int32, torch.float32, torch.int16
        S = sh.n_slots
        self.logits = torch.empty((T, E), dtype=f32, device=dev)
        self.x = torch.empty((T, D), dtype=i16, device=dev)
        self.scale = torch.empty((E,), dtype=f32, device=dev)
        self.idx = torch.empty((T, k), dtype=i32, device=dev)
        self.gates = torch.empty((T, k), dtype=f32, device=dev)
        self.slot_map = torch.empty((T, k), dtype=i32, device=dev)
        self.occ = torch.empty((max(sh.n_pools, 1),), dtype=i32, device=dev)
        self.recv_x = torch.empty((S, D), dtype=i16, device=dev)
        self.recv_hdr = torch.empty((S,), dtype=i32, device=dev)
        self.recv_row = torch.empty((S,), dtype=i32, device=dev)
        self.bucket_slot = torch.empty((max(sh.bucket_len, 1),), dtype=i32, device=dev)
        self.expert_counts = torch.empty((2, sh.local_experts), dtype=i32, device=dev)
        self.ret_x = torch.empty((S, D), dtype=i16, device=dev)
        self.ret_hdr = torch.empty((S,), dtype=i32, device=dev)
        self.out = torch.empty((T, D), dtype=f32, device=dev)
        self.counters = torch.zeros((mp.COUNTERS_BYTES // 8,), dtype=torch.int64, device=dev)
        self.workspace = torch.empty((max(sh.workspace_bytes, 256),), dtype=torch.uint8,
                                     device=dev)
        self.host_expert_counts = np.zeros((2, sh.local_experts), np.int32)
        self.peers = mp.moe_pw_ep_peers()
        self.set_peer(gpu, self.addresses())

    def addresses(self) -> tuple[int, int, int, int]:
        """This GPU's receive and return pools as (recv_x, recv_hdr, ret_x, ret_hdr)."""
        return (self.recv_x.data_ptr(), self.recv_hdr.data_ptr(), self.ret_x.data_ptr(),
                self.ret_hdr.data_ptr())

    def set_peer(self, h: int, addrs):
        """Entry h of the peer table: GPU h's pools as this GPU addresses them."""
        self.peers.recv_x[h], self.peers.recv_hdr[h], self.peers.ret_x[h], self.peers.ret_hdr[h] = (
            addrs)

    # the steps, on this GPU's share
    def route(self, stream=None):
        mp.moe_pw_ep_route(self.cfg, self.n_gpus, self.gpu, self.logits, self.idx, self.gates,
                           stream)

    def assign(self, stream=None):
        mp.moe_pw_ep_assign(self.cfg, self.n_gpus, self.gpu, self.idx, self.slot_map, self.occ,
                            self.counters, self.workspace, stream)

    def pack(self, wave_mask=ALL_WAVES, stream=None):
        mp.moe_pw_ep_pack(self.cfg, self.n_gpus, self.gpu, self.peers, self.x, self.idx,
                          self.slot_map, self.occ, wave_mask, self.counters, stream)

    def bucket(self, wave_mask=ALL_WAVES, stream=None):
        mp.moe_pw_ep_bucket(self.cfg, self.n_gpus, self.gpu, self.recv_hdr, self.recv_row,
                            self.bucket_slot, self.expert_counts, wave_mask, self.counters,
                            stream)

    def expert(self, wave_mask=ALL_WAVES, stream=None):
        mp.moe_pw_ep_expert(self.cfg, self.n_gpus, self.gpu, self.peers, self.recv_x,
                            self.recv_hdr, self.recv_row, self.scale, wave_mask, stream)

    def combine(self, stream=None):
        mp.moe_pw_ep_combine(self.cfg, self.n_gpus, self.gpu, self.ret_x, self.ret_hdr,
                             self.slot_map, self.gates, self.out, self.counters, stream)

    def stats(self, stream=None, raise_on_device_error: bool = True) -> mp.moe_pw_drop_stats:
        return mp.moe_pw_ep_stats(self.cfg, self.n_gpus, self.gpu, self.counters,
                                  self.expert_counts, self.host_expert_counts, stream,
                                  raise_on_device_error)

    def run_op(self, name: str, wave_mask: int, stream=None):
        if name in ("pack", "bucket", "expert"):
            getattr(self, name)(wave_mask, stream)
        else:
            getattr(self, name)(stream)


def run_step(b: EpBuffers, barrier, stream_a, stream_b, overlap: bool = True, events=None):
    """One step of this GPU in an expert-parallel run of several processes.

    barrier(stream) must enqueue, on that stream, a point that every GPU
    passes only once every GPU's work before it on that stream is complete
    (a one-element all-reduce).  Stream b waits for the start of each phase
    on stream a, and stream a waits for stream b before each barrier.
    events: optional list that receives a timing event recorded on stream a
    after each phase's barrier (len(phases) events, the last after combine)."""
    phases = schedule(b.cfg.W, overlap)
    for i, phase in enumerate(phases):
        start = torch.cuda.Event()
        start.record(stream_a)
        stream_b.wait_event(start)
        for s, name, mask in phase:
            b.run_op(name, mask, stream_a if s == "a" else stream_b)
        done_b = torch.cuda.Event()
        done_b.record(stream_b)
        stream_a.wait_event(done_b)
        if i + 1 < len(phases):
            barrier(stream_a)
        if events is not None:
            ev = torch.cuda.Event(enable_timing=True)
            ev.record(stream_a)
            events.append(ev)


def emulate_step(bufs: list[EpBuffers], overlap: bool = True, stream=None):
    """One step of an n-GPU run emulated on one GPU: the shares' buffers all
    live on this GPU, the peer tables hold their plain addresses, and each
    phase runs for every share in turn on one stream before the next phase
    starts, which stands in for the barrier.  No kernel waits on another."""
    for b in bufs:
        for h, o in enumerate(bufs):
            b.set_peer(h, o.addresses())
    for phase in schedule(bufs[0].cfg.W, overlap):
        for b in bufs:
            for _, name, mask in phase:
                b.run_op(name, mask, stream)


class PeerLinks:
    """CUDA IPC links of this process's pools to the other GPUs' processes:
    each process exports its four pool arrays, the descriptions are gathered
    over ``group`` (``all_gather_object``), and every other process's arrays
    are opened here and written into this GPU's peer table.  ``close()``
    unmaps them; call it before the buffers of the other processes are
    freed."""

    def __init__(self, b: EpBuffers, all_gather_object, export=None, open_=None, close=None):
        self._export = export or mp.moe_pw_ipc_export
        self._open = open_ or mp.moe_pw_ipc_open
        self._close = close or mp.moe_pw_ipc_close
        mine = [bytes(self._export(t)) for t in (b.recv_x, b.recv_hdr, b.ret_x, b.ret_hdr)]
        gathered = [None] * b.n_gpus
        all_gather_object(gathered, (b.gpu, mine))
        self.opened = []
        for h, (gpu, descs) in enumerate(gathered):
            assert gpu == h, "ranks must gather in GPU order"
            if h == b.gpu:
                continue
            addrs = []
            for d in descs:
                handle = mp.moe_pw_ipc_handle.from_buffer_copy(d)
                ptr = self._open(handle)
                self.opened.append((ptr, handle))
                addrs.append(ptr)
            b.set_peer(h, tuple(addrs))

    def close(self):
        for ptr, handle in self.opened:
            self._close(ptr, handle)
        self.opened = []
