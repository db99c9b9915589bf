"""Reassembling the per-GPU shares of an expert-parallel run into the
single-batch layout, so the oracle's arrays can be compared with them
directly.  Only index relabelling lives here (the layouts of include/moe_pw.h,
"Expert parallelism over several GPUs"); no arithmetic of the method.  Across
GPUs the rows of slots whose header is -1 are not sent, so their payload is
not defined there: those rows are set to the single-GPU reading (zeros)
before the comparison, and the headers, compared in full, must mark them.
"""
from types import SimpleNamespace

import numpy as np
import torch


def recv_to_global(R: int, Rn: int, W: int, C_s: int, h: int) -> np.ndarray:
    """Global slot of every receive slot of GPU h."""
    return np.arange(R * R * W * C_s, dtype=np.int64).reshape(R, R, W, C_s)[
        :, h * Rn:(h + 1) * Rn].reshape(-1)


def _n(t):
    return t.detach().cpu().numpy()


def assemble(cfg, shares, stats):
    """shares: EpBuffers of GPUs 0..n-1 (after a step); stats: their
    moe_pw_drop_stats.  Returns (b, st) shaped like the single-GPU Buffers /
    moe_pw_drop_stats that tests/test_gpu_parity.py's checks take."""
    n = len(shares)
    sh0 = shares[0].share
    R, W, C_s, D, L = cfg.R, cfg.W, sh0.C_s, cfg.D, cfg.L
    Rn = R // n
    S_loc = sh0.n_slots
    S = n * S_loc
    E = cfg.E
    b = SimpleNamespace()
    cat = lambda name: np.concatenate([_n(getattr(s, name)) for s in shares])
    b.idx = cat("idx")
    b.gates = cat("gates")
    sm = [np.where(_n(s.slot_map) >= 0, _n(s.slot_map).astype(np.int64) + g * S_loc, -1)
          for g, s in enumerate(shares)]
    b.slot_map = np.concatenate(sm).astype(np.int32)
    b.occ = np.concatenate([_n(s.occ)[: sh0.n_pools] for s in shares])
    pool_x = np.zeros((R, R, W, C_s, D), np.int16)
    pool_hdr = np.zeros((R, R, W, C_s), np.int32)
    recv_row = np.zeros((R, R, W, C_s), np.int32)
    bucket = np.zeros((E, sh0.C_r), np.int32)
    counts = np.zeros((2, E), np.int32)
    host_counts = np.zeros((2, E), np.int32)
    for h, s in enumerate(shares):
        sl = slice(h * Rn, (h + 1) * Rn)
        pool_x[:, sl] = _n(s.recv_x).reshape(R, Rn, W, C_s, D)
        pool_hdr[:, sl] = _n(s.recv_hdr).reshape(R, Rn, W, C_s)
        recv_row[:, sl] = _n(s.recv_row).reshape(R, Rn, W, C_s)
        m = recv_to_global(R, Rn, W, C_s, h)
        bs = _n(s.bucket_slot)[: sh0.bucket_len].reshape(Rn * L, sh0.C_r).astype(np.int64)
        bucket[h * Rn * L:(h + 1) * Rn * L] = np.where(bs >= 0, m[np.maximum(bs, 0)], -1)
        counts[:, h * Rn * L:(h + 1) * Rn * L] = _n(s.expert_counts)
        host_counts[:, h * Rn * L:(h + 1) * Rn * L] = s.host_expert_counts
    # across GPUs the rows of empty and of receiver-dropped slots are not
    # sent (their headers say so); the single-GPU reading has zeros there
    pool_x[pool_hdr < 0] = 0
    b.pool_x = pool_x.reshape(S, D)
    b.pool_hdr = pool_hdr.reshape(S)
    b.recv_row = recv_row.reshape(S)
    b.bucket_slot = bucket.reshape(-1)
    b.expert_counts = counts
    b.host_expert_counts = host_counts
    b.ret_x = cat("ret_x")
    b.ret_hdr = cat("ret_hdr")
    b.ret_x[b.ret_hdr < 0] = 0
    b.out = cat("out")
    for k, v in list(vars(b).items()):
        if isinstance(v, np.ndarray) and k != "host_expert_counts":
            setattr(b, k, torch.from_numpy(np.ascontiguousarray(v)))
    st = SimpleNamespace(
        assignments=sum(x.assignments for x in stats),
        kept=sum(x.kept for x in stats),
        sender_dropped=sum(x.sender_dropped for x in stats),
        receiver_dropped=sum(x.receiver_dropped for x in stats),
        error=int(np.bitwise_or.reduce([x.error for x in stats])))
    return b, st
