"""Thin Python binding of libmoe_pw.so (include/moe_pw.h), via ctypes.

Each ``moe_pw_*`` function has the C entry point's name and arguments; it only
turns torch tensors into device pointers, picks the current CUDA stream and
raises ``MoePwError`` on a non-zero return code.  Every step of the path runs
in the library's CUDA kernels; there is no fallback.  PyTorch provides device
memory and streams.

``Buffers`` allocates every array of the path for a config (plumbing) and
``run_step`` chains route -> dispatch -> expert -> combine on one stream.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_pw.so")

MOE_PW_OK, MOE_PW_EINVAL, MOE_PW_EUNSUPPORTED, MOE_PW_ECUDA, MOE_PW_EDEVICE, MOE_PW_ENOMEM = (
    0, -1, -2, -3, -4, -5)
MOE_PW_POOLED, MOE_PW_RAGGED = 0, 1
DEVERR_EXPERT_ID, DEVERR_HEADER, DEVERR_TIMEOUT, DEVERR_SLOT = 1, 2, 4, 8


class MoePwError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed: {code} ({msg})")
        self.code = code


class moe_pw_config(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("E", ctypes.c_int32), ("k", ctypes.c_int32),
                ("D", ctypes.c_int32), ("R", ctypes.c_int32), ("L", ctypes.c_int32),
                ("W", ctypes.c_int32), ("P", ctypes.c_int32), ("cf_send_pct", ctypes.c_int32),
                ("cf_recv_pct", ctypes.c_int32), ("mode", ctypes.c_int32)]


class moe_pw_sizes(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("C_s", "C_r", "n_pools", "n_slots", "occ_len",
                                              "bucket_len", "workspace_bytes", "total_bytes")]


class moe_pw_counters(ctypes.Structure):
    _fields_ = [("sender_dropped", ctypes.c_uint64), ("receiver_dropped", ctypes.c_uint64),
                ("kept", ctypes.c_uint64), ("max_occ", ctypes.c_int32),
                ("max_fill", ctypes.c_int32), ("error", ctypes.c_int32),
                ("work", ctypes.c_int32)]


class moe_pw_drop_stats(ctypes.Structure):
    _fields_ = [("assignments", ctypes.c_int64), ("kept", ctypes.c_int64),
                ("sender_dropped", ctypes.c_int64), ("receiver_dropped", ctypes.c_int64),
                ("max_occ", ctypes.c_int32), ("max_fill", ctypes.c_int32),
                ("error", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class moe_pw_device_buffers(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "logits", "x", "scale", "idx", "gates", "slot_map", "occ", "pool_x", "pool_hdr",
        "recv_row", "bucket_slot", "expert_counts", "ret_x", "ret_hdr", "out", "counters",
        "workspace")] + [("workspace_bytes", ctypes.c_size_t)]


EP_MAX_GPUS = 64  # MOE_PW_EP_MAX_GPUS


class moe_pw_ep(ctypes.Structure):
    _fields_ = [("n_gpus", ctypes.c_int32), ("gpu", ctypes.c_int32)]


class moe_pw_ep_peers(ctypes.Structure):
    _fields_ = [("recv_x", ctypes.c_void_p * EP_MAX_GPUS),
                ("recv_hdr", ctypes.c_void_p * EP_MAX_GPUS),
                ("ret_x", ctypes.c_void_p * EP_MAX_GPUS),
                ("ret_hdr", ctypes.c_void_p * EP_MAX_GPUS)]


class moe_pw_ep_sizes(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("tokens", "first_token", "C_s", "C_r", "n_pools",
                                              "n_slots", "local_experts", "bucket_len",
                                              "workspace_bytes", "total_bytes")]


class moe_pw_ipc_handle(ctypes.Structure):
    _fields_ = [("handle", ctypes.c_ubyte * 64), ("offset", ctypes.c_uint64)]


# name -> argument types (after the config pointer); every function returns int
_VP, _SZ, _I64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int64
_CFG = ctypes.POINTER(moe_pw_config)
SIGNATURES = {
    "moe_pw_version": [],
    "moe_pw_strerror": [ctypes.c_int],
    "moe_pw_plan": [_CFG, _I64, ctypes.POINTER(moe_pw_sizes)],
    "moe_pw_route": [_CFG, _VP, _VP, _VP, _VP],
    "moe_pw_assign": [_CFG, _VP, _VP, _VP, _VP, _VP, _SZ, _VP],
    "moe_pw_assign_noalloc": [_CFG, _VP, _VP, _VP, _VP, _VP],
    "moe_pw_pack": [_CFG, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP],
    "moe_pw_bucket": [_CFG, _VP, _VP, _VP, _VP, _VP, _VP, _VP],
    "moe_pw_route_assign": [_CFG, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP],
    "moe_pw_route_assign_plan": [_CFG, ctypes.POINTER(ctypes.c_int32)],
    "moe_pw_route_assign_form": [_CFG, ctypes.c_int32, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP,
                                 _SZ, _VP],
    "moe_pw_assign_headers": [_CFG, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP],
    "moe_pw_pack_bucket": [_CFG, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP],
    "moe_pw_dispatch": [_CFG, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP],
    "moe_pw_expert": [_CFG, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP],
    "moe_pw_combine": [_CFG, _VP, _VP, _VP, _VP, _VP, _VP, _VP],
    "moe_pw_combine_bf16": [_CFG, _VP, _VP, _VP, _VP, _VP, _VP, _VP],
    "moe_pw_combine_bf16_rows": [_CFG, _VP, _VP, _VP, _VP, _I64, _I64, _VP, _VP, _VP],
    "moe_pw_combine_backward": [_CFG, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP],
    "moe_pw_dispatch_backward": [_CFG, _VP, _VP, _VP, _VP, _VP, _VP],
    "moe_pw_project": [_VP, _VP, _VP, _I64, ctypes.c_int32, ctypes.c_int32, _VP, _VP],
    "moe_pw_project_add": [_VP, _VP, _VP, _VP, _I64, ctypes.c_int32, ctypes.c_int32, _VP, _VP],
    "moe_pw_project_pack": [_CFG, _VP, _VP, ctypes.c_int32, _VP, _VP, _VP, _VP, _VP, _VP, _VP],
    "moe_pw_stats": [_CFG, _VP, _VP, ctypes.POINTER(moe_pw_drop_stats), _VP, _VP],
    "moe_pw_selftest_wait_timeout": [_VP, ctypes.c_int32, _VP],
    "moe_pw_seq_balance_plan": [_CFG, _I64, ctypes.POINTER(ctypes.c_int64)],
    "moe_pw_seq_balance": [_CFG, _I64, ctypes.c_float, _VP, _VP, _VP, _VP, _VP, _VP,
                           ctypes.c_int32, _VP, _SZ, _VP],
    "moe_pw_step_host": [_CFG, _VP, _VP, _VP, _VP, _VP, ctypes.POINTER(moe_pw_device_buffers),
                         _VP, _VP, _VP],
    "moe_pw_ep_plan": [_CFG, ctypes.POINTER(moe_pw_ep), _I64, ctypes.POINTER(moe_pw_ep_sizes)],
    "moe_pw_ep_route": [_CFG, ctypes.POINTER(moe_pw_ep), _VP, _VP, _VP, _VP],
    "moe_pw_ep_assign": [_CFG, ctypes.POINTER(moe_pw_ep), _VP, _VP, _VP, _VP, _VP, _SZ, _VP],
    "moe_pw_ep_pack": [_CFG, ctypes.POINTER(moe_pw_ep), ctypes.POINTER(moe_pw_ep_peers), _VP, _VP,
                       _VP, _VP, ctypes.c_uint32, _VP, _VP],
    "moe_pw_ep_bucket": [_CFG, ctypes.POINTER(moe_pw_ep), _VP, _VP, _VP, _VP, ctypes.c_uint32,
                         _VP, _VP],
    "moe_pw_ep_expert": [_CFG, ctypes.POINTER(moe_pw_ep), ctypes.POINTER(moe_pw_ep_peers), _VP,
                         _VP, _VP, _VP, ctypes.c_uint32, _VP],
    "moe_pw_ep_combine": [_CFG, ctypes.POINTER(moe_pw_ep), _VP, _VP, _VP, _VP, _VP, _VP, _VP],
    "moe_pw_ep_stats": [_CFG, ctypes.POINTER(moe_pw_ep), _VP, _VP,
                        ctypes.POINTER(moe_pw_drop_stats), _VP, _VP],
    "moe_pw_ipc_export": [_VP, ctypes.POINTER(moe_pw_ipc_handle)],
    "moe_pw_ipc_open": [ctypes.POINTER(moe_pw_ipc_handle), ctypes.POINTER(ctypes.c_void_p)],
    "moe_pw_ipc_close": [_VP, ctypes.POINTER(moe_pw_ipc_handle)],
}

_lib = None


def load_library(path: str = LIB_PATH):
    """Load libmoe_pw.so.  Raises if it has not been built: there is no
    fallback implementation of any step."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise ImportError(f"{path} is missing; build it with "
                              "`python -m combine_moe_pw_b200.build` (nvcc, sm_100a)")
        lib = ctypes.CDLL(path)
        for name, args in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = ctypes.c_char_p if name == "moe_pw_strerror" else ctypes.c_int
        _lib = lib
    return _lib


def _check(name: str, rc: int):
    if rc != MOE_PW_OK:
        raise MoePwError(name, rc, load_library().moe_pw_strerror(rc).decode())


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


@dataclass(frozen=True)
class Config:
    """Python mirror of ``moe_pw_config``."""

    T: int
    E: int
    k: int
    D: int
    R: int
    L: int
    W: int
    P: int
    cf_send_pct: int = 110
    cf_recv_pct: int = 115
    mode: int = MOE_PW_POOLED

    @classmethod
    def from_workload(cls, w) -> "Config":
        return cls(T=w.T, E=w.E, k=w.k, D=w.D, R=w.R, L=w.L, W=w.W, P=w.P,
                   cf_send_pct=w.cf_send_pct, cf_recv_pct=w.cf_recv_pct, mode=w.mode)

    def c(self) -> moe_pw_config:
        return moe_pw_config(self.T, self.E, self.k, self.D, self.R, self.L, self.W, self.P,
                             self.cf_send_pct, self.cf_recv_pct, self.mode)


def _cfg(cfg) -> moe_pw_config:
    return cfg.c() if isinstance(cfg, Config) else cfg


def moe_pw_version() -> int:
    return load_library().moe_pw_version()


def moe_pw_plan(cfg, budget_bytes: int = 0) -> moe_pw_sizes:
    out = moe_pw_sizes()
    c = _cfg(cfg)
    _check("moe_pw_plan", load_library().moe_pw_plan(ctypes.byref(c), budget_bytes,
                                                     ctypes.byref(out)))
    return out


def moe_pw_route(cfg, logits, idx, gates, stream=None):
    c = _cfg(cfg)
    _check("moe_pw_route", load_library().moe_pw_route(
        ctypes.byref(c), _ptr(logits), _ptr(idx), _ptr(gates), _stream(stream)))


def moe_pw_assign(cfg, idx, slot_map, occ, counters, workspace, workspace_bytes=None, stream=None):
    c = _cfg(cfg)
    wsb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check("moe_pw_assign", load_library().moe_pw_assign(
        ctypes.byref(c), _ptr(idx), _ptr(slot_map), _ptr(occ), _ptr(counters), _ptr(workspace),
        wsb, _stream(stream)))


NOALLOC_SCRATCH_BYTES = 4 << 20  # MOE_PW_NOALLOC_SCRATCH_BYTES


def moe_pw_assign_noalloc(cfg, idx, slot_map, occ, counters, stream=None):
    """moe_pw_assign without a workspace argument: the library's built-in
    scratch array is used (see include/moe_pw.h for its limits)."""
    c = _cfg(cfg)
    _check("moe_pw_assign_noalloc", load_library().moe_pw_assign_noalloc(
        ctypes.byref(c), _ptr(idx), _ptr(slot_map), _ptr(occ), _ptr(counters), _stream(stream)))


def moe_pw_pack(cfg, x, idx, slot_map, occ, pool_x, pool_hdr, counters, stream=None):
    c = _cfg(cfg)
    _check("moe_pw_pack", load_library().moe_pw_pack(
        ctypes.byref(c), _ptr(x), _ptr(idx), _ptr(slot_map), _ptr(occ), _ptr(pool_x),
        _ptr(pool_hdr), _ptr(counters), _stream(stream)))


def moe_pw_bucket(cfg, pool_hdr, occ, recv_row, bucket_slot, expert_counts, counters, stream=None):
    c = _cfg(cfg)
    _check("moe_pw_bucket", load_library().moe_pw_bucket(
        ctypes.byref(c), _ptr(pool_hdr), _ptr(occ), _ptr(recv_row), _ptr(bucket_slot),
        _ptr(expert_counts), _ptr(counters), _stream(stream)))


def moe_pw_route_assign(cfg, logits, idx, gates, slot_map, occ, pool_hdr, counters, workspace,
                        workspace_bytes=None, stream=None):
    """moe_pw_route + moe_pw_assign_headers, one clustered launch where the
    batch allows (pooled mode)."""
    c = _cfg(cfg)
    wsb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check("moe_pw_route_assign", load_library().moe_pw_route_assign(
        ctypes.byref(c), _ptr(logits), _ptr(idx), _ptr(gates), _ptr(slot_map), _ptr(occ),
        _ptr(pool_hdr), _ptr(counters), _ptr(workspace), wsb, _stream(stream)))


RA_SEPARATE, RA_CLUSTER = 0, 1  # MOE_PW_RA_*


def moe_pw_route_assign_form(cfg, form, logits, idx, gates, slot_map, occ, pool_hdr, counters,
                             workspace, workspace_bytes=None, stream=None):
    """moe_pw_route_assign in a given form (RA_*), or -1 for the default;
    raises MoePwError (MOE_PW_EUNSUPPORTED) if the form does not fit."""
    c = _cfg(cfg)
    wsb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check("moe_pw_route_assign_form", load_library().moe_pw_route_assign_form(
        ctypes.byref(c), form, _ptr(logits), _ptr(idx), _ptr(gates), _ptr(slot_map), _ptr(occ),
        _ptr(pool_hdr), _ptr(counters), _ptr(workspace), wsb, _stream(stream)))


def moe_pw_route_assign_plan(cfg) -> int:
    """The form moe_pw_route_assign takes for this batch on the current
    device: RA_SEPARATE or RA_CLUSTER."""
    c = _cfg(cfg)
    form = ctypes.c_int32(0)
    _check("moe_pw_route_assign_plan",
           load_library().moe_pw_route_assign_plan(ctypes.byref(c), ctypes.byref(form)))
    return int(form.value)


def moe_pw_assign_headers(cfg, idx, slot_map, occ, pool_hdr, counters, workspace,
                          workspace_bytes=None, stream=None):
    """moe_pw_assign that also writes the kept slots' headers (pooled mode)."""
    c = _cfg(cfg)
    wsb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check("moe_pw_assign_headers", load_library().moe_pw_assign_headers(
        ctypes.byref(c), _ptr(idx), _ptr(slot_map), _ptr(occ), _ptr(pool_hdr), _ptr(counters),
        _ptr(workspace), wsb, _stream(stream)))


def moe_pw_pack_bucket(cfg, x, idx, slot_map, occ, pool_x, pool_hdr, recv_row, bucket_slot,
                       expert_counts, counters, stream=None):
    """Pack and receiver bucketing in one launch; pool_hdr must hold the
    kept slots' headers from moe_pw_assign_headers."""
    c = _cfg(cfg)
    _check("moe_pw_pack_bucket", load_library().moe_pw_pack_bucket(
        ctypes.byref(c), _ptr(x), _ptr(idx), _ptr(slot_map), _ptr(occ), _ptr(pool_x),
        _ptr(pool_hdr), _ptr(recv_row), _ptr(bucket_slot), _ptr(expert_counts), _ptr(counters),
        _stream(stream)))


def moe_pw_dispatch(cfg, x, idx, slot_map, occ, pool_x, pool_hdr, recv_row, bucket_slot,
                    expert_counts, counters, workspace, workspace_bytes=None, stream=None):
    c = _cfg(cfg)
    wsb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check("moe_pw_dispatch", load_library().moe_pw_dispatch(
        ctypes.byref(c), _ptr(x), _ptr(idx), _ptr(slot_map), _ptr(occ), _ptr(pool_x),
        _ptr(pool_hdr), _ptr(recv_row), _ptr(bucket_slot), _ptr(expert_counts), _ptr(counters),
        _ptr(workspace), wsb, _stream(stream)))


def moe_pw_expert(cfg, pool_x, pool_hdr, recv_row, scale, ret_x, ret_hdr, counters,
                  stream=None):
    c = _cfg(cfg)
    _check("moe_pw_expert", load_library().moe_pw_expert(
        ctypes.byref(c), _ptr(pool_x), _ptr(pool_hdr), _ptr(recv_row), _ptr(scale), _ptr(ret_x),
        _ptr(ret_hdr), _ptr(counters), _stream(stream)))


def moe_pw_combine(cfg, ret_x, ret_hdr, slot_map, gates, out, counters, stream=None):
    c = _cfg(cfg)
    _check("moe_pw_combine", load_library().moe_pw_combine(
        ctypes.byref(c), _ptr(ret_x), _ptr(ret_hdr), _ptr(slot_map), _ptr(gates), _ptr(out),
        _ptr(counters), _stream(stream)))


def moe_pw_combine_bf16(cfg, ret_x, ret_hdr, slot_map, gates, out, counters, stream=None):
    c = _cfg(cfg)
    _check("moe_pw_combine_bf16", load_library().moe_pw_combine_bf16(
        ctypes.byref(c), _ptr(ret_x), _ptr(ret_hdr), _ptr(slot_map), _ptr(gates), _ptr(out),
        _ptr(counters), _stream(stream)))


def moe_pw_combine_bf16_rows(cfg, ret_x, ret_hdr, slot_map, gates, first_token: int,
                             n_tokens: int, out, counters, stream=None):
    c = _cfg(cfg)
    _check("moe_pw_combine_bf16_rows", load_library().moe_pw_combine_bf16_rows(
        ctypes.byref(c), _ptr(ret_x), _ptr(ret_hdr), _ptr(slot_map), _ptr(gates), first_token,
        n_tokens, _ptr(out), _ptr(counters), _stream(stream)))


def moe_pw_combine_backward(cfg, dout, ret_x, ret_hdr, slot_map, idx, gates, d_ret, dgates,
                            dlogits, counters, stream=None):
    c = _cfg(cfg)
    _check("moe_pw_combine_backward", load_library().moe_pw_combine_backward(
        ctypes.byref(c), _ptr(dout), _ptr(ret_x), _ptr(ret_hdr), _ptr(slot_map), _ptr(idx),
        _ptr(gates), _ptr(d_ret), _ptr(dgates), _ptr(dlogits), _ptr(counters), _stream(stream)))


def moe_pw_dispatch_backward(cfg, d_pool, recv_row, slot_map, dx, counters, stream=None):
    c = _cfg(cfg)
    _check("moe_pw_dispatch_backward", load_library().moe_pw_dispatch_backward(
        ctypes.byref(c), _ptr(d_pool), _ptr(recv_row), _ptr(slot_map), _ptr(dx), _ptr(counters),
        _stream(stream)))


def moe_pw_project(A, Bt, C, M: int, N: int, K: int, counters, stream=None):
    """C = bf16(A @ Bt^T) on the tensor cores (bf16 operands, fp32 accumulation)."""
    _check("moe_pw_project", load_library().moe_pw_project(
        _ptr(A), _ptr(Bt), _ptr(C), M, N, K, _ptr(counters), _stream(stream)))


def moe_pw_project_add(A, Bt, add, C, M: int, N: int, K: int, counters, stream=None):
    """C = bf16(A @ Bt^T + add): the up-projection merged with the shared path."""
    _check("moe_pw_project_add", load_library().moe_pw_project_add(
        _ptr(A), _ptr(Bt), _ptr(add), _ptr(C), M, N, K, _ptr(counters), _stream(stream)))


def moe_pw_project_pack(cfg, h, w_down_t, model_width: int, idx, slot_map, occ, pool_x, pool_hdr,
                        counters, stream=None):
    """Down-projection fused with the pack (see include/moe_pw.h)."""
    c = _cfg(cfg)
    _check("moe_pw_project_pack", load_library().moe_pw_project_pack(
        ctypes.byref(c), _ptr(h), _ptr(w_down_t), model_width, _ptr(idx), _ptr(slot_map),
        _ptr(occ), _ptr(pool_x), _ptr(pool_hdr), _ptr(counters), _stream(stream)))


def moe_pw_stats(cfg, counters, stream=None, raise_on_device_error: bool = True,
                 expert_counts=None, host_expert_counts=None) -> moe_pw_drop_stats:
    """Drop statistics.  With ``expert_counts`` (device i32 [2, E]) and
    ``host_expert_counts`` (a C-contiguous numpy int32 [2, E] array) the
    per-expert arrivals and kept rows are copied into the latter as well."""
    c = _cfg(cfg)
    out = moe_pw_drop_stats()
    hp = None
    if host_expert_counts is not None:
        assert host_expert_counts.dtype == np.int32 and host_expert_counts.flags.c_contiguous
        assert host_expert_counts.size >= 2 * c.E
        hp = host_expert_counts.ctypes.data
    rc = load_library().moe_pw_stats(ctypes.byref(c), _ptr(counters), _ptr(expert_counts),
                                     ctypes.byref(out), hp, _stream(stream))
    if rc == MOE_PW_EDEVICE and not raise_on_device_error:
        return out
    _check("moe_pw_stats", rc)
    return out


def moe_pw_selftest_wait_timeout(counters, polls: int = 4096, stream=None):
    """Run the bounded-wait self-test (see include/moe_pw.h)."""
    _check("moe_pw_selftest_wait_timeout", load_library().moe_pw_selftest_wait_timeout(
        _ptr(counters), polls, _stream(stream)))


def moe_pw_seq_balance_plan(cfg, seq_len: int) -> int:
    c = _cfg(cfg)
    n = ctypes.c_int64()
    _check("moe_pw_seq_balance_plan", load_library().moe_pw_seq_balance_plan(
        ctypes.byref(c), seq_len, ctypes.byref(n)))
    return int(n.value)


def moe_pw_seq_balance(cfg, seq_len: int, alpha: float, logits, idx, f, P, loss, workspace,
                       dlogits=None, accumulate: bool = False, stream=None):
    """Sequence-level balance term and (with dlogits) its gradient; see
    include/moe_pw.h."""
    c = _cfg(cfg)
    _check("moe_pw_seq_balance", load_library().moe_pw_seq_balance(
        ctypes.byref(c), seq_len, alpha, _ptr(logits), _ptr(idx), _ptr(f), _ptr(P), _ptr(loss),
        _ptr(dlogits), 1 if accumulate else 0, _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def moe_pw_step_host(cfg, h_logits, h_x, h_scale, h_out, h_counters,
                     dev: moe_pw_device_buffers, compute=None, copy_in=None, copy_out=None):
    """One step from host buffers to host buffers, enqueued on three streams
    (see include/moe_pw.h).  Host arrays: pinned torch CPU tensors."""
    c = _cfg(cfg)
    s_c = _stream(compute)
    s_i = s_c if copy_in is None else _stream(copy_in)
    s_o = s_c if copy_out is None else _stream(copy_out)
    _check("moe_pw_step_host", load_library().moe_pw_step_host(
        ctypes.byref(c), _ptr(h_logits), _ptr(h_x), _ptr(h_scale), _ptr(h_out),
        _ptr(h_counters), ctypes.byref(dev), s_c, s_i, s_o))


def _ep(n_gpus: int, gpu: int) -> moe_pw_ep:
    return moe_pw_ep(n_gpus, gpu)


def moe_pw_ep_plan(cfg, n_gpus: int, gpu: int, budget_bytes: int = 0) -> moe_pw_ep_sizes:
    out = moe_pw_ep_sizes()
    c, e = _cfg(cfg), _ep(n_gpus, gpu)
    _check("moe_pw_ep_plan", load_library().moe_pw_ep_plan(ctypes.byref(c), ctypes.byref(e),
                                                           budget_bytes, ctypes.byref(out)))
    return out


def moe_pw_ep_route(cfg, n_gpus, gpu, logits, idx, gates, stream=None):
    c, e = _cfg(cfg), _ep(n_gpus, gpu)
    _check("moe_pw_ep_route", load_library().moe_pw_ep_route(
        ctypes.byref(c), ctypes.byref(e), _ptr(logits), _ptr(idx), _ptr(gates), _stream(stream)))


def moe_pw_ep_assign(cfg, n_gpus, gpu, idx, slot_map, occ, counters, workspace, stream=None):
    c, e = _cfg(cfg), _ep(n_gpus, gpu)
    wsb = workspace.numel() * workspace.element_size()
    _check("moe_pw_ep_assign", load_library().moe_pw_ep_assign(
        ctypes.byref(c), ctypes.byref(e), _ptr(idx), _ptr(slot_map), _ptr(occ), _ptr(counters),
        _ptr(workspace), wsb, _stream(stream)))


def moe_pw_ep_pack(cfg, n_gpus, gpu, peers: moe_pw_ep_peers, x, idx, slot_map, occ, wave_mask,
                   counters, stream=None):
    c, e = _cfg(cfg), _ep(n_gpus, gpu)
    _check("moe_pw_ep_pack", load_library().moe_pw_ep_pack(
        ctypes.byref(c), ctypes.byref(e), ctypes.byref(peers), _ptr(x), _ptr(idx), _ptr(slot_map),
        _ptr(occ), wave_mask, _ptr(counters), _stream(stream)))


def moe_pw_ep_bucket(cfg, n_gpus, gpu, recv_hdr, recv_row, bucket_slot, expert_counts, wave_mask,
                     counters, stream=None):
    c, e = _cfg(cfg), _ep(n_gpus, gpu)
    _check("moe_pw_ep_bucket", load_library().moe_pw_ep_bucket(
        ctypes.byref(c), ctypes.byref(e), _ptr(recv_hdr), _ptr(recv_row), _ptr(bucket_slot),
        _ptr(expert_counts), wave_mask, _ptr(counters), _stream(stream)))


def moe_pw_ep_expert(cfg, n_gpus, gpu, peers: moe_pw_ep_peers, recv_x, recv_hdr, recv_row, scale,
                     wave_mask, stream=None):
    c, e = _cfg(cfg), _ep(n_gpus, gpu)
    _check("moe_pw_ep_expert", load_library().moe_pw_ep_expert(
        ctypes.byref(c), ctypes.byref(e), ctypes.byref(peers), _ptr(recv_x), _ptr(recv_hdr),
        _ptr(recv_row), _ptr(scale), wave_mask, _stream(stream)))


def moe_pw_ep_combine(cfg, n_gpus, gpu, ret_x, ret_hdr, slot_map, gates, out, counters,
                      stream=None):
    c, e = _cfg(cfg), _ep(n_gpus, gpu)
    _check("moe_pw_ep_combine", load_library().moe_pw_ep_combine(
        ctypes.byref(c), ctypes.byref(e), _ptr(ret_x), _ptr(ret_hdr), _ptr(slot_map), _ptr(gates),
        _ptr(out), _ptr(counters), _stream(stream)))


def moe_pw_ep_stats(cfg, n_gpus, gpu, counters, expert_counts=None, host_expert_counts=None,
                    stream=None, raise_on_device_error: bool = True) -> moe_pw_drop_stats:
    c, e = _cfg(cfg), _ep(n_gpus, gpu)
    out = moe_pw_drop_stats()
    hp = None
    if host_expert_counts is not None:
        assert host_expert_counts.dtype == np.int32 and host_expert_counts.flags.c_contiguous
        hp = host_expert_counts.ctypes.data
    rc = load_library().moe_pw_ep_stats(ctypes.byref(c), ctypes.byref(e), _ptr(counters),
                                        _ptr(expert_counts), ctypes.byref(out), hp,
                                        _stream(stream))
    if rc == MOE_PW_EDEVICE and not raise_on_device_error:
        return out
    _check("moe_pw_ep_stats", rc)
    return out


def moe_pw_ipc_export(t) -> moe_pw_ipc_handle:
    h = moe_pw_ipc_handle()
    _check("moe_pw_ipc_export", load_library().moe_pw_ipc_export(_ptr(t), ctypes.byref(h)))
    return h


def moe_pw_ipc_open(h: moe_pw_ipc_handle) -> int:
    p = ctypes.c_void_p()
    _check("moe_pw_ipc_open", load_library().moe_pw_ipc_open(ctypes.byref(h), ctypes.byref(p)))
    return int(p.value)


def moe_pw_ipc_close(ptr: int, h: moe_pw_ipc_handle):
    _check("moe_pw_ipc_close", load_library().moe_pw_ipc_close(ptr, ctypes.byref(h)))


COUNTERS_BYTES = ctypes.sizeof(moe_pw_counters)


class Buffers:
    """Every device array of the path for one config, allocated with torch.

    Layouts follow include/moe_pw.h.  bf16 arrays are stored as int16 tensors
    holding the raw bits (``.view(torch.bfloat16)`` gives the values)."""

    def __init__(self, cfg: Config, device="cuda", budget_bytes: int = 0):
        self.cfg = cfg
        self.sizes = s = moe_pw_plan(cfg, budget_bytes)
        dev = torch.device(device)
        T, E, k, D = cfg.T, cfg.E, cfg.k, cfg.D
        i32, f32, i16 = torch.int32, torch.float32, torch.int16
        self.logits = torch.empty((T, E), dtype=f32, device=dev)
        self.x = torch.empty((T, D), dtype=i16, device=dev)
        self.scale = torch.empty((E,), dtype=f32, device=dev)
        self.idx = torch.empty((T, k), dtype=i32, device=dev)
        self.gates = torch.empty((T, k), dtype=f32, device=dev)
        self.slot_map = torch.empty((T, k), dtype=i32, device=dev)
        self.occ = torch.empty((max(s.occ_len, 1),), dtype=i32, device=dev)
        self.pool_x = torch.empty((s.n_slots, D), dtype=i16, device=dev)
        self.pool_hdr = torch.empty((s.n_slots,), dtype=i32, device=dev)
        self.recv_row = torch.empty((s.n_slots,), dtype=i32, device=dev)
        self.bucket_slot = torch.empty((max(s.bucket_len, 1),), dtype=i32, device=dev)
        self.expert_counts = torch.empty((2, E), dtype=i32, device=dev)
        self.host_expert_counts = np.zeros((2, E), np.int32)
        self.ret_x = torch.empty((s.n_slots, D), dtype=i16, device=dev)
        self.ret_hdr = torch.empty((s.n_slots,), dtype=i32, device=dev)
        self.out = torch.empty((T, D), dtype=f32, device=dev)
        self.counters = torch.zeros((COUNTERS_BYTES // 8,), dtype=torch.int64, device=dev)
        self.workspace = torch.empty((max(s.workspace_bytes, 256),), dtype=torch.uint8, device=dev)

    def device_buffers(self) -> moe_pw_device_buffers:
        """The device arrays as the C struct moe_pw_step_host takes."""
        d = moe_pw_device_buffers()
        for name in ("logits", "x", "scale", "idx", "gates", "slot_map", "occ", "pool_x",
                     "pool_hdr", "recv_row", "bucket_slot", "expert_counts", "ret_x", "ret_hdr",
                     "out", "counters", "workspace"):
            setattr(d, name, getattr(self, name).data_ptr())
        d.workspace_bytes = self.workspace.numel()
        return d

    def route(self, stream=None):
        moe_pw_route(self.cfg, self.logits, self.idx, self.gates, stream)

    def dispatch(self, stream=None):
        moe_pw_dispatch(self.cfg, self.x, self.idx, self.slot_map, self.occ, self.pool_x,
                        self.pool_hdr, self.recv_row, self.bucket_slot, self.expert_counts,
                        self.counters, self.workspace, stream=stream)

    def assign(self, stream=None):
        moe_pw_assign(self.cfg, self.idx, self.slot_map, self.occ, self.counters, self.workspace,
                      stream=stream)

    def route_assign(self, stream=None, form: int = -1):
        """Route + assignment with the kept slots' headers; form: RA_* or -1
        for the library's choice."""
        moe_pw_route_assign_form(self.cfg, form, self.logits, self.idx, self.gates, self.slot_map,
                                 self.occ, self.pool_hdr, self.counters, self.workspace,
                                 stream=stream)

    def assign_headers(self, stream=None):
        moe_pw_assign_headers(self.cfg, self.idx, self.slot_map, self.occ, self.pool_hdr,
                              self.counters, self.workspace, stream=stream)

    def pack_bucket(self, stream=None):
        moe_pw_pack_bucket(self.cfg, self.x, self.idx, self.slot_map, self.occ, self.pool_x,
                           self.pool_hdr, self.recv_row, self.bucket_slot, self.expert_counts,
                           self.counters, stream)

    def pack(self, stream=None):
        moe_pw_pack(self.cfg, self.x, self.idx, self.slot_map, self.occ, self.pool_x,
                    self.pool_hdr, self.counters, stream)

    def bucket(self, stream=None):
        moe_pw_bucket(self.cfg, self.pool_hdr, self.occ, self.recv_row, self.bucket_slot,
                      self.expert_counts, self.counters, stream)

    def expert(self, stream=None):
        moe_pw_expert(self.cfg, self.pool_x, self.pool_hdr, self.recv_row, self.scale,
                      self.ret_x, self.ret_hdr, self.counters, stream)

    def combine(self, stream=None):
        moe_pw_combine(self.cfg, self.ret_x, self.ret_hdr, self.slot_map, self.gates, self.out,
                       self.counters, stream)

    def stats(self, stream=None, raise_on_device_error: bool = True) -> moe_pw_drop_stats:
        """Drop statistics; the per-expert arrivals and kept rows land in
        ``self.host_expert_counts`` (numpy int32 [2, E])."""
        return moe_pw_stats(self.cfg, self.counters, stream, raise_on_device_error,
                            self.expert_counts, self.host_expert_counts)

    def alloc_backward(self):
        """Gradient buffers: dout (input), d_ret / d_pool (gradient pools),
        dgates, dlogits, dx."""
        dev, T, E, k, D = self.out.device, self.cfg.T, self.cfg.E, self.cfg.k, self.cfg.D
        n = self.sizes.n_slots
        self.dout = torch.empty((T, D), dtype=torch.float32, device=dev)
        self.d_ret = torch.empty((n, D), dtype=torch.int16, device=dev)
        self.d_pool = torch.empty((n, D), dtype=torch.int16, device=dev)
        self.d_pool_hdr = torch.empty((n,), dtype=torch.int32, device=dev)
        self.dgates = torch.empty((T, k), dtype=torch.float32, device=dev)
        self.dlogits = torch.empty((T, E), dtype=torch.float32, device=dev)
        self.dx = torch.empty((T, D), dtype=torch.float32, device=dev)

    def run_backward(self, stream=None):
        """combine backward -> expert backward (the same scale op on the
        gradient pool) -> pack backward."""
        moe_pw_combine_backward(self.cfg, self.dout, self.ret_x, self.ret_hdr, self.slot_map,
                                self.idx, self.gates, self.d_ret, self.dgates, self.dlogits,
                                self.counters, stream)
        moe_pw_expert(self.cfg, self.d_ret, self.pool_hdr, self.recv_row, self.scale,
                      self.d_pool, self.d_pool_hdr, self.counters, stream)
        moe_pw_dispatch_backward(self.cfg, self.d_pool, self.recv_row, self.slot_map, self.dx,
                                 self.counters, stream)

    OVERLAP_BLOCK_TOKENS = 16384  # block size for the overlapped routed layer

    def run_routed_layer(self, h, w_down_t, w_up_t, model_width: int, latent_bf16, out_model,
                         stream=None, shared_out=None, overlap: bool = False):
        """The whole routed branch from model width back to model width:
        route -> assign -> down-projection fused with the pack -> bucket ->
        expert op -> combine (bf16 latent) -> up-projection.  h: bf16 [T, Dm],
        w_down_t: bf16 [D, Dm], w_up_t: bf16 [Dm, D], latent_bf16: bf16 [T, D]
        (scratch), out_model: bf16 [T, Dm].  With shared_out (bf16 [T, Dm],
        the shared experts' output) the up-projection's epilogue adds it: the
        merge of the two paths.  With overlap (and at least two blocks of
        OVERLAP_BLOCK_TOKENS tokens) the combine and the up-projection run
        block by block on two streams (run_routed_layer_pipelined), the two
        block buffers taken from latent_bf16; the bytes are the same.  Off by
        default: on the rack batch the GEMMs run at the power cap, and with the
        combine beside them the overlap gained 1 ms in one run and lost 0.5 ms
        in another."""
        cfg = self.cfg
        blk = self.OVERLAP_BLOCK_TOKENS
        if overlap and cfg.T >= 2 * blk:
            self.run_routed_layer_pipelined(h, w_down_t, w_up_t, model_width, out_model,
                                            shared_out=shared_out, chunk_tokens=blk,
                                            stream=stream,
                                            latent_chunks=[latent_bf16[:blk], latent_bf16[blk:2 * blk]])
            return
        self.route(stream)
        self.assign(stream)
        moe_pw_project_pack(cfg, h, w_down_t, model_width, self.idx, self.slot_map, self.occ,
                            self.pool_x, self.pool_hdr, self.counters, stream)
        self.bucket(stream)
        self.expert(stream)
        moe_pw_combine_bf16(cfg, self.ret_x, self.ret_hdr, self.slot_map, self.gates, latent_bf16,
                            self.counters, stream)
        if shared_out is None:
            moe_pw_project(latent_bf16, w_up_t, out_model, cfg.T, model_width, cfg.D,
                           self.counters, stream)
        else:
            moe_pw_project_add(latent_bf16, w_up_t, shared_out, out_model, cfg.T, model_width,
                               cfg.D, self.counters, stream)

    def run_routed_layer_pipelined(self, h, w_down_t, w_up_t, model_width: int, out_model,
                                   shared_out=None, chunk_tokens: int = 8192, stream=None,
                                   side_stream=None, latent_chunks=None):
        """run_routed_layer with the combine and the up-projection overlapped
        block by block: the combine of token block c + 1 (HBM-bound) runs on
        one stream while the up-projection of block c (tensor-bound) runs on
        another, and the bf16 latent passes through two buffers of
        chunk_tokens rows (latent_chunks, allocated here if not given) instead
        of a whole-batch array.  Same kernels, same per-row arithmetic: the
        output equals run_routed_layer's bit for bit."""
        cfg = self.cfg
        dev = self.out.device
        s0 = stream if stream is not None else torch.cuda.current_stream(dev)
        if side_stream is None:
            if getattr(self, "_side", None) is None:
                self._side = torch.cuda.Stream(dev)
            side_stream = self._side
        s1 = side_stream
        if latent_chunks is None:
            # kept with the buffers: the side stream may still read them after return
            key = ("latent_chunks", chunk_tokens)
            if getattr(self, "_chunks_key", None) != key:
                self._chunks = [torch.empty((chunk_tokens, cfg.D), dtype=torch.int16, device=dev)
                                for _ in range(2)]
                self._chunks_key = key
            latent_chunks = self._chunks
        self.route(s0)
        self.assign(s0)
        moe_pw_project_pack(cfg, h, w_down_t, model_width, self.idx, self.slot_map, self.occ,
                            self.pool_x, self.pool_hdr, self.counters, s0)
        self.bucket(s0)
        self.expert(s0)
        n_chunks = (cfg.T + chunk_tokens - 1) // chunk_tokens
        freed = [None, None]
        for c in range(n_chunks):
            t0 = c * chunk_tokens
            n = min(chunk_tokens, cfg.T - t0)
            lat = latent_chunks[c % 2]
            if freed[c % 2] is not None:
                s0.wait_event(freed[c % 2])
            moe_pw_combine_bf16_rows(cfg, self.ret_x, self.ret_hdr, self.slot_map, self.gates,
                                     t0, n, lat, self.counters, s0)
            ready = torch.cuda.Event()
            ready.record(s0)
            s1.wait_event(ready)
            rows = out_model[t0:t0 + n]
            if shared_out is None:
                moe_pw_project(lat, w_up_t, rows, n, model_width, cfg.D, self.counters, s1)
            else:
                moe_pw_project_add(lat, w_up_t, shared_out[t0:t0 + n], rows, n, model_width,
                                   cfg.D, self.counters, s1)
            done = torch.cuda.Event()
            done.record(s1)
            freed[c % 2] = done
        for ev in freed:
            if ev is not None:
                s0.wait_event(ev)

    def run_step(self, stream=None):
        """route -> dispatch (assign, pack, bucket) -> expert -> combine.
        Pooled mode: route and assignment in one launch, then the pack and the
        bucketing in one launch."""
        if self.cfg.mode == MOE_PW_POOLED:
            self.route_assign(stream)
            self.pack_bucket(stream)
        else:
            self.route(stream)
            self.dispatch(stream)
        self.expert(stream)
        self.combine(stream)

    def capture_step(self):
        """One forward step (``run_step``) recorded as a CUDA graph on these
        buffers.  Every call of the step is asynchronous on its stream with no
        host synchronisation, so the whole step captures; ``graph.replay()``
        then runs it with one launch from the host.  The graph reads the
        buffers' current contents when it runs: copy new logits, x and scales
        into them and replay.  The step runs once eagerly first (on the
        capture stream) so that every per-device setup is done before capture."""
        side = torch.cuda.Stream(device=self.out.device)
        side.wait_stream(torch.cuda.current_stream(self.out.device))
        with torch.cuda.stream(side):
            self.run_step()
        torch.cuda.current_stream(self.out.device).wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            self.run_step()
        return graph


class Pipeline:
    """Streams batches from pinned host memory through the path with the host
    copies of neighbouring batches overlapped with compute.

    ``depth`` device buffer sets are used in turn.  Batch i's inputs go up on
    the copy-in stream while batch i-1 computes on its own stream and batch
    i-2's output comes down on the copy-out stream (PCIe is full duplex and
    the copy engines run beside the SMs).  Events order each buffer set's
    reuse: inputs are overwritten only after the compute that read them, the
    output only after its copy to the host.  Nothing blocks the host; call
    ``synchronize()`` before reading results."""

    def __init__(self, cfg: Config, device="cuda", depth: int = 2):
        dev = torch.device(device)
        self.cfg, self.depth, self.n = cfg, depth, 0
        self.bufs = [Buffers(cfg, dev) for _ in range(depth)]
        self.s_in = torch.cuda.Stream(dev)
        self.s_out = torch.cuda.Stream(dev)
        self.s_comp = [torch.cuda.Stream(dev) for _ in range(depth)]
        self.inputs_free = [None] * depth   # compute of the last batch in set b has read its inputs
        self.output_free = [None] * depth   # last output of set b is on the host
        self.h_counters = [torch.empty_like(b.counters, device="cpu").pin_memory() for b in self.bufs]
        self.dev = [b.device_buffers() for b in self.bufs]

    def submit(self, h_logits, h_x, h_scale, h_out):
        """Queue one batch: pinned host logits f32 [T,E], x bf16 bits [T,D],
        scale f32 [E]; the result lands in pinned host h_out f32 [T,D].  The
        library's moe_pw_step_host enqueues the upload, the path and the
        download; this only orders the reuse of each buffer set."""
        k = self.n % self.depth
        b, sc = self.bufs[k], self.s_comp[k]
        if self.inputs_free[k] is not None:
            self.s_in.wait_event(self.inputs_free[k])   # inputs read by the last compute
        if self.output_free[k] is not None:
            sc.wait_event(self.output_free[k])          # output read by the last download
        moe_pw_step_host(self.cfg, h_logits, h_x, h_scale, h_out, self.h_counters[k],
                         self.dev[k], sc, self.s_in, self.s_out)
        done = torch.cuda.Event()
        done.record(sc)
        self.inputs_free[k] = done
        out_done = torch.cuda.Event()
        out_done.record(self.s_out)
        self.output_free[k] = out_done
        self.n += 1
        return k

    def synchronize(self):
        for s in [self.s_in, self.s_out, *self.s_comp]:
            s.synchronize()

    def stats(self, k: int) -> moe_pw_counters:
        """Counters of the last batch that used buffer set k (after synchronize)."""
        return moe_pw_counters.from_buffer_copy(self.h_counters[k].numpy().tobytes())
