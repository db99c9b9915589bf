"""CPU oracle for pooled-wave MoE dispatch/combine (ctypes wrapper over oracle.c).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py``; never by the library.  It shares no code
with the CUDA path and takes no input from it.

Every function here is argument marshalling around the single-threaded C
definitions in ``oracle.c``; the arithmetic lives there, each step citing the
page passage it follows.  ``run()`` chains the stages in the method's order:
route -> sender assignment -> pack -> (exchange = index relabel) -> receiver
bucketing -> per-expert op -> combine.

Parity status: every stage is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_*.py`` (brute force on tiny inputs, closed forms, library
routines, invariants); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")


def build(force: bool = False) -> str:
    """Compile oracle.c (plain gcc, no FMA contraction, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Geom(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("T_s", ctypes.c_int64),
                ("R", ctypes.c_int32), ("L", ctypes.c_int32), ("W", ctypes.c_int32),
                ("P", ctypes.c_int32), ("E", ctypes.c_int32), ("k", ctypes.c_int32),
                ("D", ctypes.c_int32), ("pad", ctypes.c_int32),
                ("C_s", ctypes.c_int64), ("C_r", ctypes.c_int64)]


@dataclass
class Geom:
    """Batch geometry.  ``T_s`` is the number of tokens per source shard; the
    sources present are ``T // T_s`` (all R of them for a full batch)."""

    T: int
    T_s: int
    R: int
    L: int
    W: int
    P: int
    k: int
    D: int
    C_s: int
    C_r: int

    @property
    def E(self) -> int:
        return self.R * self.L

    @property
    def n_src(self) -> int:
        return self.T // self.T_s

    @property
    def n_pools(self) -> int:
        return self.n_src * self.R * self.W

    @property
    def n_slots(self) -> int:
        return self.n_pools * self.C_s

    def c(self) -> _Geom:
        return _Geom(self.T, self.T_s, self.R, self.L, self.W, self.P, self.E, self.k,
                     self.D, 0, self.C_s, self.C_r)


_lib = None


def _configure(lib):
    """Declare the C signatures on a loaded oracle library."""
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
    gp = ctypes.POINTER(_Geom)
    lib.orc_capacity.argtypes = [i64, i64, i32, i32, i32, i32, i32,
                                 ctypes.POINTER(i64), ctypes.POINTER(i64)]
    lib.orc_route.argtypes = [gp, vp, vp, vp]
    lib.orc_assign_pooled.argtypes = [gp, vp, vp, vp, vp]
    lib.orc_assign_pooled.restype = i64
    lib.orc_pack.argtypes = [gp, i64, vp, vp, vp, vp, vp]
    lib.orc_pack_headers.argtypes = [gp, i64, vp, vp, vp]
    lib.orc_bucket.argtypes = [gp, vp, vp, vp, vp, vp, vp]
    lib.orc_bucket.restype = i64
    lib.orc_assign_ragged.argtypes = [gp, vp, vp, vp, vp, vp]
    lib.orc_bucket_ragged.argtypes = [gp, i64, vp, vp, vp, vp]
    lib.orc_kept.argtypes = [gp, vp]
    lib.orc_kept.restype = i64
    lib.orc_expert_pooled.argtypes = [gp, i64, vp, vp, vp, vp, vp, vp]
    lib.orc_expert_ragged.argtypes = [gp, i64, vp, vp, vp, vp, vp]
    lib.orc_combine.argtypes = [gp, vp, vp, vp, vp, vp]
    lib.orc_combine_tokens.argtypes = [gp, vp, vp, vp, vp, vp, vp, vp, i64, vp, vp]
    lib.orc_combine_mag.argtypes = [gp, vp, vp, vp, vp, vp]
    lib.orc_combine_backward.argtypes = [gp, i64, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.orc_dispatch_backward.argtypes = [gp, vp, vp, vp, vp]
    lib.orc_backward_tokens.argtypes = [gp, vp, vp, vp, vp, vp, vp, vp, vp, i64, vp, vp, vp, vp]
    lib.orc_project.argtypes = [vp, vp, i64, i64, i64, vp, vp, vp, vp]
    lib.orc_seq_balance.argtypes = [gp, i64, ctypes.c_double, vp, vp, vp, vp, vp, vp]
    lib.orc_bf16_round.argtypes = [vp, vp, i64]
    lib.orc_expert_product.argtypes = [vp, vp, vp, i64]
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _configure(ctypes.CDLL(build()))
    return _lib


class variant:
    """Context manager that routes every oracle call to another build of
    oracle.c (the tests use it to plant mistakes and check a pin catches them)."""

    def __init__(self, so_path: str):
        self.lib = _configure(ctypes.CDLL(so_path))

    def __enter__(self):
        global _lib
        self.saved, _lib = _load(), self.lib
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


def _p(a: np.ndarray) -> int:
    assert a.flags.c_contiguous, "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


# Integer outputs are handed to the C code pre-filled with this value, so an
# entry that a C function forgets to write cannot pass for a plausible one
# (np.empty could hold zeros or -1 by chance).
POISON = -0x5A5A5A5B


def _out_i32(shape) -> np.ndarray:
    return np.full(shape, POISON, np.int32)


def capacity(T: int, T_s: int, E: int, k: int, P: int, cf_send_pct: int, cf_recv_pct: int):
    """(C_s, C_r) as defined in oracle.c (ceil of factor x uniform-routing mean)."""
    cs, cr = ctypes.c_int64(), ctypes.c_int64()
    if _load().orc_capacity(T, T_s, E, k, P, cf_send_pct, cf_recv_pct,
                            ctypes.byref(cs), ctypes.byref(cr)) != 0:
        raise ValueError("bad capacity arguments")
    return int(cs.value), int(cr.value)


def geom_for(w, T: int | None = None, T_s: int | None = None) -> Geom:
    """Geometry of workload ``w`` (a ``synth.Workload``).  ``T``/``T_s`` select a
    sample of source shards; capacities always come from the full batch."""
    T_full, Ts_full = w.T, w.T // w.R
    C_s, C_r = capacity(T_full, Ts_full, w.E, w.k, w.P, w.cf_send_pct, w.cf_recv_pct)
    return Geom(T=T_full if T is None else T, T_s=Ts_full if T_s is None else T_s,
                R=w.R, L=w.L, W=w.W, P=w.P, k=w.k, D=w.D, C_s=C_s, C_r=C_r)


def route(g: Geom, logits: np.ndarray):
    lg = _c(logits, np.float32).reshape(g.T, g.E)
    idx = _out_i32((g.T, g.k))
    gates = np.empty((g.T, g.k), np.float64)
    gc = g.c()
    _load().orc_route(ctypes.byref(gc), _p(lg), _p(idx), _p(gates))
    return idx, gates


def assign_pooled(g: Geom, idx: np.ndarray):
    idx = _c(idx, np.int32)
    slot_map = _out_i32((g.T, g.k))
    occ = _out_i32((g.n_src, g.R, g.W))
    slot_tok = _out_i32((g.n_slots,))
    gc = g.c()
    dropped = _load().orc_assign_pooled(ctypes.byref(gc), _p(idx), _p(slot_map), _p(occ),
                                        _p(slot_tok))
    return slot_map, occ, slot_tok, int(dropped)


def assign_ragged(g: Geom, idx: np.ndarray):
    idx = _c(idx, np.int32)
    slot_map = _out_i32((g.T, g.k))
    row_off = _out_i32((g.E + 1,))
    row_cnt = _out_i32((g.E,))
    slot_tok = _out_i32((g.T * g.k,))
    gc = g.c()
    _load().orc_assign_ragged(ctypes.byref(gc), _p(idx), _p(slot_map), _p(row_off),
                              _p(row_cnt), _p(slot_tok))
    return slot_map, row_off, row_cnt, slot_tok


def pack(g: Geom, n_slots: int, x: np.ndarray, idx: np.ndarray, slot_map: np.ndarray):
    x = _c(x, np.uint16)
    pool_x = np.empty((n_slots, g.D), np.uint16)
    pool_hdr = _out_i32((n_slots,))
    gc = g.c()
    _load().orc_pack(ctypes.byref(gc), n_slots, _p(x), _p(_c(idx, np.int32)),
                     _p(_c(slot_map, np.int32)), _p(pool_x), _p(pool_hdr))
    return pool_x, pool_hdr


def pack_headers(g: Geom, n_slots: int, idx: np.ndarray, slot_map: np.ndarray) -> np.ndarray:
    pool_hdr = _out_i32((n_slots,))
    gc = g.c()
    _load().orc_pack_headers(ctypes.byref(gc), n_slots, _p(_c(idx, np.int32)),
                             _p(_c(slot_map, np.int32)), _p(pool_hdr))
    return pool_hdr


def kept(g: Geom, bucket_cnt: np.ndarray) -> int:
    """Rows every expert accepted (the drop statistics' "kept")."""
    gc = g.c()
    return int(_load().orc_kept(ctypes.byref(gc), _p(_c(bucket_cnt, np.int32))))


def bucket_ragged(g: Geom, row_hdr: np.ndarray):
    """Dropless receiver: (recv_row, arrivals, bucket_cnt) of every row."""
    row_hdr = _c(row_hdr, np.int32)
    recv_row = _out_i32((row_hdr.size,))
    arrivals = _out_i32((g.E,))
    bucket_cnt = _out_i32((g.E,))
    gc = g.c()
    _load().orc_bucket_ragged(ctypes.byref(gc), row_hdr.size, _p(row_hdr), _p(recv_row),
                              _p(arrivals), _p(bucket_cnt))
    return recv_row, arrivals, bucket_cnt


def bucket(g: Geom, pool_hdr: np.ndarray, occ: np.ndarray):
    recv_row = _out_i32((g.n_slots,))
    bucket_slot = _out_i32((g.E, g.C_r))
    arrivals = _out_i32((g.E,))
    bucket_cnt = _out_i32((g.E,))
    gc = g.c()
    dropped = _load().orc_bucket(ctypes.byref(gc), _p(_c(pool_hdr, np.int32)),
                                 _p(_c(occ, np.int32)), _p(recv_row), _p(bucket_slot),
                                 _p(arrivals), _p(bucket_cnt))
    return recv_row, bucket_slot, arrivals, bucket_cnt, int(dropped)


def expert_pooled(g: Geom, pool_x, bucket_slot, bucket_cnt, scale):
    n = pool_x.shape[0]
    ret_x = np.empty_like(pool_x)
    ret_hdr = _out_i32((n,))
    gc = g.c()
    _load().orc_expert_pooled(ctypes.byref(gc), n, _p(_c(pool_x, np.uint16)),
                              _p(_c(bucket_slot, np.int32)), _p(_c(bucket_cnt, np.int32)),
                              _p(_c(scale, np.float32)), _p(ret_x), _p(ret_hdr))
    return ret_x, ret_hdr


def expert_ragged(g: Geom, rows, row_hdr, scale):
    n = rows.shape[0]
    ret_x = np.empty_like(rows)
    ret_hdr = _out_i32((n,))
    gc = g.c()
    _load().orc_expert_ragged(ctypes.byref(gc), n, _p(_c(rows, np.uint16)),
                              _p(_c(row_hdr, np.int32)), _p(_c(scale, np.float32)),
                              _p(ret_x), _p(ret_hdr))
    return ret_x, ret_hdr


def combine(g: Geom, ret_x, ret_hdr, slot_map, gates, with_mag: bool = False):
    out = np.empty((g.T, g.D), np.float64)
    gc = g.c()
    args = (_p(_c(ret_x, np.uint16)), _p(_c(ret_hdr, np.int32)), _p(_c(slot_map, np.int32)),
            _p(_c(gates, np.float64)))
    _load().orc_combine(ctypes.byref(gc), *args, _p(out))
    if not with_mag:
        return out
    mag = np.empty((g.T, g.D), np.float64)
    _load().orc_combine_mag(ctypes.byref(gc), *args, _p(mag))
    return out, mag


def combine_tokens(g: Geom, x, idx, gates, slot_map, recv_row, scale, tokens):
    tokens = _c(tokens, np.int64)
    out = np.empty((tokens.size, g.D), np.float64)
    mag = np.empty((tokens.size, g.D), np.float64)
    gc = g.c()
    _load().orc_combine_tokens(ctypes.byref(gc), _p(_c(x, np.uint16)), _p(_c(idx, np.int32)),
                               _p(_c(gates, np.float64)), _p(_c(slot_map, np.int32)),
                               _p(_c(recv_row, np.int32)), _p(_c(scale, np.float32)),
                               _p(tokens), tokens.size, _p(out), _p(mag))
    return out, mag


def run_headers(w, logits: np.ndarray) -> dict:
    """The integer part of the path (route, assignment, headers, bucketing)
    plus the gates, without materialising any pool rows.  Rows are checked
    per slot / per token with ``combine_tokens`` and ``expert_product``."""
    g = geom_for(w)
    r = {"geom": g}
    r["idx"], r["gates"] = route(g, logits)
    if w.mode == 0:
        r["slot_map"], r["occ"], r["slot_tok"], r["sender_dropped"] = assign_pooled(g, r["idx"])
        r["pool_hdr"] = pack_headers(g, g.n_slots, r["idx"], r["slot_map"])
        (r["recv_row"], r["bucket_slot"], r["arrivals"], r["bucket_cnt"],
         r["receiver_dropped"]) = bucket(g, r["pool_hdr"], r["occ"])
    else:
        r["slot_map"], r["row_off"], r["row_cnt"], r["slot_tok"] = assign_ragged(g, r["idx"])
        n_rows = g.T * g.k
        r["pool_hdr"] = pack_headers(g, n_rows, r["idx"], r["slot_map"])
        r["recv_row"], r["arrivals"], r["bucket_cnt"] = bucket_ragged(g, r["pool_hdr"])
        r["sender_dropped"] = r["receiver_dropped"] = 0
    r["kept"] = kept(g, r["bucket_cnt"])
    return r


def combine_backward(g: Geom, dout, ret_x, ret_hdr, slot_map, idx, gates):
    """(d_ret bf16 bits [n_slots, D], dgate f64 [T, k], dlogits f64 [T, E])."""
    n = ret_x.shape[0]
    d_ret = np.empty((n, g.D), np.uint16)
    dgate = np.empty((g.T, g.k), np.float64)
    dlogits = np.empty((g.T, g.E), np.float64)
    gc = g.c()
    _load().orc_combine_backward(ctypes.byref(gc), n, _p(_c(dout, np.float32)),
                                 _p(_c(ret_x, np.uint16)), _p(_c(ret_hdr, np.int32)),
                                 _p(_c(slot_map, np.int32)), _p(_c(idx, np.int32)),
                                 _p(_c(gates, np.float64)), _p(d_ret), _p(dgate), _p(dlogits))
    return d_ret, dgate, dlogits


def dispatch_backward(g: Geom, d_pool, recv_row, slot_map):
    """dx f64 [T, D]."""
    dx = np.empty((g.T, g.D), np.float64)
    gc = g.c()
    _load().orc_dispatch_backward(ctypes.byref(gc), _p(_c(d_pool, np.uint16)),
                                  _p(_c(recv_row, np.int32)), _p(_c(slot_map, np.int32)), _p(dx))
    return dx


def backward_tokens(g: Geom, x, idx, gates, slot_map, recv_row, scale, dout, tokens):
    """Per-token backward (see orc_backward_tokens): d_ret rows [n, k, D] bf16
    bits, dgate [n, k], dlogits [n, E], dx [n, D]."""
    tokens = _c(tokens, np.int64)
    n = tokens.size
    d_ret = np.empty((n, g.k, g.D), np.uint16)
    dgate = np.empty((n, g.k), np.float64)
    dlogits = np.empty((n, g.E), np.float64)
    dx = np.empty((n, g.D), np.float64)
    gc = g.c()
    _load().orc_backward_tokens(ctypes.byref(gc), _p(_c(x, np.uint16)), _p(_c(idx, np.int32)),
                                _p(_c(gates, np.float64)), _p(_c(slot_map, np.int32)),
                                _p(_c(recv_row, np.int32)), _p(_c(scale, np.float32)),
                                _p(_c(dout, np.float32)), _p(tokens), n, _p(d_ret), _p(dgate),
                                _p(dlogits), _p(dx))
    return d_ret, dgate, dlogits, dx


def run_backward(w, r: dict, dout: np.ndarray, scale: np.ndarray) -> dict:
    """Backward of ``run``'s forward for a given dL/dout: combine backward,
    the expert op's backward (the same scale op on the gradient pool, the
    bf16 rounding passed straight through) and the pack transpose."""
    g = r["geom"]
    b = {}
    b["d_ret"], b["dgate"], b["dlogits"] = combine_backward(
        g, dout, r["ret_x"], r["ret_hdr"], r["slot_map"], r["idx"], r["gates"])
    if w.mode == 0:
        b["d_pool"], _ = expert_pooled(g, b["d_ret"], r["bucket_slot"], r["bucket_cnt"], scale)
    else:
        b["d_pool"], _ = expert_ragged(g, b["d_ret"], r["pool_hdr"], scale)
    b["dx"] = dispatch_backward(g, b["d_pool"], r["recv_row"], r["slot_map"])
    return b


def project(A: np.ndarray, Bt: np.ndarray, exact: bool = False, add: np.ndarray | None = None):
    """C = bf16(A @ Bt^T [+ add]) (bf16 bits); with exact=True also the
    double sums and sum |terms|."""
    A, Bt = _c(A, np.uint16), _c(Bt, np.uint16)
    M, K = A.shape
    N = Bt.shape[0]
    assert Bt.shape[1] == K
    if add is not None:
        add = _c(add, np.uint16)
        assert add.shape == (M, N)
    C = np.empty((M, N), np.uint16)
    Ce = np.empty((M, N), np.float64) if exact else None
    mag = np.empty((M, N), np.float64) if exact else None
    _load().orc_project(_p(A), _p(Bt), M, N, K, _p(add) if add is not None else None, _p(C),
                        _p(Ce) if exact else None, _p(mag) if exact else None)
    return (C, Ce, mag) if exact else C


def seq_balance(g: Geom, seq_len: int, alpha: float, logits, idx, with_grad: bool = True):
    """Sequence-level balance term (see orc_seq_balance): f, P [n_seq, E],
    loss [n_seq] and, with_grad, dlogits [T, E]."""
    lg = _c(logits, np.float32).reshape(g.T, g.E)
    ix = _c(idx, np.int32).reshape(g.T, g.k)
    n_seq = g.T // seq_len
    f = np.empty((n_seq, g.E), np.float64)
    P = np.empty((n_seq, g.E), np.float64)
    loss = np.empty((n_seq,), np.float64)
    dl = np.empty((g.T, g.E), np.float64) if with_grad else None
    gc = g.c()
    _load().orc_seq_balance(ctypes.byref(gc), seq_len, alpha, _p(lg), _p(ix), _p(f), _p(P),
                            _p(loss), _p(dl) if with_grad else None)
    return (f, P, loss, dl) if with_grad else (f, P, loss)


def bf16_round(a: np.ndarray) -> np.ndarray:
    a = _c(a, np.float32)
    out = np.empty(a.shape, np.uint16)
    _load().orc_bf16_round(_p(a), _p(out), a.size)
    return out


def expert_product(s: np.ndarray, x: np.ndarray) -> np.ndarray:
    s, x = _c(s, np.float32), _c(x, np.uint16)
    assert s.shape == x.shape
    y = np.empty(x.shape, np.uint16)
    _load().orc_expert_product(_p(s), _p(x), _p(y), x.size)
    return y


def run(w, logits: np.ndarray, x: np.ndarray, scale: np.ndarray, T: int | None = None,
        with_mag: bool = False) -> dict:
    """Whole path for workload ``w`` (optionally only its first ``T`` tokens,
    i.e. the first T // T_s source shards).  Returns every intermediate."""
    g = geom_for(w, T=T)
    lg = logits[: g.T]
    xx = x[: g.T]
    r = {"geom": g}
    r["idx"], r["gates"] = route(g, lg)
    if w.mode == 0:
        r["slot_map"], r["occ"], r["slot_tok"], r["sender_dropped"] = assign_pooled(g, r["idx"])
        r["pool_x"], r["pool_hdr"] = pack(g, g.n_slots, xx, r["idx"], r["slot_map"])
        (r["recv_row"], r["bucket_slot"], r["arrivals"], r["bucket_cnt"],
         r["receiver_dropped"]) = bucket(g, r["pool_hdr"], r["occ"])
        r["ret_x"], r["ret_hdr"] = expert_pooled(g, r["pool_x"], r["bucket_slot"],
                                                 r["bucket_cnt"], scale)
    else:
        r["slot_map"], r["row_off"], r["row_cnt"], r["slot_tok"] = assign_ragged(g, r["idx"])
        n_rows = g.T * g.k
        r["pool_x"], r["pool_hdr"] = pack(g, n_rows, xx, r["idx"], r["slot_map"])
        r["recv_row"], r["arrivals"], r["bucket_cnt"] = bucket_ragged(g, r["pool_hdr"])
        r["sender_dropped"] = r["receiver_dropped"] = 0
        r["ret_x"], r["ret_hdr"] = expert_ragged(g, r["pool_x"], r["pool_hdr"], scale)
    res = combine(g, r["ret_x"], r["ret_hdr"], r["slot_map"], r["gates"], with_mag=with_mag)
    if with_mag:
        r["out"], r["mag"] = res
    else:
        r["out"] = res
    r["kept"] = kept(g, r["bucket_cnt"])
    return r
