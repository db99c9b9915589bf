"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the CPU oracle.

The generator (``synth.c``) is counter-based, so every value depends only on
(seed, stream, index).  This module holds the workload recipes (shapes and
distributions) and nothing of the routing/packing/combining arithmetic.

Workload recipes follow the shapes of the Marin 535B-A23B MoE layer described in
"Marin 开始公开训练 535B 参数 MoE 模型" (lamjinlab blog), section 二: 384 routed
experts, top-8 routing, 64 expert-parallel ranks with 6 experts each, three
waves, a 3072-wide latent, sender/receiver capacity factors 1.10 / 1.15.  The
pages measure on a trained router; these synthetic logits stand in for it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, replace

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")

LOGIT_IID, LOGIT_SEQBIAS, LOGIT_ZIPF = 0, 1, 2
MODE_POOLED, MODE_RAGGED = 0, 1


@dataclass(frozen=True)
class Workload:
    """Shape and input distribution of one synthetic batch."""

    name: str
    T: int            # tokens in the batch
    R: int            # expert-parallel ranks (logical shards on one GPU)
    L: int            # routed experts per rank
    W: int            # waves per (source, destination) pair
    P: int            # experts carried per wave (L == W * P)
    k: int            # experts chosen per token
    D: int            # latent width, bf16 elements
    seq_len: int      # tokens per sequence (drives the per-sequence logit bias)
    logit_kind: int   # LOGIT_IID / LOGIT_SEQBIAS / LOGIT_ZIPF
    sigma_b: float = 0.5
    cf_send_pct: int = 110   # <= 0: unbounded
    cf_recv_pct: int = 115   # <= 0: unbounded
    mode: int = MODE_POOLED
    seed: int = 0
    scale_lo: float = 0.5
    scale_hi: float = 1.5

    @property
    def E(self) -> int:
        return self.R * self.L

    @property
    def assignments(self) -> int:
        return self.T * self.k

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


_PAGES = dict(R=64, L=6, W=3, P=2, k=8, D=3072)

WORKLOADS = {
    # small parity case: 8 logical ranks x 6 = 48 experts, 2048 = 8 x 256 tokens, iid logits
    "tiny": Workload("tiny", T=2048, R=8, L=6, W=3, P=2, k=8, D=128, seq_len=256,
                     logit_kind=LOGIT_IID),
    # one layer at the pages' shapes: 65,536 = 16 x 4096 tokens
    "layer": Workload("layer", T=65536, seq_len=4096, logit_kind=LOGIT_SEQBIAS, **_PAGES),
    # rack-scale token batch on one GPU: 262,144 = 64 x 4096 tokens
    "rack": Workload("rack", T=262144, seq_len=4096, logit_kind=LOGIT_SEQBIAS, **_PAGES),
    # long context: 262,144 = 4 x 65,536 tokens (fewer sequences -> more imbalance)
    "long": Workload("long", T=262144, seq_len=65536, logit_kind=LOGIT_SEQBIAS, **_PAGES),
    # dropless ragged variant: 262,144 = 32 x 8192 tokens, Zipf(1) expert popularity
    "ragged": Workload("ragged", T=262144, seq_len=8192, logit_kind=LOGIT_ZIPF,
                       cf_send_pct=0, cf_recv_pct=0, mode=MODE_RAGGED, **_PAGES),
}


def build(force: bool = False) -> str:
    """Compile the generator with gcc (OpenMP) next to this file."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64, i32, u64, f64, vp = (ctypes.c_int64, ctypes.c_int32, ctypes.c_uint64,
                                  ctypes.c_double, ctypes.c_void_p)
        lib.synth_logits.argtypes = [ctypes.c_int, i64, i32, i64, f64, u64, vp]
        lib.synth_x_bf16.argtypes = [i64, i32, u64, vp]
        lib.synth_logits_rows.argtypes = [ctypes.c_int, i64, i64, i32, i64, f64, u64, vp]
        lib.synth_x_bf16_rows.argtypes = [i64, i64, i32, u64, vp]
        lib.synth_scales.argtypes = [i32, f64, f64, u64, vp]
        lib.synth_dout_f32.argtypes = [i64, i32, u64, vp]
        lib.synth_matrix_bf16.argtypes = [i64, i64, f64, u64, u64, vp]
        lib.synth_u64.argtypes = [u64, u64, u64]
        lib.synth_u64.restype = u64
        lib.synth_normal.argtypes = [u64, u64, u64]
        lib.synth_normal.restype = f64
        _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags.c_contiguous
    return a.ctypes.data


def logits(w: Workload, out: np.ndarray | None = None) -> np.ndarray:
    """Router logits fp32 [T, E] for workload ``w``."""
    out = np.empty((w.T, w.E), np.float32) if out is None else out
    assert out.dtype == np.float32 and out.shape == (w.T, w.E)
    rc = _load().synth_logits(w.logit_kind, w.T, w.E, w.seq_len, w.sigma_b, w.seed, _ptr(out))
    if rc != 0:
        raise ValueError(f"synth_logits failed for {w}")
    return out


def logits_rows(w: Workload, t0: int, n: int) -> np.ndarray:
    """Rows [t0, t0 + n) of ``logits(w)`` (one GPU's share of a batch)."""
    out = np.empty((n, w.E), np.float32)
    if _load().synth_logits_rows(w.logit_kind, t0, n, w.E, w.seq_len, w.sigma_b, w.seed,
                                 _ptr(out)) != 0:
        raise ValueError(f"synth_logits_rows failed for {w}")
    return out


def x_bf16_rows(w: Workload, t0: int, n: int) -> np.ndarray:
    """Rows [t0, t0 + n) of ``x_bf16(w)``."""
    out = np.empty((n, w.D), np.uint16)
    if _load().synth_x_bf16_rows(t0, n, w.D, w.seed, _ptr(out)) != 0:
        raise ValueError("synth_x_bf16_rows failed")
    return out


def x_bf16(w: Workload, out: np.ndarray | None = None) -> np.ndarray:
    """Latent rows as raw bf16 bits, uint16 [T, D]."""
    out = np.empty((w.T, w.D), np.uint16) if out is None else out
    assert out.dtype == np.uint16 and out.shape == (w.T, w.D)
    if _load().synth_x_bf16(w.T, w.D, w.seed, _ptr(out)) != 0:
        raise ValueError(f"synth_x_bf16 failed for {w}")
    return out


def dout(w: Workload, out: np.ndarray | None = None) -> np.ndarray:
    """Upstream gradient dL/dout for the backward, fp32 [T, D] ~ N(0, 1)."""
    out = np.empty((w.T, w.D), np.float32) if out is None else out
    assert out.dtype == np.float32 and out.shape == (w.T, w.D)
    if _load().synth_dout_f32(w.T, w.D, w.seed, _ptr(out)) != 0:
        raise ValueError("synth_dout_f32 failed")
    return out


# named matrices for the latent projections (stream ids >= 16)
STREAM_H, STREAM_W_DOWN, STREAM_W_UP = 16, 17, 18
MODEL_WIDTH = 6144  # model state width of the pages' layer (latent = half of it)


def matrix_bf16(rows: int, cols: int, std: float, stream: int, seed: int = 0) -> np.ndarray:
    """bf16 bits [rows, cols] ~ N(0, std^2) from a named stream."""
    out = np.empty((rows, cols), np.uint16)
    if _load().synth_matrix_bf16(rows, cols, std, seed, stream, _ptr(out)) != 0:
        raise ValueError("synth_matrix_bf16 failed")
    return out


def projection_inputs(w: Workload, model_width: int = MODEL_WIDTH):
    """Model-width activations h [T, Dm] ~ N(0,1) and random-init projection
    weights, both stored K-major for the GEMM: w_down_t [D, Dm] (h @ w_down_t^T
    gives the latent) and w_up_t [Dm, D] (latent @ w_up_t^T gives model width),
    each ~ N(0, 1/fan_in)."""
    h = matrix_bf16(w.T, model_width, 1.0, STREAM_H, w.seed)
    w_down_t = matrix_bf16(w.D, model_width, model_width ** -0.5, STREAM_W_DOWN, w.seed)
    w_up_t = matrix_bf16(model_width, w.D, w.D ** -0.5, STREAM_W_UP, w.seed)
    return h, w_down_t, w_up_t


def scales(w: Workload) -> np.ndarray:
    """Per-expert op scales s_e ~ U(scale_lo, scale_hi), fp32 [E]."""
    out = np.empty((w.E,), np.float32)
    if _load().synth_scales(w.E, w.scale_lo, w.scale_hi, w.seed, _ptr(out)) != 0:
        raise ValueError("synth_scales failed")
    return out


def raw_u64(seed: int, stream: int, i: int) -> int:
    return int(_load().synth_u64(seed, stream, i))


def raw_normal(seed: int, stream: int, n: int) -> float:
    return float(_load().synth_normal(seed, stream, n))


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    """Reinterpret bf16 bits (uint16) as fp32 values (exact widening)."""
    return (a.astype(np.uint32) << 16).view(np.float32)
