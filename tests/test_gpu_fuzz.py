"""Seeded random small configurations: the whole GPU path against the whole
oracle, with the same bar as tests/test_gpu_parity.py (bit-exact integer and
byte outputs, gates within 1e-6 relative, combine within 1e-6 of its scale).

Each case draws its geometry (ranks, experts per rank, waves, top-k, width,
tokens per source, capacity factors, pooled or dropless mode, logit
distribution) from a fixed seed, so a failure names a case that reproduces.
The draws cover shapes the named workloads do not: one-token sources, widths
that are not a multiple of 128 bytes, P up to 6, k up to 12, factors below
the mean load (heavy drops) and far above it.
"""
import numpy as np
import pytest

import oracle
from combine_moe_pw_b200 import synth
from fuzz_cases import random_wide_workload, random_workload
from test_gpu_parity import _inputs, check_full, run_gpu

N_CASES = 24
N_BACKWARD = 12
N_PROJECT = 12
N_WIDE = 8


def test_draws_are_varied():
    ws = [random_workload(i) for i in range(N_CASES)]
    assert len({(w.R, w.L, w.W, w.P, w.k, w.D) for w in ws}) > N_CASES // 2
    assert any(w.mode == synth.MODE_RAGGED for w in ws)
    assert any(w.cf_send_pct and w.cf_send_pct < 100 for w in ws)
    wide = [random_wide_workload(i) for i in range(N_WIDE)]
    assert len({w.D for w in wide}) > 1 and len({(w.R, w.L, w.k) for w in wide}) > N_WIDE // 2


@pytest.mark.gpu
@pytest.mark.parametrize("i", range(N_CASES))
def test_random_config_full_parity(i):
    w = random_workload(i)
    lg, x, s = _inputs(w)
    b, st = run_gpu(w, lg, x, s)
    check_full(w, lg, x, s, b, st)


@pytest.mark.gpu
@pytest.mark.parametrize("i", range(N_WIDE))
def test_random_wide_config_full_parity(i):
    """Seeded draws at 1024 to 6144 bf16 per row (the pack's and the expert
    op's shared-memory rings then hold few rows per block)."""
    w = random_wide_workload(i)
    lg, x, s = _inputs(w)
    b, st = run_gpu(w, lg, x, s)
    check_full(w, lg, x, s, b, st)


@pytest.mark.gpu
@pytest.mark.parametrize("i", range(N_BACKWARD))
def test_random_config_backward(i):
    """The backward (combine, expert op, pack) on further seeded draws, with
    the bounds of tests/test_gpu_backward.py."""
    from test_gpu_backward import check_backward, run_both
    w = random_workload(N_CASES + i)
    b, st, r, ob, dout = run_both(w)
    check_backward(w, b, st, r, ob, dout)


def random_gemm(i: int):
    rng = np.random.default_rng(9000 + i)
    return (int(rng.integers(1, 700)), 8 * int(rng.integers(1, 130)),
            8 * int(rng.integers(1, 260)))


@pytest.mark.gpu
@pytest.mark.parametrize("i", range(N_PROJECT))
def test_random_projection(i):
    """moe_pw_project on seeded shapes (M 1..699, N and K multiples of 8 up to
    1032 and 2072: ragged row, column and K tails of the 256-row pair tiles),
    with the bound of tests/test_gpu_project.py; bf16 codes may differ from
    the oracle's (which sums in double) on at most 2% of the elements or 3 of
    them, whichever is more."""
    from test_gpu_project import _f64, gpu_project
    M, N, K = random_gemm(i)
    A = synth.matrix_bf16(M, K, 1.0, 50 + i)
    Bt = synth.matrix_bf16(N, K, K ** -0.5, 80 + i)
    C, _ = gpu_project(A, Bt)
    Cr, Ce, mag = oracle.project(A, Bt, exact=True)
    got = _f64(C)
    assert np.all(np.isfinite(got))
    assert np.all(np.abs(got - Ce) <= 2.0 ** -8 * np.abs(Ce) + 2.0 ** -20 * mag + 1e-30)
    assert (C != Cr).sum() <= max(0.02 * C.size, 3)
