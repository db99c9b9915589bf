"""Pins for the oracle's latent projection: a plain matrix product with bf16
operands, summed exactly enough in double, rounded fp32 -> bf16."""
import numpy as np
import torch

import oracle
from combine_moe_pw_b200 import synth


def _f64(u16):
    return (u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_project_matches_numpy_matmul():
    A = synth.matrix_bf16(37, 200, 1.0, 20)
    Bt = synth.matrix_bf16(24, 200, 200 ** -0.5, 21)
    C, Ce, mag = oracle.project(A, Bt, exact=True)
    ref = _f64(A) @ _f64(Bt).T
    np.testing.assert_allclose(Ce, ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(mag, np.abs(_f64(A)) @ np.abs(_f64(Bt)).T, rtol=1e-12)
    # rounding: fp32 then bf16 nearest-even, as torch does it
    expect = torch.from_numpy(ref.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
    np.testing.assert_array_equal(C, expect.view(np.uint16))


def test_project_identity_and_zero():
    K = 64
    eye = torch.eye(K, dtype=torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    A = synth.matrix_bf16(5, K, 1.0, 22)
    np.testing.assert_array_equal(oracle.project(A, eye), A)
    np.testing.assert_array_equal(oracle.project(A, np.zeros((3, K), np.uint16)), 0)


def test_projection_inputs_shapes():
    w = synth.WORKLOADS["tiny"].with_(T=16)
    h, wd, wu = synth.projection_inputs(w, model_width=256)
    assert h.shape == (16, 256) and wd.shape == (w.D, 256) and wu.shape == (256, w.D)
    assert abs(_f64(wd).std() - 256 ** -0.5) < 0.01


def test_project_with_shared_path_merge():
    """The merge with the shared path: bf16(A @ Bt^T + add), formed exactly
    and rounded once, against numpy's float64 product plus the addend and
    torch's fp32 -> bf16 rounding; add = 0 gives the plain projection."""
    A = synth.matrix_bf16(29, 136, 1.0, 23)
    Bt = synth.matrix_bf16(40, 136, 136 ** -0.5, 24)
    add = synth.matrix_bf16(29, 40, 1.0, 25)
    C, Ce, mag = oracle.project(A, Bt, exact=True, add=add)
    ref = _f64(A) @ _f64(Bt).T + _f64(add)
    np.testing.assert_allclose(Ce, ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(mag, np.abs(_f64(A)) @ np.abs(_f64(Bt)).T + np.abs(_f64(add)),
                               rtol=1e-12)
    expect = torch.from_numpy(ref.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
    np.testing.assert_array_equal(C, expect.view(np.uint16))
    np.testing.assert_array_equal(oracle.project(A, Bt, add=np.zeros((29, 40), np.uint16)),
                                  oracle.project(A, Bt))
    # a zero product leaves the addend itself
    np.testing.assert_array_equal(oracle.project(np.zeros_like(A), Bt, add=add), add)
