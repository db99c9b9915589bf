"""Shared pytest configuration.

Markers:
  gpu  - needs a CUDA device (B200, sm_100a) and the built CUDA library.
Everything unmarked runs on a CPU-only host.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device and the built CUDA library")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device on this host")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


@pytest.fixture(scope="session")
def tiny_inputs():
    from combine_moe_pw_b200 import synth
    w = synth.WORKLOADS["tiny"]
    return w, synth.logits(w), synth.x_bf16(w), synth.scales(w)


@pytest.fixture(scope="session")
def tiny_oracle(tiny_inputs):
    import oracle
    w, lg, x, s = tiny_inputs
    return oracle.run(w, lg, x, s, with_mag=True)
