"""Host-only pin of the tcgen05 descriptor encoders (umma.cuh): compiled as
plain host code with nvcc and compared bit for bit with CUTLASS's
cute::UMMA::SmemDescriptor / InstrDescriptor unions.  No GPU needed."""
import glob
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CANDIDATES = glob.glob("/opt/prime-rl/.venv/lib/python3.12/site-packages/*/data/cutlass/include") + \
    glob.glob("/opt/prime-rl/.venv/lib/python3.12/site-packages/*/3rdparty/cutlass/include")


@pytest.mark.skipif(not CANDIDATES, reason="no CUTLASS headers in this image")
def test_descriptor_encoders_match_cutlass(tmp_path):
    exe = tmp_path / "umma_check"
    subprocess.check_call(["/usr/local/cuda/bin/nvcc", "-std=c++17", "-I", CANDIDATES[0], "-I",
                           os.path.join(ROOT, "combine_moe_pw_b200", "csrc"), "-o", str(exe),
                           os.path.join(ROOT, "tests", "host", "umma_desc_check.cu")],
                          stderr=subprocess.DEVNULL)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "OK", out.stdout
