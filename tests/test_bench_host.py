"""Host-side helpers of bench.py on CPU: the DRAM-traffic figure scaled from a
committed small-case profile (and refused once a profiled source changes),
and the CPU baseline's sample accounting."""
import os
import shutil

import pytest

import bench
from combine_moe_pw_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROFILE = "pack_bucket_kernel_small_case_traffic.txt"


def _profiled_sources(text):
    return [ln.split(":", 1)[1].strip() for ln in text.splitlines()
            if ln.startswith("source_file:")]


def _ratio(text):
    return float([ln for ln in text.splitlines()
                  if ln.startswith("traffic_per_algorithmic_byte:")][0].split(":")[1])


def _copy_tree(tmp_path):
    """profiles/ and the profiled sources, in a scratch root."""
    text = open(os.path.join(ROOT, "profiles", PROFILE)).read()
    os.makedirs(tmp_path / "profiles")
    shutil.copy(os.path.join(ROOT, "profiles", PROFILE), tmp_path / "profiles" / PROFILE)
    for f in _profiled_sources(text):
        os.makedirs(os.path.dirname(tmp_path / f), exist_ok=True)
        shutil.copy(os.path.join(ROOT, f), tmp_path / f)
    return text


def test_traffic_scales_with_algorithmic_bytes(tmp_path, monkeypatch):
    text = _copy_tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert len(_profiled_sources(text)) >= 1
    got = bench.traffic_from_profiles("pack_bucket_kernel", 1.0e10)
    assert got == pytest.approx(_ratio(text) * 1.0e10)


def test_traffic_refused_when_a_profiled_source_changed(tmp_path, monkeypatch):
    text = _copy_tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    for f in _profiled_sources(text):  # each source on its own
        path = tmp_path / f
        keep = path.read_bytes()
        path.write_bytes(keep + b"\n// changed\n")
        assert bench.traffic_from_profiles("pack_bucket_kernel", 1.0e10) is None
        path.write_bytes(keep)
    assert bench.traffic_from_profiles("pack_bucket_kernel", 1.0e10) is not None


def test_traffic_none_without_a_profile(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_from_profiles("pack_bucket_kernel", 1.0e10) is None


def test_committed_traffic_profiles_match_their_sources():
    """Every committed traffic record still names the sources as they are, so
    the bench line's traffic figure is not silently dropped."""
    for name in os.listdir(os.path.join(ROOT, "profiles")):
        if not name.endswith("_small_case_traffic.txt"):
            continue
        kernel = name[: -len("_small_case_traffic.txt")]
        assert bench.traffic_from_profiles(kernel, 1.0) is not None, name


def test_cpu_sample_counts_every_run():
    w = synth.WORKLOADS["tiny"]
    units, seconds = bench.cpu_oracle_sample(w, 2, reps=3)
    assert units == 3 * 2 * (w.T // w.R) * w.k
    assert seconds > 0
