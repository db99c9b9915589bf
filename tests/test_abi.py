"""The C ABI on a CPU-only host: the library loads, exports every entry point
include/moe_pw.h declares, and its host-only logic (moe_pw_plan, argument
validation) behaves.  No kernel is launched here."""
import os
import re

import pytest

import oracle
from combine_moe_pw_b200 import build as cbuild
from combine_moe_pw_b200 import moe_pw as mp
from combine_moe_pw_b200 import synth

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "moe_pw.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_pw_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    cbuild.build()
    return mp.load_library()


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert "moe_pw_dispatch" in names and len(names) >= 11
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(mp.SIGNATURES), "binding and header disagree"


def test_version_and_strerror(lib):
    assert mp.moe_pw_version() == 10000
    assert lib.moe_pw_strerror(mp.MOE_PW_ENOMEM).decode().startswith("buffers exceed")


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_plan_capacities_agree_with_oracle(lib, name):
    w = synth.WORKLOADS[name]
    s = mp.moe_pw_plan(mp.Config.from_workload(w))
    if w.mode == synth.MODE_POOLED:
        cs, cr = oracle.capacity(w.T, w.T // w.R, w.E, w.k, w.P, w.cf_send_pct, w.cf_recv_pct)
        assert (s.C_s, s.C_r) == (cs, cr)
        assert s.n_slots == w.R * w.R * w.W * cs
        assert s.occ_len == w.R * w.R * w.W and s.bucket_len == w.E * cr
    else:
        assert s.n_slots == w.T * w.k and s.occ_len == w.E + 1 and s.bucket_len == 0


def test_plan_rack_sizes(lib):
    s = mp.moe_pw_plan(mp.Config.from_workload(synth.WORKLOADS["rack"]))
    assert (s.C_s, s.C_r, s.n_slots) == (188, 6281, 2310144)
    assert 30e9 < s.total_bytes < 40e9  # x, both pool sets, logits, out
    assert s.workspace_bytes % 256 == 0 and s.workspace_bytes < 4 << 20


def test_plan_budget_refuses(lib):
    cfg = mp.Config.from_workload(synth.WORKLOADS["rack"])
    with pytest.raises(mp.MoePwError) as ei:
        mp.moe_pw_plan(cfg, budget_bytes=16 << 30)
    assert ei.value.code == mp.MOE_PW_ENOMEM


@pytest.mark.parametrize("bad,code", [
    (dict(T=2049), mp.MOE_PW_EINVAL),          # T % R != 0
    (dict(E=50), mp.MOE_PW_EINVAL),            # E != R*L
    (dict(P=4), mp.MOE_PW_EINVAL),             # L != W*P
    (dict(k=0), mp.MOE_PW_EINVAL),
    (dict(k=49), mp.MOE_PW_EINVAL),            # k > E
    (dict(mode=2), mp.MOE_PW_EINVAL),
    (dict(T=-8), mp.MOE_PW_EINVAL),
    (dict(D=100), mp.MOE_PW_EUNSUPPORTED),     # D % 8
    (dict(D=12296), mp.MOE_PW_EUNSUPPORTED),   # D too wide
])
def test_plan_rejects(lib, bad, code):
    base = mp.Config.from_workload(synth.WORKLOADS["tiny"])
    cfg = mp.Config(**{**base.__dict__, **bad})
    with pytest.raises(mp.MoePwError) as ei:
        mp.moe_pw_plan(cfg)
    assert ei.value.code == code


def test_k_above_32_unsupported(lib):
    w = synth.WORKLOADS["layer"]
    cfg = mp.Config(**{**mp.Config.from_workload(w).__dict__, "k": 33})
    with pytest.raises(mp.MoePwError) as ei:
        mp.moe_pw_plan(cfg)
    assert ei.value.code == mp.MOE_PW_EUNSUPPORTED


def test_null_pointers_rejected_before_any_launch(lib):
    cfg = mp.Config.from_workload(synth.WORKLOADS["tiny"])
    for fn, args in [
        (mp.moe_pw_route, (0, 0, 0)),
        (mp.moe_pw_expert, (0, 0, 0, 0, 0, 0, 0)),
        (mp.moe_pw_combine, (0, 0, 0, 0, 0, 0)),
    ]:
        with pytest.raises(mp.MoePwError) as ei:
            fn(cfg, *[None] * len(args), stream=0)
        assert ei.value.code == mp.MOE_PW_EINVAL


def test_empty_batch_plans(lib):
    base = mp.Config.from_workload(synth.WORKLOADS["tiny"])
    s = mp.moe_pw_plan(mp.Config(**{**base.__dict__, "T": 0}))
    assert s.n_slots == 0 and s.C_s == 0 and s.C_r == 0


def test_misaligned_pointers_rejected_before_any_launch(lib):
    cfg = mp.Config.from_workload(synth.WORKLOADS["tiny"])
    good, odd = 1 << 20, (1 << 20) + 4  # placeholder addresses, never dereferenced
    with pytest.raises(mp.MoePwError) as ei:
        mp.moe_pw_route(cfg, odd, good, good, stream=0)      # logits need 16-byte alignment
    assert ei.value.code == mp.MOE_PW_EUNSUPPORTED
    with pytest.raises(mp.MoePwError) as ei:
        mp.moe_pw_combine(cfg, good, good, good, good, odd + 8, good, stream=0)
    assert ei.value.code == mp.MOE_PW_EUNSUPPORTED
    with pytest.raises(mp.MoePwError) as ei:
        mp.moe_pw_project(good, good, good, 128, 264, 100, good, stream=0)  # K % 8 != 0
    assert ei.value.code == mp.MOE_PW_EUNSUPPORTED
    with pytest.raises(mp.MoePwError) as ei:
        mp.moe_pw_selftest_wait_timeout(good + 4, 16, stream=0)
    assert ei.value.code == mp.MOE_PW_EUNSUPPORTED


@pytest.mark.parametrize("k,chunks_per_source", [(1, 1), (8, 1), (32, 4)])
def test_workspace_follows_the_chunk_rule(lib, k, chunks_per_source):
    """Ranking chunks hold 2048 assignments (2048 // k tokens, never more than
    a source's tokens): the workspace is the per-chunk counts plus the
    per-source totals, each padded to 256 bytes."""
    base = mp.Config.from_workload(synth.WORKLOADS["tiny"])  # 8 sources x 256 tokens
    cfg = mp.Config(**{**base.__dict__, "k": k})
    s = mp.moe_pw_plan(cfg)
    bins = cfg.R * cfg.W
    pad = lambda b: (b + 255) // 256 * 256
    assert s.workspace_bytes == pad(4 * cfg.R * chunks_per_source * bins) + pad(4 * cfg.R * bins)


def test_fused_dispatch_entries_validate_before_any_launch(lib):
    """The fused dispatch halves are pooled-mode calls: a ragged config is
    refused, and so are missing or misaligned buffers, all on the host."""
    tiny = mp.Config.from_workload(synth.WORKLOADS["tiny"])
    ragged = mp.Config(**{**tiny.__dict__, "mode": synth.MODE_RAGGED, "cf_send_pct": 0,
                          "cf_recv_pct": 0})
    good, odd = 1 << 20, (1 << 20) + 4  # placeholder addresses, never dereferenced
    ws = mp.moe_pw_plan(tiny).workspace_bytes
    with pytest.raises(mp.MoePwError) as ei:
        mp.moe_pw_assign_headers(ragged, good, good, good, good, good, good, ws, stream=0)
    assert ei.value.code == mp.MOE_PW_EUNSUPPORTED
    with pytest.raises(mp.MoePwError) as ei:
        mp.moe_pw_pack_bucket(ragged, *[good] * 10, stream=0)
    assert ei.value.code == mp.MOE_PW_EUNSUPPORTED
    with pytest.raises(mp.MoePwError) as ei:
        mp.moe_pw_assign_headers(tiny, good, good, good, None, good, good, ws, stream=0)
    assert ei.value.code == mp.MOE_PW_EINVAL
    with pytest.raises(mp.MoePwError) as ei:
        mp.moe_pw_assign_headers(tiny, good, good, good, good, good, good, ws - 256, stream=0)
    assert ei.value.code == mp.MOE_PW_EINVAL
    with pytest.raises(mp.MoePwError) as ei:
        mp.moe_pw_pack_bucket(tiny, *[good] * 6, None, *[good] * 3, stream=0)  # no recv_row
    assert ei.value.code == mp.MOE_PW_EINVAL
    with pytest.raises(mp.MoePwError) as ei:
        mp.moe_pw_pack_bucket(tiny, odd + 8, *[good] * 9, stream=0)  # x needs 16 bytes
    assert ei.value.code == mp.MOE_PW_EUNSUPPORTED


def test_route_assign_entries_validate_before_any_launch(lib):
    """moe_pw_route_assign(_form): pooled mode only, a known form, buffers
    present and aligned, a large enough workspace: all checked on the host."""
    tiny = mp.Config.from_workload(synth.WORKLOADS["tiny"])
    ragged = mp.Config(**{**tiny.__dict__, "mode": synth.MODE_RAGGED, "cf_send_pct": 0,
                          "cf_recv_pct": 0})
    good, odd = 1 << 20, (1 << 20) + 4  # placeholder addresses, never dereferenced
    ws = mp.moe_pw_plan(tiny).workspace_bytes
    args = [good] * 7  # logits, idx, gates, slot_map, occ, pool_hdr, counters
    with pytest.raises(mp.MoePwError) as ei:
        mp.moe_pw_route_assign_form(ragged, -1, *args, good, ws, stream=0)
    assert ei.value.code == mp.MOE_PW_EUNSUPPORTED
    for form in (-2, 2, 7):
        with pytest.raises(mp.MoePwError) as ei:
            mp.moe_pw_route_assign_form(tiny, form, *args, good, ws, stream=0)
        assert ei.value.code == mp.MOE_PW_EINVAL
    with pytest.raises(mp.MoePwError) as ei:
        mp.moe_pw_route_assign_form(tiny, -1, good, good, good, None, good, good, good, good, ws,
                                    stream=0)  # no slot_map
    assert ei.value.code == mp.MOE_PW_EINVAL
    with pytest.raises(mp.MoePwError) as ei:
        mp.moe_pw_route_assign_form(tiny, -1, *args, good, ws - 256, stream=0)  # workspace short
    assert ei.value.code == mp.MOE_PW_EINVAL
    with pytest.raises(mp.MoePwError) as ei:
        mp.moe_pw_route_assign_form(tiny, -1, odd + 8, *args[1:], good, ws, stream=0)
    assert ei.value.code == mp.MOE_PW_EUNSUPPORTED  # logits need 16 bytes
