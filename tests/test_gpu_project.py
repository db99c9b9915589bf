"""Latent projection on the tensor cores (tcgen05) against the CPU oracle.

Tolerance (derived): the device accumulates K bf16 products in fp32 and
rounds to bf16; the oracle sums in double.  |gpu - exact| <= 2^-8 |exact| (bf16
rounding, one ulp margin) + 2^-20 * sum_k |a_k b_k| (fp32 accumulation: K
roundings of partial sums, K <= 6144 < 2^13 gives K * 2^-24 < 2^-11 of the
magnitude; the bound leaves room), and the bf16 codes must agree on almost
every element.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
from combine_moe_pw_b200 import moe_pw as mp
from combine_moe_pw_b200 import synth

pytestmark = pytest.mark.gpu


def _f64(u16):
    return (u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _ctr():
    return torch.zeros((mp.COUNTERS_BYTES // 8,), dtype=torch.int64, device="cuda")


def gpu_project(A, Bt):
    M, K = A.shape
    N = Bt.shape[0]
    a = torch.from_numpy(A.view(np.int16)).cuda()
    b = torch.from_numpy(Bt.view(np.int16)).cuda()
    c = torch.full((M, N), 0x7FC0, dtype=torch.int16, device="cuda")  # NaN poison
    ctr = _ctr()
    mp.moe_pw_project(a, b, c, M, N, K, ctr)
    torch.cuda.synchronize()
    assert mp.moe_pw_stats(mp.Config(T=0, E=8, k=1, D=8, R=1, L=8, W=1, P=8), ctr).error == 0
    return c.cpu().numpy().view(np.uint16), ctr


def check_project(A, Bt, C):
    Cr, Ce, mag = oracle.project(A, Bt, exact=True)
    got = _f64(C)
    assert np.all(np.isfinite(got))
    assert np.all(np.abs(got - Ce) <= 2.0 ** -8 * np.abs(Ce) + 2.0 ** -20 * mag + 1e-30)
    assert (C != Cr).mean() < 0.02


def test_single_tile():
    A = synth.matrix_bf16(128, 64, 1.0, 30)
    Bt = synth.matrix_bf16(256, 64, 0.125, 31)
    C, ctr = gpu_project(A, Bt)
    check_project(A, Bt, C)


@pytest.mark.parametrize("M,N,K", [(256, 512, 128), (300, 264, 200), (1, 8, 8), (129, 264, 4096),
                                   (640, 3072, 256), (512, 768, 1024)])
def test_shapes(M, N, K):
    A = synth.matrix_bf16(M, K, 1.0, 32)
    Bt = synth.matrix_bf16(N, K, K ** -0.5, 33)
    C, ctr = gpu_project(A, Bt)
    check_project(A, Bt, C)


def test_identity_weights_copy_rows():
    K = 256
    A = synth.matrix_bf16(384, K, 1.0, 34)
    eye = torch.eye(K, dtype=torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    C, _ = gpu_project(A, eye)
    np.testing.assert_array_equal(C, A)


def _pack_inputs(w, Dm):
    lg = synth.logits(w)
    h, wd, _ = synth.projection_inputs(w, Dm)
    return lg, h, wd


@pytest.mark.parametrize("name,Dm", [("tiny", 256), ("pages_small", 1024)])
def test_project_pack_matches_two_step_and_oracle(name, Dm):
    w = (synth.WORKLOADS["tiny"] if name == "tiny" else
         synth.Workload("pages_small", T=64 * 64, R=64, L=6, W=3, P=2, k=8, D=512, seq_len=1024,
                        logit_kind=synth.LOGIT_SEQBIAS))
    lg, h, wd = _pack_inputs(w, Dm)
    cfg = mp.Config.from_workload(w)
    b = mp.Buffers(cfg)
    b.logits.copy_(torch.from_numpy(lg))
    hd = torch.from_numpy(h.view(np.int16)).cuda()
    wdd = torch.from_numpy(wd.view(np.int16)).cuda()
    b.route()
    b.assign()
    # two-step: x = project(h), then pack
    mp.moe_pw_project(hd, wdd, b.x, w.T, w.D, Dm, b.counters)
    b.pack()
    ref_pool = b.pool_x.clone()
    ref_hdr = b.pool_hdr.clone()
    x_gpu = b.x.cpu().numpy().view(np.uint16)
    # fused
    b.pool_x.fill_(0x1234)
    b.pool_hdr.fill_(-7)
    mp.moe_pw_project_pack(cfg, hd, wdd, Dm, b.idx, b.slot_map, b.occ, b.pool_x, b.pool_hdr,
                           b.counters)
    st = b.stats()
    assert st.error == 0
    assert torch.equal(b.pool_x, ref_pool) and torch.equal(b.pool_hdr, ref_hdr)
    # the projection itself against the oracle, and the pools against an
    # oracle pack of the GPU's x (integer work: bit-exact)
    check_project(h, wd, x_gpu)
    r = oracle.run_headers(w, lg)
    np.testing.assert_array_equal(b.pool_hdr.cpu().numpy(), r["pool_hdr"])
    pool = b.pool_x.cpu().numpy().view(np.uint16)
    full = r["slot_tok"] >= 0
    np.testing.assert_array_equal(pool[full], x_gpu[r["slot_tok"][full]])
    assert not pool[~full].any()


def test_down_projection_full_size_sampled():
    """Rack batch: h [262144, 6144] x w_down^T -> [262144, 3072], rows sampled."""
    w = synth.WORKLOADS["rack"]
    h, wd, _ = synth.projection_inputs(w)
    hd = torch.from_numpy(h.view(np.int16)).cuda()
    wdd = torch.from_numpy(wd.view(np.int16)).cuda()
    c = torch.empty((w.T, w.D), dtype=torch.int16, device="cuda")
    ctr = _ctr()
    mp.moe_pw_project(hd, wdd, c, w.T, w.D, h.shape[1], ctr)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([np.random.default_rng(5).integers(0, w.T, 24), [0, w.T - 1]]))
    C = c[torch.from_numpy(rows).cuda()].cpu().numpy().view(np.uint16)
    check_project(h[rows], wd, C)


@pytest.mark.parametrize("name,Dm", [("tiny", 256), ("pages_small", 1024)])
def test_routed_layer_against_oracle_chain(name, Dm):
    """h -> (down-projection + pack) -> bucket -> expert -> combine (bf16) ->
    up-projection, against the oracle's chain on its own intermediates.
    Where the chains may part: a bf16 rounding of the projected or combined
    latent can land one ulp apart (double vs fp32 sums), so the bound is
    2^-6 of sum_k |latent_k w_nk| plus 2^-8 of the value, and almost every
    element must agree far more closely."""
    w = (synth.WORKLOADS["tiny"] if name == "tiny" else
         synth.Workload("pages_small", T=64 * 64, R=64, L=6, W=3, P=2, k=8, D=512, seq_len=1024,
                        logit_kind=synth.LOGIT_SEQBIAS))
    lg, s = synth.logits(w), synth.scales(w)
    h, wd, wu = synth.projection_inputs(w, Dm)
    b = mp.Buffers(mp.Config.from_workload(w))
    b.logits.copy_(torch.from_numpy(lg))
    b.scale.copy_(torch.from_numpy(s))
    lat = torch.empty((w.T, w.D), dtype=torch.int16, device="cuda")
    out = torch.empty((w.T, Dm), dtype=torch.int16, device="cuda")
    b.run_routed_layer(torch.from_numpy(h.view(np.int16)).cuda(),
                       torch.from_numpy(wd.view(np.int16)).cuda(),
                       torch.from_numpy(wu.view(np.int16)).cuda(), Dm, lat, out)
    assert b.stats().error == 0
    # oracle chain
    x, _, xmag = oracle.project(h, wd, exact=True)
    r = oracle.run(w, lg, x, s)
    lat_ref = oracle.bf16_round(r["out"].astype(np.float32))
    out_ref, out_exact, mag = oracle.project(lat_ref, wu, exact=True)
    got = _f64(out.cpu().numpy().view(np.uint16))
    err = np.abs(got - out_exact)
    assert np.all(err <= 2.0 ** -6 * mag + 2.0 ** -8 * np.abs(out_exact) + 1e-30)
    assert (err <= 2.0 ** -8 * np.abs(out_exact) + 2.0 ** -18 * mag).mean() > 0.99
    # the bf16 latent: every term of a token's combine is a multiple of the same
    # x_i, latent_i = x_i * sum_j g_j s_j, so its error follows x_i's: the
    # projection's own bound (2^-8 |x| + 2^-20 sum_k |h_k w_ik|, the second term
    # for near-cancelling sums) and one bf16 ulp each for the expert row and
    # the latent
    got_lat = _f64(lat.cpu().numpy().view(np.uint16))
    ref_lat = r["out"]
    xf = _f64(x)
    keep = r["slot_map"] >= 0
    keep &= r["recv_row"][np.where(keep, r["slot_map"], 0)] >= 0
    c = (r["gates"] * s[r["idx"]] * keep).sum(axis=1, keepdims=True)
    bound = (2.0 ** -6 * np.abs(xf) + 2.0 ** -19 * xmag) * c + 1e-30
    bad = np.abs(got_lat - ref_lat) > bound
    if bad.any():
        t, i = np.argwhere(bad)[0]
        raise AssertionError(f"latent[{t},{i}] got {got_lat[t, i]!r} ref {ref_lat[t, i]!r} "
                             f"x {xf[t, i]!r} c {c[t, 0]!r} bad {bad.sum()}")


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (300, 264, 200), (1, 8, 8),
                                   (129, 1032, 2072), (515, 512, 3072)])
def test_project_add_merges_shared_path(M, N, K):
    """C = bf16(A @ Bt^T + add) against the oracle's merge, with the
    projection's bound (its magnitude now includes |add|); then in place
    (add is C) with the same bytes."""
    A = synth.matrix_bf16(M, K, 1.0, 60)
    Bt = synth.matrix_bf16(N, K, K ** -0.5, 61)
    S = synth.matrix_bf16(M, N, 1.0, 62)
    a = torch.from_numpy(A.view(np.int16)).cuda()
    b = torch.from_numpy(Bt.view(np.int16)).cuda()
    sh = torch.from_numpy(S.view(np.int16)).cuda()
    c = torch.full((M, N), 0x7FC0, dtype=torch.int16, device="cuda")
    ctr = _ctr()
    mp.moe_pw_project_add(a, b, sh, c, M, N, K, ctr)
    inplace = sh.clone()
    mp.moe_pw_project_add(a, b, inplace, inplace, M, N, K, ctr)
    torch.cuda.synchronize()
    assert mp.moe_pw_stats(mp.Config(T=0, E=8, k=1, D=8, R=1, L=8, W=1, P=8), ctr).error == 0
    C = c.cpu().numpy().view(np.uint16)
    Cr, Ce, mag = oracle.project(A, Bt, exact=True, add=S)
    got = _f64(C)
    assert np.all(np.isfinite(got))
    assert np.all(np.abs(got - Ce) <= 2.0 ** -8 * np.abs(Ce) + 2.0 ** -20 * mag + 1e-30)
    assert (C != Cr).mean() < 0.02
    assert torch.equal(inplace, c)


def test_routed_layer_with_shared_merge():
    """The routed branch ending in the merge: the up-projection's epilogue
    adds the shared path's output.  Against the oracle's chain extended by
    the same merge, with the routed-layer bound."""
    w = synth.WORKLOADS["tiny"]
    Dm = 256
    lg, s = synth.logits(w), synth.scales(w)
    h, wd, wu = synth.projection_inputs(w, Dm)
    S = synth.matrix_bf16(w.T, Dm, 1.0, 63)
    b = mp.Buffers(mp.Config.from_workload(w))
    b.logits.copy_(torch.from_numpy(lg))
    b.scale.copy_(torch.from_numpy(s))
    lat = torch.empty((w.T, w.D), dtype=torch.int16, device="cuda")
    out = torch.empty((w.T, Dm), dtype=torch.int16, device="cuda")
    b.run_routed_layer(torch.from_numpy(h.view(np.int16)).cuda(),
                       torch.from_numpy(wd.view(np.int16)).cuda(),
                       torch.from_numpy(wu.view(np.int16)).cuda(), Dm, lat, out,
                       shared_out=torch.from_numpy(S.view(np.int16)).cuda())
    assert b.stats().error == 0
    x = oracle.project(h, wd)
    r = oracle.run(w, lg, x, s)
    lat_ref = oracle.bf16_round(r["out"].astype(np.float32))
    _, out_exact, mag = oracle.project(lat_ref, wu, exact=True, add=S)
    got = _f64(out.cpu().numpy().view(np.uint16))
    err = np.abs(got - out_exact)
    assert np.all(err <= 2.0 ** -6 * mag + 2.0 ** -8 * np.abs(out_exact) + 1e-30)
    assert (err <= 2.0 ** -8 * np.abs(out_exact) + 2.0 ** -18 * mag).mean() > 0.99


@pytest.mark.parametrize("chunk", [1000, 2048, 4096])
def test_pipelined_routed_layer_equals_sequential(chunk):
    """The routed layer with the combine and the up-projection overlapped in
    token blocks (two latent buffers, two streams): the same bytes as the
    sequential chain, with and without the shared-path merge; block sizes
    that divide the batch and one that leaves a ragged last block."""
    w = synth.Workload("pages_small", T=64 * 64, R=64, L=6, W=3, P=2, k=8, D=512, seq_len=1024,
                       logit_kind=synth.LOGIT_SEQBIAS)
    Dm = 1024
    lg, s = synth.logits(w), synth.scales(w)
    h, wd, wu = (torch.from_numpy(a.view(np.int16)).cuda() for a in synth.projection_inputs(w, Dm))
    S = torch.from_numpy(synth.matrix_bf16(w.T, Dm, 1.0, 64).view(np.int16)).cuda()
    b = mp.Buffers(mp.Config.from_workload(w))
    b.logits.copy_(torch.from_numpy(lg))
    b.scale.copy_(torch.from_numpy(s))
    lat = torch.empty((w.T, w.D), dtype=torch.int16, device="cuda")
    for shared in (None, S):
        ref = torch.empty((w.T, Dm), dtype=torch.int16, device="cuda")
        b.run_routed_layer(h, wd, wu, Dm, lat, ref, shared_out=shared, overlap=False)
        got = torch.full((w.T, Dm), 0x7FC0, dtype=torch.int16, device="cuda")
        b.run_routed_layer_pipelined(h, wd, wu, Dm, got, shared_out=shared, chunk_tokens=chunk)
        torch.cuda.synchronize()
        assert torch.equal(got, ref)
    assert b.stats().error == 0


def test_combine_rows_is_the_combine_of_those_tokens():
    w = synth.WORKLOADS["tiny"]
    lg = synth.logits(w)
    b = mp.Buffers(mp.Config.from_workload(w))
    b.logits.copy_(torch.from_numpy(lg))
    b.x.copy_(torch.from_numpy(synth.x_bf16(w).view(np.int16)))
    b.scale.copy_(torch.from_numpy(synth.scales(w)))
    b.run_step()
    full = torch.empty((w.T, w.D), dtype=torch.int16, device="cuda")
    mp.moe_pw_combine_bf16(b.cfg, b.ret_x, b.ret_hdr, b.slot_map, b.gates, full, b.counters)
    part = torch.full((300, w.D), 0x7FC0, dtype=torch.int16, device="cuda")
    mp.moe_pw_combine_bf16_rows(b.cfg, b.ret_x, b.ret_hdr, b.slot_map, b.gates, 1001, 300, part,
                                b.counters)
    torch.cuda.synchronize()
    assert torch.equal(part, full[1001:1301])
    with pytest.raises(mp.MoePwError):
        mp.moe_pw_combine_bf16_rows(b.cfg, b.ret_x, b.ret_hdr, b.slot_map, b.gates, w.T - 5, 6,
                                    part, b.counters)


_FALLBACK_SHAPES = [(300, 264, 200), (129, 264, 4096), (512, 768, 1024), (1, 8, 8)]

_FALLBACK_CHILD = r"""
import sys, numpy as np, torch
sys.path.insert(0, {root!r})
from combine_moe_pw_b200 import moe_pw as mp, synth
out = {{}}
for M, N, K in {shapes!r}:
    A = synth.matrix_bf16(M, K, 1.0, 40)
    Bt = synth.matrix_bf16(N, K, K ** -0.5, 41)
    a = torch.from_numpy(A.view(np.int16)).cuda()
    b = torch.from_numpy(Bt.view(np.int16)).cuda()
    c = torch.full((M, N), 0x7FC0, dtype=torch.int16, device="cuda")
    ctr = torch.zeros((mp.COUNTERS_BYTES // 8,), dtype=torch.int64, device="cuda")
    mp.moe_pw_project(a, b, c, M, N, K, ctr)
    torch.cuda.synchronize()
    assert int(ctr[4].item()) & 0xFFFFFFFF == 0
    out[f"{{M}}_{{N}}_{{K}}"] = c.cpu().numpy()
np.savez({path!r}, **out)
"""


def test_one_sm_fallback_matches_pair_kernel(tmp_path):
    """The one-SM kernel (the fallback where a cluster of two cannot be
    launched; selected here with MOE_PW_GEMM_PAIR=0 in a child process) and
    the default two-SM kernel: the same MMA steps in the same K order per
    output element, so bit-identical products."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    path = str(tmp_path / "one_sm.npz")
    code = _FALLBACK_CHILD.format(root=root, shapes=_FALLBACK_SHAPES, path=path)
    env = {**os.environ, "MOE_PW_GEMM_PAIR": "0"}
    subprocess.run([sys.executable, "-c", code], env=env, check=True, timeout=600)
    one_sm = np.load(path)
    for M, N, K in _FALLBACK_SHAPES:
        A = synth.matrix_bf16(M, K, 1.0, 40)
        Bt = synth.matrix_bf16(N, K, K ** -0.5, 41)
        C, _ = gpu_project(A, Bt)
        check_project(A, Bt, C)
        np.testing.assert_array_equal(C, one_sm[f"{M}_{N}_{K}"].view(np.uint16))


def test_routed_layer_overlap_on_large_batches():
    """At two or more blocks of 16,384 tokens run_routed_layer(overlap=True)
    overlaps the combine and the up-projection, using its latent scratch for
    the two block buffers: the same bytes as the sequential chain."""
    w = synth.Workload("two_blocks", T=64 * 600, R=64, L=6, W=3, P=2, k=8, D=256, seq_len=600,
                       logit_kind=synth.LOGIT_SEQBIAS)
    Dm = 512
    h, wd, wu = (torch.from_numpy(a.view(np.int16)).cuda() for a in synth.projection_inputs(w, Dm))
    S = torch.from_numpy(synth.matrix_bf16(w.T, Dm, 1.0, 65).view(np.int16)).cuda()
    b = mp.Buffers(mp.Config.from_workload(w))
    b.logits.copy_(torch.from_numpy(synth.logits(w)))
    b.scale.copy_(torch.from_numpy(synth.scales(w)))
    lat = torch.empty((w.T, w.D), dtype=torch.int16, device="cuda")
    ref = torch.empty((w.T, Dm), dtype=torch.int16, device="cuda")
    b.run_routed_layer(h, wd, wu, Dm, lat, ref, shared_out=S, overlap=False)
    got = torch.full((w.T, Dm), 0x7FC0, dtype=torch.int16, device="cuda")
    assert w.T >= 2 * b.OVERLAP_BLOCK_TOKENS
    b.run_routed_layer(h, wd, wu, Dm, lat, got, shared_out=S, overlap=True)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)
