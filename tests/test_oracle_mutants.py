"""Planted mistakes: each test builds a copy of oracle.c with one plausible bug
(a flipped tie-break, an off-by-one capacity, a wrong wave index, a shifted
gate, truncating bf16 rounding, ...) and checks that the pins in the other
oracle test files reject it.  This shows the pins are not satisfied by any
oracle, only by a correct one.  Everything runs on the CPU.
"""
import os
import subprocess

import numpy as np
import pytest

import oracle
from combine_moe_pw_b200 import synth

import test_oracle_backward as tb
import test_oracle_combine as tc
import test_oracle_dispatch as td
import test_oracle_headers as th
import test_oracle_route as tr
import test_oracle_seq_balance as tsb

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "oracle.c")


def _mutant(tmp_path, old, new):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor not found: {old!r}"
    path = tmp_path / "mut.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-ffp-contract=off",
                           "-o", str(so), str(path), "-lm"])
    return oracle.variant(str(so))


def _tiny():
    w = synth.WORKLOADS["tiny"]
    return w, synth.logits(w), synth.x_bf16(w), synth.scales(w)


def _tiny_run():
    w, lg, x, s = _tiny()
    return oracle.run(w, lg, x, s, with_mag=True)


def _bw_case():
    w, lg, x, s = _tiny()
    r = oracle.run(w, lg, x, s)
    dout = synth.dout(w)
    return w, lg, x, s, r, dout, oracle.run_backward(w, r, dout, s)


MUTANTS = [
    ("softmax_backward_sign", "gates[t * k + j] * (dgate[t * k + j] - weighted)",
     "gates[t * k + j] * (weighted - dgate[t * k + j])",
     lambda: tb.test_backward_with_exact_rows(_bw_case())),
    ("grad_row_without_gate", "d_ret[slot * D + i] = f32_to_bf16_rne(gj * dt[i]);",
     "d_ret[slot * D + i] = f32_to_bf16_rne(dt[i]);",
     lambda: tb.test_backward_matches_autograd(_bw_case())),
    ("dispatch_backward_skips_last_choice", "for (int32_t j = 0; j < g->k; ++j) {\n            const int64_t slot = slot_map[t * g->k + j];\n            if (slot < 0 || recv_row[slot] < 0) continue;",
     "for (int32_t j = 0; j + 1 < g->k; ++j) {\n            const int64_t slot = slot_map[t * g->k + j];\n            if (slot < 0 || recv_row[slot] < 0) continue;",
     lambda: tb.test_backward_matches_autograd(_bw_case())),
    ("ties_to_higher_index", "l[e] > l[best]", "l[e] >= l[best]",
     lambda: tr.test_topk_matches_full_sort(48, 8)),
    ("gate_sum_skips_first", "den += ex[j];", "if (j) den += ex[j];",
     lambda: tr.test_gates_match_library_softmax(_tiny())),
    ("capacity_floor", "return (a + b - 1) / b;", "return a / b;",
     lambda: [td.test_capacity_golden(c) for c in __import__("json").load(
         open(os.path.join(td.GOLDEN, "capacities.json")))["cases"]]),
    ("sender_keeps_one_fewer", "if (rank < g->C_s) {", "if (rank < g->C_s - 1) {",
     lambda: td.test_sender_assignment_brute_force(1.5)),
    ("sender_rank_off_by_one", "const int64_t rank = count[p]++;", "const int64_t rank = ++count[p] - (p == 0 ? 0 : 1);",
     lambda: td.test_sender_assignment_brute_force(0.0)),
    ("wave_index_modulo", "*w = (e % g->L) / g->P;", "*w = (e % g->L) % g->W;",
     lambda: td.test_closed_form_every_token_picks_experts_0_to_7(_tiny())),
    ("receiver_keeps_one_fewer", "if (r < g->C_r) {", "if (r + 1 < g->C_r) {",
     lambda: td.test_receiver_bucketing_brute_force()),
    ("header_is_rank_not_expert", "pool_hdr[slot] = idx[t * g->k + j];", "pool_hdr[slot] = j;",
     lambda: td.test_invariants_tiny(_tiny(), _tiny_run())),
    ("bf16_truncates", "return (uint16_t)((v.u + 0x7FFFu + ((v.u >> 16) & 1u)) >> 16);",
     "return (uint16_t)(v.u >> 16);",
     lambda: tc.test_bf16_round_matches_torch()),
    ("combine_shifted_gate", "const double gj = gates[t * g->k + j];\n            for (int64_t i = 0; i < D; ++i) o[i] +=",
     "const double gj = gates[t * g->k + (j + 1) % g->k];\n            for (int64_t i = 0; i < D; ++i) o[i] +=",
     lambda: tc.test_combine_matches_einsum(_tiny_run())),
    ("pack_headers_writes_rank", "if (slot >= 0) pool_hdr[slot] = idx[t * g->k + j];",
     "if (slot >= 0) pool_hdr[slot] = j;",
     lambda: th.test_run_headers_equals_run("tiny")),
    ("pack_headers_skips_empty_reset", "for (int64_t q = 0; q < n_slots; ++q) pool_hdr[q] = -1;",
     "",
     lambda: th.test_run_headers_equals_run("tiny")),
    ("ragged_receiver_counts_from_one", "recv_row[q] = arrivals[e]++;",
     "recv_row[q] = ++arrivals[e];",
     lambda: th.test_ragged_receiver_rows_brute_force()),
    ("balance_share_not_scaled", "fs[e] *= (double)E / ((double)k * (double)seq_len);",
     "fs[e] /= (double)seq_len;",
     lambda: tsb.test_perfect_balance_gives_alpha_for_any_logits()),
    ("balance_prob_not_averaged", "Ps[e] /= (double)seq_len;", "Ps[e] /= 1.0;",
     lambda: tsb.test_f_and_P_against_library_routines()),
    ("balance_gradient_sign", "p[e] * (fs[e] - dot);", "p[e] * (dot - fs[e]);",
     lambda: tsb.test_gradient_matches_autograd_and_rows_sum_to_zero()),
    ("ragged_rows_by_token_desc", "const int32_t row = next[e]++;",
     "const int32_t row = row_off[e] + row_cnt[e] - 1 - (next[e]++ - row_off[e]);",
     lambda: td.test_ragged_assignment()),
]


@pytest.mark.parametrize("name,old,new,check", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pin_rejects_planted_mistake(tmp_path, name, old, new, check):
    check()  # the pin passes on the real oracle
    with _mutant(tmp_path, old, new):
        with pytest.raises(AssertionError):
            check()
