"""Planted mistakes in the oracle must fail at least one pin.

Each mutant is a one-spot edit of ``oracle/mep_oracle.c`` (a dropped term, a
wrong index, a swapped loop, a wrong comparison), compiled with gcc into a
temporary library and run through every pin in ``oracle_pins``.  All mutants
keep every memory access in bounds.  CPU only.
"""
import os

import pytest

import oracle
import oracle_pins

MUTANTS = {
    "maxvio_drops_minus_one": (
        "return (double)((int64_t)m * E) / (double)NK - 1.0;",
        "return (double)((int64_t)m * E) / (double)NK;"),
    "maxvio_tbar_over_tokens": (
        "return (double)((int64_t)m * E) / (double)NK - 1.0;",
        "return (double)((int64_t)m * E) / (double)(NK / K) - 1.0;"),
    "maxvio_min_not_max": (
        "if (counts[e] > m)", "if (counts[e] < m || m == 0)"),
    "sort_k_major": (
        "for (int64_t g = 0; g < N; ++g) {\n        for (int k = 0; k < K; ++k) {",
        "for (int k = 0; k < K; ++k) {\n        for (int64_t g = 0; g < N; ++g) {"),
    "sort_fills_expert_backwards": (
        "int32_t p = expert_offset[e] + counts[e];",
        "int32_t p = expert_offset[e + 1] - 1 - counts[e];"),
    "segment_cut_by_rank_only": (
        "if (r != prev_r || e != prev_e) {", "if (r != prev_r) {"),
    "segment_start_global": (
        "seg[4 * ns + 2] = (int32_t)(p - (int64_t)r * SK);",
        "seg[4 * ns + 2] = (int32_t)p;"),
    "home_modulo_ranks": ("if (r != e / B)", "if (r != e % R)"),
    "replica_flag_inverted": ("if (r != e / B)", "if (r == e / B)"),
    "rank_ptr_off_by_one": (
        "while (s < ns && seg[4 * s + 1] < r)", "while (s < ns && seg[4 * s + 1] <= r)"),
    "dispatch_token_mod_k": (
        "int64_t g = src_pair[p] / K;", "int64_t g = src_pair[p] % K;"),
    "combine_weight_transposed": (
        "double term = (double)w[g * K + k]", "double term = (double)w[k * ntok + g]"),
    "combine_drops_last_k": (
        "for (int k = 0; k < K; ++k) {\n                int64_t p = slot[g * K + k];",
        "for (int k = 0; k < K - 1; ++k) {\n                int64_t p = slot[g * K + k];"),
    "bf16_ties_away": (
        "if (rem > 0.5 || (rem == 0.5 && fmod(n, 2.0) != 0.0))", "if (rem >= 0.5)"),
    "bf16_truncates": (
        "if (rem > 0.5 || (rem == 0.5 && fmod(n, 2.0) != 0.0))", "if (0)"),
    "bf16_widen_wrong_shift": ("uint32_t u = (uint32_t)b << 16;", "uint32_t u = (uint32_t)b << 15;"),
    "reduce_skips_first_segment": (
        "for (int32_t s = expert_seg_ptr[e]; s < expert_seg_ptr[e + 1]; ++s)",
        "for (int32_t s = expert_seg_ptr[e] + 1; s < expert_seg_ptr[e + 1]; ++s)"),
    "reduce_uses_next_expert": (
        "for (int32_t s = expert_seg_ptr[e]; s < expert_seg_ptr[e + 1]; ++s)",
        "for (int32_t s = expert_seg_ptr[e]; s < expert_seg_ptr[e + 1] && e + 1 < E; ++s)"),
    "combine_bwd_first_weight_only": (
        "double wk = (double)w[g * K + k];", "double wk = (double)w[g * K];"),
    "combine_bwd_gradw_uses_grad_out_twice": (
        "double term = go * (double)ora_bf16_to_f32(y[p * H + h]);  /* exact */",
        "double term = go * go;"),
    "combine_bwd_row_by_pair_not_slot": (
        "grad_y[p * H + h] = ora_f64_to_bf16(prod);",
        "grad_y[(g * K + k) * H + h] = ora_f64_to_bf16(prod);"),
    "dispatch_bwd_drops_last_k": (
        "for (int k = 0; k < K; ++k) {\n                double v = (double)ora_bf16_to_f32(grad_buf",
        "for (int k = 0; k < K - 1; ++k) {\n                double v = (double)ora_bf16_to_f32(grad_buf"),
    "prefetch_uses_rank_not_expert": (
        "int32_t e = seg[4 * replica_seg[j] + 0];", "int32_t e = seg[4 * replica_seg[j] + 1];"),
    "home_first_fill_ignores_room_order": (
        "pre[e] = (int32_t)fill;", "pre[e] = (int32_t)(C - fill - take);"),
    "home_first_overflow_before_home": (
        "p = (int64_t)r * C + F[r] + (q - D[r]);", "p = (int64_t)r * C + (q - D[r]);"),
    "home_first_replica_flag_by_slot_rank": (
        "if (seg[4 * a + 1] != seg[4 * a] / B)", "if (seg[4 * a + 1] != seg[4 * a] % R)"),
    "capped_home_fill_largest_first": (
        "if (counts[e2] < counts[e] || (counts[e2] == counts[e] && e2 < e))",
        "if (counts[e2] > counts[e] || (counts[e2] == counts[e] && e2 < e))"),
    "capped_items_ascending": (
        "while (at > 0 && (O[item[at - 1]] < O[e] ||",
        "while (at > 0 && (O[item[at - 1]] > O[e] ||"),
    "capped_rooms_ascending": (
        "while (at > 0 && (D[room[at - 1]] < D[r] ||",
        "while (at > 0 && (D[room[at - 1]] > D[r] ||"),
    "capped_one_round_too_many": (
        "if (round < B - 2 && left[j] >= O[e]) {", "if (round < B - 1 && left[j] >= O[e]) {"),
    "capped_filler_threshold_inclusive": (
        "if (O[e] >= dmax)\n                continue;", "if (O[e] > dmax)\n                continue;"),
    "capped_replicas_over_home_slots": ("rfill[r] = F[r];", "rfill[r] = 0;"),
    "capped_last_pairs_stay_home": (
        "        if (i < h[e]) {\n            p = (int64_t)(e / Bh) * C + hpre[e] + i;\n"
        "        } else {\n            int32_t q = i - h[e];",
        "        if (i >= O[e]) {\n            p = (int64_t)(e / Bh) * C + hpre[e] + (i - O[e]);\n"
        "        } else {\n            int32_t q = i;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    before, after = MUTANTS[name]
    src = open(oracle.SRC).read()
    assert src.count(before) == 1, f"mutation site for {name} not found exactly once"
    mpath = tmp_path / "mutant.c"
    mpath.write_text(src.replace(before, after))
    lib = oracle.build(str(mpath), str(tmp_path / "libmutant.so"))
    ora = oracle.Oracle(lib)
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(ora)
        except AssertionError:
            failed.append(pin.__name__)
        except oracle.OracleError:
            failed.append(pin.__name__)
    assert failed, f"no pin catches mutant {name}"


def test_unmutated_oracle_passes_every_pin():
    ora = oracle.get()
    for pin in oracle_pins.ALL_PINS:
        pin(ora)
    assert os.path.exists(oracle.LIB)
