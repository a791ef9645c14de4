"""The pins catch plausible mistakes in the oracle.

Each case below plants one mistake in a copy of the oracle's C source (on
the CPU: a text substitution, compiled to a temporary library) and requires
at least one pin of tests/oracle_pins.py to fail on it.  The mistakes are
the ones a reader of the pages could make: a dropped term, a wrong sign, a
wrong index, swapped operands, the other rounding rule, the other reading of
the residual.
"""
import os

import pytest

import oracle
import oracle_pins

MUTANTS = {
    "owner_fixup_dropped": (
        "m_fast[orow + j] = fadd(m_fast[orow + j], fmul(one_m_bf, er));", ""),
    "owner_index_shifted": (
        "const int owner = (int)((col * G) / chunk);",
        "const int owner = (int)(((col * G) / chunk + 1) % P);"),
    "correction_subtracted": ("v = fadd(v, c);", "v = fsub(v, c);"),
    "alpha_on_slow_ema": (
        "float c = fadd(fmul(alpha, m_fast[row + j]),\n"
        "                                   fmul(one_m_alpha, m_slow[row + j]));",
        "float c = fadd(fmul(one_m_alpha, m_fast[row + j]),\n"
        "                                   fmul(alpha, m_slow[row + j]));"),
    "ties_away_from_zero": ("float r = rintf(fdiv(v[j], scale));",
                            "float r = roundf(fdiv(v[j], scale));"),
    "scale_over_eight": ("scale = fdiv(a, levels);", "scale = fdiv(a, levels + 1.0f);"),
    "nibbles_swapped": ("bytes[j] = (uint8_t)(lo | (hi << 4));",
                        "bytes[j] = (uint8_t)(hi | (lo << 4));"),
    "no_clamp": ("if (r > levels) r = levels;", ""),
    "ema_decay_swapped": (
        "m_fast[row + j] = fadd(fmul(bf, m_fast[row + j]),\n"
        "                                           fmul(one_m_bf, e));",
        "m_fast[row + j] = fadd(fmul(one_m_bf, m_fast[row + j]),\n"
        "                                           fmul(bf, e));"),
    "slow_ema_not_updated": (
        "m_slow[row + j] = fadd(fmul(bs, m_slow[row + j]),\n"
        "                                           fmul(one_m_bs, e));", ""),
    "residual_against_raw_input": (
        "float e = fsub(xt[j], d);",
        "float e = fsub(eo_bf16_to_f32(x[row + j]), d);"),
    "requant_error_against_fp32": (
        "float er = fsub(sum[j], eo_bf16_to_f32(yb));",
        "float er = fsub(sum[j], eo_dequant(k[j], scale2));"),
    "sum_not_requantized": (
        "uint16_t yb = requantize ? eo_f32_to_bf16_rne(eo_dequant(k[j], scale2))",
        "uint16_t yb = requantize ? eo_f32_to_bf16_rne(sum[j])"),
    "sum_skips_last_rank": ("sum[j] = fadd(sum[j], d);",
                            "if (r < P - 1 || P == 1) sum[j] = fadd(sum[j], d);"),
    "rs_output_requantized": (": eo_f32_to_bf16_rne(sum[j]);",
                              ": eo_f32_to_bf16_rne(fmul(sum[j], 1.0078125f));"),
    "rs_residual_not_folded": (
        "/* 9. the owner alone also folds the requantization error in */\n"
        "            if (prm->compensate) {",
        "/* 9. the owner alone also folds the requantization error in */\n"
        "            if (prm->compensate && requantize) {"),
    "levels_off_by_one_for_8bit": ("const int L = prm->bits == 8 ? 127 : 7;",
                                   "const int L = prm->bits == 8 ? 128 : 7;"),
    "pack8_as_nibbles": ("bytes[j] = (uint8_t)k[j];", "bytes[j] = (uint8_t)(k[j] & 0x0f);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_fails_a_pin(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(oracle.SOURCE).read()
    assert src.count(old) == 1, "mutation site not found: " + name
    path = os.path.join(tmp_path, "mutant.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    mut = oracle.Oracle(oracle.compile_source(path, os.path.join(tmp_path, "mutant.so")))
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(mut)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
            break
    assert failed, "no pin catches the mutant " + name
