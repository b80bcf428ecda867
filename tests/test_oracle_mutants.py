"""Plant plausible mistakes in a copy of the oracle and check that the pins
catch every one.  The mistakes are planted on the CPU, in a temporary copy
of the oracle's C source; the real oracle is never modified."""
import os

import pytest

import oracle
from oracle import build as obuild
from tests import pins

# (name, original text, replacement)
MUTANTS = [
    ("taps_reversed", "w[(int64_t)j * C + c]", "w[(int64_t)(W - 1 - j) * C + c]"),
    ("dropped_oldest_tap", "for (int j = 0; j < W; ++j) {", "for (int j = 1; j < W; ++j) {"),
    ("state_rows_reversed", "s[(W - 1 + q) * state_row_stride + c]", "s[(-1 - q) * state_row_stride + c]"),
    ("sign_flip", "acc += oracle_bf16_to_double", "acc -= oracle_bf16_to_double"),
    ("eps_outside_sqrt", "1.0 / sqrt(ss / (double)D + eps)", "1.0 / (sqrt(ss / (double)D) + eps)"),
    ("sum_not_mean", "1.0 / sqrt(ss / (double)D + eps)", "1.0 / sqrt(ss + eps)"),
    ("gamma_by_head", "(double)gh[d]", "(double)gh[h % D]"),
    ("gamma_head_stride_ignored", "const float* gh = gamma + (int64_t)h * gamma_head_stride;",
     "const float* gh = gamma;"),
    ("ring_write_row_shifted", "const int64_t row = (pos0 + q) % n;", "const int64_t row = (pos0 + q + 1) % n;"),
    ("ring_read_ignores_position", "const int64_t row = (pos0 + j) % n;", "const int64_t row = j % n;"),
    ("state_keeps_oldest", "int64_t q = L - n + j;", "int64_t q = j;"),
    ("v_uses_k_taps", "(which == 0 ? conv_w_k : conv_w_v)", "(conv_w_k)"),
    ("v_state_in_k_half", "st + (which == 0 ? 0 : C)", "st + 0"),
    ("slot_offset_dropped", "int64_t off = slot % page_size;", "int64_t off = 0;"),
    ("round_truncates", "r = ldexp(rint(ldexp(ax, -q)), q);", "r = ldexp(floor(ldexp(ax, -q)), q);"),
    ("negative_slot_written", "if (slot < 0) continue;", "if (slot < 0) slot = 0;"),
    ("head_stride_dropped", "(int64_t)h * stride_head;", "0;"),
    ("mx_emax_7", "s = (e - 1) - 8;", "s = (e - 1) - 7;"),
    ("mx_ceil_log2", "s = (e - 1) - 8;", "s = e - 8;"),
    ("e4m3_overflow_nan", "if (a >= 448.0) return (uint8_t)(sign | 0x7E);", "if (a >= 448.0) return (uint8_t)(sign | 0x7F);"),
    ("e4m3_truncates", "double r = ldexp(rint(ldexp(a, -q)), q);", "double r = ldexp(floor(ldexp(a, -q)), q);"),
    ("e4m3_subnormal_grid", "if (q < -9) q = -9;", "if (q < -10) q = -10;"),
    ("eps_dropped", "1.0 / sqrt(ss / (double)D + eps)", "1.0 / sqrt(ss / (double)D)"),
    ("gamma_in_sum_of_squares", "ss += yh[d] * yh[d];",
     "ss += yh[d] * yh[d] * (double)gh[d] * (double)gh[d];"),
    ("state_indices_ignored", "state_indices ? state_indices[i] : i", "i"),
]


def _mutant_lib(tmp_path, name, old, new):
    src = open(obuild.SRC).read()
    assert src.count(old) >= 1, f"mutant {name}: pattern not found"
    mutated = src.replace(old, new)
    path = os.path.join(str(tmp_path), f"mut_{name}.c")
    with open(path, "w") as f:
        f.write(mutated)
    out = os.path.join(str(tmp_path), f"libmut_{name}.so")
    obuild.build(src=path, out=out)
    return oracle.load(out)


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new):
    lib = _mutant_lib(tmp_path, name, old, new)
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(lib)
        except (AssertionError, oracle.OracleError):
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake {name}"
