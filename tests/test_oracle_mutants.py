"""Sensitivity of the oracle pins: each plausible mistake planted in a copy of the C oracle
(a flipped sign, a dropped term, an off-by-one, a transposed index) must make at least one
pin fail.  Mistakes are planted on the CPU, in a temporary build; the regular build is
untouched.  CPU only."""
import ctypes
import os
import subprocess
import tempfile

import pytest

import oracle
from oracle import build as obuild
import tests.test_oracle_pins as pins

MUTANTS = {
    "rope sign": ("x[i] = a * c - b * s;", "x[i] = a * c + b * s;"),
    "rope frequency exponent": ("pow(base, -2.0 * (double)i / (double)D)", "pow(base, -1.0 * (double)i / (double)D)"),
    "rope position offset": ("double ang = (double)t * theta;", "double ang = (double)(t + 1) * theta;"),
    "rms drops eps": ("sqrt(ss / (double)D + eps)", "sqrt(ss / (double)D)"),
    "rms sum instead of mean": ("sqrt(ss / (double)D + eps)", "sqrt(ss + eps)"),
    "window off by one": ("convention == 0 ? (diff < W)", "convention == 0 ? (diff <= W)"),
    "diagonal masked": ("if (diff < 0) return 0;", "if (diff <= 0) return 0;"),
    "scale 1/D": ("const double scale = 1.0 / sqrt((double)D);", "const double scale = 1.0 / (double)D;"),
    "gate without factor 2": ("double gate = 2.0 / (1.0 + exp(-z));", "double gate = 1.0 / (1.0 + exp(-z));"),
    "gate sign": ("double gate = 2.0 / (1.0 + exp(-z));", "double gate = 2.0 / (1.0 + exp(z));"),
    "Wg transposed": ("bf16_to_double(Wg[c * H + h])", "bf16_to_double(Wg[h * 32 + c])"),
    "ve head offset dropped": ("(size_t)id * (size_t)H * D + (size_t)h * D", "(size_t)id * (size_t)H * D"),
    "lse drops max": ("*lse = M + log(L);", "*lse = log(L);"),
    "bf16 rounding truncates": ("double r = nearbyint(ldexp(m, 8));", "double r = trunc(ldexp(m, 8));"),
    "rope second component swapped": ("x[i + half] = a * s + b * c;", "x[i + half] = b * s + a * c;"),
    "gqa head mapping modulo": ("const int hk = h / G;", "const int hk = h % Hkv;"),
}

PIN_FUNCS = [
    lambda: pins.test_oracle_matches_bruteforce(2, 3, 2, 8, 0, True),
    lambda: pins.test_oracle_matches_bruteforce(1, 70, 3, 128, 5, True),
    lambda: pins.test_no_prologue_equals_torch_sdpa(9),
    pins.test_window_one_is_identity_on_v_prime,
    pins.test_row_zero_is_gated_v0_and_its_single_score,
    pins.test_zero_queries_give_uniform_weights,
    pins.test_hand_derived_two_token_case,
    pins.test_rope_d2_is_rotation_by_t_radians,
    pins.test_rope_d4_second_pair_uses_base_power,
    pins.test_rms_unit_when_eps_zero_and_closed_form_otherwise,
    pins.test_gate_is_two_sigmoid_per_head_in_open_interval,
    pins.test_round_bf16_ties_to_even_without_double_rounding,
    lambda: pins.test_gqa_equals_multihead_with_repeated_kv_heads(6, 2, 13, True),
]


def _failing_pins():
    failed = 0
    for f in PIN_FUNCS:
        try:
            f()
        except (AssertionError, ValueError, FloatingPointError):
            failed += 1
    return failed


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    old, new = MUTANTS[name]
    src = open(obuild.SRC).read()
    assert src.count(old) == 1, f"mutation anchor not found: {old!r}"
    with tempfile.TemporaryDirectory() as tmp:
        c = os.path.join(tmp, "mutant.c")
        so = os.path.join(tmp, "libmutant.so")
        open(c, "w").write(src.replace(old, new))
        subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fPIC",
                        "-shared", "-o", so, c, "-lm"], check=True)
        oracle._swap_library(so)
        try:
            assert _failing_pins() >= 1, f"no pin caught the planted mistake: {name}"
        finally:
            oracle._swap_library(None)


def test_unmutated_oracle_passes_every_pin():
    assert _failing_pins() == 0
