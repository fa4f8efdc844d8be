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
import tests.test_oracle_backward_pins as bpins
import tests.test_oracle_pins as pins
import tests.test_oracle_doc_pins as dpins
import tests.test_oracle_qkv_pins as qpins

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


# Mistakes in the backward (the gradient of the layer); the forward stays correct.
BACKWARD_MUTANTS = {
    "bwd row pass drops delta": ("p * (dot_d(gi, vp + (size_t)j * D, D) - dl) + p * gl",
                                 "p * dot_d(gi, vp + (size_t)j * D, D) + p * gl"),
    "bwd key pass drops delta": ("p * (dot_d(gi, vj, D) - delta[i]) + p * gl",
                                 "p * dot_d(gi, vj, D) + p * gl"),
    "bwd row pass drops dlse": ("- dl) + p * gl;", "- dl);"),
    "bwd key pass drops dlse": ("- delta[i]) + p * gl;", "- delta[i]);"),
    "bwd rms correction sign": ("dx[d] = r * dy[d] - coef * xr[d];", "dx[d] = r * dy[d] + coef * xr[d];"),
    "bwd rms r squared": ("const double coef = r * r * r * xdy", "const double coef = r * r * xdy"),
    "bwd rope not transposed": (
        "    for (int i = half; i < D; ++i) g[i] = -g[i];\n    rope_inplace(g, D, t, base);\n"
        "    for (int i = half; i < D; ++i) g[i] = -g[i];\n",
        "    rope_inplace(g, D, t, base);\n"),
    "bwd gate derivative without 1 - sigma": ("dgate * 2.0 * sig * (1.0 - sig)", "dgate * 2.0 * sig"),
    "bwd ve gradient without gate": ("dve_out[d] = 2.0 * sig * dvt[d];", "dve_out[d] = dvt[d];"),
    "bwd dx reads Wg transposed": (
        "acc += dz[(size_t)bt * Hkv + hk] * bf16_to_double(Wg[(size_t)c * Hkv + hk]);",
        "acc += dz[(size_t)bt * Hkv + hk] * bf16_to_double(Wg[(size_t)hk * 32 + c]);"),
    "bwd dWg reads x with stride 32": ("bf16_to_double(x[(size_t)bt * C + c])",
                                       "bf16_to_double(x[(size_t)bt * 32 + c])"),
    "bwd key pass window off by one": ("return window_convention == 0 ? W - 1 : W;",
                                       "return window_convention == 0 ? W : W;"),
    "bwd gqa group sum dropped": (
        "            memset(dkh, 0, sizeof(double) * TD);\n            memset(dvp, 0, sizeof(double) * TD);\n\n"
        "            for (int g = 0; g < G; ++g) {\n",
        "            for (int g = 0; g < G; ++g) {\n"
        "            memset(dkh, 0, sizeof(double) * TD);\n            memset(dvp, 0, sizeof(double) * TD);\n"),
    "bwd dk without scale": ("dkj[d] += ds * qi[d] * inv_sqrt_d;", "dkj[d] += ds * qi[d];"),
    "bwd dv weighted by dS": ("dvj[d] += p * gi[d];", "dvj[d] += ds * gi[d];"),
    "bwd dq from queries": ("dqi[d] += ds * kh[(size_t)j * D + d] * inv_sqrt_d;",
                            "dqi[d] += ds * qi[d] * inv_sqrt_d;"),
    "bwd keys not rounded in parity mode": ("                    round_bf16, kh + (size_t)t * D);",
                                            "                    0, kh + (size_t)t * D);"),
}

BACKWARD_PIN_FUNCS = [
    lambda: bpins.test_backward_matches_central_differences(1, 7, 1, 8, 3, True, True, True, True),
    lambda: bpins.test_backward_matches_central_differences(2, 5, 2, 4, 2, False, True, True, True),
    lambda: bpins.test_backward_matches_torch_autograd(4, 2, 5, True),
    lambda: bpins.test_parity_mode_backward_is_straight_through_rounding(2),
    bpins.test_window_one_closed_form,
    bpins.test_lse_only_cotangent_leaves_values_untouched,
    lambda: bpins.test_rms_scale_invariance_makes_dq_orthogonal_to_q(True),
    lambda: bpins.test_gqa_gradients_are_group_sums_of_repeated_head_gradients(6, 2),
]


# Mistakes in the fused projection + prologue (every planted index stays inside its array).
QKV_MUTANTS = {
    "proj weight row stride": ("const uint16_t* w = Wqkv + (size_t)n * C;", "const uint16_t* w = Wqkv + (size_t)n * (C - 1);"),
    "proj k rows start at Hkv D": ("const int n0 = part == 0 ? 0 : H * D;", "const int n0 = part == 0 ? 0 : Hkv * D;"),
    "proj v reads the k rows": ("proj_dot(xr, Wqkv, C, (H + Hkv) * D + h * D + d)", "proj_dot(xr, Wqkv, C, H * D + h * D + d)"),
    "proj gate column reversed": ("bf16_to_double(Wg[c * Hkv + h]);\n                    gate = 2.0",
                                  "bf16_to_double(Wg[c * Hkv + (Hkv - 1 - h)]);\n                    gate = 2.0"),
    "proj rope position from b": ("if (use_rope) rope_inplace(row, D, t, rope_base);", "if (use_rope) rope_inplace(row, D, b, rope_base);"),
}

DOC_MUTANTS = {
    "doc compared with the first position": ("doc_b[j] == doc_b[i]", "doc_b[j] == doc_b[0]"),
    "previous document leaks in": ("doc_b[j] == doc_b[i]", "(doc_b[j] == doc_b[i] || doc_b[j] + 1 == doc_b[i])"),
    "backward key pass ignores documents": ("if (doc_b != NULL && doc_b[i] != doc_b[j]) continue;", ";"),
}

DOC_PIN_FUNCS = [
    lambda: dpins.test_documents_match_bruteforce(7, True),
    dpins.test_each_document_is_the_layer_on_its_own_slice,
    dpins.test_first_row_of_each_document_is_its_own_value,
    lambda: dpins.test_gradient_with_documents_matches_central_differences(3),
    dpins.test_gradient_of_each_document_is_the_gradient_on_its_own_slice,
]

QKV_PIN_FUNCS = [
    lambda: qpins.test_permutation_weights_reduce_to_the_prologue_bit_for_bit(2, 2, 16, True, False),
    lambda: qpins.test_permutation_weights_reduce_to_the_prologue_bit_for_bit(4, 2, 8, True, True),
    qpins.test_projection_alone_equals_numpy_matmul,
    qpins.test_doubling_the_weights_leaves_the_normalised_rows_unchanged,
]


def _failing_pins(funcs=None):
    failed = 0
    for f in (PIN_FUNCS if funcs is None else funcs):
        try:
            f()
        except (AssertionError, ValueError, FloatingPointError):
            failed += 1
    return failed


def _scratch():
    """Mutant builds go to a git-ignored directory inside the repository."""
    d = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), ".pytest_cache", "mutants")
    os.makedirs(d, exist_ok=True)
    return d


def _build_mutant(old, new, tmp):
    src = open(obuild.SRC).read()
    assert src.count(old) == 1, f"mutation anchor not found: {old!r}"
    c = os.path.join(tmp, "mutant.c")
    so = os.path.join(tmp, "libmutant.so")
    open(c, "w").write(src.replace(old, new))
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fPIC",
                    "-shared", "-o", so, c, "-lm"], check=True)
    return so


@pytest.mark.parametrize("name", sorted(BACKWARD_MUTANTS))
def test_planted_backward_mistake_is_caught(name):
    old, new = BACKWARD_MUTANTS[name]
    with tempfile.TemporaryDirectory(dir=_scratch()) as tmp:
        oracle._swap_library(_build_mutant(old, new, tmp))
        try:
            assert _failing_pins(BACKWARD_PIN_FUNCS) >= 1, f"no pin caught the planted mistake: {name}"
        finally:
            oracle._swap_library(None)


@pytest.mark.parametrize("name", sorted(QKV_MUTANTS))
def test_planted_projection_mistake_is_caught(name):
    old, new = QKV_MUTANTS[name]
    with tempfile.TemporaryDirectory(dir=_scratch()) as tmp:
        oracle._swap_library(_build_mutant(old, new, tmp))
        try:
            assert _failing_pins(QKV_PIN_FUNCS) >= 1, f"no pin caught the planted mistake: {name}"
        finally:
            oracle._swap_library(None)


@pytest.mark.parametrize("name", sorted(DOC_MUTANTS))
def test_planted_document_mask_mistake_is_caught(name):
    old, new = DOC_MUTANTS[name]
    with tempfile.TemporaryDirectory(dir=_scratch()) as tmp:
        oracle._swap_library(_build_mutant(old, new, tmp))
        try:
            assert _failing_pins(DOC_PIN_FUNCS) >= 1, f"no pin caught the planted mistake: {name}"
        finally:
            oracle._swap_library(None)


def test_unmutated_projection_passes_every_projection_pin():
    assert _failing_pins(QKV_PIN_FUNCS) == 0


def test_unmutated_backward_passes_every_backward_pin():
    assert _failing_pins(BACKWARD_PIN_FUNCS) == 0


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    old, new = MUTANTS[name]
    src = open(obuild.SRC).read()
    assert src.count(old) == 1, f"mutation anchor not found: {old!r}"
    with tempfile.TemporaryDirectory(dir=_scratch()) as tmp:
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
