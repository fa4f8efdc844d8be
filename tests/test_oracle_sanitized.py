"""The C oracle is memory-safe and free of undefined behaviour on the pins' inputs: a copy built
with AddressSanitizer (out-of-bounds and use-after-free) and one built with UBSan (-fno-sanitize-
recover, so any report aborts) each run a set of pins in a child process.  CPU only."""
import os
import shutil
import subprocess
import sys
import tempfile

import pytest

from oracle import build as obuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PINS = """
import sys
import oracle
oracle._swap_library(sys.argv[1])
import tests.test_oracle_pins as pins
import tests.test_oracle_backward_pins as bpins
import tests.test_oracle_doc_pins as dpins
import tests.test_oracle_qkv_pins as qpins
pins.test_oracle_matches_bruteforce(1, 70, 3, 128, 5, True)
pins.test_oracle_matches_bruteforce(2, 3, 2, 8, 0, True)
pins.test_window_one_is_identity_on_v_prime()
pins.test_gqa_equals_multihead_with_repeated_kv_heads(6, 2, 13, True)
bpins.test_backward_matches_central_differences(1, 7, 1, 8, 3, True, True, True, True)
bpins.test_gqa_gradients_are_group_sums_of_repeated_head_gradients(6, 2)
dpins.test_documents_match_bruteforce(7, True)
dpins.test_gradient_with_documents_matches_central_differences(3)
qpins.test_permutation_weights_reduce_to_the_prologue_bit_for_bit(4, 2, 8, True, True)
print("pins ok under", oracle._lib._name)
"""


def _runtime(name):
    gcc = shutil.which("gcc")
    if gcc is None:
        return None
    p = subprocess.run([gcc, f"-print-file-name={name}"], capture_output=True, text=True).stdout.strip()
    return p if os.path.isabs(p) and os.path.exists(p) else None


# A one-element heap overflow planted in the row buffer of the attention step: the address
# sanitizer run must report it (the check is not vacuous).
OVERFLOW = ("            double* o = (double*)malloc(sizeof(double) * (size_t)D);",
            "            double* o = (double*)malloc(sizeof(double) * (size_t)(D - 1));")


def _run_pins(kind, src_text):
    rt = _runtime("libasan.so" if kind == "address" else "libubsan.so")
    if rt is None:
        pytest.skip(f"no {kind} sanitizer runtime")
    scratch = os.path.join(ROOT, ".pytest_cache", "sanitized")
    os.makedirs(scratch, exist_ok=True)
    with tempfile.TemporaryDirectory(dir=scratch) as tmp:
        c = os.path.join(tmp, "oracle_san.c")
        so = os.path.join(tmp, "liboracle_san.so")
        open(c, "w").write(src_text)
        flags = ["-fsanitize=address", "-fno-omit-frame-pointer"] if kind == "address" else \
            ["-fsanitize=undefined,bounds", "-fno-sanitize-recover=all"]
        subprocess.run(["gcc", "-O1", "-g", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
                        *flags, "-o", so, c, "-lm"], check=True)
        env = dict(os.environ, ASAN_OPTIONS="detect_leaks=0")
        # the runtime goes first; libstdc++ with it, so the sanitizer finds the C++ runtime it wraps
        env["LD_PRELOAD"] = " ".join(p for p in (rt, _runtime("libstdc++.so")) if p)
        return subprocess.run([sys.executable, "-c", PINS, so], cwd=ROOT, env=env, capture_output=True,
                              text=True, timeout=600)


@pytest.mark.parametrize("kind", ["address", "undefined"])
def test_oracle_pins_under_a_sanitizer(kind):
    r = _run_pins(kind, open(obuild.SRC).read())
    assert r.returncode == 0 and "pins ok under" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]


def test_planted_overflow_is_reported():
    src = open(obuild.SRC).read()
    assert src.count(OVERFLOW[0]) == 1
    r = _run_pins("address", src.replace(*OVERFLOW))
    assert r.returncode != 0 and "heap-buffer-overflow" in r.stderr, r.stderr[-2000:]
