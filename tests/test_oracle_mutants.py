"""Plants plausible mistakes in a copy of the oracle and checks that the pins
in test_oracle_pins.py catch every one of them (the oracle itself is never
modified; each mutant is compiled from a patched copy in a temp directory)."""
import ctypes
import os
import subprocess

import pytest

import oracle
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "kda_oracle.c")

# (name, exact text in kda_oracle.c, replacement)
MUTANTS = [
    ("erase_sign_flipped", "u[j] = bt * ((double)vt[j] - sk);", "u[j] = bt * ((double)vt[j] + sk);"),
    ("erase_dropped", "if (c->erase)\n", "if (0)\n"),
    ("beta_not_applied", "u[j] = bt * ((double)vt[j] - sk);", "u[j] = ((double)vt[j] - sk);"),
    ("decay_on_value_columns", "for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= alpha[i];",
     "for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= alpha[j % dk];"),
    ("no_log_decay_floor", "if (l < c->la_floor) l = c->la_floor;\n            alpha[i] = exp(l);",
     "alpha[i] = exp(l);"),
    ("read_before_write", "for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * (double)qt[i];",
     "for (int i = 0; i < dk; ++i) acc += (S[(size_t)i * dv + j] - (double)kt[i] * u[j]) * (double)qt[i];"),
]

CHECKS = [
    lambda: [pins.test_hand_worked_examples(c) for c in pins.json.load(open(pins.GOLDEN))["cases"]],
    lambda: pins.test_erase_write_invariant(16),
    lambda: pins.test_repeated_key_geometric_convergence(0.5),
    lambda: pins.test_beta_zero_pure_decay(),
    lambda: pins.test_gated_linear_attention_closed_form(),
    lambda: pins.test_log_decay_floor(),
    lambda: pins.test_linear_attention_reduction_bruteforce(),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor not found: {name}"
    mut = src.replace(old, new, 1)
    c_path = tmp_path / "mut.c"
    so_path = tmp_path / "libmut.so"
    c_path.write_text(mut)
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-o", str(so_path), str(c_path),
                    "-lm", "-lpthread"], check=True)
    saved = oracle._lib
    oracle._lib = oracle._setup(ctypes.CDLL(str(so_path)))
    caught = 0
    try:
        for chk in CHECKS:
            try:
                chk()
            except AssertionError:
                caught += 1
    finally:
        oracle._lib = saved
    assert caught >= 1, f"no pin caught mutant {name}"
