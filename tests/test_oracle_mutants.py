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


# mistakes in the backward sweep, caught by the finite-difference and closed-form pins
BWD_MUTANTS = [
    ("dbeta_scaled_by_beta", "db += du[j] * r[j];", "db += du[j] * r[j] * bt;"),
    ("state_gradient_not_decayed", "G[(size_t)i * dv + j] = al[i] * dSp[(size_t)i * dv + j];",
     "G[(size_t)i * dv + j] = dSp[(size_t)i * dv + j];"),
    ("erase_term_dropped_from_dk", "c->dk_out[ti * dk + i] = acc_u - acc_r;", "c->dk_out[ti * dk + i] = acc_u;"),
    ("clamp_passes_everything", "((double)lt[i] >= c->la_floor) ? 1.0 : 0.0", "1.0"),
    ("dq_from_decayed_previous_state", "for (int j = 0; j < dv; ++j) acc += St[(size_t)i * dv + j] * dot[j];",
     "for (int j = 0; j < dv; ++j) acc += al[i] * Sprev[(size_t)i * dv + j] * dot[j];"),
    ("erase_gradient_sign", "const double g = G[(size_t)i * dv + j] - (double)kt[i] * dr[j];",
     "const double g = G[(size_t)i * dv + j] + (double)kt[i] * dr[j];"),
]

BWD_CHECKS = [
    lambda: pins.test_backward_matches_finite_differences(),
    lambda: pins.test_backward_clamp_blocks_gradient(),
    lambda: pins.test_backward_of_one_token_closed_form(),
]


@pytest.mark.parametrize("name,old,new", BWD_MUTANTS, ids=[m[0] for m in BWD_MUTANTS])
def test_backward_pins_catch_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not found: {name}"
    c_path = tmp_path / "mut.c"
    so_path = tmp_path / "libmut.so"
    c_path.write_text(src.replace(old, new, 1))
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-o", str(so_path), str(c_path),
                    "-lm", "-lpthread"], check=True)
    saved = oracle._lib
    oracle._lib = oracle._setup(ctypes.CDLL(str(so_path)))
    caught = 0
    try:
        for chk in BWD_CHECKS:
            try:
                chk()
            except AssertionError:
                caught += 1
    finally:
        oracle._lib = saved
    assert caught >= 1, f"no pin caught mutant {name}"
