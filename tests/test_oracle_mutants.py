"""The oracle's pins must catch plausible mistakes.

Each mutant below is a copy of ``oracle/kda_oracle.c`` with one planted
mistake (a dropped term, a wrong sign, a wrong order or index), built on the
CPU into a temporary library. The pins of ``test_oracle.py`` run against it,
and at least one of them must fail. Nothing here touches a GPU.
"""
import os
import subprocess

import pytest

import oracle
import test_oracle as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "kda_oracle.c")

DECAY = "S[i * dv + j] *= a;"
UPDATE = "S[i * dv + j] += kt[i] * u[j];"
WRITE = "u[j] = bw * widen(v, row * dv + j, in_dtype) - be * r[j];"
READ = "o += S[i * dv + j] * qt[i];"
LOAD_S0 = "S[e] = s0[e];"

MUTANTS = {
    "erase_sign_flipped": [(WRITE, "u[j] = bw * widen(v, row * dv + j, in_dtype) + be * r[j];")],
    "decay_dropped": [(DECAY, "(void)a;")],
    "write_not_weighted": [(WRITE, "u[j] = widen(v, row * dv + j, in_dtype) - be * r[j];")],
    "erase_not_weighted": [(WRITE, "u[j] = bw * widen(v, row * dv + j, in_dtype) - r[j];")],
    "decay_after_update": [
        (DECAY, "(void)a;"),
        (UPDATE, "S[i * dv + j] = (S[i * dv + j] + kt[i] * u[j]) * exp((double)log_alpha[row * dk + i]);"),
    ],
    "read_before_update": [(READ, "o += (S[i * dv + j] - kt[i] * u[j]) * qt[i];")],
    "read_with_key": [(READ, "o += S[i * dv + j] * kt[i];")],
    "gate_channel_reversed": [
        ("double a = exp((double)log_alpha[row * dk + i]);",
         "double a = exp((double)log_alpha[row * dk + (dk - 1 - i)]);")],
    "initial_state_transposed": [(LOAD_S0, "S[e] = s0[(e % dv) * dk + e / dv];")],
}

PINS = [
    pins.test_linear_attention_special_case,
    pins.test_gated_linear_attention_closed_form,
    pins.test_gdn_scalar_gate_special_case,
    pins.test_deltanet_basis_keys_overwrite_rows,
    pins.test_beta_zero_is_pure_decay,
    lambda: pins.test_bruteforce_transition_products(7, 4, 6),
    pins.test_handworked_example,
]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    src = open(SRC).read()
    for old, new in MUTANTS[name]:
        assert src.count(old) == 1, f"mutation site not found: {old}"
        src = src.replace(old, new)
    path = tmp_path / f"{name}.c"
    path.write_text(src)
    lib = tmp_path / f"lib{name}.so"
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c99", "-o", str(lib),
                    str(path), "-lm"], check=True)
    caught = []
    with oracle.swapped_library(str(lib)):
        for pin in PINS:
            try:
                pin()
            except AssertionError:
                caught.append(getattr(pin, "__name__", "bruteforce"))
    assert caught, f"no pin caught mutant {name}"
