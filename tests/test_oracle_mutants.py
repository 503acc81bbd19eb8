"""Plants plausible mistakes in copies of the oracle and checks the pins catch each.

The copies are compiled from ``oracle/gdr_oracle.c`` with one textual change each
and run on the CPU only.
"""
import os
import subprocess

import pytest

import oracle
import oracle_pins as P

SRC = os.path.join(os.path.dirname(oracle.library_path()), "gdr_oracle.c")

MUTANTS = {
    "erase_sign": ("- e[c] * z[j] + vv[c]", "+ e[c] * z[j] + vv[c]"),
    "no_decay": ("S[(size_t)c * dk + j] * w[j] - e[c]", "S[(size_t)c * dk + j] - e[c]"),
    "gdn2_u_without_alpha": ("u[j] = w[j] * e1[tk + j] * k[tk + j];", "u[j] = e1[tk + j] * k[tk + j];"),
    "readout_with_key": ("S[(size_t)c * dk + j] * q[tk + j]", "S[(size_t)c * dk + j] * k[tk + j]"),
    "rwkv7_z_scaled": ("z[j] = e1[tk + j]; }", "z[j] = cc * e1[tk + j]; }"),
    "write_gate_dropped": ("if (e2) for (int c = 0; c < dv; ++c) vv[c] *= e2[tv + c];", ""),
    "state_in_transposed": ("S0[so + (size_t)j * dv + c]", "S0[so + (size_t)c * dv + j]"),
    "write_key_swapped": ("vv[c] * k[tk + j]", "vv[c] * q[tk + j]"),
}


def _compile(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    lib = tmp_path / f"lib{name}.so"
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-shared", "-fPIC", "-o", str(lib),
                           str(path), "-lm"])
    return oracle.load_library(str(lib))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    lib = _compile(tmp_path, name, *MUTANTS[name])

    def fwd(form, q, k, v, log_w, e1, e2, S0):
        return oracle.forward(form, q, k, v, log_w, e1, e2, S0, lib=lib)

    caught = []
    for pin in P.ALL_PINS:
        try:
            pin(fwd)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin detects mutant {name}"
