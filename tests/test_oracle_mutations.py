"""Plant plausible mistakes in a copy of the oracle and check that the pins catch each.

Every mutation below is a one-token slip of the kind a restatement of the
recurrence could contain (a dropped term, a sign, a wrong index or operand).
The copy is compiled into a temporary directory; the real oracle is untouched.
"""
import os
import subprocess

import pytest

import oracle
from oracle_pins import PINS

MUTATIONS = {
    "drop_decay": ("S[c * Dv + j] *= a;", "S[c * Dv + j] *= 1.0;"),
    "delta_sign": ("S[c * Dv + j] += bt * kt[c] * (vt[j] - y[j]);",
                   "S[c * Dv + j] += bt * kt[c] * (vt[j] + y[j]);"),
    "retrieve_with_q": ("y[j] += S[c * Dv + j] * kt[c];", "y[j] += S[c * Dv + j] * qt[c];"),
    # the delta rule applied to the state before its decay (retrieval from S_{t-1})
    "retrieve_before_decay": ("y[j] += S[c * Dv + j] * kt[c];",
                              "y[j] += S[c * Dv + j] * kt[c] / exp(gt[c]);"),
    "drop_beta": ("S[c * Dv + j] += bt * kt[c] * (vt[j] - y[j])", "S[c * Dv + j] += kt[c] * (vt[j] - y[j])"),
    "output_with_k": ("ot[j] += S[c * Dv + j] * qt[c];", "ot[j] += S[c * Dv + j] * kt[c];"),
    "ckpt_off_by_one": ("(t + 1 - t0) % p->ckpt_interval", "(t + 2 - t0) % p->ckpt_interval"),
    "gate_transposed": ("exp(Gam[r * Dk + c] - Gam[i * Dk + c])",
                        "exp(Gam[i * Dk + c] - Gam[r * Dk + c])"),
    "beta_row_index": ("(i < r) ? B_(r) * m", "(i < r) ? B_(i) * m"),
    "p_strict": ("P[r * C + i] = (i <= r) ? pr : 0.0;", "P[r * C + i] = (i < r) ? pr : 0.0;"),
    "carry_no_decay": ("double s = exp(gl) * S[c * Dv + j];", "double s = S[c * Dv + j];"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name, tmp_path):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "kda_oracle.c")).read()
    old, new = MUTATIONS[name]
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    path = tmp_path / "mut.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", str(so),
                           str(path), "-lm"])
    lib = oracle.load(str(so))
    caught = []
    for pin, (fn, bound) in PINS.items():
        try:
            err = fn(lib)
        except Exception:
            err = float("inf")
        if not err <= bound:
            caught.append(pin)
    assert caught, f"no pin caught mutation {name}"
