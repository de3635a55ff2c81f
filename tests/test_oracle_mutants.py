"""Planted mistakes in the oracle must be caught by the pins.

Each mutant is a plausible slip in ``oracle/kda_oracle.c`` (a dropped term, a
wrong sign, a wrong operand or order).  The test writes a patched copy of the C
source to a temporary directory, compiles it, and runs every pin in
``pins.py`` against it; at least one pin must fail.  The real oracle is never
modified.
"""
import os

import pytest

import oracle
from tests import pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "kda_oracle.c")

MUTANTS = {
    # the decay is used without exponentiating log alpha (first-order slip)
    "decay_not_exponentiated": [("const double a = exp(la[i]);", "const double a = 1.0 + la[i];")],
    # the erase term enters with the wrong sign
    "erase_sign": [("S[i * dv + j] += bk * (vt[j] - y[j]);", "S[i * dv + j] += bk * (vt[j] + y[j]);")],
    # beta scales the write but not the erase
    "beta_only_on_write": [("S[i * dv + j] += bk * (vt[j] - y[j]);",
                            "S[i * dv + j] += bk * vt[j] - kt[i] * y[j];")],
    # beta applied twice
    "beta_squared": [("const double bk = bt * kt[i];", "const double bk = bt * bt * kt[i];")],
    # the prediction S^T k uses q instead of k
    "prediction_uses_q": [("acc += kt[i] * S[i * dv + j];", "acc += qt[i] * S[i * dv + j];")],
    # the read-out uses k instead of q
    "readout_uses_k": [("acc += qt[i] * S[i * dv + j];", "acc += kt[i] * S[i * dv + j];")],
    # the token's decay is taken from the previous token
    "decay_off_by_one": [("const double *la = J->log_alpha + th * dk;",
                          "const double *la = J->log_alpha + (t > bos ? th - H : th) * dk;")],
    # the initial state is ignored
    "ignores_S0": [("if (J->S0)", "if (0 && J->S0)")],
    # the read-out is taken before the update (o_t = S_{t-1}^T q_t)
    "readout_before_update": [
        ("        /* step 2: S <- Diag(alpha_t) S, alpha_t = exp(log_alpha_t) (step 1) */",
         "        { double *ot0 = J->o + th * dv;\n"
         "          for (int j = 0; j < dv; ++j) { double s = 0.0;\n"
         "            for (int i = 0; i < dk; ++i) s += qt[i] * S[i * dv + j]; ot0[j] = s; } }\n"),
        ("            ot[j] = acc;", "            (void)acc; (void)ot;"),
    ],
    # the decay is applied after the delta-rule correction instead of before it
    "decay_after_correction": [
        ("        /* step 2: S <- Diag(alpha_t) S, alpha_t = exp(log_alpha_t) (step 1) */\n"
         "        for (int i = 0; i < dk; ++i) {\n"
         "            const double a = exp(la[i]);\n"
         "            for (int j = 0; j < dv; ++j)\n"
         "                S[i * dv + j] *= a;\n"
         "        }\n", ""),
        ("        /* step 4: o_t = S_t^T q_t */",
         "        for (int i = 0; i < dk; ++i) { const double a = exp(la[i]);\n"
         "            for (int j = 0; j < dv; ++j) S[i * dv + j] *= a; }\n"),
    ],
}


def _mutant_library(name, edits, tmp_path):
    with open(SRC) as f:
        text = f.read()
    for old, new in edits:
        assert text.count(old) == 1, f"mutant {name}: anchor not unique/missing: {old!r}"
        text = text.replace(old, new)
    src = tmp_path / f"{name}.c"
    src.write_text(text)
    out = str(tmp_path / f"lib{name}.so")
    oracle.compile_c(str(src), out)
    return oracle.load_library(out)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    lib = _mutant_library(name, MUTANTS[name], tmp_path)

    def run(q, k, v, la, b, cu, S0):
        return oracle.prefill(q, k, v, la, b, cu, S0=S0, lib=lib)

    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(run)
        except AssertionError:
            failed.append(getattr(pin, "__name__", "pin"))
    assert failed, f"no pin caught mutant {name}"
