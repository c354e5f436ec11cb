"""The oracle's pins have teeth: plausible mistakes planted in a copy of the oracle
(on the CPU, in a temporary build) must each make at least one pin fail."""
import ctypes
import os
import subprocess
import tempfile

import pytest

import oracle
from oracle import oracle as orc
import tests.test_oracle_pins as P

SRC = os.path.join(os.path.dirname(orc.__file__), "falcon_oracle.c")

# (name, original text, mutated text) or (name, [(original, mutated), ...])
MUTANTS = [
    ("same-step pairing (k_t instead of k_{t-1})",
     "pair_key(X + (size_t)m * dk, k, kprev, t - m, dk, same_step(rule));",
     "pair_key(X + (size_t)m * dk, k, kprev, t - m + 1, dk, same_step(rule));"),
    ("no decay in the recurrence",
     "S[i] *= a; /* Sbar = alpha_t S */", "(void)a;"),
    ("normaliser ignores the key norm",
     "return den > 0.0 ? eta / den : 0.0;", "return eta / (1.0 + eps);"),
    ("wrong sign of the regression step",
     "S[(size_t)i * dk + c] -= ri * X[(size_t)m * dk + c];",
     "S[(size_t)i * dk + c] += ri * X[(size_t)m * dk + c];"),
    ("halved inner-product write",
     "S[(size_t)i * dk + c] += yi * X[(size_t)m * dk + c];",
     "S[(size_t)i * dk + c] += 0.5 * yi * X[(size_t)m * dk + c];"),
    ("read before write in the recurrence (o_t = Sbar q_t)",
     [("for (int i = 0; i < dv; ++i) o[(size_t)t * dv + i] = dotd(S + (size_t)i * dk, q + (size_t)t * dk, dk);", ""),
      ("S[i] *= a; /* Sbar = alpha_t S */",
       "S[i] *= a;\n        for (int i = 0; i < dv; ++i) o[(size_t)t * dv + i] = dotd(S + (size_t)i * dk, q + (size_t)t * dk, dk);")]),
    ("residual taken at the undecayed state",
     "R[(size_t)m * dv + i] = dotd(S + (size_t)i * dk, X + (size_t)m * dk, dk) - yi;",
     "R[(size_t)m * dv + i] = (a != 0.0 ? 1.0 / a : 0.0) * dotd(S + (size_t)i * dk, X + (size_t)m * dk, dk) - yi;"),
    ("window residuals applied one by one",
     "for (int m = 0; m < w; ++m)\n                for (int i = 0; i < dv; ++i) {\n                    const double ri",
     "for (int m = 0; m < w; ++m)\n                for (int i = 0; i < dv; ++i) {\n                    if (m > 0) R[(size_t)m * dv + i] = dotd(S + (size_t)i * dk, X + (size_t)m * dk, dk) - ((t - m) >= 0 ? v[(size_t)(t - m) * dv + i] : 0.0);\n                    const double ri"),
    ("chunk form: decay exponent flipped",
     "const double l = beta[s] * exp(g[s] - g[s2])", "const double l = beta[s] * exp(g[s2] - g[s])"),
    ("chunk form: exclusive read (before write)",
     "for (int e2 = 0; e2 < (i + 1) * w; ++e2) {", "for (int e2 = 0; e2 < i * w; ++e2) {"),
    ("chunk form: state passing drops the decay",
     "const double f = exp(gl - g[s2]);", "const double f = 1.0;"),
]


def _build_mutant(tmpdir, edits):
    src = open(SRC).read()
    for original, mutated in edits:
        assert original in src, f"mutation anchor not found: {original[:60]}"
        src = src.replace(original, mutated, 1)
    mpath = os.path.join(tmpdir, "m.c")
    open(mpath, "w").write(src)
    lib = os.path.join(tmpdir, "libm.so")
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c99", "-o", lib, mpath, "-lm"],
                   check=True)
    return lib


PIN_CALLS = [
    lambda: P.test_hand_worked_example("falcon1", "recurrent"),
    lambda: P.test_hand_worked_example("falcon3", "recurrent"),
    lambda: P.test_hand_worked_example("falcon1a", "chunk2"),
    lambda: P.test_hand_worked_example("falcon1", "chunk2"),
    lambda: P.test_falcon1_hand_expanded_first_three_steps(),
    lambda: P.test_falcon1a_is_gated_linear_attention(),
    lambda: P.test_kaczmarz_interpolation_any_decay(0),
    lambda: P.test_decay_only_when_eta_zero(oracle.RULE_1, 1),
    lambda: P.test_step_is_normalised_gradient_step(oracle.RULE_1, 1),
    lambda: P.test_step_is_normalised_gradient_step(oracle.RULE_3, 3),
    lambda: P.test_falcon3_orthonormal_window_closed_form(),
    lambda: P.test_three_forms_agree(oracle.RULE_1, 1, 4),
    lambda: P.test_three_forms_agree(oracle.RULE_3, 3, 4),
    lambda: P.test_three_forms_agree(oracle.RULE_1A, 1, 4),
]


def _edits(m):
    return m[1] if len(m) == 2 else [(m[1], m[2])]


@pytest.mark.parametrize("mutant", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(mutant, monkeypatch):
    name = mutant[0]
    with tempfile.TemporaryDirectory() as d:
        libpath = _build_mutant(d, _edits(mutant))
        good = orc._load()
        bad = ctypes.CDLL(libpath)
        for fn in ("falcon_oracle_recurrent", "falcon_oracle_chunk", "falcon_oracle_masked",
                   "falcon_oracle_max_threads"):
            getattr(bad, fn).argtypes = getattr(good, fn).argtypes
            getattr(bad, fn).restype = getattr(good, fn).restype
        monkeypatch.setattr(orc, "_lib", bad)
        caught = 0
        for call in PIN_CALLS:
            try:
                call()
            except AssertionError:
                caught += 1
        assert caught > 0, f"no pin caught the mutant: {name}"
