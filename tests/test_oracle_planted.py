"""Planted mistakes in the oracle (on the CPU) must be caught by its pins.

Each mutation is a plausible slip in the fp64 loop -- a flipped rotation sense,
an exclusive instead of inclusive angle sum, a dropped or mis-indexed term, a
wrong group mapping.  A copy of the oracle source with the slip is compiled to
a temporary library and run through the pins of test_oracle_pins; at least one
pin must fail for every mutation.
"""
import glob
import json
import os

import numpy as np
import pytest

import oracle
from tests.test_oracle_pins import GOLDEN, quadratic_form, rand_problem, test_impulse_closed_form

MUTATIONS = {
    "rotation sense": [("out[2 * i] = c * re - s * im;", "out[2 * i] = c * re + s * im;"),
                       ("out[2 * i + 1] = s * re + c * im;", "out[2 * i + 1] = -s * re + c * im;")],
    "exclusive angle": [("rotate_pairs(j->B + tg * N, phi, N, Bbar);",
                         "rotate_pairs(j->B + tg * N, phi_prev, N, Bbar);"),
                        ("rotate_pairs(j->C + tg * N, phi, N, Cbar);",
                         "rotate_pairs(j->C + tg * N, phi_prev, N, Cbar);")],
    "dropped beta term": [("+ be * Bpbar[n] * xp[p] + ga * Bbar[n] * x[p];\n\n    const double dh",
                           "+ ga * Bbar[n] * x[p];\n\n    const double dh")],
    "beta uses current B": [("be * Bpbar[n] * xp[p] + ga * Bbar[n] * x[p];\n\n    const double dh",
                             "be * Bbar[n] * xp[p] + ga * Bbar[n] * x[p];\n\n    const double dh")],
    "no decay": [("S[n * P + p] = alpha * S[n * P + p] + be * Bpbar[n] * xp[p] + ga * Bbar[n] * x[p];\n\n    const double dh",
                  "S[n * P + p] = S[n * P + p] + be * Bpbar[n] * xp[p] + ga * Bbar[n] * x[p];\n\n    const double dh")],
    "pairs swapped": [("const double re = v[2 * i];", "const double re = v[2 * i + 1];"),
                      ("const double im = v[2 * i + 1];", "const double im = v[2 * i];")],
    "group mapping": [("const int64_t g = h / (H / G);\n  const int64_t NH",
                       "const int64_t g = h % G;\n  const int64_t NH")],
    "D on previous x": [("j->Y[th * P + p] = acc + dh * x[p];", "j->Y[th * P + p] = acc + dh * xp[p];")],
    "previous B not rotated": [("rotate_pairs(Bp, phi_prev, N, Bpbar);", "rotate_pairs(Bp, phi, N, Bpbar);")],
}


def pins_pass() -> bool:
    ok = True
    for path in sorted(glob.glob(os.path.join(GOLDEN, "worked_*.json"))):
        with open(path) as f:
            g = json.load(f)
        out = oracle.oracle_fwd(**{k: np.array(v, dtype=np.float64) for k, v in g["inputs"].items()})
        for k, v in g["expected"].items():
            ok &= bool(np.allclose(out[k], np.array(v), rtol=0, atol=g["atol"]))
    p = rand_problem(np.random.default_rng(0), L=9)
    out = oracle.oracle_fwd(**p)
    Yq, hTq = quadratic_form(p)
    ok &= bool(np.allclose(out["Y"], Yq, rtol=1e-10, atol=1e-12))
    ok &= bool(np.allclose(out["hT"], hTq, rtol=1e-10, atol=1e-12))
    try:
        test_impulse_closed_form(True)
    except AssertionError:
        ok = False
    return ok


def test_unmodified_source_passes_pins():
    assert pins_pass()


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, tmp_path):
    src = oracle.source_text()
    for old, new in MUTATIONS[name]:
        assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
        src = src.replace(old, new)
    lib = oracle.compile_variant(src, str(tmp_path / "liboracle_mut.so"))
    with oracle.use_library(lib):
        assert not pins_pass(), f"planted mistake '{name}' passed every pin"
