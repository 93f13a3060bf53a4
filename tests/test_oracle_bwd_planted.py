"""Planted mistakes in the oracle's backward (on the CPU) must be caught by the
finite-difference pins of test_oracle_bwd.

Each mutation is a plausible slip in the adjoint sweep: a dropped term, the
state gradient not carried back through the decay, a missing chain-rule factor,
a wrong sign or transposition in the rotation adjoint, a gradient sent to the
wrong token.  A copy of the oracle source with the slip is compiled to a
temporary library; the directional finite-difference check must fail.
"""
import numpy as np
import pytest

import oracle
from tests.test_oracle_bwd import GRADS, INPUTS, fd_directional, make_case

MUTATIONS = {
    "dropped beta adjoint": [("dBpbar[n] = be * gxp;", "dBpbar[n] = 0.0;")],
    "decay not carried back": [("for (int64_t e = 0; e < NP; ++e) gS[e] *= a;", "")],
    "dlogdecay without alpha": [("j->dlogdecay[th] = a * da;", "j->dlogdecay[th] = da;")],
    "angle adjoint sign": [("dphi_acc[i] += -d0 * vbar[2 * i + 1] + d1 * vbar[2 * i];",
                            "dphi_acc[i] += d0 * vbar[2 * i + 1] + d1 * vbar[2 * i];")],
    "rotation adjoint not transposed": [("dv_acc[2 * i] += c * d0 + s * d1;",
                                         "dv_acc[2 * i] += c * d0 - s * d1;"),
                                        ("dv_acc[2 * i + 1] += -s * d0 + c * d1;",
                                         "dv_acc[2 * i + 1] += s * d0 + c * d1;")],
    "x gradient from the previous B": [("dx[p] += ga * gb;", "dx[p] += ga * gbp;")],
    "previous-x gradient to the current token": [("j->dX[(th - H) * P + p] += be * gbp;",
                                                  "dx[p] += be * gbp;")],
    "output gradient misses the state": [("gS[n * P + p] += Cbar[n] * dy[p];",
                                          "gS[n * P + p] += 0.0 * Cbar[n] * dy[p];")],
}


def fd_pins_pass() -> bool:
    inp, dY, dhT = make_case(1)
    grads = oracle.oracle_bwd(**inp, dY=dY, dhT=dhT)
    rng = np.random.default_rng(101)
    for key in INPUTS:
        v = rng.standard_normal(inp[key].shape)
        fd = fd_directional(inp, dY, dhT, key, v)
        an = float((grads[GRADS[key]] * v).sum())
        if abs(fd - an) > 1e-6 * max(1.0, abs(fd)):
            return False
    return True


def test_unmodified_backward_passes_pins():
    assert fd_pins_pass()


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_backward_mistake_is_caught(name, tmp_path):
    src = oracle.source_text()
    for old, new in MUTATIONS[name]:
        assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
        src = src.replace(old, new)
    lib = oracle.compile_variant(src, str(tmp_path / "liboracle_mut.so"))
    with oracle.use_library(lib):
        assert not fd_pins_pass(), f"planted mistake '{name}' passed every pin"
