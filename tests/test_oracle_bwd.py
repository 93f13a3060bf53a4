"""Pins for the oracle's backward (CPU only).

The backward is checked against the forward oracle, which is separately written
code: for L = <dY, Y> + <dhT, hT>, central finite differences of the forward
along random directions must equal <grad, direction> for every input, and
single entries are checked the same way.  fp64 central differences with a step
of 1e-5 carry an error of order step^2 times third derivatives, about 1e-9
relative here, so a 1e-6 relative tolerance catches any dropped term, wrong
sign or transposed index while leaving room for rounding.
"""
import numpy as np
import pytest

import oracle

INPUTS = ("X", "logdecay", "beta", "gamma", "B", "C", "theta", "D", "h0",
          "angle0", "xprev0", "bprev0")
GRADS = {k: "d" + k for k in INPUTS}


def make_case(seed, b=2, L=9, H=4, G=2, P=3, N=4, beta=True, theta=True, cache=True):
    rng = np.random.default_rng(seed)
    inp = {
        "X": rng.standard_normal((b, L, H, P)),
        "logdecay": -np.abs(rng.standard_normal((b, L, H))) * 0.7,
        "beta": rng.uniform(0.05, 0.6, (b, L, H)) if beta else None,
        "gamma": rng.uniform(0.05, 0.9, (b, L, H)),
        "B": rng.standard_normal((b, L, G, N)),
        "C": rng.standard_normal((b, L, G, N)),
        "theta": rng.standard_normal((b, L, H, N // 2)) * 0.4 if theta else None,
        "D": rng.standard_normal(H),
        "h0": rng.standard_normal((b, H, N, P)) * 0.5,
        "angle0": rng.uniform(-3, 3, (b, H, N // 2)) if cache else None,
        "xprev0": rng.standard_normal((b, H, P)) if cache else None,
        "bprev0": rng.standard_normal((b, G, N)) if cache else None,
    }
    dY = rng.standard_normal((b, L, H, P))
    dhT = rng.standard_normal((b, H, N, P))
    return inp, dY, dhT


def objective(inp, dY, dhT):
    out = oracle.oracle_fwd(**inp)
    return float((out["Y"] * dY).sum() + (out["hT"] * dhT).sum())


def fd_directional(inp, dY, dhT, key, v, eps=1e-5):
    plus = dict(inp)
    minus = dict(inp)
    plus[key] = inp[key] + eps * v
    minus[key] = inp[key] - eps * v
    return (objective(plus, dY, dhT) - objective(minus, dY, dhT)) / (2 * eps)


@pytest.mark.parametrize("seed,flags", [(1, {}), (2, {"beta": False}), (3, {"theta": False}),
                                        (4, {"cache": False}), (5, {"G": 4, "H": 4}),
                                        (6, {"G": 1, "H": 3, "L": 13})])
def test_bwd_matches_finite_differences(seed, flags):
    inp, dY, dhT = make_case(seed, **flags)
    grads = oracle.oracle_bwd(**inp, dY=dY, dhT=dhT)
    rng = np.random.default_rng(100 + seed)
    for key in INPUTS:
        if inp[key] is None:
            continue
        for _ in range(2):
            v = rng.standard_normal(inp[key].shape)
            fd = fd_directional(inp, dY, dhT, key, v)
            an = float((grads[GRADS[key]] * v).sum())
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (key, fd, an)


def test_bwd_single_entries():
    inp, dY, dhT = make_case(11, L=6)
    grads = oracle.oracle_bwd(**inp, dY=dY, dhT=dhT)
    rng = np.random.default_rng(7)
    for key in INPUTS:
        for _ in range(3):
            idx = tuple(int(rng.integers(0, s)) for s in inp[key].shape)
            v = np.zeros_like(inp[key])
            v[idx] = 1.0
            fd = fd_directional(inp, dY, dhT, key, v)
            assert abs(fd - grads[GRADS[key]][idx]) <= 1e-6 * max(1.0, abs(fd)), (key, idx)


def test_bwd_absent_inputs_are_derivatives_at_zero():
    # an input passed as None behaves as zero: its gradient equals the gradient
    # of an explicit zero tensor
    inp, dY, dhT = make_case(21, beta=False, theta=False, cache=False)
    g_none = oracle.oracle_bwd(**inp, dY=dY, dhT=dhT)
    b, L, H, P = inp["X"].shape
    G, N = inp["B"].shape[2], inp["B"].shape[3]
    zeros = dict(inp, beta=np.zeros((b, L, H)), theta=np.zeros((b, L, H, N // 2)),
                 angle0=np.zeros((b, H, N // 2)), xprev0=np.zeros((b, H, P)),
                 bprev0=np.zeros((b, G, N)))
    g_zero = oracle.oracle_bwd(**zeros, dY=dY, dhT=dhT)
    for k in g_none:
        np.testing.assert_allclose(g_none[k], g_zero[k], rtol=0, atol=0)


def test_bwd_is_linear_in_the_upstream_gradients():
    inp, dY, dhT = make_case(31)
    g1 = oracle.oracle_bwd(**inp, dY=dY, dhT=None)
    g2 = oracle.oracle_bwd(**inp, dY=np.zeros_like(dY), dhT=dhT)
    g12 = oracle.oracle_bwd(**inp, dY=dY, dhT=dhT)
    for k in g12:
        np.testing.assert_allclose(g12[k], g1[k] + g2[k], rtol=1e-12, atol=1e-12)
    g0 = oracle.oracle_bwd(**inp, dY=np.zeros_like(dY), dhT=None)
    for k in g0:
        assert not np.any(g0[k])


def test_bwd_empty_sequence_passes_dhT_to_dh0():
    inp, dY, dhT = make_case(41, L=0)
    g = oracle.oracle_bwd(**inp, dY=dY, dhT=dhT)
    np.testing.assert_array_equal(g["dh0"], dhT)
    assert not np.any(g["dangle0"]) and not np.any(g["dbprev0"])


def test_bwd_does_not_depend_on_thread_count():
    inp, dY, dhT = make_case(51, b=3, H=4, G=2)
    g1 = oracle.oracle_bwd(**inp, dY=dY, dhT=dhT, nthreads=1)
    g4 = oracle.oracle_bwd(**inp, dY=dY, dhT=dhT, nthreads=4)
    for k in g1:
        np.testing.assert_array_equal(g1[k], g4[k])
