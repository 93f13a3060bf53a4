"""Pins for the oracle's MIMO rank-R scan (CPU only).

The MIMO code is checked against the SISO oracle, which is separately written:
  - at R = 1 it is the SISO recurrence ("TorchMamba" README, "Models": SISO ->
    MIMO at R = 1 is structural);
  - for any R it is a sum of R^2 SISO scans ("TorchMamba" README, "Math notes",
    MIMO: training is R^2 SISO calls).  The state is linear in its inputs, so
    h = sum_r h(x_r, B_r), and output column r' reads it through C_r'.  Hence
    Y[..., r'] = sum_r SISO(x_r, B_r, C_r').Y with D applied once (r = r') and
    h0 carried once (r = 0), and hT = sum_r SISO(x_r, B_r, C_0, h0 if r = 0).hT.
  - a forward over L tokens equals a forward over the first tokens followed by
    decode steps on its cache.
"""
import numpy as np
import pytest

import oracle


def make_mimo(seed, b=2, L=11, H=4, G=2, P=3, N=4, R=3, beta=True, theta=True, cache=True):
    rng = np.random.default_rng(seed)
    return {
        "X": rng.standard_normal((b, L, H, P, R)),
        "logdecay": -np.abs(rng.standard_normal((b, L, H))) * 0.6,
        "beta": rng.uniform(0.05, 0.5, (b, L, H)) if beta else None,
        "gamma": rng.uniform(0.05, 0.9, (b, L, H)),
        "B": rng.standard_normal((b, L, G, N, R)),
        "C": rng.standard_normal((b, L, G, N, R)),
        "theta": rng.standard_normal((b, L, H, N // 2)) * 0.4 if theta else None,
        "D": rng.standard_normal(H),
        "h0": rng.standard_normal((b, H, N, P)) * 0.5,
        "angle0": rng.uniform(-3, 3, (b, H, N // 2)) if cache else None,
        "xprev0": rng.standard_normal((b, H, P, R)) if cache else None,
        "bprev0": rng.standard_normal((b, G, N, R)) if cache else None,
    }


def siso_slice(inp, r_in, r_out, with_D, with_h0):
    s = {k: v for k, v in inp.items() if k not in ("X", "B", "C", "xprev0", "bprev0", "D", "h0")}
    s["X"] = inp["X"][..., r_in]
    s["B"] = inp["B"][..., r_in]
    s["C"] = inp["C"][..., r_out]
    s["xprev0"] = None if inp["xprev0"] is None else inp["xprev0"][..., r_in]
    s["bprev0"] = None if inp["bprev0"] is None else inp["bprev0"][..., r_in]
    s["D"] = inp["D"] if with_D else None
    s["h0"] = inp["h0"] if with_h0 else None
    return s


def test_rank_one_is_siso():
    inp = make_mimo(1, R=1)
    m = oracle.oracle_mimo_fwd(**inp)
    s = oracle.oracle_fwd(**siso_slice(inp, 0, 0, True, True))
    np.testing.assert_allclose(m["Y"][..., 0], s["Y"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(m["hT"], s["hT"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(m["angleT"], s["angleT"], rtol=0, atol=1e-15)


@pytest.mark.parametrize("seed,kw", [(2, {}), (3, {"R": 4, "G": 1}), (4, {"beta": False}),
                                     (5, {"theta": False, "cache": False}), (6, {"R": 2, "L": 1})])
def test_mimo_is_a_sum_of_rank_squared_siso_scans(seed, kw):
    inp = make_mimo(seed, **kw)
    R = inp["X"].shape[-1]
    m = oracle.oracle_mimo_fwd(**inp)
    Y = np.zeros_like(m["Y"])
    for ro in range(R):
        for ri in range(R):
            Y[..., ro] += oracle.oracle_fwd(**siso_slice(inp, ri, ro, ri == ro, ri == 0))["Y"]
    hT = sum(oracle.oracle_fwd(**siso_slice(inp, ri, 0, False, ri == 0))["hT"] for ri in range(R))
    scale = np.sqrt(np.mean(m["Y"] ** 2))
    np.testing.assert_allclose(m["Y"], Y, rtol=0, atol=1e-11 * scale)
    np.testing.assert_allclose(m["hT"], hT, rtol=0, atol=1e-11 * np.sqrt(np.mean(hT ** 2)))


def test_forward_equals_prefill_then_steps():
    inp = make_mimo(7, L=10)
    full = oracle.oracle_mimo_fwd(**inp)
    L1 = 6
    pre = {k: (v[:, :L1] if k in ("X", "logdecay", "beta", "gamma", "B", "C", "theta") and v is not None
               else v) for k, v in inp.items()}
    p = oracle.oracle_mimo_fwd(**pre)
    cache = {"angle": p["angleT"].copy(), "ssm": p["hT"].copy(), "x_prev": p["xprevT"].copy(),
             "b_prev": p["bprevT"].copy()}
    for t in range(L1, 10):
        y = oracle.oracle_mimo_step(cache, inp["X"][:, t], inp["logdecay"][:, t],
                                    inp["beta"][:, t], inp["gamma"][:, t], inp["B"][:, t],
                                    inp["C"][:, t], inp["theta"][:, t], inp["D"])
        np.testing.assert_allclose(y, full["Y"][:, t], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(cache["ssm"], full["hT"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(cache["x_prev"], full["xprevT"], rtol=0, atol=0)
    np.testing.assert_allclose(cache["b_prev"], full["bprevT"], rtol=0, atol=0)


MUTATIONS = {
    "rank columns rotated by the previous angle": [
        ("rotate_pairs_col(B, phi, N, R, Bbar);", "rotate_pairs_col(B, phi_prev, N, R, Bbar);")],
    "output reads the previous state": [
        ("y[p * R + r] = acc + dh * x[p * R + r];", "y[p * R + r] = dh * x[p * R + r];")],
    "rank sum over the wrong axis": [
        ("ug += Bbar[n * R + r] * x[p * R + r];", "ug += Bbar[n * R + r] * x[p * R + (R - 1 - r)];")],
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mimo_mistake_is_caught(name, tmp_path):
    src = oracle.source_text()
    for old, new in MUTATIONS[name]:
        assert src.count(old) == 1, old
        src = src.replace(old, new)
    lib = oracle.compile_variant(src, str(tmp_path / "liboracle_mut.so"))
    with oracle.use_library(lib):
        with pytest.raises(AssertionError):
            test_mimo_is_a_sum_of_rank_squared_siso_scans(2, {})
