"""Pins for the oracle of the Mamba-3 SISO block (CPU only).

Each pin is computed here from the block's definition in a form the oracle
does not use, so that a plausible mistake in the oracle fails at least one:

  - one token from an empty cache: the beta term and the rotation drop out
    (both B and C of the token turn by the same angle, and a rotation keeps
    dot products), so y = (gamma (C'.B') + D) x in closed form;
  - two tokens whose second x is zero (u_2 in the null space of the x rows of
    in_proj): y_2 = (alpha_2 gamma_1 + beta_2) (C'_2 . R(-theta_2) B'_1) x_1,
    pairwise, with theta_2 = Delta_2 theta_raw_2 -- this pins A_log, the beta
    weight, the step scaling of the angle and the rotation sense;
  - the QK-norm makes the block blind to a positive rescaling of the B (or C)
    rows of in_proj (with eps = 0);
  - a forward over L tokens equals a forward over the first tokens followed by
    decode steps on the block cache ("TorchMamba" README, "API reference":
    forward, prefill and step of every block);
  - planted mistakes in a copy of the oracle module each break one pin.
"""
import types

import numpy as np
import pytest

from oracle import block as ob
from selective_state_space_m3ssd_b200.synth import BLOCKS, make_block


def _np(wts):
    return {k: (v.double().numpy() if hasattr(v, "double") else v) for k, v in wts.items()}


def setup(seed, **kw):
    s = BLOCKS["small"].with_(seed=seed, **kw)
    u, w = make_block(s)
    return s, u.double().numpy(), _np(w)


def _sp(v):
    return np.log1p(np.exp(-abs(v))) + max(v, 0.0)


def _sig(v):
    return 1.0 / (1.0 + np.exp(-v))


def _parts(s, w, uvec):
    """The in_proj outputs of one token, by head (independent index arithmetic)."""
    H, P, N, G = s.nheads, s.headdim, s.dstate, s.ngroups
    v = w["W_in"] @ uvec
    base_B, base_C = 2 * H * P, 2 * H * P + G * N
    base_dt = 2 * H * P + 2 * G * N
    out = []
    for h in range(H):
        g = h // (H // G)
        Braw = v[base_B + g * N: base_B + (g + 1) * N]
        Craw = v[base_C + g * N: base_C + (g + 1) * N]
        rB = np.sqrt(np.sum(Braw ** 2) / N + w["eps"])
        rC = np.sqrt(np.sum(Craw ** 2) / N + w["eps"])
        delta = _sp(v[base_dt + h] + w["dt_bias"][h])
        lam = _sig(v[base_dt + H + h])
        th0 = base_dt + 2 * H + h * (N // 2)
        out.append({
            "z": v[h * P:(h + 1) * P], "x": v[H * P + h * P: H * P + (h + 1) * P],
            "B": Braw / rB * w["B_norm_w"] + w["B_bias"][h],
            "C": Craw / rC * w["C_norm_w"] + w["C_bias"][h],
            "delta": delta, "lam": lam, "theta_raw": v[th0: th0 + N // 2],
        })
    return out


def pin_one_token(mod, seed=1):
    s, u, w = setup(seed, seqlen=1)
    out, _ = mod.oracle_block_fwd(u, w, s.nheads, s.headdim, s.dstate, s.ngroups)
    for bb in range(s.batch):
        gated = []
        for h, p in enumerate(_parts(s, w, u[bb, 0])):
            y = (p["lam"] * p["delta"] * np.dot(p["C"], p["B"]) + w["D"][h]) * p["x"]
            gated.append(y * p["z"] * _sig(p["z"]))
        want = w["W_out"] @ np.concatenate(gated)
        np.testing.assert_allclose(out[bb, 0], want, rtol=1e-10, atol=1e-10 * np.abs(want).max())


def pin_two_tokens(mod, seed=2):
    # d_model above H P, so that the x rows of in_proj have a null space
    s, u, w = setup(seed, seqlen=2, d_model=48)
    H, P, N, G = s.nheads, s.headdim, s.dstate, s.ngroups
    assert s.d_model > H * P
    Wx = w["W_in"][H * P: 2 * H * P]
    # second token in the null space of the x rows: x_2 = 0
    proj = np.eye(s.d_model) - Wx.T @ np.linalg.solve(Wx @ Wx.T, Wx)
    u = u.copy()
    for bb in range(s.batch):
        u[bb, 1] = proj @ u[bb, 1]
    out, _ = mod.oracle_block_fwd(u, w, H, P, N, G)
    for bb in range(s.batch):
        p1s, p2s = _parts(s, w, u[bb, 0]), _parts(s, w, u[bb, 1])
        gated = []
        for h in range(H):
            p1, p2 = p1s[h], p2s[h]
            assert np.abs(p2["x"]).max() < 1e-12
            a2 = np.exp(-np.exp(w["A_log"][h]) * p2["delta"])
            g1 = p1["lam"] * p1["delta"]
            b2 = (1.0 - p2["lam"]) * p2["delta"] * a2
            ang = p2["delta"] * p2["theta_raw"]  # phi_2 - phi_1
            dot = 0.0
            for i in range(N // 2):
                c, sn = np.cos(ang[i]), np.sin(ang[i])
                b0, b1 = p1["B"][2 * i], p1["B"][2 * i + 1]
                rb0, rb1 = c * b0 + sn * b1, -sn * b0 + c * b1   # R(-ang) B'_1
                dot += p2["C"][2 * i] * rb0 + p2["C"][2 * i + 1] * rb1
            y2 = (a2 * g1 + b2) * dot * p1["x"]
            gated.append(y2 * p2["z"] * _sig(p2["z"]))
        want = w["W_out"] @ np.concatenate(gated)
        assert np.abs(want).max() > 1e-3
        np.testing.assert_allclose(out[bb, 1], want, rtol=1e-9, atol=1e-9 * np.abs(want).max())


def pin_norm_scale_invariance(mod, seed=3):
    s, u, w = setup(seed, seqlen=9)
    H, P, N, G = s.nheads, s.headdim, s.dstate, s.ngroups
    w = dict(w, eps=0.0)
    ref, _ = mod.oracle_block_fwd(u, w, H, P, N, G)
    for lo in (2 * H * P, 2 * H * P + G * N):   # the B rows, then the C rows
        w2 = dict(w, W_in=w["W_in"].copy())
        w2["W_in"][lo: lo + G * N] *= 3.7
        got, _ = mod.oracle_block_fwd(u, w2, H, P, N, G)
        np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-11 * np.abs(ref).max())


def pin_forward_equals_prefill_then_steps(mod, seed=4):
    s, u, w = setup(seed, seqlen=12)
    H, P, N, G = s.nheads, s.headdim, s.dstate, s.ngroups
    full, fc = mod.oracle_block_fwd(u, w, H, P, N, G)
    _, cache = mod.oracle_block_fwd(u[:, :7], w, H, P, N, G)
    for t in range(7, 12):
        o = mod.oracle_block_step(u[:, t], w, H, P, N, G, cache)
        np.testing.assert_allclose(o, full[:, t], rtol=1e-11, atol=1e-11 * np.abs(full).max())
    for k in ("ssm", "x_prev", "b_prev"):
        np.testing.assert_allclose(cache[k], fc[k], rtol=1e-11, atol=1e-12)


PINS = [pin_one_token, pin_two_tokens, pin_norm_scale_invariance,
        pin_forward_equals_prefill_then_steps]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_block_oracle_pin(pin):
    pin(ob)


def test_block_cache_continues_a_sequence():
    # a forward from a cache equals the tail of the forward over the whole sequence
    s, u, w = setup(5, seqlen=10)
    H, P, N, G = s.nheads, s.headdim, s.dstate, s.ngroups
    full, _ = ob.oracle_block_fwd(u, w, H, P, N, G)
    _, c = ob.oracle_block_fwd(u[:, :4], w, H, P, N, G)
    tail, _ = ob.oracle_block_fwd(u[:, 4:], w, H, P, N, G, cache=c)
    np.testing.assert_allclose(tail, full[:, 4:], rtol=1e-11, atol=1e-11 * np.abs(full).max())


MUTATIONS = {
    "gate by sigmoid instead of SiLU": ("return v * sigmoid(v)", "return sigmoid(v)"),
    "head bias before the norm": (
        'Bh = store(bc_norm(s["B"], f("B_norm_w"), eps))[..., grp, :] + f("B_bias")',
        'Bh = store(bc_norm(s["B"][..., grp, :] + f("B_bias"), f("B_norm_w"), eps))'),
    "norm dropped on C": (
        'Ch = store(bc_norm(s["C"], f("C_norm_w"), eps))[..., grp, :] + f("C_bias")',
        'Ch = store(s["C"] * f("C_norm_w"))[..., grp, :] + f("C_bias")'),
    "dt bias dropped": ('delta = softplus(s["dt"] + f("dt_bias"))', 'delta = softplus(s["dt"])'),
    "angle not scaled by the step": ('theta = delta[..., None] * s["theta"]',
                                     'theta = s["theta"]'),
    "beta without the decay": ("beta = (1.0 - lam) * delta * np.exp(logdecay)",
                               "beta = (1.0 - lam) * delta"),
    "A_log used as A": ('A = -np.exp(f("A_log"))', 'A = -f("A_log")'),
    "x and z swapped": ('("z", H * P, (H, P)), ("x", H * P, (H, P))',
                        '("x", H * P, (H, P)), ("z", H * P, (H, P))'),
}


def _mutant(old, new):
    src = open(ob.__file__).read()
    assert src.count(old) == 1, old
    mod = types.ModuleType("oracle._block_mutant")
    mod.__package__ = "oracle"
    mod.__file__ = ob.__file__
    exec(compile(src.replace(old, new), ob.__file__, "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_block_mistake_is_caught(name):
    mod = _mutant(*MUTATIONS[name])
    caught = 0
    for pin in PINS:
        try:
            pin(mod)
        except AssertionError:
            caught += 1
    assert caught >= 1, name
