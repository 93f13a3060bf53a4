"""Pins of the fp64 oracle to things other than itself (CPU only).

Each check is an independent statement of what the scan must produce:
  * hand-worked examples (tests/golden/*.json, derivations inside);
  * a brute-force quadratic (matrix) form on L <= 16, built from explicit
    products of alpha, gamma and beta and complex-number rotations
    ("TorchMamba" README: trap_rope_matrix, size-guarded at L <= 16);
  * the two-SSD identity ("VikramLex/mamba3-minimal", "Two-SSD Decomposition");
  * the lambda = 1, theta = 0 reduction to the scalar-decay SSD recurrence and
    to its quadratic dual ("TorchMamba" README: reductions M2 -> SISO, and
    "Math notes" M2: Y = (L o C B^T) X);
  * forward over L == L unrolled decode steps from the same cache
    ("Crate burn_mamba", "Two execution modes");
  * closed forms for a single impulse under constant decay, with and without a
    constant rotation;
  * invariances (angle0 shift, theta + 2 pi, linearity in X, norm of rotation).
"""
import glob
import json
import math
import os

import numpy as np
import pytest

import oracle
from selective_state_space_m3ssd_b200.synth import WORKLOADS, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RTOL64, ATOL64 = 1e-10, 1e-12  # fp64 tolerances ("TorchMamba" README, "Verification")


def rand_problem(rng, b=2, L=9, H=4, P=3, N=6, G=2, with_cache=True, with_h0=True):
    """Small random problem with every optional input present."""
    p = {
        "X": rng.standard_normal((b, L, H, P)),
        "logdecay": -rng.uniform(0.05, 1.5, (b, L, H)),
        "beta": rng.uniform(0.0, 0.8, (b, L, H)),
        "gamma": rng.uniform(0.1, 1.0, (b, L, H)),
        "B": rng.standard_normal((b, L, G, N)) / math.sqrt(N),
        "C": rng.standard_normal((b, L, G, N)) / math.sqrt(N),
        "theta": rng.standard_normal((b, L, H, N // 2)),
        "D": rng.standard_normal(H),
    }
    if with_h0:
        p["h0"] = rng.standard_normal((b, H, N, P)) * 0.3
    if with_cache:
        p["angle0"] = rng.uniform(-3, 3, (b, H, N // 2))
        p["xprev0"] = rng.standard_normal((b, H, P))
        p["bprev0"] = rng.standard_normal((b, G, N)) / math.sqrt(N)
    return p


# ----------------------------------------------------------------------------
# Independent forms (written from the definitions, not from the oracle source)
# ----------------------------------------------------------------------------

def as_complex(v):
    """Adjacent pairs (2i, 2i+1) of the last axis as complex numbers."""
    return v[..., 0::2] + 1j * v[..., 1::2]


def as_real(z):
    out = np.empty(z.shape[:-1] + (2 * z.shape[-1],))
    out[..., 0::2] = z.real
    out[..., 1::2] = z.imag
    return out


def quadratic_form(p):
    """Dense (L x L) form of the scan; every coefficient is an explicit product."""
    X = p["X"]
    b, L, H, P = X.shape
    G, N = p["B"].shape[2], p["B"].shape[3]
    if L > 16:
        raise ValueError("quadratic form is size-guarded at L <= 16")
    beta = p.get("beta")
    beta = np.zeros((b, L, H)) if beta is None else beta
    theta = p.get("theta")
    theta = np.zeros((b, L, H, N // 2)) if theta is None else theta
    D = p.get("D")
    D = np.zeros(H) if D is None else D
    h0 = p.get("h0")
    h0 = np.zeros((b, H, N, P)) if h0 is None else h0
    angle0 = p.get("angle0")
    angle0 = np.zeros((b, H, N // 2)) if angle0 is None else angle0
    xprev0 = p.get("xprev0")
    xprev0 = np.zeros((b, H, P)) if xprev0 is None else xprev0
    bprev0 = p.get("bprev0")
    bprev0 = np.zeros((b, G, N)) if bprev0 is None else bprev0

    Y = np.zeros((b, L, H, P))
    hT = np.zeros((b, H, N, P))
    for bi in range(b):
        for h in range(H):
            g = h // (H // G)
            alpha = np.exp(p["logdecay"][bi, :, h])
            ga, be = p["gamma"][bi, :, h], beta[bi, :, h]

            def prod(lo, hi):  # alpha_lo * ... * alpha_hi, empty product = 1
                return float(np.prod(alpha[lo:hi + 1])) if hi >= lo else 1.0

            phi = angle0[bi, h] + np.cumsum(theta[bi, :, h], axis=0)       # (L, N/2)
            Bz = as_complex(p["B"][bi, :, g]) * np.exp(1j * phi)             # (L, N/2)
            Cz = as_complex(p["C"][bi, :, g]) * np.exp(1j * phi)
            Bm1 = as_complex(bprev0[bi, g]) * np.exp(1j * angle0[bi, h])   # (N/2,)
            Cr = as_real(Cz)
            # coefficient of Bbar_s x_s^T inside h_t
            W = np.zeros((L, L))
            for t in range(L):
                for s in range(t + 1):
                    W[t, s] = ga[s] * prod(s + 1, t)
                    if s + 1 <= t:
                        W[t, s] += be[s + 1] * prod(s + 2, t)
            gram = np.real(np.conj(Cz) @ Bz.T)                              # (L, L)
            gram_m1 = np.real(np.conj(Cz) @ Bm1)                            # (L,)
            x = X[bi, :, h]
            for t in range(L):
                y = (W[t, :t + 1] * gram[t, :t + 1]) @ x[:t + 1]
                y = y + be[0] * prod(1, t) * gram_m1[t] * xprev0[bi, h]
                y = y + prod(0, t) * (Cr[t] @ h0[bi, h])
                Y[bi, t, h] = y + D[h] * x[t]
            Br = as_real(Bz)
            hT[bi, h] = prod(0, L - 1) * h0[bi, h] + be[0] * prod(1, L - 1) * np.outer(
                as_real(Bm1), xprev0[bi, h])
            for s in range(L):
                hT[bi, h] += W[L - 1, s] * np.outer(Br[s], x[s])
    return Y, hT


def ssd_recurrent(X, logdecay, gamma, B, C):
    """Scalar-decay SSD recurrence h = a h + B (gamma x)^T, y = C^T h (G = 1)."""
    b, L, H, P = X.shape
    N = B.shape[-1]
    h = np.zeros((b, H, N, P))
    Y = np.zeros_like(X)
    for t in range(L):
        a = np.exp(logdecay[:, t])[:, :, None, None]
        u = gamma[:, t][:, :, None] * X[:, t]                      # (b,H,P)
        h = a * h + B[:, t, 0][:, None, :, None] * u[:, :, None, :]
        Y[:, t] = np.einsum("bn,bhnp->bhp", C[:, t, 0], h)
    return Y, h


def ssd_quadratic(X, logdecay, gamma, B, C):
    """Quadratic dual Y = (Lmask o C B^T)(gamma X) with Lmask[t,s] = exp(cs_t - cs_s)."""
    b, L, H, P = X.shape
    Y = np.zeros_like(X)
    for bi in range(b):
        CB = C[bi, :, 0] @ B[bi, :, 0].T
        for h in range(H):
            cs = np.cumsum(logdecay[bi, :, h])
            Lm = np.tril(np.exp(cs[:, None] - cs[None, :]))
            Y[bi, :, h] = (Lm * CB) @ (gamma[bi, :, h, None] * X[bi, :, h])
    return Y


def rel_err(a, ref):
    return float(np.max(np.abs(a - ref)) / max(np.sqrt(np.mean(ref ** 2)), 1e-300))


# ----------------------------------------------------------------------------
# Tests
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("path", sorted(glob.glob(os.path.join(GOLDEN, "worked_*.json"))))
def test_hand_worked_examples(path):
    with open(path) as f:
        g = json.load(f)
    inp = {k: np.array(v, dtype=np.float64) for k, v in g["inputs"].items()}
    out = oracle.oracle_fwd(**inp)
    for k, v in g["expected"].items():
        np.testing.assert_allclose(out[k], np.array(v), rtol=0, atol=g["atol"], err_msg=k)


@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("L", [1, 2, 7, 16])
def test_quadratic_form(seed, L):
    rng = np.random.default_rng(seed)
    p = rand_problem(rng, L=L)
    out = oracle.oracle_fwd(**p)
    Yq, hTq = quadratic_form(p)
    np.testing.assert_allclose(out["Y"], Yq, rtol=RTOL64, atol=ATOL64)
    np.testing.assert_allclose(out["hT"], hTq, rtol=RTOL64, atol=ATOL64)
    phi = p["angle0"] + p["theta"].sum(axis=1)
    np.testing.assert_allclose(out["angleT"], phi, rtol=RTOL64, atol=ATOL64)
    np.testing.assert_array_equal(out["xprevT"], p["X"][:, -1])
    np.testing.assert_array_equal(out["bprevT"], p["B"][:, -1])


def test_quadratic_form_without_optional_inputs():
    rng = np.random.default_rng(5)
    p = rand_problem(rng, L=12, with_cache=False, with_h0=False)
    p["beta"] = None
    p["theta"] = None
    p["D"] = None
    out = oracle.oracle_fwd(**p)
    Yq, hTq = quadratic_form(p)
    np.testing.assert_allclose(out["Y"], Yq, rtol=RTOL64, atol=ATOL64)
    np.testing.assert_allclose(out["hT"], hTq, rtol=RTOL64, atol=ATOL64)


def test_quadratic_form_on_tiny_workload_slice():
    w = WORKLOADS["tiny"].with_(seqlen=16)
    inp = make_inputs(w)
    p = {k: (None if v is None else v.double().numpy()) for k, v in inp.items()}
    out = oracle.oracle_fwd(**p)
    Yq, hTq = quadratic_form(p)
    np.testing.assert_allclose(out["Y"], Yq, rtol=RTOL64, atol=ATOL64)
    np.testing.assert_allclose(out["hT"], hTq, rtol=RTOL64, atol=ATOL64)


@pytest.mark.parametrize("seed", [3, 4])
def test_two_ssd_identity(seed):
    """Full scan == SSD(gamma x, B~, C~) + SSD(beta x_{t-1}, B~_{t-1}, C~) with the
    rotations applied outside the oracle and beta/theta absent in both calls."""
    rng = np.random.default_rng(seed)
    p = rand_problem(rng, b=2, L=23, H=4, P=3, N=6, G=2)
    full = oracle.oracle_fwd(**p)
    b, L, H, P = p["X"].shape
    G, N = p["B"].shape[2:]
    hg = np.arange(H) // (H // G)
    phi = p["angle0"][:, None] + np.cumsum(p["theta"], axis=1)              # (b,L,H,N/2)
    Bt = as_real(as_complex(p["B"][:, :, hg]) * np.exp(1j * phi))             # (b,L,H,N)
    Ct = as_real(as_complex(p["C"][:, :, hg]) * np.exp(1j * phi))
    Bm1 = as_real(as_complex(p["bprev0"][:, hg]) * np.exp(1j * p["angle0"]))  # (b,H,N)
    X_shift = np.concatenate([p["xprev0"][:, None], p["X"][:, :-1]], axis=1)
    B_shift = np.concatenate([Bm1[:, None], Bt[:, :-1]], axis=1)
    one = oracle.oracle_fwd(p["X"], p["logdecay"], None, p["gamma"], Bt, Ct, None, p["D"], p["h0"])
    two = oracle.oracle_fwd(X_shift, p["logdecay"], None, p["beta"], B_shift, Ct, None, None, None)
    np.testing.assert_allclose(full["Y"], one["Y"] + two["Y"], rtol=RTOL64, atol=ATOL64)
    np.testing.assert_allclose(full["hT"], one["hT"] + two["hT"], rtol=RTOL64, atol=ATOL64)


def test_ssd_reduction_recurrent_and_quadratic():
    """lambda = 1 (beta absent) and theta = 0: the scan is the scalar-decay SSD."""
    w = WORKLOADS["tiny"].with_(has_beta=False, has_theta=False, seqlen=40, nheads=3)
    inp = make_inputs(w)
    p = {k: (None if v is None else v.double().numpy()) for k, v in inp.items()}
    out = oracle.oracle_fwd(p["X"], p["logdecay"], None, p["gamma"], p["B"], p["C"])
    Yr, hr = ssd_recurrent(p["X"], p["logdecay"], p["gamma"], p["B"], p["C"])
    np.testing.assert_allclose(out["Y"], Yr, rtol=RTOL64, atol=ATOL64)
    np.testing.assert_allclose(out["hT"], hr, rtol=RTOL64, atol=ATOL64)
    Yq = ssd_quadratic(p["X"], p["logdecay"], p["gamma"], p["B"], p["C"])
    np.testing.assert_allclose(out["Y"], Yq, rtol=1e-9, atol=1e-12)
    # zero arrays take the same values as absent ones
    z = oracle.oracle_fwd(p["X"], p["logdecay"], np.zeros_like(p["gamma"]), p["gamma"], p["B"],
                          p["C"], np.zeros(p["X"].shape[:3] + (p["B"].shape[-1] // 2,)))
    np.testing.assert_array_equal(z["Y"], out["Y"])


@pytest.mark.parametrize("split", [0, 1, 5, 17])
def test_forward_equals_prefill_plus_steps(split):
    """Forward over L == forward over a prefix, then unrolled decode steps from
    the returned cache ("Crate burn_mamba", "Two execution modes"; "TorchMamba"
    README, parity tests with B=2, L=17, prefix=9)."""
    rng = np.random.default_rng(11)
    p = rand_problem(rng, b=2, L=17, H=4, P=3, N=6, G=2)
    full = oracle.oracle_fwd(**p)
    pre = {k: (v[:, :split] if k in ("X", "logdecay", "beta", "gamma", "B", "C", "theta") else v)
           for k, v in p.items()}
    pf = oracle.oracle_fwd(**pre)
    cache = {"angle": pf["angleT"].copy(), "ssm": pf["hT"].copy(),
             "x_prev": pf["xprevT"].copy(), "b_prev": pf["bprevT"].copy()}
    ys = [pf["Y"]]
    for t in range(split, 17):
        y = oracle.oracle_step(cache, p["X"][:, t], p["logdecay"][:, t], p["beta"][:, t],
                               p["gamma"][:, t], p["B"][:, t], p["C"][:, t], p["theta"][:, t],
                               p["D"])
        ys.append(y[:, None])
    Y = np.concatenate(ys, axis=1)
    np.testing.assert_allclose(Y, full["Y"], rtol=RTOL64, atol=ATOL64)
    np.testing.assert_allclose(cache["ssm"], full["hT"], rtol=RTOL64, atol=ATOL64)
    np.testing.assert_allclose(cache["angle"], full["angleT"], rtol=RTOL64, atol=ATOL64)
    np.testing.assert_array_equal(cache["x_prev"], full["xprevT"])
    np.testing.assert_array_equal(cache["b_prev"], full["bprevT"])


@pytest.mark.parametrize("with_theta", [False, True])
def test_impulse_closed_form(with_theta):
    """Constant alpha, beta, gamma; B_t = b for all t; x_0 = e_p, x_t = 0 after.
    h_0 = gamma R(w) b e_p^T and for t >= 1
        h_t = (gamma alpha^t + beta alpha^(t-1)) R(w) b e_p^T
    (the beta term first acts at t = 1 and carries Bbar_0 = R(phi_0) b).
    With a constant per-pair angle step w, phi_t = (t+1) w and
        y_t = (gamma alpha^t + beta alpha^(t-1)) * C^T R(-t w) b   (t >= 1),
    where (R(-x) b)_{2i} = cos x b_{2i} + sin x b_{2i+1},
          (R(-x) b)_{2i+1} = -sin x b_{2i} + cos x b_{2i+1}."""
    L, N, P, pidx = 12, 6, 3, 1
    alpha, beta, gamma = 0.7, 0.3, 0.9
    rng = np.random.default_rng(2)
    bvec = rng.standard_normal(N)
    cvec = rng.standard_normal(N)
    w = rng.uniform(-1, 1, N // 2) if with_theta else np.zeros(N // 2)
    X = np.zeros((1, L, 1, P))
    X[0, 0, 0, pidx] = 1.0
    p = {"X": X, "logdecay": np.full((1, L, 1), math.log(alpha)),
         "beta": np.full((1, L, 1), beta), "gamma": np.full((1, L, 1), gamma),
         "B": np.tile(bvec, (1, L, 1, 1)), "C": np.tile(cvec, (1, L, 1, 1)),
         "theta": np.tile(w, (1, L, 1, 1))}
    out = oracle.oracle_fwd(**p)
    y = out["Y"][0, :, 0]
    for t in range(L):
        coef = gamma * alpha ** t + (beta * alpha ** (t - 1) if t >= 1 else 0.0)
        x = t * w
        rb = np.empty(N)
        rb[0::2] = np.cos(x) * bvec[0::2] + np.sin(x) * bvec[1::2]
        rb[1::2] = -np.sin(x) * bvec[0::2] + np.cos(x) * bvec[1::2]
        expect = np.zeros(P)
        expect[pidx] = coef * float(cvec @ rb)
        np.testing.assert_allclose(y[t], expect, rtol=1e-12, atol=1e-14)
    # final state in closed form as well: coef * R(w) b e_p^T
    coef = gamma * alpha ** (L - 1) + beta * alpha ** (L - 2)
    rwb = np.empty(N)
    rwb[0::2] = np.cos(w) * bvec[0::2] - np.sin(w) * bvec[1::2]
    rwb[1::2] = np.sin(w) * bvec[0::2] + np.cos(w) * bvec[1::2]
    hT = np.zeros((N, P))
    hT[:, pidx] = coef * rwb
    np.testing.assert_allclose(out["hT"][0, 0], hT, rtol=1e-12, atol=1e-14)


def test_angle0_shift_invariance():
    """Only relative angles reach Y; a constant added to angle0 (h0 = 0) leaves
    Y unchanged and rotates hT by the same constant."""
    rng = np.random.default_rng(7)
    p = rand_problem(rng, L=13, with_h0=False)
    c = rng.uniform(-4, 4, p["angle0"].shape)
    a = oracle.oracle_fwd(**p)
    q = dict(p)
    q["angle0"] = p["angle0"] + c
    bq = oracle.oracle_fwd(**q)
    np.testing.assert_allclose(bq["Y"], a["Y"], rtol=1e-10, atol=1e-12)
    rot = as_real(as_complex(np.swapaxes(a["hT"], -1, -2)) * np.exp(1j * c)[:, :, None, :])
    np.testing.assert_allclose(bq["hT"], np.swapaxes(rot, -1, -2), rtol=1e-10, atol=1e-12)


def test_theta_two_pi_and_linearity():
    rng = np.random.default_rng(8)
    p = rand_problem(rng, L=11, with_h0=False, with_cache=False)
    a = oracle.oracle_fwd(**p)
    q = dict(p)
    q["theta"] = p["theta"].copy()
    q["theta"][:, 4] += 2 * math.pi
    np.testing.assert_allclose(oracle.oracle_fwd(**q)["Y"], a["Y"], rtol=1e-9, atol=1e-12)
    # linear in X with zero initial state and zero previous token
    X2 = rng.standard_normal(p["X"].shape)
    q = dict(p)
    q["X"] = 2.0 * p["X"] - 3.0 * X2
    r = dict(p)
    r["X"] = X2
    lin = 2.0 * a["Y"] - 3.0 * oracle.oracle_fwd(**r)["Y"]
    np.testing.assert_allclose(oracle.oracle_fwd(**q)["Y"], lin, rtol=1e-10, atol=1e-12)


def test_theta_changes_output():
    """Differ-guard: a silently dropped rotation must be visible."""
    w = WORKLOADS["tiny"]
    inp = make_inputs(w)
    a = oracle.oracle_fwd(**inp)
    q = dict(inp)
    q["theta"] = None
    b = oracle.oracle_fwd(**q)
    assert rel_err(b["Y"] - inp["D"].double().numpy()[None, None, :, None] * inp["X"].double().numpy(),
                   a["Y"] - inp["D"].double().numpy()[None, None, :, None] * inp["X"].double().numpy()) > 1e-2


def test_single_pair_rotation_is_local():
    """Only pair i rotating: components outside pair i of B and C never mix with it."""
    rng = np.random.default_rng(9)
    p = rand_problem(rng, b=1, L=6, H=1, P=2, N=6, G=1, with_cache=False, with_h0=False)
    p["theta"] = np.zeros_like(p["theta"])
    p["theta"][..., 1] = 0.9  # pair (2, 3) only
    out = oracle.oracle_fwd(**p)
    Yq, _ = quadratic_form(p)
    np.testing.assert_allclose(out["Y"], Yq, rtol=RTOL64, atol=ATOL64)
    # zeroing B, C on pair 1 gives the unrotated result
    q = dict(p)
    q["B"] = p["B"].copy()
    q["C"] = p["C"].copy()
    q["B"][..., 2:4] = 0
    q["C"][..., 2:4] = 0
    r = dict(q)
    r["theta"] = None
    np.testing.assert_allclose(oracle.oracle_fwd(**q)["Y"], oracle.oracle_fwd(**r)["Y"],
                               rtol=RTOL64, atol=ATOL64)


def test_empty_sequence_returns_initial_cache():
    rng = np.random.default_rng(10)
    p = rand_problem(rng, L=0)
    out = oracle.oracle_fwd(**p)
    assert out["Y"].shape[1] == 0
    np.testing.assert_array_equal(out["hT"], p["h0"])
    np.testing.assert_array_equal(out["angleT"], p["angle0"])
    np.testing.assert_array_equal(out["xprevT"], p["xprev0"])
    np.testing.assert_array_equal(out["bprevT"], p["bprev0"])


def test_thread_count_does_not_change_results():
    rng = np.random.default_rng(12)
    p = rand_problem(rng, b=3, L=20, H=4)
    a = oracle.oracle_fwd(**p, nthreads=1)
    b = oracle.oracle_fwd(**p, nthreads=5)
    np.testing.assert_array_equal(a["Y"], b["Y"])
    np.testing.assert_array_equal(a["hT"], b["hT"])
