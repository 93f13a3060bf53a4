"""fp64 oracle of the Mamba-3 SISO block around the scan -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module; the CUDA library never calls it.

The block, in the order the pages give it ("VikramLex/mamba3-minimal" README,
"Architecture", the Mamba3 SSM box; "TorchMamba" README, "API reference",
``Mamba3SisoBlock`` with its ``forward``/``prefill``/``step`` and the
``Mamba3SisoCache(angle, ssm, x_prev, b_prev)``):

  1. in_proj: one linear map of the block input u to (z, x, B, C, dt, lam, theta);
  2. B and C: QK-norm (an RMS norm over the state axis), then a learnable bias
     that is head-specific and channel-wise ("Learnable BC Bias" row of the
     mamba3-minimal innovations table), then the data-dependent rotation inside
     the scan;
  3. the trapezoidal scan (the SISO recurrence of ``oracle_fwd``), with D x;
  4. y * SiLU(z), then out_proj.

Readings where the pages are silent (each one stated in full below):
  - in_proj and out_proj are bias-free linear maps; the block's ``bias=True``
    is the BC bias, which replaces the removed short convolution ("TorchMamba"
    README, "Math notes", M3 SISO);
  - in_proj output columns are [z (H P) | x (H P) | B (G N) | C (G N) | dt (H) |
    lam (H) | theta (H N/2)], heads outermost inside each part;
  - Delta = softplus(dt + dt_bias); A = -exp(A_log); logdecay = Delta A;
    lambda = sigmoid(lam); gamma = lambda Delta; beta = (1 - lambda) Delta
    exp(logdecay) (the trapezoid weights of the workload recipe);
    theta_dt = Delta theta (the scan takes the angle increment already scaled);
  - the norm is x / sqrt(mean(x^2) + eps) times a learnable weight of length N,
    applied per group; the head bias is added after it, so each head gets its
    own B and C (the scan runs with G = H) and the cache's b_prev is per head.

Storage precision: the pages' numerics policy ("TorchMamba" README,
"Behavioral notes": bf16 computes in fp32 and each output is downcast to the
input dtype) makes the tensors a bf16 block hands from one step to the next
bf16.  ``store`` (default: none) is applied to exactly those hand-offs -- the
in_proj output (z, x, B, C, dt, lam, theta), the QK-normed group vectors of B
and C (the scan's bf16 inputs; the head bias is added after them), the scan
output y and the gated product (out_proj's input) -- so that a test can
compare against a device path that stores them in bf16; everything else stays
fp64.

Numerical pins: ``tests/test_oracle_block.py`` (closed forms for one and two
tokens, the scale invariance of the norm, forward == prefill + steps, and
planted mistakes).
"""
from __future__ import annotations

import numpy as np

from . import oracle_fwd, oracle_step


def in_proj_width(H: int, P: int, N: int, G: int) -> int:
    """Number of in_proj outputs: z, x, B, C, dt, lam, theta."""
    return 2 * H * P + 2 * G * N + 2 * H + H * (N // 2)


def _split(zx, H, P, N, G):
    """Columns of the in_proj output (..., width) into named parts."""
    o = 0
    parts = {}
    for name, size, shape in (("z", H * P, (H, P)), ("x", H * P, (H, P)), ("B", G * N, (G, N)),
                              ("C", G * N, (G, N)), ("dt", H, (H,)), ("lam", H, (H,)),
                              ("theta", H * (N // 2), (H, N // 2))):
        parts[name] = zx[..., o:o + size].reshape(zx.shape[:-1] + shape)
        o += size
    return parts


def softplus(v):
    return np.logaddexp(0.0, v)


def sigmoid(v):
    return 0.5 * (1.0 + np.tanh(0.5 * v))


def silu(v):
    return v * sigmoid(v)


def bc_norm(v, w, eps):
    """RMS norm over the last (state) axis, times the learnable weight."""
    return v / np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + eps) * w


def _keep(v):
    return v


def scan_inputs(u, wts, H, P, N, G, store=_keep):
    """Steps 1-2 of the block: the scan's inputs from the block input u (..., d_model)."""
    f = lambda k: np.asarray(wts[k], dtype=np.float64)
    zx = store(np.asarray(u, dtype=np.float64) @ f("W_in").T)
    s = _split(zx, H, P, N, G)
    delta = softplus(s["dt"] + f("dt_bias"))
    A = -np.exp(f("A_log"))
    logdecay = delta * A
    lam = sigmoid(s["lam"])
    gamma = lam * delta
    beta = (1.0 - lam) * delta * np.exp(logdecay)
    theta = delta[..., None] * s["theta"]
    eps = float(wts["eps"])
    grp = np.arange(H) // (H // G)
    Bh = store(bc_norm(s["B"], f("B_norm_w"), eps))[..., grp, :] + f("B_bias")
    Ch = store(bc_norm(s["C"], f("C_norm_w"), eps))[..., grp, :] + f("C_bias")
    return {"z": s["z"], "X": store(s["x"]), "logdecay": logdecay, "beta": beta, "gamma": gamma,
            "B": Bh, "C": Ch, "theta": theta}


def new_block_cache(b, H, P, N):
    """A zero block cache: angle (b,H,N/2), ssm (b,H,N,P), x_prev (b,H,P) and the
    per-head b_prev (b,H,N), all float64."""
    return {"angle": np.zeros((b, H, N // 2)), "ssm": np.zeros((b, H, N, P)),
            "x_prev": np.zeros((b, H, P)), "b_prev": np.zeros((b, H, N))}


def oracle_block_fwd(u, wts, H, P, N, G, cache=None, store=_keep):
    """Block forward over a sequence: u (b, L, d_model) -> out (b, L, d_model).

    ``cache`` (optional, a dict as from :func:`new_block_cache`) is the state
    the sequence continues from; ``store`` rounds the bf16 hand-offs (see the
    module notes).  Returns (out, cache after the last token)."""
    u = np.asarray(u, dtype=np.float64)
    b = u.shape[0]
    si = scan_inputs(u, wts, H, P, N, G, store)
    c = cache if cache is not None else new_block_cache(b, H, P, N)
    r = oracle_fwd(si["X"], si["logdecay"], si["beta"], si["gamma"], si["B"], si["C"],
                   si["theta"], np.asarray(wts["D"], dtype=np.float64), c["ssm"],
                   angle0=c["angle"], xprev0=c["x_prev"], bprev0=c["b_prev"])
    gated = store(store(r["Y"]) * silu(si["z"]))
    out = gated.reshape(gated.shape[:2] + (H * P,)) @ np.asarray(wts["W_out"], dtype=np.float64).T
    return out, {"angle": r["angleT"], "ssm": r["hT"], "x_prev": r["xprevT"],
                 "b_prev": r["bprevT"]}


def oracle_block_step(u_t, wts, H, P, N, G, cache, store=_keep):
    """One decode step of the block: u_t (b, d_model) -> out_t (b, d_model);
    ``cache`` (float64 arrays) is updated in place."""
    u_t = np.asarray(u_t, dtype=np.float64)
    si = scan_inputs(u_t, wts, H, P, N, G, store)
    y = oracle_step(cache, si["X"], si["logdecay"], si["beta"], si["gamma"], si["B"], si["C"],
                    si["theta"], np.asarray(wts["D"], dtype=np.float64))
    gated = store(store(y) * silu(si["z"]))
    return gated.reshape(gated.shape[:1] + (H * P,)) @ np.asarray(wts["W_out"],
                                                                  dtype=np.float64).T
