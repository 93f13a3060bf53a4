"""Seeded synthetic inputs for the Mamba-3 SISO scan (no scan arithmetic here).

The recipe is the one the workloads are specified with: per (b, t, h) a step
size Delta = softplus(N(-2, 1)), per head A_h ~ U(1, 16), logdecay = -Delta*A_h,
lambda = sigmoid(N(0, 1)), gamma = lambda*Delta, beta = (1 - lambda)*Delta*exp(logdecay)
(the exponential-trapezoidal coefficients), theta = Delta*omega with
omega ~ N(0, 1) per (b, t, h, pair), B, C ~ N(0, 1/N) per (b, t, g, n),
X ~ N(0, 1), D ~ N(0, 1) per head, and optionally h0 ~ N(0, var).

The draw order is fixed (X, Delta-noise, A, lambda-noise, B, C, omega, D, h0),
so a seed names one input set.  bf16 tensors are rounded once, here, and both
the CUDA library and the oracle consume the rounded values.

This module is shared by the tests, the benchmark and the smoke check; it
computes only the inputs, never a step of the scan.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    dtype: str            # "f32" or "bf16": dtype of X, B, C and Y
    has_beta: bool        # False: lambda = 1, the exact two-term path (beta absent)
    has_theta: bool       # False: real-only path (theta absent)
    h0_var: float | None  # None: h0 absent (zero)
    seed: int

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen


# The five synthetic workloads of the scan.  Sizes follow the model shapes they
# stand for (d_model 768 / 1024 / 1536 with expand 2 and head dim 64).
WORKLOADS = {
    "tiny": Workload("tiny siso trap+rope b1 L64 H2 P8 N8 fp32", 1, 64, 2, 8, 8, 1,
                     "f32", True, True, None, 1000),
    "ssd": Workload("mamba-2 ssd reduction b8 L4096 H24 P64 N128 bf16", 8, 4096, 24, 64, 128, 1,
                    "bf16", False, False, None, 1001),
    "siso": Workload("full siso trap+rope fwd b8 L4096 H32 P64 N128 bf16", 8, 4096, 32, 64, 128, 1,
                     "bf16", True, True, 0.1, 1002),
    "long": Workload("long-sequence siso fwd b2 L32768 H48 P64 N128 bf16", 2, 32768, 48, 64, 128, 1,
                     "bf16", True, True, None, 1003),
    "decode": Workload("batched decode b256 H32 P64 N128 fp32, 512-token prefill + 1000 steps",
                       256, 512 + 1000, 32, 64, 128, 1, "f32", True, True, None, 1004),
}
DECODE_PREFILL = 512
DECODE_STEPS = 1000


def rank_workload(w: Workload, rank: int) -> Workload:
    """The workload rank ``rank`` of a weak-scaling run processes: the same
    shapes with its own seed (independent batches, no exchange between ranks)."""
    return w.with_(seed=w.seed + 7919 * rank)


def torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def make_inputs(w: Workload, device: str | torch.device = "cpu") -> dict:
    """Draw one input set for workload ``w`` on ``device`` (seeded by ``w.seed``).

    Returns a dict of tensors: X (b,L,H,P), logdecay/gamma (b,L,H) fp32,
    beta (b,L,H) fp32 or None, B/C (b,L,G,N), theta (b,L,H,N/2) fp32 or None,
    D (H) fp32, h0 (b,H,N,P) fp32 or None.  X/B/C have dtype ``w.dtype``.
    """
    b, L, H, P, N, G = w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups
    if N % 2 or H % G:
        raise ValueError("N must be even and H divisible by G")
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed)
    f32 = dict(dtype=torch.float32, device=dev, generator=gen)

    X = torch.randn(b, L, H, P, **f32)
    dt_noise = torch.randn(b, L, H, **f32)
    A = torch.rand(H, **f32) * 15.0 + 1.0
    lam_noise = torch.randn(b, L, H, **f32)
    B = torch.randn(b, L, G, N, **f32) * (1.0 / math.sqrt(N))
    C = torch.randn(b, L, G, N, **f32) * (1.0 / math.sqrt(N))
    omega = torch.randn(b, L, H, N // 2, **f32)
    D = torch.randn(H, **f32)
    h0 = None
    if w.h0_var is not None:
        h0 = torch.randn(b, H, N, P, **f32) * math.sqrt(w.h0_var)

    delta = torch.nn.functional.softplus(dt_noise - 2.0)
    del dt_noise
    logdecay = -delta * A.view(1, 1, H)
    if w.has_beta:
        lam = torch.sigmoid(lam_noise)
        gamma = lam * delta
        beta = (1.0 - lam) * delta * torch.exp(logdecay)
        del lam
    else:
        gamma = delta.clone()
        beta = None
    del lam_noise
    theta = None
    if w.has_theta:
        theta = omega.mul_(delta.unsqueeze(-1))
    del omega, delta

    xd = torch_dtype(w.dtype)
    return {"X": X.to(xd), "logdecay": logdecay, "beta": beta, "gamma": gamma,
            "B": B.to(xd), "C": C.to(xd), "theta": theta, "D": D, "h0": h0}


# The rank-4 MIMO prefill at the siso workload's shape.
MIMO_WORKLOADS = {
    "mimo": (Workload("mimo rank-4 trap+rope fwd b8 L4096 H32 P64 N128 R4 bf16", 8, 4096, 32, 64, 128,
                      1, "bf16", True, True, 0.1, 1005), 4),
}


def make_mimo_inputs(w: Workload, rank: int, device: str | torch.device = "cpu") -> dict:
    """One MIMO input set: the scalar inputs (logdecay, beta, gamma, theta, D, h0)
    drawn as for the SISO workload ``w``, then X (b,L,H,P,R) ~ N(0, 1) and B, C
    (b,L,G,N,R) ~ N(0, 1/N) per rank column from a second stream (seed + 1)."""
    scal = make_inputs(w.with_(headdim=1), device)  # its X, B, C and h0 are discarded
    b, L, H, P, N, G, R = w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups, rank
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed + 1)
    f32 = dict(dtype=torch.float32, device=dev, generator=gen)
    xd = torch_dtype(w.dtype)
    X = torch.randn(b, L, H, P, R, **f32).to(xd)
    B = (torch.randn(b, L, G, N, R, **f32) * (1.0 / math.sqrt(N))).to(xd)
    C = (torch.randn(b, L, G, N, R, **f32) * (1.0 / math.sqrt(N))).to(xd)
    h0 = None
    if w.h0_var is not None:
        h0 = torch.randn(b, H, N, P, **f32) * math.sqrt(w.h0_var)
    return {"X": X, "logdecay": scal["logdecay"], "beta": scal["beta"], "gamma": scal["gamma"],
            "B": B, "C": C, "theta": scal["theta"], "D": scal["D"], "h0": h0}


def slice_inputs(inp: dict, b: slice | int, t: slice | int | None = None, heads=None,
                 ngroups: int = 1) -> dict:
    """Cut a sub-problem out of an input set: batch rows ``b``, time ``t`` and
    a subset of heads (with their groups).  Used to run the oracle on sampled
    sequences of a large workload; it only indexes, it computes nothing."""
    def bs(x):
        return x[b:b + 1] if isinstance(b, int) else x[b]

    def ts(x):
        if t is None:
            return x
        return x[:, t:t + 1] if isinstance(t, int) else x[:, t]

    out = {}
    H = inp["X"].shape[2]
    hs = list(range(H)) if heads is None else list(heads)
    gs = sorted({h // (H // ngroups) for h in hs})
    for k, v in inp.items():
        if v is None:
            out[k] = None
        elif k in ("X", "logdecay", "beta", "gamma", "theta"):
            out[k] = ts(bs(v))[:, :, hs]
        elif k in ("B", "C"):
            out[k] = ts(bs(v))[:, :, gs]
        elif k == "D":
            out[k] = v[hs]
        elif k == "h0":
            out[k] = bs(v)[:, hs]
        else:
            out[k] = v
    return out


# ---- the Mamba-3 SISO block around the scan -----------------------------------

@dataclass(frozen=True)
class BlockShape:
    name: str
    batch: int
    seqlen: int
    d_model: int
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    seed: int

    def with_(self, **kw) -> "BlockShape":
        return replace(self, **kw)

    @property
    def in_proj_width(self) -> int:
        H, P, N, G = self.nheads, self.headdim, self.dstate, self.ngroups
        return 2 * H * P + 2 * G * N + 2 * H + H * (N // 2)


# The block at the model size of the full siso workload: d_model 1024, expand 2
# (32 heads of 64), N = 128, one B/C group.
BLOCKS = {
    "small": BlockShape("siso block b2 L70 d_model 32 H4 P8 N8 G2", 2, 70, 32, 4, 8, 8, 2, 2000),
    "model": BlockShape("siso block b8 L4096 d_model 1024 H32 P64 N128 G1", 8, 4096, 1024, 32, 64,
                        128, 1, 2001),
}


def make_block(s: BlockShape, device: str | torch.device = "cpu") -> tuple[torch.Tensor, dict]:
    """Random-init weights of the block and one input sequence, seeded by ``s.seed``.

    u (b, L, d_model) ~ N(0, 1); W_in (width, d_model) ~ N(0, 1/d_model) and
    W_out (d_model, H P) ~ N(0, 1/(H P)), all three rounded to bf16 once;
    dt_bias ~ U(-4, -2), A_log = log U(1, 16), D ~ N(0, 1) per head; the norm
    weights (N) and the head-specific B/C biases (H, N) ~ U(0.5, 1.5) (the pages
    initialise the biases to ones; random values exercise them); eps = 1e-6.
    """
    g = torch.Generator().manual_seed(s.seed)
    b, L, dm, H, P, N = s.batch, s.seqlen, s.d_model, s.nheads, s.headdim, s.dstate
    bf = torch.bfloat16
    u = torch.randn(b, L, dm, generator=g).to(bf)
    W_in = (torch.randn(s.in_proj_width, dm, generator=g) / math.sqrt(dm)).to(bf)
    W_out = (torch.randn(dm, H * P, generator=g) / math.sqrt(H * P)).to(bf)
    wts = {
        "W_in": W_in,
        "W_out": W_out,
        "dt_bias": torch.rand(H, generator=g) * 2.0 - 4.0,
        "A_log": torch.log(torch.rand(H, generator=g) * 15.0 + 1.0),
        "D": torch.randn(H, generator=g),
        "B_norm_w": torch.rand(N, generator=g) + 0.5,
        "C_norm_w": torch.rand(N, generator=g) + 0.5,
        "B_bias": torch.rand(H, N, generator=g) + 0.5,
        "C_bias": torch.rand(H, N, generator=g) + 0.5,
        "eps": 1e-6,
    }
    if str(device) != "cpu":
        u = u.to(device)
        wts = {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in wts.items()}
    return u, wts
