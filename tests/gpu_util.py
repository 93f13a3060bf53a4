"""Helpers for the GPU parity tests: move seeded inputs to the device, call
the library through its binding and measure the error against the oracle."""
import numpy as np
import torch

import selective_state_space_m3ssd_b200 as m3


def rel_max_err(got, ref) -> float:
    """max |got - ref| / RMS(ref): the parity metric of the scan."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    return float(np.max(np.abs(got - ref))) / max(rms, 1e-30)


def bf16_half_ulp(x):
    """Half the spacing of bf16 numbers at |x| (8 significant bits)."""
    a = np.maximum(np.abs(np.asarray(x, dtype=np.float64)), 2.0 ** -126)
    return np.ldexp(1.0, (np.floor(np.log2(a)) - 8).astype(np.int64))


def rel_max_err_out(got, ref, out_bf16: bool) -> float:
    """Parity metric for an output rounded to its storage dtype: the error
    beyond the final rounding (half a bf16 ulp of the larger of the two values,
    which any result returned in bf16 carries), max over elements, over
    RMS(ref).  For fp32 outputs this is rel_max_err."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    if out_bf16:
        err = np.maximum(err - bf16_half_ulp(np.maximum(np.abs(got), np.abs(ref))), 0.0)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    return float(np.max(err)) / max(rms, 1e-30)


def rel_close_err(got, ref, rtol: float, out_bf16: bool) -> float:
    """max over elements of (|got - ref| - rtol |ref|), beyond the final bf16
    rounding as in rel_max_err_out, over RMS(ref): an allclose-style metric
    (absolute bar in units of the RMS, relative slack per element) for
    heavy-tailed outputs."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref) - rtol * np.abs(ref)
    if out_bf16:
        err = err - bf16_half_ulp(np.maximum(np.abs(got), np.abs(ref)))
    rms = float(np.sqrt(np.mean(ref ** 2)))
    return float(max(np.max(err), 0.0)) / max(rms, 1e-30)


def rms_rel_err(got, ref) -> float:
    """RMS(got - ref) / RMS(ref)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.sqrt(np.mean((got - ref) ** 2) / max(np.mean(ref ** 2), 1e-300)))


def angle_err(got, ref) -> float:
    """Max |got - ref| of angles modulo 2 pi (the library stores them reduced)."""
    d = np.asarray(got, dtype=np.float64) - np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs((d + np.pi) % (2 * np.pi) - np.pi)))


def to_dev(inp: dict, device="cuda") -> dict:
    return {k: (None if v is None else v.to(device).contiguous()) for k, v in inp.items()}


def np64(t):
    return None if t is None else t.detach().to("cpu").double().numpy()


def gpu_fwd(inp: dict, **kw):
    d = to_dev(inp)
    extra = {k: d.pop(k) for k in ("angle0", "xprev0", "bprev0") if k in d}
    Y, hT, cache = m3.fwd(d["X"], d["logdecay"], d["beta"], d["gamma"], d["B"], d["C"],
                          d["theta"], d["D"], d["h0"], **extra, **kw)
    torch.cuda.synchronize()
    out = {"Y": np64(Y), "hT": np64(hT)}
    if cache is not None:
        out.update({"angleT": np64(cache["angle"]), "xprevT": np64(cache["x_prev"]),
                    "bprevT": np64(cache["b_prev"])})
    return out
