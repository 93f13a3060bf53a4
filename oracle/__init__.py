"""fp64 CPU oracle of the Mamba-3 SISO selective scan -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it and
shares no code with it.

``oracle_fwd`` and ``oracle_step`` wrap the plain C loops in ``m3ssd_oracle.c``
(sequential in t, fp64, host libm sin/cos/exp).  Inputs may be numpy arrays or
CPU torch tensors of any float dtype; they are converted to float64 exactly
(a bf16 or fp32 value is representable in fp64), so the oracle sees the very
values the GPU sees.

Pins: the oracle is checked against independent forms in
``tests/test_oracle_pins.py`` (brute-force quadratic form, the two-SSD
identity, the scalar-decay SSD reduction, forward == unrolled steps, closed
forms, invariances and hand-worked examples in ``tests/golden/``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "m3ssd_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None
_lock = threading.Lock()


class _Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in
                ("batch", "seqlen", "nheads", "headdim", "dstate", "ngroups")]


class _MimoDims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in
                ("batch", "seqlen", "nheads", "headdim", "dstate", "ngroups", "rank")]


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` with gcc (plain -O2, IEEE semantics, no fast-math)."""
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
               "-ffp-contract=off", "-o", tmp, _SRC, "-lm", "-lpthread"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _bind(path: str):
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    lib.oracle_fwd.argtypes = [ctypes.POINTER(_Dims)] + [dp] * 17 + [ctypes.c_int]
    lib.oracle_fwd.restype = ctypes.c_int
    lib.oracle_step.argtypes = [ctypes.POINTER(_Dims)] + [dp] * 13
    lib.oracle_step.restype = ctypes.c_int
    lib.oracle_bwd.argtypes = [ctypes.POINTER(_Dims)] + [dp] * 26 + [ctypes.c_int]
    lib.oracle_bwd.restype = ctypes.c_int
    lib.oracle_mimo_fwd.argtypes = [ctypes.POINTER(_MimoDims)] + [dp] * 17 + [ctypes.c_int]
    lib.oracle_mimo_fwd.restype = ctypes.c_int
    lib.oracle_mimo_step.argtypes = [ctypes.POINTER(_MimoDims)] + [dp] * 13
    lib.oracle_mimo_step.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = _bind(_LIB_PATH)
    return _lib


def compile_variant(source_text: str, out_path: str) -> str:
    """Compile a modified copy of the oracle source (used only by the tests that
    plant a mistake in the oracle and check that a pin catches it)."""
    src = out_path + ".c"
    with open(src, "w") as f:
        f.write(source_text)
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
                    "-ffp-contract=off", "-o", out_path, src, "-lm", "-lpthread"], check=True)
    return out_path


class use_library:
    """Context manager: route oracle_fwd/oracle_step through another build of
    the oracle source (a planted-mistake variant) for the duration of a test."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        _load()
        self._saved = _lib
        _lib = _bind(self.path)
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self._saved
        return False


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def _f64(a):
    """Exact conversion of an input array to a C-contiguous float64 ndarray."""
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    if a is None:
        return ctypes.POINTER(ctypes.c_double)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def oracle_fwd(X, logdecay, beta, gamma, B, C, theta=None, D=None, h0=None,
               angle0=None, xprev0=None, bprev0=None, nthreads: int | None = None):
    """Sequential fp64 forward.

    Shapes: X (b,L,H,P); logdecay, beta, gamma (b,L,H); B, C (b,L,G,N);
    theta (b,L,H,N/2); D (H); h0 (b,H,N,P); angle0 (b,H,N/2); xprev0 (b,H,P);
    bprev0 (b,G,N).  ``beta``/``theta``/``D``/``h0``/the three cache inputs may
    be None (zero).  Returns a dict with Y, hT, angleT, xprevT, bprevT (float64).
    """
    X, logdecay, beta, gamma = _f64(X), _f64(logdecay), _f64(beta), _f64(gamma)
    B, C, theta, D, h0 = _f64(B), _f64(C), _f64(theta), _f64(D), _f64(h0)
    angle0, xprev0, bprev0 = _f64(angle0), _f64(xprev0), _f64(bprev0)
    b, L, H, P = X.shape
    G, N = B.shape[2], B.shape[3]
    if N % 2 or H % G:
        raise ValueError("oracle_fwd: N must be even and H divisible by G")
    if B.shape != (b, L, G, N) or C.shape != (b, L, G, N):
        raise ValueError("oracle_fwd: B/C shape")
    if logdecay.shape != (b, L, H) or gamma.shape != (b, L, H):
        raise ValueError("oracle_fwd: logdecay/gamma shape")
    if beta is not None and beta.shape != (b, L, H):
        raise ValueError("oracle_fwd: beta shape")
    if theta is not None and theta.shape != (b, L, H, N // 2):
        raise ValueError("oracle_fwd: theta shape")
    d = _Dims(b, L, H, P, N, G)
    Y = np.zeros((b, L, H, P))
    hT = np.zeros((b, H, N, P))
    angleT = np.zeros((b, H, N // 2))
    xprevT = np.zeros((b, H, P))
    bprevT = np.zeros((b, G, N))
    if xprev0 is not None:
        xprevT[:] = xprev0
    if bprev0 is not None:
        bprevT[:] = bprev0
    rc = _load().oracle_fwd(ctypes.byref(d), _ptr(X), _ptr(logdecay), _ptr(beta), _ptr(gamma),
                            _ptr(B), _ptr(C), _ptr(theta), _ptr(D), _ptr(h0), _ptr(angle0),
                            _ptr(xprev0), _ptr(bprev0), _ptr(Y), _ptr(hT), _ptr(angleT),
                            _ptr(xprevT), _ptr(bprevT),
                            int(nthreads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"oracle_fwd failed with code {rc}")
    if L == 0:
        angleT[:] = 0.0 if angle0 is None else angle0
        if h0 is not None:
            hT[:] = h0
    return {"Y": Y, "hT": hT, "angleT": angleT, "xprevT": xprevT, "bprevT": bprevT}


def oracle_bwd(X, logdecay, beta, gamma, B, C, theta=None, D=None, h0=None,
               angle0=None, xprev0=None, bprev0=None, *, dY, dhT=None,
               nthreads: int | None = None):
    """Reverse-mode derivatives of :func:`oracle_fwd` (fp64, sequential in t).

    ``dY`` (b,L,H,P) and ``dhT`` (b,H,N,P, None = 0) are the upstream
    gradients of Y and hT.  Returns a dict with dX, dlogdecay, dbeta, dgamma,
    dB, dC, dtheta, dD, dh0, dangle0, dxprev0, dbprev0 (float64, each shaped
    like its input; an input passed as None is read as zero and its gradient is
    the derivative there).
    """
    X, logdecay, beta, gamma = _f64(X), _f64(logdecay), _f64(beta), _f64(gamma)
    B, C, theta, D, h0 = _f64(B), _f64(C), _f64(theta), _f64(D), _f64(h0)
    angle0, xprev0, bprev0 = _f64(angle0), _f64(xprev0), _f64(bprev0)
    dY, dhT = _f64(dY), _f64(dhT)
    b, L, H, P = X.shape
    G, N = B.shape[2], B.shape[3]
    if N % 2 or H % G:
        raise ValueError("oracle_bwd: N must be even and H divisible by G")
    if dY.shape != X.shape:
        raise ValueError("oracle_bwd: dY shape")
    if dhT is not None and dhT.shape != (b, H, N, P):
        raise ValueError("oracle_bwd: dhT shape")
    d = _Dims(b, L, H, P, N, G)
    out = {"dX": np.zeros((b, L, H, P)), "dlogdecay": np.zeros((b, L, H)),
           "dbeta": np.zeros((b, L, H)), "dgamma": np.zeros((b, L, H)),
           "dB": np.zeros((b, L, G, N)), "dC": np.zeros((b, L, G, N)),
           "dtheta": np.zeros((b, L, H, N // 2)), "dD": np.zeros((H,)),
           "dh0": np.zeros((b, H, N, P)), "dangle0": np.zeros((b, H, N // 2)),
           "dxprev0": np.zeros((b, H, P)), "dbprev0": np.zeros((b, G, N))}
    o = out
    rc = _load().oracle_bwd(ctypes.byref(d), _ptr(X), _ptr(logdecay), _ptr(beta), _ptr(gamma),
                            _ptr(B), _ptr(C), _ptr(theta), _ptr(D), _ptr(h0), _ptr(angle0),
                            _ptr(xprev0), _ptr(bprev0), _ptr(dY), _ptr(dhT),
                            _ptr(o["dX"]), _ptr(o["dlogdecay"]), _ptr(o["dbeta"]),
                            _ptr(o["dgamma"]), _ptr(o["dB"]), _ptr(o["dC"]), _ptr(o["dtheta"]),
                            _ptr(o["dD"]), _ptr(o["dh0"]), _ptr(o["dangle0"]),
                            _ptr(o["dxprev0"]), _ptr(o["dbprev0"]),
                            int(nthreads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"oracle_bwd failed with code {rc}")
    if L == 0 and dhT is not None:
        out["dh0"][:] = dhT
    return out


def oracle_step(cache, x_t, logdecay_t, beta_t, gamma_t, B_t, C_t, theta_t=None, D=None):
    """One decode step; ``cache`` is a dict of float64 arrays angle, ssm, x_prev,
    b_prev that is updated in place.  Returns y_t (b,H,P) float64."""
    x_t, logdecay_t, beta_t, gamma_t = _f64(x_t), _f64(logdecay_t), _f64(beta_t), _f64(gamma_t)
    B_t, C_t, theta_t, D = _f64(B_t), _f64(C_t), _f64(theta_t), _f64(D)
    for k in ("angle", "ssm", "x_prev", "b_prev"):
        a = cache[k]
        if not (isinstance(a, np.ndarray) and a.dtype == np.float64 and a.flags.c_contiguous):
            raise ValueError(f"oracle_step: cache[{k!r}] must be a C-contiguous float64 ndarray")
    b, H, P = x_t.shape
    G, N = B_t.shape[1], B_t.shape[2]
    d = _Dims(b, 1, H, P, N, G)
    y = np.zeros((b, H, P))
    rc = _load().oracle_step(ctypes.byref(d), _ptr(x_t), _ptr(logdecay_t), _ptr(beta_t),
                             _ptr(gamma_t), _ptr(B_t), _ptr(C_t), _ptr(theta_t), _ptr(D),
                             _ptr(cache["angle"]), _ptr(cache["ssm"]), _ptr(cache["x_prev"]),
                             _ptr(cache["b_prev"]), _ptr(y))
    if rc != 0:
        raise RuntimeError(f"oracle_step failed with code {rc}")
    return y


def oracle_mimo_fwd(X, logdecay, beta, gamma, B, C, theta=None, D=None, h0=None,
                    angle0=None, xprev0=None, bprev0=None, nthreads: int | None = None):
    """Sequential fp64 MIMO forward.

    Shapes: X (b,L,H,P,R); logdecay, beta, gamma (b,L,H); B, C (b,L,G,N,R);
    theta (b,L,H,N/2); D (H); h0 (b,H,N,P); angle0 (b,H,N/2);
    xprev0 (b,H,P,R); bprev0 (b,G,N,R).  Returns Y, hT, angleT, xprevT, bprevT.
    """
    X, logdecay, beta, gamma = _f64(X), _f64(logdecay), _f64(beta), _f64(gamma)
    B, C, theta, D, h0 = _f64(B), _f64(C), _f64(theta), _f64(D), _f64(h0)
    angle0, xprev0, bprev0 = _f64(angle0), _f64(xprev0), _f64(bprev0)
    b, L, H, P, R = X.shape
    G, N = B.shape[2], B.shape[3]
    if N % 2 or H % G or B.shape != (b, L, G, N, R) or C.shape != (b, L, G, N, R):
        raise ValueError("oracle_mimo_fwd: shapes")
    d = _MimoDims(b, L, H, P, N, G, R)
    Y = np.zeros((b, L, H, P, R))
    hT = np.zeros((b, H, N, P)) if h0 is None else h0.copy()
    angleT = np.zeros((b, H, N // 2)) if angle0 is None else angle0.copy()
    xprevT = np.zeros((b, H, P, R)) if xprev0 is None else xprev0.copy()
    bprevT = np.zeros((b, G, N, R)) if bprev0 is None else bprev0.copy()
    rc = _load().oracle_mimo_fwd(ctypes.byref(d), _ptr(X), _ptr(logdecay), _ptr(beta),
                                 _ptr(gamma), _ptr(B), _ptr(C), _ptr(theta), _ptr(D), _ptr(h0),
                                 _ptr(angle0), _ptr(xprev0), _ptr(bprev0), _ptr(Y), _ptr(hT),
                                 _ptr(angleT), _ptr(xprevT), _ptr(bprevT),
                                 int(nthreads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"oracle_mimo_fwd failed with code {rc}")
    return {"Y": Y, "hT": hT, "angleT": angleT, "xprevT": xprevT, "bprevT": bprevT}


def oracle_mimo_step(cache, x_t, logdecay_t, beta_t, gamma_t, B_t, C_t, theta_t=None, D=None):
    """One MIMO decode step; ``cache`` holds float64 arrays angle (b,H,N/2),
    ssm (b,H,N,P), x_prev (b,H,P,R), b_prev (b,G,N,R), updated in place.
    Returns y_t (b,H,P,R)."""
    x_t, logdecay_t, beta_t, gamma_t = _f64(x_t), _f64(logdecay_t), _f64(beta_t), _f64(gamma_t)
    B_t, C_t, theta_t, D = _f64(B_t), _f64(C_t), _f64(theta_t), _f64(D)
    for k in ("angle", "ssm", "x_prev", "b_prev"):
        a = cache[k]
        if not (isinstance(a, np.ndarray) and a.dtype == np.float64 and a.flags.c_contiguous):
            raise ValueError(f"oracle_mimo_step: cache[{k!r}] must be a C-contiguous float64 ndarray")
    b, H, P, R = x_t.shape
    G, N = B_t.shape[1], B_t.shape[2]
    d = _MimoDims(b, 1, H, P, N, G, R)
    y = np.zeros((b, H, P, R))
    rc = _load().oracle_mimo_step(ctypes.byref(d), _ptr(x_t), _ptr(logdecay_t), _ptr(beta_t),
                                  _ptr(gamma_t), _ptr(B_t), _ptr(C_t), _ptr(theta_t), _ptr(D),
                                  _ptr(cache["angle"]), _ptr(cache["ssm"]), _ptr(cache["x_prev"]),
                                  _ptr(cache["b_prev"]), _ptr(y))
    if rc != 0:
        raise RuntimeError(f"oracle_mimo_step failed with code {rc}")
    return y


def new_cache(b, H, P, N, G):
    """A zero cache of float64 arrays (angle, ssm, x_prev, b_prev)."""
    return {"angle": np.zeros((b, H, N // 2)), "ssm": np.zeros((b, H, N, P)),
            "x_prev": np.zeros((b, H, P)), "b_prev": np.zeros((b, G, N))}
