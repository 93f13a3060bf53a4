"""B200-native Mamba-3 SISO selective scan: Python binding of ``libm3ssd``.

The binding only marshals arguments (device pointers, sizes, the current CUDA
stream) into the C ABI declared in ``include/m3ssd.h``; every step of the scan
runs in the library's CUDA kernels.  Importing this package does not load the
library; the first call does, and raises ``LibraryMissing`` if it has not been
built (``python -m selective_state_space_m3ssd_b200.build``).  There is no
other implementation behind these functions.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libm3ssd.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_NONFINITE, ERR_TIMEOUT = range(7)
F32, BF16 = 0, 1
CHECK_FINITE = 1  # m3ssd_dims.flags: scan the outputs for NaN / infinity

_lib = None
_lock = threading.Lock()


class LibraryMissing(RuntimeError):
    pass


class M3SSDError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} (status {status})")
        self.status = status


class M3SSDInvalidArgument(M3SSDError, ValueError):
    pass


class Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64),
                ("nheads", ctypes.c_int64), ("headdim", ctypes.c_int64),
                ("dstate", ctypes.c_int64), ("ngroups", ctypes.c_int64),
                ("chunk", ctypes.c_int32), ("x_dtype", ctypes.c_int32),
                ("flags", ctypes.c_uint32), ("reserved", ctypes.c_uint32)]


class FwdExtra(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("angle0", "xprev0", "bprev0", "angleT", "xprevT", "bprevT")]


GRAD_NAMES = ("dX", "dlogdecay", "dbeta", "dgamma", "dB", "dC", "dtheta", "dD", "dh0",
              "dangle0", "dxprev0", "dbprev0")


class BwdGrads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in GRAD_NAMES]


class Cache(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("angle", "ssm", "x_prev", "b_prev")]


class BlockDims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in
                ("batch", "seqlen", "d_model", "nheads", "headdim", "dstate", "ngroups")]


BLOCK_WEIGHT_NAMES = ("W_in", "W_out", "dt_bias", "A_log", "D", "B_norm_w", "C_norm_w",
                      "B_bias", "C_bias")


class BlockWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in BLOCK_WEIGHT_NAMES] + [("eps", ctypes.c_float)]


def load(path: str | None = None):
    """Load ``libm3ssd.so`` (once) and declare the C signatures.

    With ``path``, load that build of the library and return its handle with
    the signatures declared; the module's own calls keep using the in-tree
    library (assign the handle to ``_lib`` to route them to the other build).
    """
    global _lib
    with _lock:
        if _lib is not None and path is None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise LibraryMissing(
                f"{p} is not built; run `python -m selective_state_space_m3ssd_b200.build`")
        lib = ctypes.CDLL(p)
        vp, sz = ctypes.c_void_p, ctypes.c_size_t
        lib.m3ssd_fwd_workspace_size.argtypes = [ctypes.POINTER(Dims)]
        lib.m3ssd_fwd_workspace_size.restype = sz
        lib.m3ssd_fwd.argtypes = [ctypes.POINTER(Dims)] + [vp] * 11 + \
            [ctypes.POINTER(FwdExtra), vp, sz, vp]
        lib.m3ssd_fwd.restype = ctypes.c_int
        lib.m3ssd_step.argtypes = [ctypes.POINTER(Dims)] + [vp] * 8 + \
            [ctypes.POINTER(Cache), vp, vp]
        lib.m3ssd_step.restype = ctypes.c_int
        lib.m3ssd_mimo_fwd.argtypes = [ctypes.POINTER(Dims), ctypes.c_int32] + [vp] * 11 + \
            [ctypes.POINTER(FwdExtra), vp]
        lib.m3ssd_mimo_fwd.restype = ctypes.c_int
        lib.m3ssd_mimo_step.argtypes = [ctypes.POINTER(Dims), ctypes.c_int32] + [vp] * 8 + \
            [ctypes.POINTER(Cache), vp, vp]
        lib.m3ssd_mimo_step.restype = ctypes.c_int
        lib.m3ssd_bwd_workspace_size.argtypes = [ctypes.POINTER(Dims)]
        lib.m3ssd_bwd_workspace_size.restype = sz
        lib.m3ssd_bwd.argtypes = [ctypes.POINTER(Dims)] + [vp] * 9 + \
            [ctypes.POINTER(FwdExtra), vp, vp, ctypes.POINTER(BwdGrads), vp, sz, vp]
        lib.m3ssd_bwd.restype = ctypes.c_int
        lib.m3ssd_bwd_noalloc.argtypes = [ctypes.POINTER(Dims)] + [vp] * 9 + \
            [ctypes.POINTER(FwdExtra), vp, vp, ctypes.POINTER(BwdGrads), vp]
        lib.m3ssd_bwd_noalloc.restype = ctypes.c_int
        lib.m3ssd_block_workspace_size.argtypes = [ctypes.POINTER(BlockDims)]
        lib.m3ssd_block_workspace_size.restype = sz
        lib.m3ssd_block_fwd.argtypes = [ctypes.POINTER(BlockDims), ctypes.POINTER(BlockWeights),
                                        vp, vp, ctypes.POINTER(Cache), ctypes.POINTER(Cache),
                                        vp, sz, vp]
        lib.m3ssd_block_fwd.restype = ctypes.c_int
        lib.m3ssd_block_step.argtypes = [ctypes.POINTER(BlockDims), ctypes.POINTER(BlockWeights),
                                         vp, vp, ctypes.POINTER(Cache), vp, sz, vp]
        lib.m3ssd_block_step.restype = ctypes.c_int
        lib.m3ssd_gemm_bf16.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_int64, ctypes.c_void_p]
        lib.m3ssd_gemm_bf16.restype = ctypes.c_int
        lib.m3ssd_status_string.argtypes = [ctypes.c_int]
        lib.m3ssd_status_string.restype = ctypes.c_char_p
        lib.m3ssd_abi_version.argtypes = []
        lib.m3ssd_abi_version.restype = ctypes.c_int
        lib.m3ssd_device_wait_timeouts.argtypes = [ctypes.POINTER(ctypes.c_uint32)]
        lib.m3ssd_device_wait_timeouts.restype = ctypes.c_int
        lib.m3ssd_nonfinite_outputs.argtypes = []
        lib.m3ssd_nonfinite_outputs.restype = ctypes.c_int
        lib.m3ssd_test_set_wait_limit.argtypes = [ctypes.c_uint64]
        lib.m3ssd_test_set_wait_limit.restype = ctypes.c_int
        lib.m3ssd_test_drop_next_gram_signal.argtypes = []
        lib.m3ssd_test_drop_next_gram_signal.restype = ctypes.c_int
        i64, i32p = ctypes.c_int64, ctypes.POINTER(ctypes.c_int32)
        lib.m3ssd_test_fwd_split_plan.argtypes = [i64, i64, i64, ctypes.c_int32, i32p, i32p]
        lib.m3ssd_test_fwd_split_plan.restype = ctypes.c_int
        if path is None:
            _lib = lib
        return lib


def status_string(status: int) -> str:
    return load().m3ssd_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status == OK:
        return
    if status == ERR_INVALID_ARG:
        raise M3SSDInvalidArgument(status, what)
    raise M3SSDError(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(device):
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _xdtype(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise ValueError(f"X/B/C must be bf16 or fp32, got {t.dtype}")


def _need_shape(t, name, dtype=None, shape=None):
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _need(t, name, dtype=None, shape=None, device=None):
    if t is None:
        return
    _need_shape(t, name, dtype, shape)
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def device_wait_timeouts() -> int:
    """Bounded device-side waits that ran out since the last call (synchronises)."""
    n = ctypes.c_uint32(0)
    _check(load().m3ssd_device_wait_timeouts(ctypes.byref(n)), "m3ssd_device_wait_timeouts")
    return int(n.value)


def nonfinite_outputs() -> bool:
    """Whether any output checked under CHECK_FINITE since the last call held a
    NaN or an infinity (synchronises; clears the record)."""
    st = load().m3ssd_nonfinite_outputs()
    if st == ERR_NONFINITE:
        return True
    _check(st, "m3ssd_nonfinite_outputs")
    return False


def set_wait_limit_for_tests(nanoseconds: int):
    """Testing hook: the chunked forward's bounded waits give up after this many
    nanoseconds (0 restores the default 2 s).  Synchronous; not while work is
    in flight."""
    _check(load().m3ssd_test_set_wait_limit(int(nanoseconds)), "m3ssd_test_set_wait_limit")


def drop_next_gram_signal_for_tests():
    """Testing hook: the next chunked-forward sequence leaves out one completion
    signal, so one of its bounded waits runs out (reported by
    device_wait_timeouts; that launch's outputs are undefined)."""
    _check(load().m3ssd_test_drop_next_gram_signal(), "m3ssd_test_drop_next_gram_signal")


def fwd_split_plan(batch: int, seqlen: int, nheads: int, sms: int) -> tuple:
    """(segments, chunks per segment) of the chunked bf16 forward's sequence
    split for this shape on a device with ``sms`` SMs; (1, 0) means no split."""
    nseg, segc = ctypes.c_int32(), ctypes.c_int32()
    _check(load().m3ssd_test_fwd_split_plan(int(batch), int(seqlen), int(nheads), int(sms),
                                            ctypes.byref(nseg), ctypes.byref(segc)),
           "m3ssd_test_fwd_split_plan")
    return nseg.value, segc.value


def make_dims(batch, seqlen, nheads, headdim, dstate, ngroups, x_dtype, chunk=0, flags=0) -> Dims:
    return Dims(batch, seqlen, nheads, headdim, dstate, ngroups, chunk, x_dtype, flags, 0)


def fwd_workspace_size(dims: Dims) -> int:
    return int(load().m3ssd_fwd_workspace_size(ctypes.byref(dims)))


def fwd(X, logdecay, beta, gamma, B, C, theta=None, D=None, h0=None, *, Y=None,
        want_hT: bool = True, hT=None, angle0=None, xprev0=None, bprev0=None,
        want_cache: bool = False, chunk: int = 0, workspace=None, check_finite: bool = False):
    """Forward scan through ``m3ssd_fwd`` on the current CUDA stream.

    Shapes as in ``include/m3ssd.h``.  Returns ``(Y, hT, cache_out)`` where
    ``cache_out`` is a dict with angleT/xprevT/bprevT when ``want_cache``.
    Output tensors are allocated by torch unless passed in.  ``check_finite``
    sets CHECK_FINITE (see :func:`nonfinite_outputs`).
    """
    import torch
    b, L, H, P = X.shape
    G, N = B.shape[2], B.shape[3]
    dev = X.device
    f32 = torch.float32
    _need(X, "X", device=dev)
    xd = X.dtype
    _need(logdecay, "logdecay", f32, (b, L, H), dev)
    _need(beta, "beta", f32, (b, L, H), dev)
    _need(gamma, "gamma", f32, (b, L, H), dev)
    _need(B, "B", xd, (b, L, G, N), dev)
    _need(C, "C", xd, (b, L, G, N), dev)
    _need(theta, "theta", f32, (b, L, H, N // 2), dev)
    _need(D, "D", f32, (H,), dev)
    _need(h0, "h0", f32, (b, H, N, P), dev)
    _need(angle0, "angle0", f32, (b, H, N // 2), dev)
    _need(xprev0, "xprev0", f32, (b, H, P), dev)
    _need(bprev0, "bprev0", f32, (b, G, N), dev)
    if Y is None:
        Y = torch.empty_like(X)
    _need(Y, "Y", xd, (b, L, H, P), dev)
    if hT is None and want_hT:
        hT = torch.empty(b, H, N, P, dtype=f32, device=dev)
    _need(hT, "hT", f32, (b, H, N, P), dev)
    cache_out = None
    extra = None
    if want_cache or angle0 is not None or xprev0 is not None or bprev0 is not None:
        if want_cache:
            cache_out = {"angle": torch.empty(b, H, N // 2, dtype=f32, device=dev),
                         "x_prev": torch.empty(b, H, P, dtype=f32, device=dev),
                         "b_prev": torch.empty(b, G, N, dtype=f32, device=dev)}
        extra = FwdExtra(
            *(None if t is None else t.data_ptr() for t in (angle0, xprev0, bprev0)),
            *(None if cache_out is None else cache_out[k].data_ptr()
              for k in ("angle", "x_prev", "b_prev")))
    dims = make_dims(b, L, H, P, N, G, _xdtype(X), chunk, CHECK_FINITE if check_finite else 0)
    ws_bytes = fwd_workspace_size(dims)
    if ws_bytes and workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    st = load().m3ssd_fwd(ctypes.byref(dims), _ptr(X), _ptr(logdecay), _ptr(beta), _ptr(gamma),
                          _ptr(B), _ptr(C), _ptr(theta), _ptr(D), _ptr(h0), _ptr(Y), _ptr(hT),
                          None if extra is None else ctypes.byref(extra), _ptr(workspace),
                          0 if workspace is None else workspace.numel() * workspace.element_size(),
                          _stream_handle(dev))
    _check(st, "m3ssd_fwd")
    return Y, hT, cache_out


def bwd_workspace_size(dims: Dims) -> int:
    return int(load().m3ssd_bwd_workspace_size(ctypes.byref(dims)))


def _bwd_args(X, logdecay, beta, gamma, B, C, theta, D, h0, dY, dhT, angle0, xprev0, bprev0,
              grads):
    """Validates every backward input (dtype, shape, device) and marshals the C
    arguments shared by :func:`bwd` and :func:`bwd_noalloc`."""
    import torch
    b, L, H, P = X.shape
    G, N = B.shape[2], B.shape[3]
    dev = X.device
    f32 = torch.float32
    xd = X.dtype
    checks = [(X, "X", None, None), (logdecay, "logdecay", f32, (b, L, H)),
              (beta, "beta", f32, (b, L, H)), (gamma, "gamma", f32, (b, L, H)),
              (B, "B", xd, (b, L, G, N)), (C, "C", xd, (b, L, G, N)),
              (theta, "theta", f32, (b, L, H, N // 2)), (D, "D", f32, (H,)),
              (h0, "h0", f32, (b, H, N, P)), (angle0, "angle0", f32, (b, H, N // 2)),
              (xprev0, "xprev0", f32, (b, H, P)), (bprev0, "bprev0", f32, (b, G, N)),
              (dY, "dY", xd, (b, L, H, P)), (dhT, "dhT", f32, (b, H, N, P))]
    for t, name, dt, shape in checks:  # every shape and dtype first, then placement
        if t is not None:
            _need_shape(t, name, dt, shape)
    for t, name, dt, shape in checks:
        _need(t, name, dt, shape, dev)
    shapes = {"dX": (b, L, H, P), "dlogdecay": (b, L, H), "dbeta": (b, L, H),
              "dgamma": (b, L, H), "dB": (b, L, G, N), "dC": (b, L, G, N),
              "dtheta": (b, L, H, N // 2), "dD": (H,), "dh0": (b, H, N, P),
              "dangle0": (b, H, N // 2), "dxprev0": (b, H, P), "dbprev0": (b, G, N)}
    if grads is None:
        grads = {k: torch.empty(v, dtype=f32, device=dev) for k, v in shapes.items()}
    for k in GRAD_NAMES:
        _need(grads.get(k), k, f32, shapes[k], dev)
    gs = BwdGrads(*(None if grads.get(k) is None else grads[k].data_ptr() for k in GRAD_NAMES))
    extra = None
    if angle0 is not None or xprev0 is not None or bprev0 is not None:
        extra = FwdExtra(*(None if t is None else t.data_ptr() for t in (angle0, xprev0, bprev0)),
                         None, None, None)
    dims = make_dims(b, L, H, P, N, G, _xdtype(X), 0)
    ptrs = [_ptr(t) for t in (X, logdecay, beta, gamma, B, C, theta, D, h0)]
    return dims, ptrs, extra, gs, grads


def bwd(X, logdecay, beta, gamma, B, C, theta=None, D=None, h0=None, *, dY, dhT=None,
        angle0=None, xprev0=None, bprev0=None, grads=None, workspace=None):
    """Backward of :func:`fwd` through ``m3ssd_bwd`` on the current CUDA stream.

    Takes the forward's inputs and the upstream gradients ``dY`` (dtype of X)
    and ``dhT`` (fp32 or None).  Returns a dict of fp32 gradients named as in
    ``GRAD_NAMES``, each shaped like its input (allocated by torch unless
    ``grads`` supplies them).
    """
    import torch
    dims, ptrs, extra, gs, grads = _bwd_args(X, logdecay, beta, gamma, B, C, theta, D, h0, dY,
                                             dhT, angle0, xprev0, bprev0, grads)
    ws_bytes = bwd_workspace_size(dims)
    if ws_bytes and workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=X.device)
    st = load().m3ssd_bwd(ctypes.byref(dims), *ptrs,
                          None if extra is None else ctypes.byref(extra), _ptr(dY), _ptr(dhT),
                          ctypes.byref(gs), _ptr(workspace),
                          0 if workspace is None else workspace.numel() * workspace.element_size(),
                          _stream_handle(X.device))
    _check(st, "m3ssd_bwd")
    return grads


def bwd_noalloc(X, logdecay, beta, gamma, B, C, theta=None, D=None, h0=None, *, dY,
                dhT=None, angle0=None, xprev0=None, bprev0=None, grads=None):
    """:func:`bwd` through ``m3ssd_bwd_noalloc`` (scratch inside the library;
    calls must not overlap).  Validates its inputs exactly as :func:`bwd` does
    and returns the same dict of fp32 gradients."""
    dims, ptrs, extra, gs, grads = _bwd_args(X, logdecay, beta, gamma, B, C, theta, D, h0, dY,
                                             dhT, angle0, xprev0, bprev0, grads)
    st = load().m3ssd_bwd_noalloc(ctypes.byref(dims), *ptrs,
                                  None if extra is None else ctypes.byref(extra), _ptr(dY),
                                  _ptr(dhT), ctypes.byref(gs), _stream_handle(X.device))
    _check(st, "m3ssd_bwd_noalloc")
    return grads


def new_cache(batch, nheads, headdim, dstate, ngroups, device):
    """A zeroed fp32 decode cache (angle, ssm, x_prev, b_prev) allocated by torch."""
    import torch
    z = dict(dtype=torch.float32, device=device)
    return {"angle": torch.zeros(batch, nheads, dstate // 2, **z),
            "ssm": torch.zeros(batch, nheads, dstate, headdim, **z),
            "x_prev": torch.zeros(batch, nheads, headdim, **z),
            "b_prev": torch.zeros(batch, ngroups, dstate, **z)}


def step(cache: dict, x_t, logdecay_t, beta_t, gamma_t, B_t, C_t, theta_t=None, D=None, *,
         y_t=None, check_finite: bool = False):
    """One decode step through ``m3ssd_step``; updates ``cache`` in place and
    returns y_t (b, H, P) in the dtype of x_t.  ``check_finite`` sets
    CHECK_FINITE on y_t (see :func:`nonfinite_outputs`)."""
    import torch
    b, H, P = x_t.shape
    G, N = B_t.shape[1], B_t.shape[2]
    dev = x_t.device
    f32 = torch.float32
    xd = x_t.dtype
    _need(x_t, "x_t", device=dev)
    _need(logdecay_t, "logdecay_t", f32, (b, H), dev)
    _need(beta_t, "beta_t", f32, (b, H), dev)
    _need(gamma_t, "gamma_t", f32, (b, H), dev)
    _need(B_t, "B_t", xd, (b, G, N), dev)
    _need(C_t, "C_t", xd, (b, G, N), dev)
    _need(theta_t, "theta_t", f32, (b, H, N // 2), dev)
    _need(D, "D", f32, (H,), dev)
    _need(cache["angle"], "cache.angle", f32, (b, H, N // 2), dev)
    _need(cache["ssm"], "cache.ssm", f32, (b, H, N, P), dev)
    _need(cache["x_prev"], "cache.x_prev", f32, (b, H, P), dev)
    _need(cache["b_prev"], "cache.b_prev", f32, (b, G, N), dev)
    if y_t is None:
        y_t = torch.empty_like(x_t)
    _need(y_t, "y_t", xd, (b, H, P), dev)
    c = Cache(cache["angle"].data_ptr(), cache["ssm"].data_ptr(), cache["x_prev"].data_ptr(),
              cache["b_prev"].data_ptr())
    dims = make_dims(b, 1, H, P, N, G, _xdtype(x_t), 0, CHECK_FINITE if check_finite else 0)
    st = load().m3ssd_step(ctypes.byref(dims), _ptr(x_t), _ptr(logdecay_t), _ptr(beta_t),
                           _ptr(gamma_t), _ptr(B_t), _ptr(C_t), _ptr(theta_t), _ptr(D),
                           ctypes.byref(c), _ptr(y_t), _stream_handle(dev))
    _check(st, "m3ssd_step")
    return y_t


def mimo_fwd(X, logdecay, beta, gamma, B, C, theta=None, D=None, h0=None, *, Y=None,
             want_hT: bool = True, angle0=None, xprev0=None, bprev0=None,
             want_cache: bool = False, check_finite: bool = False):
    """MIMO rank-R forward through ``m3ssd_mimo_fwd``: X (b,L,H,P,R), B, C
    (b,L,G,N,R).  Returns ``(Y, hT, cache_out)`` like :func:`fwd`, with the
    cache's x_prev (b,H,P,R) and b_prev (b,G,N,R)."""
    import torch
    b, L, H, P, R = X.shape
    G, N = B.shape[2], B.shape[3]
    dev, f32, xd = X.device, torch.float32, X.dtype
    _need(X, "X", device=dev)
    for name, t, dt, shape in (("logdecay", logdecay, f32, (b, L, H)), ("beta", beta, f32, (b, L, H)),
                               ("gamma", gamma, f32, (b, L, H)), ("B", B, xd, (b, L, G, N, R)),
                               ("C", C, xd, (b, L, G, N, R)), ("theta", theta, f32, (b, L, H, N // 2)),
                               ("D", D, f32, (H,)), ("h0", h0, f32, (b, H, N, P)),
                               ("angle0", angle0, f32, (b, H, N // 2)),
                               ("xprev0", xprev0, f32, (b, H, P, R)),
                               ("bprev0", bprev0, f32, (b, G, N, R))):
        _need(t, name, dt, shape, dev)
    Y = torch.empty_like(X) if Y is None else Y
    _need(Y, "Y", xd, (b, L, H, P, R), dev)
    hT = torch.empty(b, H, N, P, dtype=f32, device=dev) if want_hT else None
    cache_out = None
    extra = None
    if want_cache or angle0 is not None or xprev0 is not None or bprev0 is not None:
        if want_cache:
            cache_out = {"angle": torch.empty(b, H, N // 2, dtype=f32, device=dev),
                         "x_prev": torch.empty(b, H, P, R, dtype=f32, device=dev),
                         "b_prev": torch.empty(b, G, N, R, dtype=f32, device=dev)}
        extra = FwdExtra(
            *(None if t is None else t.data_ptr() for t in (angle0, xprev0, bprev0)),
            *(None if cache_out is None else cache_out[k].data_ptr()
              for k in ("angle", "x_prev", "b_prev")))
    dims = make_dims(b, L, H, P, N, G, _xdtype(X), 0, CHECK_FINITE if check_finite else 0)
    st = load().m3ssd_mimo_fwd(ctypes.byref(dims), R, _ptr(X), _ptr(logdecay), _ptr(beta),
                               _ptr(gamma), _ptr(B), _ptr(C), _ptr(theta), _ptr(D), _ptr(h0),
                               _ptr(Y), _ptr(hT), None if extra is None else ctypes.byref(extra),
                               _stream_handle(dev))
    _check(st, "m3ssd_mimo_fwd")
    return Y, hT, cache_out


def new_mimo_cache(batch, nheads, headdim, dstate, ngroups, rank, device):
    """A zeroed fp32 MIMO decode cache: angle, ssm, x_prev (b,H,P,R), b_prev (b,G,N,R)."""
    import torch
    z = dict(dtype=torch.float32, device=device)
    return {"angle": torch.zeros(batch, nheads, dstate // 2, **z),
            "ssm": torch.zeros(batch, nheads, dstate, headdim, **z),
            "x_prev": torch.zeros(batch, nheads, headdim, rank, **z),
            "b_prev": torch.zeros(batch, ngroups, dstate, rank, **z)}


def mimo_step(cache: dict, x_t, logdecay_t, beta_t, gamma_t, B_t, C_t, theta_t=None, D=None, *,
              y_t=None, check_finite: bool = False):
    """One MIMO decode step through ``m3ssd_mimo_step``: x_t (b,H,P,R), B_t, C_t
    (b,G,N,R); updates ``cache`` in place and returns y_t (b,H,P,R)."""
    import torch
    b, H, P, R = x_t.shape
    G, N = B_t.shape[1], B_t.shape[2]
    dev, f32, xd = x_t.device, torch.float32, x_t.dtype
    _need(x_t, "x_t", device=dev)
    for name, t, dt, shape in (("logdecay_t", logdecay_t, f32, (b, H)), ("beta_t", beta_t, f32, (b, H)),
                               ("gamma_t", gamma_t, f32, (b, H)), ("B_t", B_t, xd, (b, G, N, R)),
                               ("C_t", C_t, xd, (b, G, N, R)), ("theta_t", theta_t, f32, (b, H, N // 2)),
                               ("D", D, f32, (H,)),
                               ("cache.angle", cache["angle"], f32, (b, H, N // 2)),
                               ("cache.ssm", cache["ssm"], f32, (b, H, N, P)),
                               ("cache.x_prev", cache["x_prev"], f32, (b, H, P, R)),
                               ("cache.b_prev", cache["b_prev"], f32, (b, G, N, R))):
        _need(t, name, dt, shape, dev)
    y_t = torch.empty_like(x_t) if y_t is None else y_t
    _need(y_t, "y_t", xd, (b, H, P, R), dev)
    c = Cache(cache["angle"].data_ptr(), cache["ssm"].data_ptr(), cache["x_prev"].data_ptr(),
              cache["b_prev"].data_ptr())
    dims = make_dims(b, 1, H, P, N, G, _xdtype(x_t), 0, CHECK_FINITE if check_finite else 0)
    st = load().m3ssd_mimo_step(ctypes.byref(dims), R, _ptr(x_t), _ptr(logdecay_t), _ptr(beta_t),
                                _ptr(gamma_t), _ptr(B_t), _ptr(C_t), _ptr(theta_t), _ptr(D),
                                ctypes.byref(c), _ptr(y_t), _stream_handle(dev))
    _check(st, "m3ssd_mimo_step")
    return y_t


# ---- the Mamba-3 SISO block around the scan --------------------------------------

def block_in_proj_width(nheads, headdim, dstate, ngroups) -> int:
    """Rows of W_in: z, x (H P each), B, C (G N each), dt, lam (H each), theta (H N/2)."""
    return 2 * nheads * headdim + 2 * ngroups * dstate + 2 * nheads + nheads * (dstate // 2)


def _block_args(u, wts, seqlen):
    import torch
    b, dm = u.shape[0], u.shape[-1]
    H = wts["A_log"].shape[0]
    N = wts["B_norm_w"].shape[0]
    HP = wts["W_out"].shape[1]
    if HP % H:
        raise ValueError("W_out's columns must be H * P")
    P = HP // H
    width = wts["W_in"].shape[0]
    rest = width - 2 * HP - 2 * H - H * (N // 2)
    if rest <= 0 or rest % (2 * N):
        raise ValueError("W_in's rows do not match any group count")
    G = rest // (2 * N)
    dev = u.device
    f32, bf = torch.float32, torch.bfloat16
    _need(u, "u", bf, device=dev)
    _need(wts["W_in"], "W_in", bf, (width, dm), dev)
    _need(wts["W_out"], "W_out", bf, (dm, HP), dev)
    for k, shape in (("dt_bias", (H,)), ("A_log", (H,)), ("B_norm_w", (N,)), ("C_norm_w", (N,)),
                     ("B_bias", (H, N)), ("C_bias", (H, N))):
        _need(wts[k], k, f32, shape, dev)
    _need(wts.get("D"), "D", f32, (H,), dev)
    dims = BlockDims(b, seqlen, dm, H, P, N, G)
    w = BlockWeights(*[(None if wts.get(k) is None else wts[k].data_ptr())
                       for k in BLOCK_WEIGHT_NAMES], float(wts.get("eps", 1e-6)))
    return dims, w, (H, P, N, G)


def new_block_cache(batch, nheads, headdim, dstate, ngroups, device):
    """A zeroed block cache: angle (b,H,N/2), ssm (b,H,N,P), x_prev (b,H,P) and
    b_prev (b,G,N) (the normed group vector, the head bias added at use), all fp32."""
    return new_cache(batch, nheads, headdim, dstate, ngroups, device)


def _cache_struct(cache, b, H, P, N, G, dev, name):
    import torch
    f32 = torch.float32
    _need(cache["angle"], name + ".angle", f32, (b, H, N // 2), dev)
    _need(cache["ssm"], name + ".ssm", f32, (b, H, N, P), dev)
    _need(cache["x_prev"], name + ".x_prev", f32, (b, H, P), dev)
    _need(cache["b_prev"], name + ".b_prev", f32, (b, G, N), dev)
    return Cache(cache["angle"].data_ptr(), cache["ssm"].data_ptr(), cache["x_prev"].data_ptr(),
                 cache["b_prev"].data_ptr())


def block_workspace_size(dims: BlockDims) -> int:
    return int(load().m3ssd_block_workspace_size(ctypes.byref(dims)))


def block_fwd(u, wts: dict, *, cache_in=None, cache_out=None, out=None, workspace=None):
    """Forward of the Mamba-3 SISO block through ``m3ssd_block_fwd``: u (b, L,
    d_model) bf16 -> out (b, L, d_model) bf16.  ``cache_in`` / ``cache_out``
    (dicts as from :func:`new_block_cache`, may be the same dict) continue from
    and hand back the decode state.  ``workspace`` (uint8, 256-byte aligned) is
    allocated by torch when not given."""
    import torch
    b, L, dm = u.shape
    dims, w, (H, P, N, G) = _block_args(u, wts, L)
    dev = u.device
    out = torch.empty_like(u) if out is None else out
    _need(out, "out", torch.bfloat16, (b, L, dm), dev)
    ci = None if cache_in is None else _cache_struct(cache_in, b, H, P, N, G, dev, "cache_in")
    co = None if cache_out is None else _cache_struct(cache_out, b, H, P, N, G, dev, "cache_out")
    need = block_workspace_size(dims)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    st = load().m3ssd_block_fwd(ctypes.byref(dims), ctypes.byref(w), _ptr(u), _ptr(out),
                                None if ci is None else ctypes.byref(ci),
                                None if co is None else ctypes.byref(co), _ptr(workspace),
                                workspace.numel(), _stream_handle(dev))
    _check(st, "m3ssd_block_fwd")
    return out


def gemm_bf16(A, W, *, out=None):
    """``m3ssd_gemm_bf16``: A (M, K) @ W (N, K)^T in bf16 with fp32 accumulation
    on the current stream; returns out (M, N) bf16."""
    import torch
    _need(A, "A", torch.bfloat16, device=A.device)
    M, K = A.shape
    _need(W, "W", torch.bfloat16, (W.shape[0], K), A.device)
    N = W.shape[0]
    out = torch.empty(M, N, dtype=torch.bfloat16, device=A.device) if out is None else out
    _need(out, "out", torch.bfloat16, (M, N), A.device)
    st = load().m3ssd_gemm_bf16(M, N, K, _ptr(A), _ptr(W), _ptr(out), N, _stream_handle(A.device))
    _check(st, "m3ssd_gemm_bf16")
    return out


def block_step(cache: dict, u_t, wts: dict, *, out_t=None, workspace=None):
    """One decode step of the block through ``m3ssd_block_step``: u_t (b,
    d_model) bf16 -> out_t; ``cache`` is advanced in place."""
    import torch
    b, dm = u_t.shape
    dims, w, (H, P, N, G) = _block_args(u_t, wts, 1)
    dev = u_t.device
    out_t = torch.empty_like(u_t) if out_t is None else out_t
    _need(out_t, "out_t", torch.bfloat16, (b, dm), dev)
    c = _cache_struct(cache, b, H, P, N, G, dev, "cache")
    need = block_workspace_size(dims)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    st = load().m3ssd_block_step(ctypes.byref(dims), ctypes.byref(w), _ptr(u_t), _ptr(out_t),
                                 ctypes.byref(c), _ptr(workspace), workspace.numel(),
                                 _stream_handle(dev))
    _check(st, "m3ssd_block_step")
    return out_t


class PreparedFwd:
    """A forward call with its C arguments marshalled once, for loops that
    launch the same problem many times (benchmarks, graph capture).  Calling
    it enqueues ``m3ssd_fwd`` on the current stream of the tensors' device."""

    def __init__(self, X, logdecay, beta, gamma, B, C, theta=None, D=None, h0=None, *,
                 Y=None, hT=None, chunk: int = 0):
        import torch
        b, L, H, P = X.shape
        G, N = B.shape[2], B.shape[3]
        self.Y = torch.empty_like(X) if Y is None else Y
        self.hT = hT
        self._keep = (X, logdecay, beta, gamma, B, C, theta, D, h0, self.Y, hT)
        self._dims = make_dims(b, L, H, P, N, G, _xdtype(X), chunk)
        self._args = [_ptr(t) for t in self._keep]
        self.device = X.device
        ws = fwd_workspace_size(self._dims)
        self._ws = torch.empty(ws, dtype=torch.uint8, device=X.device) if ws else None
        self._lib = load()

    def __call__(self):
        st = self._lib.m3ssd_fwd(ctypes.byref(self._dims), *self._args, None, _ptr(self._ws),
                                 0 if self._ws is None else self._ws.numel(),
                                 _stream_handle(self.device))
        _check(st, "m3ssd_fwd")
        return self.Y
