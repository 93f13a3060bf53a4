"""The C-ABI library loads, exports every declared symbol and validates its
arguments on the host (no GPU needed: nothing here reaches a kernel)."""
import ctypes
import os
import re
import subprocess

import pytest

import selective_state_space_m3ssd_b200 as m3
from selective_state_space_m3ssd_b200 import build as m3build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "m3ssd.h")


@pytest.fixture(scope="module")
def lib():
    m3build.build()
    return m3.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(m3ssd_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("m3ssd_fwd", "m3ssd_step", "m3ssd_fwd_workspace_size", "m3ssd_status_string",
              "m3ssd_abi_version", "m3ssd_device_wait_timeouts"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", m3.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (m3ssd_\w+)", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, f"declared but not exported: {missing}"
    for n in declared_functions():
        assert hasattr(lib, n)


def test_header_compiles_as_c_and_cxx(tmp_path):
    src = tmp_path / "t.c"
    src.write_text('#include "m3ssd.h"\nint main(void){m3ssd_dims d={0};(void)d;'
                   'return m3ssd_abi_version()==M3SSD_ABI_VERSION?0:1;}\n')
    for cc, std in (("gcc", "-std=c99"), ("g++", "-std=c++17")):
        subprocess.run([cc, std, "-fsyntax-only", "-x", "c" if cc == "gcc" else "c++",
                        "-I", os.path.join(ROOT, "include"), str(src)], check=True)


def test_version_and_status_strings(lib):
    assert lib.m3ssd_abi_version() == 1
    assert m3.status_string(m3.OK) == "ok"
    assert "invalid" in m3.status_string(m3.ERR_INVALID_ARG)
    assert m3.status_string(99) == "unknown status"


def _dims(**kw):
    d = dict(batch=1, seqlen=8, nheads=2, headdim=8, dstate=8, ngroups=1, x_dtype=m3.F32,
             chunk=0, flags=0)
    d.update(kw)
    return m3.make_dims(d["batch"], d["seqlen"], d["nheads"], d["headdim"], d["dstate"],
                        d["ngroups"], d["x_dtype"], d["chunk"], d["flags"])


FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: every call below fails validation


def _fwd(lib, dims, X=FAKE, ld=FAKE, beta=None, gamma=FAKE, B=FAKE, C=FAKE, theta=None,
         D=None, h0=None, Y=FAKE, hT=None, extra=None, ws=None, ws_bytes=0):
    return lib.m3ssd_fwd(ctypes.byref(dims), X, ld, beta, gamma, B, C, theta, D, h0, Y, hT,
                         None if extra is None else ctypes.byref(extra), ws, ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(dstate=7), m3.ERR_INVALID_ARG),
    (dict(dstate=0), m3.ERR_INVALID_ARG),
    (dict(nheads=3, ngroups=2), m3.ERR_INVALID_ARG),
    (dict(nheads=0), m3.ERR_INVALID_ARG),
    (dict(headdim=0), m3.ERR_INVALID_ARG),
    (dict(batch=-1), m3.ERR_INVALID_ARG),
    (dict(seqlen=-5), m3.ERR_INVALID_ARG),
    (dict(x_dtype=7), m3.ERR_INVALID_ARG),
    (dict(flags=2), m3.ERR_UNSUPPORTED),
    (dict(chunk=48), m3.ERR_UNSUPPORTED),
    (dict(chunk=128), m3.ERR_UNSUPPORTED),                  # longer chunks: bf16 N128 P64 only
    (dict(chunk=256, x_dtype=m3.BF16), m3.ERR_UNSUPPORTED),
    (dict(dstate=512), m3.ERR_UNSUPPORTED),
    (dict(headdim=300), m3.ERR_UNSUPPORTED),
])
def test_fwd_rejects_bad_dims(lib, kw, status):
    assert _fwd(lib, _dims(**kw)) == status


def test_fwd_rejects_null_and_misaligned_pointers(lib):
    d = _dims()
    for name in ("X", "ld", "gamma", "B", "C", "Y"):
        assert _fwd(lib, d, **{name: None}) == m3.ERR_INVALID_ARG, name
    assert _fwd(lib, d, X=ctypes.c_void_p(0x10002)) == m3.ERR_INVALID_ARG
    assert _fwd(lib, d, theta=ctypes.c_void_p(0x10001)) == m3.ERR_INVALID_ARG
    assert _fwd(lib, _dims(x_dtype=m3.BF16), X=ctypes.c_void_p(0x10001)) == m3.ERR_INVALID_ARG
    e = m3.FwdExtra(None, None, 0x20000, None, None, 0x20000)
    assert _fwd(lib, d, extra=e) == m3.ERR_INVALID_ARG  # bprevT aliases bprev0


def test_fwd_with_no_batch_is_a_no_op(lib):
    assert _fwd(lib, _dims(batch=0), X=None, ld=None, gamma=None, B=None, C=None, Y=None) == m3.OK
    assert lib.m3ssd_fwd_workspace_size(ctypes.byref(_dims())) == 0
    assert lib.m3ssd_fwd_workspace_size(None) == 0


def test_fwd_split_plan_policy(lib):
    """The sequence split of the chunked bf16 forward: only when b*H is at most
    two thirds of the SM count (two chunk walks fit on an SM, and fewer than
    three per sequence would not pay for the segment pass), with segments of at
    least 8 chunks of 63 tokens that tile the sequence."""
    plan = m3.fwd_split_plan
    assert plan(2, 32768, 48, 148) == (3, 174)   # the long workload: 521 chunks
    assert plan(8, 4096, 32, 148) == (1, 0)      # 256 sequences fill the device
    assert plan(8, 4096, 24, 148) == (1, 0)
    assert plan(1, 4096, 1, 148) == (8, 9)       # 65 chunks, at least 8 a segment
    assert plan(1, 1529, 2, 148) == (3, 9)
    assert plan(1, 63 * 15, 1, 148) == (1, 0)    # fewer than 16 chunks
    assert plan(1, 4096, 99, 148) == (1, 0) and plan(1, 4096, 98, 148)[0] == 3
    assert plan(1, 4096, 1, 0) == (1, 0) and plan(0, 4096, 4, 148) == (1, 0)
    for b, L, H in ((1, 1008, 4), (1, 2000, 2), (2, 32768, 48), (1, 100000, 1), (3, 5000, 7)):
        nseg, segc = plan(b, L, H, 148)
        nC = -(-L // 63)
        if nseg > 1:
            assert (nseg - 1) * segc < nC <= nseg * segc and segc >= 8
            assert b * H * nseg <= 2 * 148
    n, c = ctypes.c_int32(), ctypes.c_int32()
    assert lib.m3ssd_test_fwd_split_plan(1, -1, 1, 148, ctypes.byref(n), ctypes.byref(c)) == \
        m3.ERR_INVALID_ARG
    assert lib.m3ssd_test_fwd_split_plan(1, 1, 1, 148, None, ctypes.byref(c)) == m3.ERR_INVALID_ARG


def test_fwd_workspace_is_zero_without_a_device(lib):
    """The split depends on the device's SM count; with no device there is no
    split and no workspace (the long workload's shape)."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    d = m3.make_dims(2, 32768, 48, 64, 128, 1, m3.BF16)
    assert lib.m3ssd_fwd_workspace_size(ctypes.byref(d)) == 0


def _step(lib, dims, cache=None, x=FAKE, y=FAKE):
    c = cache or m3.Cache(0x10000, 0x10000, 0x10000, 0x10000)
    return lib.m3ssd_step(ctypes.byref(dims), x, FAKE, None, FAKE, FAKE, FAKE, None, None,
                          ctypes.byref(c), y, None)


def test_step_validation(lib):
    assert _step(lib, _dims(dstate=5)) == m3.ERR_INVALID_ARG
    assert _step(lib, _dims(), x=None) == m3.ERR_INVALID_ARG
    assert _step(lib, _dims(), y=None) == m3.ERR_INVALID_ARG
    assert _step(lib, _dims(), cache=m3.Cache(0x10000, None, 0x10000, 0x10000)) == m3.ERR_INVALID_ARG
    assert _step(lib, _dims(), cache=m3.Cache(0x10000, 0x10002, 0x10000, 0x10000)) == m3.ERR_INVALID_ARG
    assert lib.m3ssd_step(ctypes.byref(_dims()), FAKE, FAKE, None, FAKE, FAKE, FAKE, None, None,
                          None, FAKE, None) == m3.ERR_INVALID_ARG
    assert _step(lib, _dims(batch=0), x=None, y=None) == m3.OK


def _bwd(lib, dims, grads=None, X=FAKE, dY=FAKE, ws=None, ws_bytes=0):
    g = grads if grads is not None else m3.BwdGrads(*([0x10000] * 6 + [None] * 6))
    return lib.m3ssd_bwd(ctypes.byref(dims), X, FAKE, None, FAKE, FAKE, FAKE, None, None, None,
                         None, dY, None, ctypes.byref(g), ws, ws_bytes, None)


def test_bwd_validation(lib):
    d = _dims()
    need = lib.m3ssd_bwd_workspace_size(ctypes.byref(d))
    assert need > 0 and lib.m3ssd_bwd_workspace_size(None) == 0
    assert need == lib.m3ssd_bwd_workspace_size(ctypes.byref(_dims()))
    assert lib.m3ssd_bwd_workspace_size(ctypes.byref(_dims(seqlen=200))) > need
    assert _bwd(lib, d) == m3.ERR_WORKSPACE                              # no workspace
    assert _bwd(lib, d, ws=FAKE, ws_bytes=need - 1) == m3.ERR_WORKSPACE  # too small
    assert _bwd(lib, d, ws=ctypes.c_void_p(0x10010), ws_bytes=need) == m3.ERR_WORKSPACE
    assert _bwd(lib, d, dY=None) == m3.ERR_INVALID_ARG
    assert _bwd(lib, d, X=ctypes.c_void_p(0x10002)) == m3.ERR_INVALID_ARG
    for k in ("dX", "dlogdecay", "dgamma", "dB", "dC"):
        g = m3.BwdGrads(*([0x10000] * 6 + [None] * 6))
        setattr(g, k, None)
        assert _bwd(lib, d, grads=g) == m3.ERR_INVALID_ARG, k
    assert lib.m3ssd_bwd(ctypes.byref(d), FAKE, FAKE, None, FAKE, FAKE, FAKE, None, None, None,
                         None, FAKE, None, None, None, 0, None) == m3.ERR_INVALID_ARG
    assert _bwd(lib, _dims(dstate=512)) == m3.ERR_UNSUPPORTED
    assert _bwd(lib, _dims(batch=0), X=None, dY=None, ws=FAKE, ws_bytes=1 << 20) == m3.OK


def test_mimo_validation(lib):
    d = _dims()
    def fwd(rank, dims=d, X=FAKE):
        return lib.m3ssd_mimo_fwd(ctypes.byref(dims), rank, X, FAKE, None, FAKE, FAKE, FAKE, None,
                                  None, None, FAKE, None, None, None)
    assert fwd(0) == m3.ERR_INVALID_ARG
    assert fwd(9) == m3.ERR_UNSUPPORTED
    assert fwd(2, X=None) == m3.ERR_INVALID_ARG
    assert fwd(2, X=ctypes.c_void_p(0x10002)) == m3.ERR_INVALID_ARG
    assert fwd(2, dims=_dims(chunk=64)) == m3.ERR_UNSUPPORTED
    assert fwd(2, dims=_dims(dstate=7)) == m3.ERR_INVALID_ARG
    assert fwd(2, dims=_dims(batch=0), X=None) == m3.OK
    c = m3.Cache(0x10000, 0x10000, 0x10000, 0x10000)
    def step(rank, cache=c, x=FAKE):
        return lib.m3ssd_mimo_step(ctypes.byref(d), rank, x, FAKE, None, FAKE, FAKE, FAKE, None,
                                   None, ctypes.byref(cache) if cache else None, FAKE, None)
    assert step(0) == m3.ERR_INVALID_ARG
    assert step(9) == m3.ERR_UNSUPPORTED
    assert step(2, cache=None) == m3.ERR_INVALID_ARG
    assert step(2, x=None) == m3.ERR_INVALID_ARG
    assert step(2, cache=m3.Cache(0x10000, None, 0x10000, 0x10000)) == m3.ERR_INVALID_ARG


def test_wait_timeout_query_rejects_null(lib):
    assert lib.m3ssd_device_wait_timeouts(None) == m3.ERR_INVALID_ARG


def test_python_binding_raises_value_error_on_invalid_args(lib):
    with pytest.raises(ValueError):
        m3._check(m3.ERR_INVALID_ARG, "m3ssd_fwd")
    with pytest.raises(m3.M3SSDError):
        m3._check(m3.ERR_UNSUPPORTED, "m3ssd_fwd")


def _block_dims(**kw):
    v = dict(batch=2, seqlen=16, d_model=64, nheads=4, headdim=16, dstate=16, ngroups=2)
    v.update(kw)
    return m3.BlockDims(**v)


def _block_weights(**kw):
    v = {n: 0x10000 for n in m3.BLOCK_WEIGHT_NAMES}
    v.update(kw)
    return m3.BlockWeights(*[v[n] for n in m3.BLOCK_WEIGHT_NAMES], 1e-6)


def test_block_validation(lib):
    d, w = _block_dims(), _block_weights()
    need = lib.m3ssd_block_workspace_size(ctypes.byref(d))
    assert need > 0
    assert lib.m3ssd_block_workspace_size(None) == 0
    assert lib.m3ssd_block_workspace_size(ctypes.byref(_block_dims(nheads=0))) == 0

    def fwd(dims=d, wts=w, u=FAKE, ws=FAKE, ws_bytes=need, cin=None):
        return lib.m3ssd_block_fwd(ctypes.byref(dims) if dims else None,
                                   ctypes.byref(wts) if wts else None, u, FAKE,
                                   ctypes.byref(cin) if cin else None, None, ws, ws_bytes, None)
    assert fwd(dims=None) == m3.ERR_INVALID_ARG
    assert fwd(wts=None) == m3.ERR_INVALID_ARG
    assert fwd(dims=_block_dims(d_model=60)) == m3.ERR_UNSUPPORTED
    assert fwd(dims=_block_dims(dstate=15)) == m3.ERR_INVALID_ARG
    assert fwd(dims=_block_dims(nheads=3)) == m3.ERR_INVALID_ARG   # H % G != 0
    assert fwd(wts=_block_weights(W_in=None)) == m3.ERR_INVALID_ARG
    assert fwd(wts=_block_weights(B_bias=None)) == m3.ERR_INVALID_ARG
    assert fwd(wts=_block_weights(W_out=0x10008)) == m3.ERR_INVALID_ARG   # not 16-byte aligned
    assert fwd(u=None) == m3.ERR_INVALID_ARG
    assert fwd(ws_bytes=need - 1) == m3.ERR_WORKSPACE
    assert fwd(ws=ctypes.c_void_p(0x10010)) == m3.ERR_WORKSPACE
    assert fwd(cin=m3.Cache(0x10000, None, 0x10000, 0x10000)) == m3.ERR_INVALID_ARG
    d0 = _block_dims(batch=0)
    assert fwd(dims=d0, u=None, ws_bytes=lib.m3ssd_block_workspace_size(ctypes.byref(d0))) == m3.OK

    c = m3.Cache(0x10000, 0x10000, 0x10000, 0x10000)
    def step(cache=c, dims=d, ws_bytes=need):
        return lib.m3ssd_block_step(ctypes.byref(dims), ctypes.byref(w), FAKE, FAKE,
                                    ctypes.byref(cache) if cache else None, FAKE, ws_bytes, None)
    assert step(cache=None) == m3.ERR_INVALID_ARG
    assert step(cache=m3.Cache(0x10000, 0x10000, None, 0x10000)) == m3.ERR_INVALID_ARG
    assert step(ws_bytes=16) == m3.ERR_WORKSPACE
    assert step(dims=_block_dims(batch=0)) == m3.OK


def test_backward_refuses_the_finite_check_flag(lib):
    d = _dims(flags=m3.CHECK_FINITE)
    g = m3.BwdGrads(*([0x10000] * 12))
    st = lib.m3ssd_bwd(ctypes.byref(d), FAKE, FAKE, None, FAKE, FAKE, FAKE, None, None, None,
                       None, FAKE, None, ctypes.byref(g), None, 0, None)
    assert st == m3.ERR_UNSUPPORTED


def test_gemm_validation_before_any_device_call(lib):
    g = lib.m3ssd_gemm_bf16
    al = ctypes.c_void_p(0x10000)
    assert g(0, 8, 8, al, al, al, 8, None) == m3.OK          # nothing to do
    assert g(8, 0, 8, al, al, al, 8, None) == m3.OK
    assert g(-1, 8, 8, al, al, al, 8, None) == m3.ERR_INVALID_ARG
    assert g(8, 8, 12, al, al, al, 8, None) == m3.ERR_INVALID_ARG       # K % 8
    assert g(8, 8, 8, al, al, al, 4, None) == m3.ERR_INVALID_ARG        # ldd < N
    assert g(8, 8, 8, None, al, al, 8, None) == m3.ERR_INVALID_ARG
    assert g(8, 8, 8, ctypes.c_void_p(0x10008), al, al, 8, None) == m3.ERR_INVALID_ARG  # A 16 B
    assert g(8, 8, 8, al, al, ctypes.c_void_p(0x10001), 8, None) == m3.ERR_INVALID_ARG  # D 2 B
