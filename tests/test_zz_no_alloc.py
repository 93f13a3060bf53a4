"""m3ssd_bwd_noalloc: the backward with the library's own fixed scratch array,
for callers that cannot allocate device memory where they call it.

Two calls in a row must both equal m3ssd_bwd run with a caller-provided
workspace (the backward is deterministic, so the comparison is exact), on every
backward path whose workspace fits in the array: the sequential kernel, the
column-split kernel, the chunked fp32 kernel and the tensor-core kernel.  A
request whose workspace exceeds the array, and invalid dims, are refused before
any device call; wrong-shaped inputs are refused by the binding as for
m3.bwd.
"""
import ctypes

import pytest
import torch

import selective_state_space_m3ssd_b200 as m3
from selective_state_space_m3ssd_b200.synth import WORKLOADS, make_inputs
from tests.gpu_util import to_dev

ARGS = ("X", "logdecay", "beta", "gamma", "B", "C", "theta", "D", "h0")
FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: every call below fails validation


def _call(lib, dims):
    g = m3.BwdGrads(*([0x10000] * 12))
    return lib.m3ssd_bwd_noalloc(None if dims is None else ctypes.byref(dims), FAKE, FAKE, None,
                                 FAKE, FAKE, FAKE, None, None, None, None, FAKE, None,
                                 ctypes.byref(g), None)


def test_noalloc_refuses_requests_larger_than_its_array():
    lib = m3.load()
    big = m3.make_dims(8, 4096, 32, 64, 128, 1, m3.BF16, 0, 0)
    assert lib.m3ssd_bwd_workspace_size(ctypes.byref(big)) > (64 << 20)
    assert _call(lib, big) == m3.ERR_UNSUPPORTED
    assert _call(lib, None) == m3.ERR_INVALID_ARG


def test_noalloc_reports_invalid_dims_before_any_device_call():
    lib = m3.load()
    assert _call(lib, m3.make_dims(1, 8, 2, 8, 7, 1, m3.F32, 0, 0)) == m3.ERR_INVALID_ARG  # odd N
    assert _call(lib, m3.make_dims(1, 8, 3, 8, 8, 2, m3.F32, 0, 0)) == m3.ERR_INVALID_ARG  # H % G
    assert _call(lib, m3.make_dims(1, 8, 2, 8, 8, 1, m3.F32, 0, 1)) == m3.ERR_UNSUPPORTED  # flags


def test_noalloc_binding_checks_every_input_shape():
    inp = make_inputs(WORKLOADS["tiny"].with_(seqlen=8))
    dY = torch.zeros_like(inp["X"])
    args = {k: inp[k] for k in ARGS}
    bad = dict(args, logdecay=inp["logdecay"][:, :4])
    with pytest.raises(ValueError, match="logdecay must have shape"):
        m3.bwd_noalloc(*[bad[k] for k in ARGS], dY=dY)
    with pytest.raises(ValueError, match="dY must have shape"):
        m3.bwd_noalloc(*[args[k] for k in ARGS], dY=dY[:, :4])


CASES = {
    # sequential backward (N = 16)
    "seq": WORKLOADS["tiny"].with_(batch=2, nheads=4, ngroups=2, headdim=16, dstate=16,
                                   seqlen=90, seed=55),
    # column-split backward (N = 128, P = 32)
    "split": WORKLOADS["tiny"].with_(batch=1, nheads=2, headdim=32, dstate=128, seqlen=70,
                                     seed=56),
    # chunked fp32 backward (N = 128, P = 64)
    "chunk": WORKLOADS["tiny"].with_(batch=1, nheads=2, headdim=64, dstate=128, seqlen=140,
                                     seed=57),
    # tensor-core backward (bf16, N = 128, P = 64)
    "tc": WORKLOADS["siso"].with_(batch=1, nheads=2, seqlen=140, seed=58),
}


@pytest.mark.gpu
@pytest.mark.parametrize("case", sorted(CASES))
def test_noalloc_twice_equals_the_workspace_entry_point(case):
    w = CASES[case]
    inp = make_inputs(w)
    gen = torch.Generator().manual_seed(3)
    dY = torch.randn(inp["X"].shape, generator=gen).to(inp["X"].dtype)
    dhT = torch.randn(w.batch, w.nheads, w.dstate, w.headdim, generator=gen)
    dims = m3.make_dims(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups,
                        m3.BF16 if w.dtype == "bf16" else m3.F32, 0, 0)
    assert 0 < m3.bwd_workspace_size(dims) <= (64 << 20)
    d = to_dev(inp)
    args = [d.get(k) for k in ARGS]
    ref = m3.bwd(*args, dY=dY.cuda(), dhT=dhT.cuda())
    first = m3.bwd_noalloc(*args, dY=dY.cuda(), dhT=dhT.cuda())
    second = m3.bwd_noalloc(*args, dY=dY.cuda(), dhT=dhT.cuda())
    torch.cuda.synchronize()
    for k in ref:
        assert torch.equal(first[k], ref[k]), k
        assert torch.equal(second[k], ref[k]), k
