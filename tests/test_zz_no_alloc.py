"""m3ssd_bwd_noalloc: the backward with the library's own fixed scratch array.

Two calls in a row must both equal m3ssd_bwd run with a caller-provided
workspace (the backward is deterministic, so the comparison is exact); a
request whose workspace exceeds the array is refused before any device call.
"""
import ctypes

import pytest
import torch

import selective_state_space_m3ssd_b200 as m3
from selective_state_space_m3ssd_b200.synth import WORKLOADS, make_inputs
from tests.gpu_util import to_dev

ARGS = ("X", "logdecay", "beta", "gamma", "B", "C", "theta", "D", "h0")


def test_noalloc_refuses_requests_larger_than_its_array():
    lib = m3.load()
    big = m3.make_dims(8, 4096, 32, 64, 128, 1, m3.BF16, 0, 0)
    assert lib.m3ssd_bwd_workspace_size(ctypes.byref(big)) > (64 << 20)
    fake = ctypes.c_void_p(0x10000)
    g = m3.BwdGrads(*([0x10000] * 12))
    st = lib.m3ssd_bwd_noalloc(ctypes.byref(big), fake, fake, None, fake, fake, fake, None, None,
                               None, None, fake, None, ctypes.byref(g), None)
    assert st == m3.ERR_UNSUPPORTED
    assert lib.m3ssd_bwd_noalloc(None, fake, fake, None, fake, fake, fake, None, None, None, None,
                                 fake, None, ctypes.byref(g), None) == m3.ERR_INVALID_ARG


@pytest.mark.gpu
def test_noalloc_twice_equals_the_workspace_entry_point():
    w = WORKLOADS["tiny"].with_(batch=2, nheads=4, ngroups=2, headdim=16, dstate=16, seqlen=90,
                                seed=55)
    inp = make_inputs(w)
    gen = torch.Generator().manual_seed(3)
    dY = torch.randn(inp["X"].shape, generator=gen)
    dhT = torch.randn(2, 4, 16, 16, generator=gen)
    d = to_dev(inp)
    args = [d.get(k) for k in ARGS]
    ref = m3.bwd(*args, dY=dY.cuda(), dhT=dhT.cuda())
    first = m3.bwd_noalloc(*args, dY=dY.cuda(), dhT=dhT.cuda())
    second = m3.bwd_noalloc(*args, dY=dY.cuda(), dhT=dhT.cuda())
    torch.cuda.synchronize()
    for k in ref:
        assert torch.equal(first[k], ref[k]), k
        assert torch.equal(second[k], ref[k]), k
