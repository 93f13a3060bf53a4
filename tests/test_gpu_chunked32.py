"""GPU parity of the chunked fp32 forward (fp32 X, B, C, Y at N = 128, P = 64;
tensor-core products on fp16 high / low operand parts) against the fp64
oracle at the fp32 bar: max |gpu - oracle| / RMS(oracle) <= 1e-4 on Y and hT.

Small cases span several chunks and ragged tails (L = 1, 63, 64, 65, 200,
320) and every path (beta / theta / D absent, cache inputs, groups); a
two-call continuation equals one pass; the decode workload's 512-token
prefill is checked on sampled sequences in the benchmark's configuration."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_m3ssd_b200 as m3
from selective_state_space_m3ssd_b200.synth import DECODE_PREFILL, WORKLOADS, make_inputs, slice_inputs
from tests.gpu_util import angle_err, gpu_fwd, np64, rel_max_err, rms_rel_err, to_dev
from tests.test_gpu_seq_step import with_cache_inputs

pytestmark = pytest.mark.gpu
TOL = 1e-4
BASE = WORKLOADS["siso"].with_(batch=2, nheads=3, dtype="f32", seed=432)


@pytest.mark.parametrize("L", [1, 63, 64, 65, 200, 320])
def test_chunked32_vs_oracle_lengths(L):
    inp = make_inputs(BASE.with_(seqlen=L))
    ref = oracle.oracle_fwd(**inp)
    got = gpu_fwd(inp, want_cache=True)
    assert rel_max_err(got["Y"], ref["Y"]) <= TOL
    assert rel_max_err(got["hT"], ref["hT"]) <= TOL
    assert angle_err(got["angleT"], ref["angleT"]) <= 1e-5
    np.testing.assert_array_equal(got["xprevT"], ref["xprevT"])
    np.testing.assert_array_equal(got["bprevT"], ref["bprevT"])


@pytest.mark.parametrize("has_beta", [False, True])
@pytest.mark.parametrize("has_theta", [False, True])
@pytest.mark.parametrize("with_D", [False, True])
def test_chunked32_paths(has_beta, has_theta, with_D):
    inp = make_inputs(BASE.with_(seqlen=190, has_beta=has_beta, has_theta=has_theta, seed=15))
    if not with_D:
        inp["D"] = None
    ref = oracle.oracle_fwd(**inp)
    got = gpu_fwd(inp)
    assert rel_max_err(got["Y"], ref["Y"]) <= TOL
    if not with_D:
        assert rms_rel_err(got["Y"], ref["Y"]) <= TOL
    assert rel_max_err(got["hT"], ref["hT"]) <= TOL


def test_chunked32_cache_inputs_and_groups():
    w = BASE.with_(seqlen=150, nheads=4, ngroups=2, seed=18)
    inp = with_cache_inputs(make_inputs(w))
    ref = oracle.oracle_fwd(**inp)
    got = gpu_fwd(inp, want_cache=True)
    assert rel_max_err(got["Y"], ref["Y"]) <= TOL
    assert rel_max_err(got["hT"], ref["hT"]) <= TOL
    assert angle_err(got["angleT"], ref["angleT"]) <= 1e-5
    np.testing.assert_array_equal(got["xprevT"], ref["xprevT"])
    np.testing.assert_array_equal(got["bprevT"], ref["bprevT"])
    assert m3.device_wait_timeouts() == 0


def test_chunked32_continuation_equals_one_pass():
    inp = make_inputs(BASE.with_(seqlen=300, seed=19))
    full = gpu_fwd(inp, want_cache=True)
    d = to_dev(inp)
    cut = 130
    part = lambda k, sl: None if d[k] is None else d[k][:, sl].contiguous()
    keys = ("X", "logdecay", "beta", "gamma", "B", "C", "theta")
    _, h1, c1 = m3.fwd(*(part(k, slice(0, cut)) for k in keys), d["D"], d["h0"], want_cache=True)
    Y2, h2, _ = m3.fwd(*(part(k, slice(cut, None)) for k in keys), d["D"], h1,
                       angle0=c1["angle"], xprev0=c1["x_prev"], bprev0=c1["b_prev"],
                       want_cache=True)
    torch.cuda.synchronize()
    assert rel_max_err(np64(Y2), full["Y"][:, cut:]) <= TOL
    assert rel_max_err(np64(h2), full["hT"]) <= TOL


def test_decode_prefill_sampled():
    """The decode workload's 512-token fp32 prefill (b256 H32), sampled."""
    w = WORKLOADS["decode"].with_(seqlen=DECODE_PREFILL)
    inp = make_inputs(w, device="cuda")
    Y, hT, _ = m3.fwd(inp["X"], inp["logdecay"], inp["beta"], inp["gamma"], inp["B"], inp["C"],
                      inp["theta"], inp["D"], inp["h0"])
    torch.cuda.synchronize()
    cpu = {k: (None if v is None else v.cpu()) for k, v in inp.items()}
    gy, ry, gh, rh = [], [], [], []
    for bi, heads in ((0, [0, 5]), (131, [17]), (255, [31])):
        ref = oracle.oracle_fwd(**slice_inputs(cpu, b=bi, heads=heads))
        gy.append(np64(Y[bi:bi + 1][:, :, heads]))
        gh.append(np64(hT[bi:bi + 1][:, heads]))
        ry.append(ref["Y"])
        rh.append(ref["hT"])
    assert rel_max_err(np.concatenate(gy, 2), np.concatenate(ry, 2)) <= TOL
    assert rel_max_err(np.concatenate(gh, 1), np.concatenate(rh, 1)) <= TOL
