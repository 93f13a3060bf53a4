"""GPU parity of the chunked bf16 tensor-core forward (N = 128, P = 64) against
the fp64 oracle: max |gpu - oracle| / RMS(oracle) <= 2e-2 on hT (fp32) and on Y
beyond the half-ulp rounding of its bf16 storage (see rel_max_err_out).

Small cases span several chunks and ragged tails (L = 1, 63, 64, 65, 200, 320)
and every specialised path (beta/theta present or absent, cache inputs, groups,
D absent so that the scan part alone is measured).  The full-size workloads
run in the same launch configuration as the benchmark and are checked on
sampled (b, h) sequences that the oracle computes one by one."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_m3ssd_b200 as m3
from selective_state_space_m3ssd_b200.synth import WORKLOADS, make_inputs, slice_inputs
from tests.gpu_util import angle_err, gpu_fwd, np64, rel_max_err, rel_max_err_out, rms_rel_err, to_dev
from tests.test_gpu_seq_step import with_cache_inputs

pytestmark = pytest.mark.gpu
TOL = 2e-2
# Scan-only outputs (D absent) are heavy tailed (max/RMS up to ~50); they are
# held to the same max bound as every other output.  The kernel's fp16 tensor-core
# operands keep their error near 2^-12 of the large diagonal terms (bf16 rotated
# operands, 2^-9, gave a max error of about 5e-2 of the RMS here).


def check_y(got, ref, with_D):
    assert rel_max_err_out(got, ref, True) <= TOL
    if not with_D:
        assert rms_rel_err(got, ref) <= TOL


BASE = WORKLOADS["siso"].with_(batch=2, nheads=3, seed=321)


@pytest.mark.parametrize("L", [1, 63, 64, 65, 200, 320])
def test_chunked_vs_oracle_lengths(L):
    inp = make_inputs(BASE.with_(seqlen=L))
    ref = oracle.oracle_fwd(**inp)
    got = gpu_fwd(inp, want_cache=True)
    assert rel_max_err_out(got["Y"], ref["Y"], True) <= TOL
    assert rel_max_err(got["hT"], ref["hT"]) <= TOL
    assert angle_err(got["angleT"], ref["angleT"]) <= 1e-5
    np.testing.assert_array_equal(got["xprevT"], ref["xprevT"])
    np.testing.assert_array_equal(got["bprevT"], ref["bprevT"])


@pytest.mark.parametrize("has_beta", [False, True])
@pytest.mark.parametrize("has_theta", [False, True])
@pytest.mark.parametrize("with_D", [False, True])
def test_chunked_paths(has_beta, has_theta, with_D):
    inp = make_inputs(BASE.with_(seqlen=190, has_beta=has_beta, has_theta=has_theta, seed=5))
    if not with_D:
        inp["D"] = None  # the scan part alone, normalised by its own RMS
    ref = oracle.oracle_fwd(**inp)
    got = gpu_fwd(inp)
    check_y(got["Y"], ref["Y"], with_D)
    assert rel_max_err(got["hT"], ref["hT"]) <= TOL


def test_no_device_wait_timed_out():
    """Every bounded tensor-core wait of the runs above completed."""
    gpu_fwd(make_inputs(BASE.with_(seqlen=130, seed=12)))
    assert m3.device_wait_timeouts() == 0


def test_theta_is_not_dropped():
    """Differ-guard: with theta the output must differ from the theta-free run."""
    inp = make_inputs(BASE.with_(seqlen=128, seed=6))
    inp["D"] = None
    a = gpu_fwd(inp)["Y"]
    q = dict(inp)
    q["theta"] = None
    b = gpu_fwd(q)["Y"]
    assert rel_max_err(b, a) > 0.2


@pytest.mark.parametrize("with_D", [False, True])
def test_chunked_with_cache_inputs_and_groups(with_D):
    w = BASE.with_(seqlen=150, nheads=4, ngroups=2, seed=8)
    inp = with_cache_inputs(make_inputs(w))
    if not with_D:
        inp["D"] = None
    ref = oracle.oracle_fwd(**inp)
    got = gpu_fwd(inp, want_cache=True)
    check_y(got["Y"], ref["Y"], with_D)
    assert rel_max_err(got["hT"], ref["hT"]) <= TOL
    assert angle_err(got["angleT"], ref["angleT"]) <= 1e-5
    np.testing.assert_array_equal(got["xprevT"], ref["xprevT"])
    np.testing.assert_array_equal(got["bprevT"], ref["bprevT"])


def test_chunked_continuation_equals_one_pass():
    """fwd(L1) then fwd(L2) from the returned cache == fwd(L1 + L2)."""
    inp = make_inputs(BASE.with_(seqlen=300, seed=9))
    full = gpu_fwd(inp, want_cache=True)
    d = to_dev(inp)
    cut = 130
    part = lambda k, sl: None if d[k] is None else d[k][:, sl].contiguous()
    keys = ("X", "logdecay", "beta", "gamma", "B", "C", "theta")
    Y1, h1, c1 = m3.fwd(*(part(k, slice(0, cut)) for k in keys), d["D"], d["h0"], want_cache=True)
    Y2, h2, c2 = m3.fwd(*(part(k, slice(cut, None)) for k in keys), d["D"], h1,
                        angle0=c1["angle"], xprev0=c1["x_prev"], bprev0=c1["b_prev"],
                        want_cache=True)
    torch.cuda.synchronize()
    Y = np.concatenate([np64(Y1), np64(Y2)], 1)
    assert rel_max_err_out(Y, full["Y"], True) <= TOL
    assert rel_max_err(np64(h2), full["hT"]) <= TOL


def _sampled_full_size(key, pairs):
    """Run the full workload on the GPU in the benchmark's launch configuration,
    recompute the sampled (b, h) sequences (full length) with the oracle and
    hold them to the bound, normalised by the RMS of all sampled oracle outputs
    (an estimate of the output RMS the bound is stated against)."""
    w = WORKLOADS[key]
    inp = make_inputs(w, device="cuda")
    d = to_dev(inp)
    Y, hT, _ = m3.fwd(d["X"], d["logdecay"], d["beta"], d["gamma"], d["B"], d["C"], d["theta"],
                      d["D"], d["h0"])
    torch.cuda.synchronize()
    cpu = {k: (None if v is None else v.cpu()) for k, v in inp.items()}
    by_b = {}
    for bi, hi in pairs:
        by_b.setdefault(bi, []).append(hi)
    gy, ry, gh, rh = [], [], [], []
    for bi, heads in sorted(by_b.items()):
        ref = oracle.oracle_fwd(**slice_inputs(cpu, b=bi, heads=heads))
        gy.append(np64(Y[bi:bi + 1][:, :, heads]))
        gh.append(np64(hT[bi:bi + 1][:, heads]))
        ry.append(ref["Y"])
        rh.append(ref["hT"])
    gy, ry = np.concatenate(gy, 2), np.concatenate(ry, 2)
    gh, rh = np.concatenate(gh, 1), np.concatenate(rh, 1)
    ey, eh = rel_max_err_out(gy, ry, True), rel_max_err(gh, rh)
    assert ey <= TOL and eh <= TOL, (key, ey, eh)


@pytest.mark.parametrize("key,pairs", [
    ("ssd", [(0, 0), (0, 9), (3, 11), (3, 17), (7, 5), (7, 23)]),
    ("siso", [(0, 0), (0, 13), (4, 17), (4, 30), (7, 2), (7, 31)]),
    ("long", [(0, 0), (0, 20), (0, 33), (1, 7), (1, 40), (1, 47)]),
])
def test_full_size_workloads_sampled(key, pairs):
    _sampled_full_size(key, pairs)
