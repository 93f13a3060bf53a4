"""GPU parity of the chunked bf16 forward at every chunk length Q in {64, 128,
256} (m3ssd_dims.chunk): the intra-chunk quadratic form spans Q rows and the
state passes between chunks.  Same bar as the 64-row kernel: max |gpu -
oracle| / RMS(oracle) <= 2e-2 on hT and on Y beyond the half-ulp rounding of
its bf16 storage (and 2e-2 in RMS with D absent).  Small cases span several
chunks with ragged tails at each Q, every path (beta / theta / D absent, cache
inputs, groups); the long workload runs at each Q in the benchmark's launch
configuration, checked on sampled sequences; the lengths agree with each
other within the bar."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_m3ssd_b200 as m3
from selective_state_space_m3ssd_b200.synth import WORKLOADS, make_inputs, slice_inputs
from tests.gpu_util import angle_err, np64, rel_max_err, rel_max_err_out, rms_rel_err, to_dev
from tests.test_gpu_seq_step import with_cache_inputs

pytestmark = pytest.mark.gpu
TOL = 2e-2
BASE = WORKLOADS["siso"].with_(batch=2, nheads=3, seed=654)
KEYS = ("X", "logdecay", "beta", "gamma", "B", "C", "theta", "D", "h0")


def run(inp, chunk, want_cache=False):
    d = to_dev(inp)
    extra = {k: d.pop(k) for k in ("angle0", "xprev0", "bprev0") if k in d}
    Y, hT, cache = m3.fwd(*(d[k] for k in KEYS), chunk=chunk, want_cache=want_cache, **extra)
    torch.cuda.synchronize()
    out = {"Y": np64(Y), "hT": np64(hT)}
    if cache is not None:
        out.update({"angleT": np64(cache["angle"]), "xprevT": np64(cache["x_prev"]),
                    "bprevT": np64(cache["b_prev"])})
    return out


@pytest.mark.parametrize("Q", [128, 256])
@pytest.mark.parametrize("L", [1, 127, 128, 129, 255, 256, 257, 600])
def test_chunk_lengths_vs_oracle(Q, L):
    inp = with_cache_inputs(make_inputs(BASE.with_(seqlen=L, seed=700 + L)))
    ref = oracle.oracle_fwd(**inp)
    got = run(inp, Q, want_cache=True)
    assert rel_max_err_out(got["Y"], ref["Y"], True) <= TOL
    assert rel_max_err(got["hT"], ref["hT"]) <= TOL
    assert angle_err(got["angleT"], ref["angleT"]) <= 1e-5
    np.testing.assert_array_equal(got["xprevT"], ref["xprevT"])
    np.testing.assert_array_equal(got["bprevT"], ref["bprevT"])


@pytest.mark.parametrize("Q", [128, 256])
@pytest.mark.parametrize("has_beta,has_theta,with_D", [(False, False, True), (True, False, False),
                                                       (False, True, False), (True, True, False)])
def test_chunk_lengths_paths(Q, has_beta, has_theta, with_D):
    inp = make_inputs(BASE.with_(seqlen=300, has_beta=has_beta, has_theta=has_theta, seed=17,
                                 nheads=4, ngroups=2))
    if not with_D:
        inp["D"] = None
    ref = oracle.oracle_fwd(**inp)
    got = run(inp, Q)
    assert rel_max_err_out(got["Y"], ref["Y"], True) <= TOL
    if not with_D:
        assert rms_rel_err(got["Y"], ref["Y"]) <= TOL
    assert rel_max_err(got["hT"], ref["hT"]) <= TOL
    assert m3.device_wait_timeouts() == 0


def test_chunk_lengths_agree():
    inp = make_inputs(BASE.with_(seqlen=1000, seed=19))
    outs = {Q: run(inp, Q) for Q in (64, 128, 256)}
    for Q in (128, 256):
        assert rel_max_err_out(outs[Q]["Y"], outs[64]["Y"], True) <= TOL
        assert rel_max_err(outs[Q]["hT"], outs[64]["hT"]) <= TOL


def test_chunk_longer_than_64_refused_off_the_bf16_path():
    inp = make_inputs(BASE.with_(seqlen=50, dtype="f32"))
    with pytest.raises(m3.M3SSDError) as e:
        run(inp, 128)
    assert e.value.status == m3.ERR_UNSUPPORTED


@pytest.mark.parametrize("Q", [64, 128, 256])
def test_long_workload_sampled_at_each_chunk_length(Q):
    w = WORKLOADS["long"]
    inp = make_inputs(w, device="cuda")
    Y, hT, _ = m3.fwd(*(inp[k] for k in KEYS), chunk=Q)
    torch.cuda.synchronize()
    cpu = {k: (None if v is None else v.cpu()) for k, v in inp.items()}
    gy, ry, gh, rh = [], [], [], []
    for bi, heads in ((0, [0]), (1, [47])):
        ref = oracle.oracle_fwd(**slice_inputs(cpu, b=bi, heads=heads))
        gy.append(np64(Y[bi:bi + 1][:, :, heads]))
        gh.append(np64(hT[bi:bi + 1][:, heads]))
        ry.append(ref["Y"])
        rh.append(ref["hT"])
    assert rel_max_err_out(np.concatenate(gy, 2), np.concatenate(ry, 2), True) <= TOL
    assert rel_max_err(np.concatenate(gh, 1), np.concatenate(rh, 1)) <= TOL
