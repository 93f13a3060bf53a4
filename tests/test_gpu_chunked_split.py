"""GPU parity of the sequence-split chunked bf16 forward against the fp64
oracle, at the bar of the unsplit kernel (max |gpu - oracle| / RMS(oracle) <=
2e-2 beyond the bf16 rounding of Y; x_prev and b_prev exact, the cache angle
within 1e-4, its sums running in another order than the unsplit walk's).

The split engages by itself for few (b, h) sequences of at least 16 chunks
(the binding passes the workspace m3ssd_fwd_workspace_size asks for); each case
first checks that it does.  Cases cover segment boundaries inside and at the
end of the sequence, a ragged last chunk, every input path (beta / theta / D
present or absent, an initial angle without theta, cache inputs, groups) and
the full long workload (b2 L32768 H48: three segments of 174 chunks), whose
sampled sequences are checked in test_gpu_chunked.py."""
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
BASE = WORKLOADS["siso"].with_(batch=1, nheads=2, seed=404)


def sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def assert_splits(w):
    nseg, segc = m3.fwd_split_plan(w.batch, w.seqlen, w.nheads, sms())
    assert nseg > 1, (w, nseg)
    d = m3.make_dims(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups, m3.BF16)
    assert m3.fwd_workspace_size(d) > 0
    return nseg, segc


def check_all(got, ref, with_D=True, cache=True):
    assert rel_max_err_out(got["Y"], ref["Y"], True) <= TOL
    if not with_D:
        assert rms_rel_err(got["Y"], ref["Y"]) <= TOL
    assert rel_max_err(got["hT"], ref["hT"]) <= TOL
    if cache:
        assert angle_err(got["angleT"], ref["angleT"]) <= 1e-4
        np.testing.assert_array_equal(got["xprevT"], ref["xprevT"])
        np.testing.assert_array_equal(got["bprevT"], ref["bprevT"])


@pytest.mark.parametrize("L", [1008, 1529, 2000, 4096])
def test_split_vs_oracle_with_cache_inputs(L):
    """1008 = 16 full chunks (two segments, no ragged tail); 1529 and 2000 end in
    a partial chunk; 4096 cuts 65 chunks into eight segments."""
    w = BASE.with_(seqlen=L, nheads=1 if L == 4096 else 2)
    assert_splits(w)
    inp = with_cache_inputs(make_inputs(w))
    ref = oracle.oracle_fwd(**inp)
    got = gpu_fwd(inp, want_cache=True)
    check_all(got, ref)


@pytest.mark.parametrize("has_beta,has_theta", [(False, False), (True, False), (False, True),
                                                (True, True)])
@pytest.mark.parametrize("with_D", [False, True])
def test_split_paths(has_beta, has_theta, with_D):
    w = BASE.with_(seqlen=1100, nheads=3, has_beta=has_beta, has_theta=has_theta, seed=41)
    assert_splits(w)
    inp = make_inputs(w)
    if not with_D:
        inp["D"] = None
    ref = oracle.oracle_fwd(**inp)
    got = gpu_fwd(inp, want_cache=True)
    check_all(got, ref, with_D)


def test_split_groups_and_cache():
    w = BASE.with_(seqlen=1300, nheads=4, ngroups=2, seed=42)
    assert_splits(w)
    inp = with_cache_inputs(make_inputs(w))
    inp["D"] = None
    ref = oracle.oracle_fwd(**inp)
    got = gpu_fwd(inp, want_cache=True)
    check_all(got, ref, with_D=False)


def test_split_start_angle_without_theta():
    """The rotation by the cache's angle alone (theta absent): the segment pass
    rotates nothing and the combine step turns every segment state by angle0."""
    w = BASE.with_(seqlen=1200, has_theta=False, seed=43)
    assert_splits(w)
    inp = with_cache_inputs(make_inputs(w))
    ref = oracle.oracle_fwd(**inp)
    got = gpu_fwd(inp, want_cache=True)
    check_all(got, ref)


def test_split_matches_unsplit_walk():
    """The same two sequences inside a batch of 64 (128 sequences: no split):
    both runs meet the bar against the oracle, and the split's error is no
    larger than the unsplit walk's beyond a margin for the different rounding
    order (its segment states accumulate whole segments in one fp32 product)."""
    w = BASE.with_(seqlen=1600, seed=44)
    assert_splits(w)
    inp = with_cache_inputs(make_inputs(w))
    ref = oracle.oracle_fwd(**inp)
    split = gpu_fwd(inp, want_cache=True)
    wide = {k: (v if v is None or k == "D" else torch.cat([v] * 64, 0)) for k, v in inp.items()}
    assert m3.fwd_split_plan(64, w.seqlen, w.nheads, sms())[0] == 1
    whole = gpu_fwd(wide, want_cache=True)
    ey_s = rel_max_err_out(split["Y"], ref["Y"], True)
    ey_w = rel_max_err_out(whole["Y"][:1], ref["Y"], True)
    eh_s = rel_max_err(split["hT"], ref["hT"])
    eh_w = rel_max_err(whole["hT"][:1], ref["hT"])
    msg = (ey_s, ey_w, eh_s, eh_w)
    assert max(msg) <= TOL, msg
    assert ey_s <= 1.5 * ey_w + 1e-3 and eh_s <= 1.5 * eh_w + 1e-3, msg
    assert angle_err(split["angleT"], whole["angleT"][:1]) <= 1e-4


def test_split_continuation_equals_one_pass():
    """A split forward of the first part, then one of the rest from its cache,
    equals one split forward over the whole sequence."""
    w = BASE.with_(seqlen=2600, seed=45)
    inp = make_inputs(w)
    full = gpu_fwd(inp, want_cache=True)
    d = to_dev(inp)
    cut = 63 * 20 + 5
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


def test_split_no_device_wait_timed_out():
    gpu_fwd(make_inputs(BASE.with_(seqlen=1400, seed=46)))
    assert m3.device_wait_timeouts() == 0


@pytest.mark.parametrize("H", [2 * 148 // 3, 2 * 148 // 3 + 1])
def test_split_threshold_sampled(H):
    """At the plan's threshold (b H = 98 sequences split into segments on 148 SMs,
    99 do not), every head's outputs match the oracle on sampled heads."""
    if sms() != 148:
        pytest.skip("threshold sizes are for a 148-SM device")
    w = BASE.with_(nheads=H, seqlen=1100, seed=47)
    splits = m3.fwd_split_plan(1, w.seqlen, H, sms())[0] > 1
    assert splits == (H <= 98)
    inp = make_inputs(w)
    got = gpu_fwd(inp)
    heads = [0, H // 2, H - 1]
    ref = oracle.oracle_fwd(**slice_inputs(inp, b=0, heads=heads))
    assert rel_max_err_out(got["Y"][:, :, heads], ref["Y"], True) <= TOL
    assert rel_max_err(got["hT"][:, heads], ref["hT"]) <= TOL


def test_split_needs_its_workspace():
    """The C ABI's contract for a shape that splits: without the workspace that
    m3ssd_fwd_workspace_size asks for the call is refused (M3SSD_ERR_WORKSPACE,
    nothing launched), with it the call succeeds and matches the binding's run."""
    import ctypes
    w = BASE.with_(seqlen=1529, seed=48)
    assert_splits(w)
    d = to_dev(make_inputs(w))
    b, L, H, P = d["X"].shape
    dims = m3.make_dims(b, L, H, P, 128, 1, m3.BF16)
    need = m3.fwd_workspace_size(dims)
    Y = torch.empty_like(d["X"])
    lib = m3.load()
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    args = [p(d[k]) for k in ("X", "logdecay", "beta", "gamma", "B", "C", "theta", "D", "h0")]
    call = lambda ws, nbytes: lib.m3ssd_fwd(ctypes.byref(dims), *args, p(Y), None, None, ws,
                                            nbytes, None)
    assert call(None, 0) == m3.ERR_WORKSPACE
    small = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    assert call(p(small), need - 256) == m3.ERR_WORKSPACE
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    assert call(p(ws), need) == m3.OK
    torch.cuda.synchronize()
    ref, _, _ = m3.fwd(d["X"], d["logdecay"], d["beta"], d["gamma"], d["B"], d["C"], d["theta"],
                       d["D"], d["h0"])
    torch.cuda.synchronize()
    assert torch.equal(Y, ref)  # the same launches on the same inputs
