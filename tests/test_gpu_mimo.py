"""MIMO rank-R forward and decode step through the C ABI against the fp64 MIMO
oracle (which is itself pinned to the SISO oracle).

Bars as the SISO sequential path: max |err| / RMS <= 1e-4 with fp32 inputs and
outputs (fp32 state and arithmetic, sequential in time); with bf16 X, B, C, Y
the inputs are rounded before either side sees them.  The output is allowed
its final bf16 rounding (half an ulp) plus 1e-4 of the RMS: the fp32
arithmetic before that rounding is the same as on the fp32 path.
"""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_m3ssd_b200 as m3
from tests.gpu_util import angle_err, rel_max_err, rel_max_err_out
from tests.test_oracle_mimo import make_mimo

pytestmark = pytest.mark.gpu
TOL = 1e-4


def prep(inp, dtype):
    """Round X, B, C to the device dtype; return (rounded fp64 inputs, device tensors)."""
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    ref, dev = {}, {}
    for k, v in inp.items():
        if v is None:
            ref[k], dev[k] = None, None
            continue
        t = torch.from_numpy(v)
        if k in ("X", "B", "C"):
            t = t.to(td)
            ref[k] = t.double().numpy()
            dev[k] = t.cuda().contiguous()
        else:
            ref[k] = v
            dev[k] = t.float().cuda().contiguous()
    return ref, dev


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("seed,kw", [(1, {}), (2, {"R": 4, "L": 70, "N": 16, "P": 16}),
                                     (3, {"R": 8, "G": 1, "N": 8}), (4, {"beta": False}),
                                     (5, {"theta": False, "cache": False}), (6, {"R": 1})])
def test_mimo_fwd_matches_oracle(dtype, seed, kw):
    ref_in, d = prep(make_mimo(seed, **kw), dtype)
    ref = oracle.oracle_mimo_fwd(**ref_in)
    Y, hT, cache = m3.mimo_fwd(d["X"], d["logdecay"], d["beta"], d["gamma"], d["B"], d["C"],
                               d["theta"], d["D"], d["h0"], angle0=d["angle0"],
                               xprev0=d["xprev0"], bprev0=d["bprev0"], want_cache=True)
    torch.cuda.synchronize()
    assert rel_max_err_out(Y.double().cpu().numpy(), ref["Y"], dtype == "bf16") <= TOL
    assert rel_max_err(hT.double().cpu().numpy(), ref["hT"]) <= TOL
    assert angle_err(cache["angle"].double().cpu().numpy(), ref["angleT"]) <= 1e-5
    np.testing.assert_array_equal(cache["x_prev"].double().cpu().numpy(), ref["xprevT"])
    np.testing.assert_array_equal(cache["b_prev"].double().cpu().numpy(), ref["bprevT"])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_mimo_prefill_then_decode_matches_oracle(dtype):
    inp = make_mimo(9, b=3, L=40, H=4, G=2, P=16, N=16, R=4)
    ref_in, d = prep(inp, dtype)
    full = oracle.oracle_mimo_fwd(**ref_in)
    L1 = 25
    pre = {k: (v[:, :L1].contiguous() if k in ("X", "logdecay", "beta", "gamma", "B", "C", "theta")
               and v is not None else v) for k, v in d.items()}
    _, hT, cache = m3.mimo_fwd(pre["X"], pre["logdecay"], pre["beta"], pre["gamma"], pre["B"],
                               pre["C"], pre["theta"], pre["D"], pre["h0"], angle0=pre["angle0"],
                               xprev0=pre["xprev0"], bprev0=pre["bprev0"], want_cache=True)
    cache["ssm"] = hT
    for t in range(L1, 40):
        y = m3.mimo_step(cache, d["X"][:, t].contiguous(), d["logdecay"][:, t].contiguous(),
                         d["beta"][:, t].contiguous(), d["gamma"][:, t].contiguous(),
                         d["B"][:, t].contiguous(), d["C"][:, t].contiguous(),
                         d["theta"][:, t].contiguous(), d["D"])
        torch.cuda.synchronize()
        assert rel_max_err_out(y.double().cpu().numpy(), full["Y"][:, t], dtype == "bf16") <= TOL, t
    assert rel_max_err(cache["ssm"].double().cpu().numpy(), full["hT"]) <= TOL
    assert angle_err(cache["angle"].double().cpu().numpy(), full["angleT"]) <= 1e-5


def test_mimo_rank_one_equals_siso_path():
    # at R = 1 the MIMO entry point computes what the SISO entry point does
    inp = make_mimo(12, b=2, L=30, H=2, G=1, P=8, N=8, R=1)
    _, d = prep(inp, "f32")
    Ym, hm, _ = m3.mimo_fwd(d["X"], d["logdecay"], d["beta"], d["gamma"], d["B"], d["C"],
                            d["theta"], d["D"], d["h0"])
    Ys, hs, _ = m3.fwd(d["X"][..., 0].contiguous(), d["logdecay"], d["beta"], d["gamma"],
                       d["B"][..., 0].contiguous(), d["C"][..., 0].contiguous(), d["theta"],
                       d["D"], d["h0"])
    torch.cuda.synchronize()
    assert rel_max_err(Ym[..., 0].double().cpu().numpy(), Ys.double().cpu().numpy()) <= 1e-5
    assert rel_max_err(hm.double().cpu().numpy(), hs.double().cpu().numpy()) <= 1e-5


def test_mimo_rejects_unsupported_rank():
    _, d = prep(make_mimo(13, R=3), "f32")
    bad = d["X"].repeat(1, 1, 1, 1, 3)  # R = 9
    with pytest.raises(m3.M3SSDError):
        m3.mimo_fwd(bad, d["logdecay"], d["beta"], d["gamma"], d["B"].repeat(1, 1, 1, 1, 3),
                    d["C"].repeat(1, 1, 1, 1, 3))


@pytest.mark.parametrize("R,aligned", [(1, True), (2, True), (3, True), (4, True), (4, False)])
def test_mimo_decode_steps_at_wide_heads(R, aligned):
    # P = 64, N = 128: the specialised step when the cache state is 16-byte
    # aligned, the general mapping when it starts 4 bytes past that
    inp = make_mimo(21 + R, b=2, L=6, H=4, G=2, P=64, N=128, R=R)
    ref_in, d = prep(inp, "bf16")
    full = oracle.oracle_mimo_fwd(**ref_in)
    L1 = 2
    pre = {k: (v[:, :L1] if k in ("X", "logdecay", "beta", "gamma", "B", "C", "theta")
               and v is not None else v) for k, v in ref_in.items()}
    p = oracle.oracle_mimo_fwd(**pre)
    n = p["hT"].size
    buf = torch.zeros(n + 4, dtype=torch.float32, device="cuda")
    ssm = buf[(0 if aligned else 1):][:n].view(p["hT"].shape)
    ssm.copy_(torch.from_numpy(p["hT"]).float())
    assert (ssm.data_ptr() % 16 == 0) == aligned
    cache = {"angle": torch.from_numpy(p["angleT"]).float().cuda(), "ssm": ssm,
             "x_prev": torch.from_numpy(p["xprevT"]).float().cuda(),
             "b_prev": torch.from_numpy(p["bprevT"]).float().cuda()}
    for t in range(L1, 6):
        y = m3.mimo_step(cache, d["X"][:, t].contiguous(), d["logdecay"][:, t].contiguous(),
                         d["beta"][:, t].contiguous(), d["gamma"][:, t].contiguous(),
                         d["B"][:, t].contiguous(), d["C"][:, t].contiguous(),
                         d["theta"][:, t].contiguous(), d["D"])
        torch.cuda.synchronize()
        assert rel_max_err_out(y.double().cpu().numpy(), full["Y"][:, t], True) <= TOL, t
    assert rel_max_err(ssm.double().cpu().numpy(), full["hT"]) <= TOL
