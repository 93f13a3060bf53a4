"""The optional non-finite check (M3SSD_CHECK_FINITE): with the flag, the
forward and the decode step scan the outputs they wrote, and
m3ssd_nonfinite_outputs reports a NaN or an infinity ("Crate burn_mamba",
DENY_NAN / DENY_INF).  A NaN or an infinity is planted in one host input."""
import math

import pytest
import torch

import selective_state_space_m3ssd_b200 as m3
from selective_state_space_m3ssd_b200.synth import WORKLOADS, make_inputs
from tests.gpu_util import to_dev

pytestmark = pytest.mark.gpu
KEYS = ("X", "logdecay", "beta", "gamma", "B", "C", "theta", "D", "h0")

CASES = {"chunked_bf16": WORKLOADS["siso"].with_(batch=1, nheads=2, seqlen=130, seed=31),
         "chunked_f32": WORKLOADS["siso"].with_(batch=1, nheads=2, seqlen=130, seed=35, dtype="f32"),
         "sequential_f32": WORKLOADS["tiny"].with_(seed=32)}


def _fwd(inp, check=True):
    d = to_dev(inp)
    m3.fwd(*(d[k] for k in KEYS), check_finite=check)
    torch.cuda.synchronize()


@pytest.mark.parametrize("case", sorted(CASES))
@pytest.mark.parametrize("bad", [math.nan, math.inf])
def test_forward_reports_a_planted_nonfinite_value(case, bad):
    inp = make_inputs(CASES[case])
    m3.nonfinite_outputs()  # clear
    _fwd(inp)
    assert not m3.nonfinite_outputs()
    for key, idx in (("X", (0, 5, 1, 3)), ("logdecay", (0, 7, 0)), ("C", (0, 9, 0, 2))):
        q = dict(inp)
        q[key] = inp[key].clone()
        q[key][idx] = bad
        _fwd(q)
        assert m3.nonfinite_outputs(), key
        assert not m3.nonfinite_outputs()  # the record was cleared
    _fwd(inp, check=False)  # unchecked calls record nothing
    assert not m3.nonfinite_outputs()


def test_step_reports_a_planted_nonfinite_value():
    w = WORKLOADS["tiny"].with_(seqlen=1, seed=33)
    d = to_dev(make_inputs(w))
    args = [d[k][:, 0].contiguous() for k in ("X", "logdecay", "beta", "gamma", "B", "C", "theta")]
    cache = m3.new_cache(w.batch, w.nheads, w.headdim, w.dstate, w.ngroups, "cuda")
    m3.nonfinite_outputs()
    m3.step(cache, *args, d["D"], check_finite=True)
    assert not m3.nonfinite_outputs()
    args[0][0, 1, 2] = math.nan
    m3.step(cache, *args, d["D"], check_finite=True)
    assert m3.nonfinite_outputs()


def test_mimo_forward_reports_a_planted_nonfinite_value():
    g = torch.Generator().manual_seed(34)
    b, L, H, P, N, G, R = 1, 40, 2, 16, 16, 1, 2
    X = torch.randn(b, L, H, P, R, generator=g)
    logdecay = -torch.rand(b, L, H, generator=g)
    gamma = torch.rand(b, L, H, generator=g)
    Bm = torch.randn(b, L, G, N, R, generator=g) * 0.3
    Cm = torch.randn(b, L, G, N, R, generator=g) * 0.3
    dev = [t.cuda() for t in (X, logdecay, gamma, Bm, Cm)]
    m3.nonfinite_outputs()
    m3.mimo_fwd(dev[0], dev[1], None, dev[2], dev[3], dev[4], check_finite=True)
    assert not m3.nonfinite_outputs()
    dev[0][0, 3, 1, 2, 1] = math.inf
    m3.mimo_fwd(dev[0], dev[1], None, dev[2], dev[3], dev[4], check_finite=True)
    assert m3.nonfinite_outputs()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_chunked_mimo_forward_reports_a_planted_nonfinite_value(dtype):
    from selective_state_space_m3ssd_b200.synth import make_mimo_inputs
    inp = make_mimo_inputs(WORKLOADS["siso"].with_(batch=1, nheads=2, seqlen=50, seed=36,
                                                   dtype=dtype), 4)
    d = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    m3.nonfinite_outputs()
    m3.mimo_fwd(*(d[k] for k in KEYS), check_finite=True)
    assert not m3.nonfinite_outputs()
    d["X"][0, 9, 1, 3, 2] = math.nan
    m3.mimo_fwd(*(d[k] for k in KEYS), check_finite=True)
    assert m3.nonfinite_outputs()
