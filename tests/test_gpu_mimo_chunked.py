"""GPU parity of the chunked bf16 tensor-core MIMO forward (N = 128, P = 64,
R = 1, 2, 4, 8; 64 (token, rank) rows per chunk) against the fp64 MIMO oracle:
max |gpu - oracle| / RMS(oracle) <= 2e-2 on hT and on Y beyond the half-ulp
rounding of its bf16 storage, the bar of the bf16 SISO chunked forward.

Small cases span several chunks (64/R - 1 tokens each) and ragged tails, with
beta / theta / cache inputs present or absent and D absent (the scan part
alone, also held to 2e-2 in RMS); a prefill through the chunked kernel is
continued by decode steps; the full rank-4 prefill workload is checked on
sampled (b, h) sequences."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_m3ssd_b200 as m3
from selective_state_space_m3ssd_b200.synth import MIMO_WORKLOADS, WORKLOADS, make_mimo_inputs
from tests.gpu_util import angle_err, rel_max_err, rel_max_err_out, rms_rel_err

pytestmark = pytest.mark.gpu
TOL = 2e-2
KEYS = ("X", "logdecay", "beta", "gamma", "B", "C", "theta", "D", "h0")
BASE = WORKLOADS["siso"].with_(batch=2, nheads=3, seed=77)


def f64(v):
    return None if v is None else v.detach().to("cpu").double().numpy()


def with_cache(inp, R, seed):
    g = torch.Generator().manual_seed(seed)
    b, _, H, P, _ = inp["X"].shape
    G, N = inp["B"].shape[2], inp["B"].shape[3]
    q = dict(inp)
    q["angle0"] = torch.rand(b, H, N // 2, generator=g) * 6 - 3
    q["xprev0"] = torch.randn(b, H, P, R, generator=g).bfloat16().float()
    q["bprev0"] = (torch.randn(b, G, N, R, generator=g) / N ** 0.5).bfloat16().float()
    return q


def run(inp, want_cache=False):
    d = {k: (None if v is None else v.cuda().contiguous()) for k, v in inp.items()}
    Y, hT, cache = m3.mimo_fwd(*(d[k] for k in KEYS), angle0=d.get("angle0"),
                               xprev0=d.get("xprev0"), bprev0=d.get("bprev0"),
                               want_cache=want_cache)
    torch.cuda.synchronize()
    return Y, hT, cache


def reference(inp):
    return oracle.oracle_mimo_fwd(**{k: f64(v) for k, v in inp.items()})


@pytest.mark.parametrize("R", [1, 2, 4, 8])
@pytest.mark.parametrize("L", [1, 7, 31, 64, 129, 200])
def test_mimo_chunked_vs_oracle_lengths(R, L):
    inp = with_cache(make_mimo_inputs(BASE.with_(seqlen=L, seed=100 + L), R), R, L)
    ref = reference(inp)
    Y, hT, cache = run(inp, want_cache=True)
    assert rel_max_err_out(f64(Y), ref["Y"], True) <= TOL
    assert rel_max_err(f64(hT), ref["hT"]) <= TOL
    assert angle_err(f64(cache["angle"]), ref["angleT"]) <= 1e-5
    np.testing.assert_array_equal(f64(cache["x_prev"]), ref["xprevT"])
    np.testing.assert_array_equal(f64(cache["b_prev"]), ref["bprevT"])


@pytest.mark.parametrize("R", [2, 4, 8])
@pytest.mark.parametrize("has_beta,has_theta,with_D", [(False, False, True), (True, False, False),
                                                       (False, True, False), (True, True, False)])
def test_mimo_chunked_paths(R, has_beta, has_theta, with_D):
    w = BASE.with_(seqlen=150, has_beta=has_beta, has_theta=has_theta, seed=9, ngroups=1)
    inp = make_mimo_inputs(w, R)
    if not with_D:
        inp["D"] = None
    ref = reference(inp)
    Y, hT, _ = run(inp)
    assert rel_max_err_out(f64(Y), ref["Y"], True) <= TOL
    if not with_D:
        assert rms_rel_err(f64(Y), ref["Y"]) <= TOL
    assert rel_max_err(f64(hT), ref["hT"]) <= TOL


def test_mimo_chunked_groups():
    w = BASE.with_(seqlen=90, nheads=4, ngroups=2, seed=10)
    inp = make_mimo_inputs(w, 4)
    ref = reference(inp)
    Y, hT, _ = run(inp)
    assert rel_max_err_out(f64(Y), ref["Y"], True) <= TOL
    assert rel_max_err(f64(hT), ref["hT"]) <= TOL
    assert m3.device_wait_timeouts() == 0


def test_mimo_chunked_prefill_then_decode():
    """The chunked kernel's cache outputs continue through m3ssd_mimo_step."""
    R, L, L1 = 4, 60, 37
    inp = with_cache(make_mimo_inputs(BASE.with_(seqlen=L, seed=11), R), R, 12)
    ref = reference(inp)
    pre = {k: (v[:, :L1] if k in ("X", "logdecay", "beta", "gamma", "B", "C", "theta") else v)
           for k, v in inp.items()}
    _, hT, cache = run(pre, want_cache=True)
    cache["ssm"] = hT
    d = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    for t in range(L1, L):
        y = m3.mimo_step(cache, *(d[k][:, t].contiguous() for k in
                                  ("X", "logdecay", "beta", "gamma", "B", "C", "theta")), d["D"])
        torch.cuda.synchronize()
        assert rel_max_err_out(f64(y), ref["Y"][:, t], True) <= TOL, t
    assert rel_max_err(f64(cache["ssm"]), ref["hT"]) <= TOL


def test_mimo_prefill_workload_sampled():
    """The rank-4 prefill workload in the benchmark's launch configuration,
    checked on sampled (b, h) sequences over their full length."""
    w, R = MIMO_WORKLOADS["mimo"]
    inp = make_mimo_inputs(w, R, "cuda")
    Y, hT, _ = m3.mimo_fwd(*(inp[k] for k in KEYS))
    torch.cuda.synchronize()
    errs = []
    for b, h in ((0, 0), (3, 17), (7, 31)):
        sub = {k: (None if v is None else v) for k, v in inp.items()}
        s = {}
        for k, v in sub.items():
            if v is None:
                s[k] = None
            elif k in ("X", "logdecay", "beta", "gamma", "theta"):
                s[k] = v[b:b + 1, :, h:h + 1]
            elif k in ("B", "C"):
                s[k] = v[b:b + 1]
            elif k == "D":
                s[k] = v[h:h + 1]
            else:
                s[k] = v[b:b + 1, h:h + 1]
        ref = reference(s)
        errs.append((f64(Y[b:b + 1, :, h:h + 1]), ref["Y"], f64(hT[b:b + 1, h:h + 1]), ref["hT"]))
    ys = np.concatenate([e[0].ravel() for e in errs])
    yr = np.concatenate([e[1].ravel() for e in errs])
    assert rel_max_err_out(ys, yr, True) <= TOL
    for e in errs:
        assert rel_max_err(e[2], e[3]) <= TOL


# ---- fp32 inputs: the chunked kernel with fp16 high / low operand parts, bar 1e-4 ----
TOL32 = 1e-4
BASE32 = BASE.with_(dtype="f32", seed=78)


@pytest.mark.parametrize("R", [1, 2, 4, 8])
@pytest.mark.parametrize("L", [1, 7, 64, 129, 200])
def test_mimo_chunked_fp32_vs_oracle(R, L):
    inp = make_mimo_inputs(BASE32.with_(seqlen=L, seed=300 + L), R)
    inp = with_cache(inp, R, L)
    inp["xprev0"] = torch.randn(inp["xprev0"].shape, generator=torch.Generator().manual_seed(L))
    ref = reference(inp)
    Y, hT, cache = run(inp, want_cache=True)
    assert rel_max_err(f64(Y), ref["Y"]) <= TOL32
    assert rel_max_err(f64(hT), ref["hT"]) <= TOL32
    assert angle_err(f64(cache["angle"]), ref["angleT"]) <= 1e-5
    np.testing.assert_array_equal(f64(cache["x_prev"]), ref["xprevT"])
    np.testing.assert_array_equal(f64(cache["b_prev"]), ref["bprevT"])


@pytest.mark.parametrize("R", [2, 4, 8])
@pytest.mark.parametrize("has_beta,has_theta,with_D", [(False, False, True), (True, True, False)])
def test_mimo_chunked_fp32_paths(R, has_beta, has_theta, with_D):
    w = BASE32.with_(seqlen=150, has_beta=has_beta, has_theta=has_theta, seed=29, nheads=4,
                     ngroups=2)
    inp = make_mimo_inputs(w, R)
    if not with_D:
        inp["D"] = None
    ref = reference(inp)
    Y, hT, _ = run(inp)
    assert rel_max_err(f64(Y), ref["Y"]) <= TOL32
    if not with_D:
        assert rms_rel_err(f64(Y), ref["Y"]) <= TOL32
    assert rel_max_err(f64(hT), ref["hT"]) <= TOL32
    assert m3.device_wait_timeouts() == 0
