"""GPU parity of the sequential fp32 forward and of the decode step against
the fp64 oracle (max |gpu - oracle| / RMS(oracle) <= 1e-4 for fp32 inputs and
<= 2e-2 for bf16 inputs)."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_m3ssd_b200 as m3
from selective_state_space_m3ssd_b200.synth import WORKLOADS, make_inputs
from tests.gpu_util import angle_err, gpu_fwd, np64, rel_max_err, rel_max_err_out, to_dev

pytestmark = pytest.mark.gpu
TOL_F32, TOL_BF16 = 1e-4, 2e-2


def with_cache_inputs(inp, seed=5):
    g = torch.Generator().manual_seed(seed)
    b, L, H, P = inp["X"].shape
    G, N = inp["B"].shape[2:]
    out = dict(inp)
    out["angle0"] = torch.rand(b, H, N // 2, generator=g) * 6 - 3
    out["xprev0"] = torch.randn(b, H, P, generator=g)
    out["bprev0"] = torch.randn(b, G, N, generator=g) / N ** 0.5
    out["h0"] = torch.randn(b, H, N, P, generator=g) * 0.3
    return out


def test_tiny_workload_fp32():
    inp = make_inputs(WORKLOADS["tiny"])
    ref = oracle.oracle_fwd(**inp)
    got = gpu_fwd(inp)
    assert rel_max_err(got["Y"], ref["Y"]) <= TOL_F32
    assert rel_max_err(got["hT"], ref["hT"]) <= TOL_F32


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("G,H", [(1, 3), (2, 4)])
def test_general_path_with_cache_inputs(dtype, G, H):
    w = WORKLOADS["tiny"].with_(batch=2, seqlen=37, nheads=H, ngroups=G, headdim=12, dstate=10,
                                dtype=dtype, seed=77)
    inp = with_cache_inputs(make_inputs(w))
    ref = oracle.oracle_fwd(**inp)
    got = gpu_fwd(inp, want_cache=True)
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    assert rel_max_err_out(got["Y"], ref["Y"], dtype == "bf16") <= tol
    assert rel_max_err(got["hT"], ref["hT"]) <= TOL_F32 * (1 if dtype == "f32" else 10)
    assert angle_err(got["angleT"], ref["angleT"]) <= 1e-5
    np.testing.assert_array_equal(got["xprevT"], ref["xprevT"])
    np.testing.assert_array_equal(got["bprevT"], ref["bprevT"])


def test_beta_theta_absent_fp32():
    w = WORKLOADS["tiny"].with_(has_beta=False, has_theta=False, seed=31)
    inp = make_inputs(w)
    ref = oracle.oracle_fwd(**inp)
    got = gpu_fwd(inp)
    assert rel_max_err(got["Y"], ref["Y"]) <= TOL_F32
    assert rel_max_err(got["hT"], ref["hT"]) <= TOL_F32


def test_empty_sequence_passes_the_cache_through():
    w = WORKLOADS["tiny"].with_(seqlen=0, batch=2)
    inp = with_cache_inputs(make_inputs(w))
    got = gpu_fwd(inp, want_cache=True)
    np.testing.assert_array_equal(got["hT"], np64(inp["h0"]))
    assert angle_err(got["angleT"], np64(inp["angle0"])) <= 1e-6
    np.testing.assert_array_equal(got["xprevT"], np64(inp["xprev0"]))
    np.testing.assert_array_equal(got["bprevT"], np64(inp["bprev0"]))


def _steps_gpu_and_oracle(w, nsteps, start_cache=True):
    inp = make_inputs(w.with_(seqlen=nsteps))
    b, L, H, P = inp["X"].shape
    G, N = inp["B"].shape[2:]
    g = torch.Generator().manual_seed(9)
    init = {"angle": torch.rand(b, H, N // 2, generator=g) * 6 - 3,
            "ssm": torch.randn(b, H, N, P, generator=g) * 0.3,
            "x_prev": torch.randn(b, H, P, generator=g),
            "b_prev": torch.randn(b, G, N, generator=g) / N ** 0.5}
    if not start_cache:
        init = {k: torch.zeros_like(v) for k, v in init.items()}
    ocache = {k: np64(v).copy() for k, v in init.items()}
    gcache = {k: v.cuda() for k, v in init.items()}
    d = to_dev(inp)
    ys_o, ys_g = [], []
    for t in range(nsteps):
        sl = lambda k: None if d[k] is None else d[k][:, t].contiguous()
        ys_g.append(np64(m3.step(gcache, sl("X"), sl("logdecay"), sl("beta"), sl("gamma"),
                                 sl("B"), sl("C"), sl("theta"), d["D"])))
        so = lambda k: None if inp[k] is None else inp[k][:, t]
        ys_o.append(oracle.oracle_step(ocache, so("X"), so("logdecay"), so("beta"), so("gamma"),
                                       so("B"), so("C"), so("theta"), inp["D"]))
    torch.cuda.synchronize()
    return np.stack(ys_g, 1), np.stack(ys_o, 1), {k: np64(v) for k, v in gcache.items()}, ocache


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("P,N,G,H", [(64, 128, 1, 4), (12, 10, 2, 4), (3, 6, 1, 2)])
def test_decode_steps(dtype, P, N, G, H):
    w = WORKLOADS["tiny"].with_(batch=3, nheads=H, ngroups=G, headdim=P, dstate=N, dtype=dtype,
                                seed=55)
    yg, yo, cg, co = _steps_gpu_and_oracle(w, 6)
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    assert rel_max_err_out(yg, yo, dtype == "bf16") <= tol
    assert rel_max_err(cg["ssm"], co["ssm"]) <= TOL_F32
    assert angle_err(cg["angle"], co["angle"]) <= 1e-5
    np.testing.assert_array_equal(cg["x_prev"], co["x_prev"])
    np.testing.assert_array_equal(cg["b_prev"], co["b_prev"])


def test_forward_equals_prefill_plus_steps_on_gpu():
    w = WORKLOADS["tiny"].with_(batch=2, seqlen=40, nheads=4, headdim=16, dstate=16, seed=21)
    inp = make_inputs(w)
    full = gpu_fwd(inp)
    d = to_dev(inp)
    split = 23
    Y, hT, cache = m3.fwd(*(None if d[k] is None else d[k][:, :split].contiguous()
                            for k in ("X", "logdecay", "beta", "gamma", "B", "C", "theta")),
                          d["D"], d["h0"], want_cache=True)
    cache["ssm"] = hT
    ys = [np64(Y)]
    for t in range(split, 40):
        ys.append(np64(m3.step(cache, *(d[k][:, t].contiguous() for k in
                                        ("X", "logdecay", "beta", "gamma", "B", "C", "theta")),
                               d["D"]))[:, None])
    torch.cuda.synchronize()
    assert rel_max_err(np.concatenate(ys, 1), full["Y"]) <= TOL_F32
    assert rel_max_err(np64(cache["ssm"]), full["hT"]) <= TOL_F32


def test_decode_workload_prefill_then_1000_steps_sampled():
    """Batched decode b256 H32 P64 N128 fp32: a 512-token prefill through
    m3ssd_fwd, then 1000 m3ssd_step calls, against the oracle over the same
    1512 tokens on sampled (b, h) sequences (outputs and final cache)."""
    from selective_state_space_m3ssd_b200.synth import DECODE_PREFILL, DECODE_STEPS, slice_inputs
    w = WORKLOADS["decode"]
    inp = make_inputs(w, device="cuda")
    Lp = DECODE_PREFILL
    keys = ("X", "logdecay", "beta", "gamma", "B", "C", "theta")
    Y, hT, cache = m3.fwd(*(inp[k][:, :Lp].contiguous() for k in keys), inp["D"], None,
                          want_cache=True)
    cache["ssm"] = hT
    ys = torch.empty(w.batch, DECODE_STEPS, w.nheads, w.headdim, device="cuda")
    for t in range(DECODE_STEPS):
        ys[:, t] = m3.step(cache, *(inp[k][:, Lp + t].contiguous() for k in keys), inp["D"])
    torch.cuda.synchronize()
    cpu = {k: (None if v is None else v.cpu()) for k, v in inp.items()}
    pairs = {0: [0, 31], 128: [7], 255: [16, 30]}
    for bi, heads in pairs.items():
        ref = oracle.oracle_fwd(**slice_inputs(cpu, b=bi, heads=heads))
        got_y = np.concatenate([np64(Y[bi:bi + 1][:, :, heads]),
                                np64(ys[bi:bi + 1][:, :, heads])], axis=1)
        assert rel_max_err(got_y, ref["Y"]) <= TOL_F32
        assert rel_max_err(np64(cache["ssm"][bi:bi + 1][:, heads]), ref["hT"]) <= TOL_F32
        assert angle_err(np64(cache["angle"][bi:bi + 1][:, heads]), ref["angleT"]) <= 1e-4
        np.testing.assert_array_equal(np64(cache["x_prev"][bi:bi + 1][:, heads]), ref["xprevT"])
        np.testing.assert_array_equal(np64(cache["b_prev"][bi:bi + 1]), ref["bprevT"])


def test_decode_workload_1000_steps_replayed_from_a_cuda_graph():
    """The decode workload as the benchmark runs it: the 1000 m3ssd_step calls
    captured in one CUDA graph (per-step inputs staged time-major so every step
    reads contiguous tensors) and replayed once after the 512-token prefill;
    sampled (b, h) outputs and the final cache against the oracle over the same
    1512 tokens ("mamba-rs" crate page, feature list: CUDA Graph capture of the
    inference step)."""
    from selective_state_space_m3ssd_b200.synth import DECODE_PREFILL, DECODE_STEPS, slice_inputs
    w = WORKLOADS["decode"]
    inp = make_inputs(w, device="cuda")
    Lp = DECODE_PREFILL
    keys = ("X", "logdecay", "beta", "gamma", "B", "C", "theta")
    Y, hT, cache = m3.fwd(*(inp[k][:, :Lp].contiguous() for k in keys), inp["D"], None,
                          want_cache=True)
    cache["ssm"] = hT
    steps = {k: inp[k][:, Lp:].transpose(0, 1).contiguous() for k in keys}  # (T, b, ...)
    ys = torch.empty(DECODE_STEPS, w.batch, w.nheads, w.headdim, device="cuda")
    # one eager step on a copy first: the library's one-time launch set-up stays
    # out of the capture
    scratch = {k: v.clone() for k, v in cache.items()}
    m3.step(scratch, *(steps[k][0] for k in keys), inp["D"], y_t=torch.empty_like(ys[0]))
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for t in range(DECODE_STEPS):
            m3.step(cache, *(steps[k][t] for k in keys), inp["D"], y_t=ys[t])
    g.replay()
    torch.cuda.synchronize()
    del g
    cpu = {k: (None if v is None else v.cpu()) for k, v in inp.items()}
    pairs = {3: [1, 30], 200: [12]}
    for bi, heads in pairs.items():
        ref = oracle.oracle_fwd(**slice_inputs(cpu, b=bi, heads=heads))
        got_y = np.concatenate([np64(Y[bi:bi + 1][:, :, heads]),
                                np64(ys[:, bi:bi + 1][:, :, heads].transpose(0, 1))], axis=1)
        assert rel_max_err(got_y, ref["Y"]) <= TOL_F32
        assert rel_max_err(np64(cache["ssm"][bi:bi + 1][:, heads]), ref["hT"]) <= TOL_F32
        assert angle_err(np64(cache["angle"][bi:bi + 1][:, heads]), ref["angleT"]) <= 1e-4
        np.testing.assert_array_equal(np64(cache["x_prev"][bi:bi + 1][:, heads]), ref["xprevT"])
        np.testing.assert_array_equal(np64(cache["b_prev"][bi:bi + 1]), ref["bprevT"])


# The largest state the sequential kernels keep in one CTA: N * P = 16384 with
# N, P <= 256 (the three corners), forward with cache in and out, then decode
# steps from the forward's cache, each against the oracle.
@pytest.mark.parametrize("P,N", [(64, 256), (256, 64), (128, 128)])
def test_general_path_maximum_state(P, N):
    w = WORKLOADS["tiny"].with_(batch=1, seqlen=21, nheads=2, ngroups=1, headdim=P, dstate=N,
                                seed=91 + P)
    inp = with_cache_inputs(make_inputs(w), seed=P + N)
    ref = oracle.oracle_fwd(**inp)
    got = gpu_fwd(inp, want_cache=True)
    assert rel_max_err(got["Y"], ref["Y"]) <= TOL_F32
    assert rel_max_err(got["hT"], ref["hT"]) <= TOL_F32
    assert angle_err(got["angleT"], ref["angleT"]) <= 1e-5
    yg, yo, cg, co = _steps_gpu_and_oracle(w, 4)
    assert rel_max_err(yg, yo) <= TOL_F32
    assert rel_max_err(cg["ssm"], co["ssm"]) <= TOL_F32


def test_state_over_the_limit_is_refused():
    # N * P = 16640 > 16384: the sequential kernels cannot hold it
    w = WORKLOADS["tiny"].with_(batch=1, seqlen=3, nheads=1, headdim=65, dstate=256, seed=3)
    inp = make_inputs(w)
    with pytest.raises(m3.M3SSDError):
        gpu_fwd(inp)
