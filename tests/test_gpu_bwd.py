"""GPU backward through the C ABI (m3ssd_bwd) against the fp64 oracle's backward.

Every gradient output is compared element by element with oracle.oracle_bwd on
the same inputs (bf16 inputs are rounded before either side sees them), by
max |err| / RMS(reference).

fp32 kernels (sequential, column-split, and the fp32 chunked kernel that takes
fp32 inputs or unaligned bf16 ones): bar 2e-4.  They recompute the forward and
sweep it back in fp32; recurrence, rotations and reductions each carry an error
of order 1e-6 of a gradient's scale, a few 1e-5 over a few hundred tokens.

The tensor-core chunked kernel (bf16 inputs, N = 128, P = 64): bar 1e-3.  Each
fp32 operand enters its products as a bf16 high part plus a bf16 residual, whose
own rounding leaves at most 2^-18 of the element; the products take
hi x hi + hi x lo + lo x hi, and lo x lo too where they feed dtheta's suffix
sums: a product term carries up to about 2^-16 relative error, some 30 times
the fp32 kernels'.  The gradients are heavy-tailed (max / RMS up to about 16), so an
element's error reaches about 1e-4 of the RMS, and dtheta and dlogdecay, suffix
sums over every later token, collect the errors of all later chunks (measured
3.2e-4 at L = 4096 for dtheta, under 1.6e-4 at L <= 400).
"""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_m3ssd_b200 as m3
from selective_state_space_m3ssd_b200.synth import WORKLOADS, make_inputs
from tests.gpu_util import np64, rel_max_err, to_dev
from tests.test_gpu_seq_step import with_cache_inputs

pytestmark = pytest.mark.gpu

TOL = 2e-4
TOL_TC = 1e-3
SMALL = WORKLOADS["tiny"].with_(batch=2, nheads=4, ngroups=2, headdim=16, dstate=16, seed=77)
ARGS = ("X", "logdecay", "beta", "gamma", "B", "C", "theta", "D", "h0")


def upstream(inp, seed, with_dhT=True):
    g = torch.Generator().manual_seed(seed)
    b, L, H, P = inp["X"].shape
    N = inp["B"].shape[3]
    dY = torch.randn(b, L, H, P, generator=g).to(inp["X"].dtype)
    dhT = torch.randn(b, H, N, P, generator=g) if with_dhT else None
    return dY, dhT


def run_both(inp, dY, dhT):
    ref = oracle.oracle_bwd(**inp, dY=dY, dhT=dhT)
    d = to_dev(inp)
    got = m3.bwd(*(d.get(k) for k in ARGS), dY=dY.cuda(), dhT=None if dhT is None else dhT.cuda(),
                 angle0=d.get("angle0"), xprev0=d.get("xprev0"), bprev0=d.get("bprev0"))
    torch.cuda.synchronize()
    return {k: np64(v) for k, v in got.items()}, ref


def check_all(got, ref, tol=TOL, skip=()):
    for k, r in ref.items():
        if k in skip:
            continue
        if np.size(r) == 0:  # an empty sequence: nothing to compare but the shape
            assert np.shape(got[k]) == np.shape(r), k
            continue
        if not np.any(r):
            assert np.max(np.abs(got[k])) == 0.0, k
            continue
        assert rel_max_err(got[k], r) <= tol, (k, rel_max_err(got[k], r))


@pytest.mark.parametrize("L", [1, 17, 64, 65, 130])
def test_bwd_fp32_lengths(L):
    inp = with_cache_inputs(make_inputs(SMALL.with_(seqlen=L)), seed=L)
    dY, dhT = upstream(inp, 10 + L)
    got, ref = run_both(inp, dY, dhT)
    check_all(got, ref)


@pytest.mark.parametrize("variant", ["no_beta", "no_theta", "no_cache", "no_dhT", "one_group"])
def test_bwd_fp32_paths(variant):
    w = SMALL.with_(seqlen=70)
    if variant == "no_beta":
        w = w.with_(has_beta=False)
    if variant == "no_theta":
        w = w.with_(has_theta=False)
    if variant == "one_group":
        w = w.with_(ngroups=1)
    inp = make_inputs(w)
    if variant != "no_cache":
        inp = with_cache_inputs(inp, seed=3)
    dY, dhT = upstream(inp, 5, with_dhT=variant != "no_dhT")
    got, ref = run_both(inp, dY, dhT)
    check_all(got, ref)


def test_bwd_bf16_siso_shape():
    # the shape of the chunked forward (N = 128, P = 64) with bf16 X, B, C, dY:
    # the tensor-core kernel
    w = WORKLOADS["siso"].with_(batch=1, nheads=2, seqlen=100, seed=88)
    inp = with_cache_inputs(make_inputs(w), seed=9)
    dY, dhT = upstream(inp, 11)
    got, ref = run_both(inp, dY, dhT)
    check_all(got, ref, tol=TOL_TC)


def test_bwd_is_deterministic():
    inp = make_inputs(SMALL.with_(seqlen=90))
    dY, dhT = upstream(inp, 21)
    d = to_dev(inp)
    args = [d.get(k) for k in ARGS]
    g1 = m3.bwd(*args, dY=dY.cuda(), dhT=dhT.cuda())
    g2 = m3.bwd(*args, dY=dY.cuda(), dhT=dhT.cuda())
    torch.cuda.synchronize()
    for k in g1:
        assert torch.equal(g1[k], g2[k]), k


def test_bwd_rejects_small_workspace():
    inp = make_inputs(SMALL.with_(seqlen=20))
    dY, _ = upstream(inp, 1)
    d = to_dev(inp)
    with pytest.raises(m3.M3SSDError):
        m3.bwd(*(d.get(k) for k in ARGS), dY=dY.cuda(),
               workspace=torch.empty(256, dtype=torch.uint8, device="cuda"))


# N = 128 and P a multiple of 16: the column-split backward (one CTA per (b, h)
# and 16-column slice, block checkpoints every 16 tokens, slice partials summed
# in a fixed order)
SPLIT = WORKLOADS["tiny"].with_(batch=2, nheads=4, ngroups=2, headdim=32, dstate=128, seed=91)


@pytest.mark.parametrize("L", [1, 15, 16, 17, 50])
def test_bwd_split_lengths(L):
    inp = with_cache_inputs(make_inputs(SPLIT.with_(seqlen=L)), seed=L)
    dY, dhT = upstream(inp, 40 + L)
    got, ref = run_both(inp, dY, dhT)
    check_all(got, ref)


@pytest.mark.parametrize("variant", ["no_beta", "no_theta", "no_cache", "no_dhT", "one_slice"])
def test_bwd_split_paths(variant):
    w = SPLIT.with_(seqlen=37)
    if variant == "no_beta":
        w = w.with_(has_beta=False)
    if variant == "no_theta":
        w = w.with_(has_theta=False)
    if variant == "one_slice":
        w = w.with_(headdim=16, ngroups=1)
    inp = make_inputs(w)
    if variant != "no_cache":
        inp = with_cache_inputs(inp, seed=8)
    dY, dhT = upstream(inp, 6, with_dhT=variant != "no_dhT")
    got, ref = run_both(inp, dY, dhT)
    check_all(got, ref)


def test_bwd_split_is_deterministic():
    inp = make_inputs(SPLIT.with_(seqlen=40))
    dY, dhT = upstream(inp, 22)
    d = to_dev(inp)
    args = [d.get(k) for k in ARGS]
    g1 = m3.bwd(*args, dY=dY.cuda(), dhT=dhT.cuda())
    g2 = m3.bwd(*args, dY=dY.cuda(), dhT=dhT.cuda())
    torch.cuda.synchronize()
    for k in g1:
        assert torch.equal(g1[k], g2[k]), k


# N = 128 and P = 64: the chunked backward (one CTA per (b, h), chunks of 63
# tokens plus the carry-in row, forward pass for the chunk-start states, then
# the chunks in reverse; group sums in a second kernel)
CHUNK = WORKLOADS["siso"].with_(batch=2, nheads=4, ngroups=2, seed=131)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("L", [0, 1, 2, 62, 63, 64, 126, 127, 200])
def test_bwd_chunk_lengths(L, dtype):
    # fp32 inputs: the fp32 chunked kernel; bf16 inputs: the tensor-core one
    inp = with_cache_inputs(make_inputs(CHUNK.with_(seqlen=L, dtype=dtype)), seed=L)
    dY, dhT = upstream(inp, 60 + L)
    got, ref = run_both(inp, dY, dhT)
    check_all(got, ref, tol=TOL_TC if dtype == "bf16" else TOL)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("variant", ["all", "no_beta", "no_theta", "no_cache", "no_dhT",
                                     "one_group"])
def test_bwd_chunk_paths(variant, dtype):
    w = CHUNK.with_(seqlen=150, dtype=dtype)
    if variant == "no_beta":
        w = w.with_(has_beta=False)
    if variant == "no_theta":
        w = w.with_(has_theta=False)
    if variant == "one_group":
        w = w.with_(ngroups=1)
    inp = make_inputs(w)
    if variant != "no_cache":
        inp = with_cache_inputs(inp, seed=12)
    dY, dhT = upstream(inp, 7, with_dhT=variant != "no_dhT")
    got, ref = run_both(inp, dY, dhT)
    check_all(got, ref, tol=TOL_TC if dtype == "bf16" else TOL)


def _offset_copy(t):
    # the same values at an address one element past a 16-byte boundary
    flat = torch.empty(t.numel() + 1, dtype=t.dtype, device=t.device)
    v = flat[1:].view(t.shape)
    v.copy_(t)
    return v


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_bwd_chunk_unaligned_inputs(dtype):
    # X, B, C, theta and dY off the 16-byte grid: the element-wise load path
    inp = with_cache_inputs(make_inputs(CHUNK.with_(seqlen=90, dtype=dtype)), seed=5)
    dY, dhT = upstream(inp, 24)
    ref = oracle.oracle_bwd(**inp, dY=dY, dhT=dhT)
    d = to_dev(inp)
    for k in ("X", "B", "C", "theta"):
        d[k] = _offset_copy(d[k])
    dYd = _offset_copy(dY.cuda())
    assert dYd.data_ptr() % 16 != 0
    got = m3.bwd(*(d.get(k) for k in ARGS), dY=dYd, dhT=dhT.cuda(), angle0=d.get("angle0"),
                 xprev0=d.get("xprev0"), bprev0=d.get("bprev0"))
    torch.cuda.synchronize()
    check_all({k: np64(v) for k, v in got.items()}, ref)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_bwd_chunk_group_sums_unaligned_outputs(dtype):
    # dB and dC one element past a 16-byte boundary take the element-wise group
    # sums; aligned ones take the four-column kernel.  Both add the same per-head
    # shares in the same order, so the results agree bit for bit.
    inp = with_cache_inputs(make_inputs(CHUNK.with_(seqlen=130, dtype=dtype)), seed=9)
    dY, dhT = upstream(inp, 31)
    d = to_dev(inp)
    args = [d.get(k) for k in ARGS]
    extra = dict(angle0=d.get("angle0"), xprev0=d.get("xprev0"), bprev0=d.get("bprev0"))
    g1 = m3.bwd(*args, dY=dY.cuda(), dhT=dhT.cuda(), **extra)
    grads = {k: (_offset_copy(torch.zeros_like(v)) if k in ("dB", "dC") else torch.empty_like(v))
             for k, v in g1.items()}
    assert grads["dB"].data_ptr() % 16 != 0 and grads["dC"].data_ptr() % 16 != 0
    m3.bwd(*args, dY=dY.cuda(), dhT=dhT.cuda(), grads=grads, **extra)
    torch.cuda.synchronize()
    for k in g1:
        assert torch.equal(g1[k], grads[k]), k


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_bwd_chunk_is_deterministic(dtype):
    inp = with_cache_inputs(make_inputs(CHUNK.with_(seqlen=140, dtype=dtype)), seed=4)
    dY, dhT = upstream(inp, 23)
    d = to_dev(inp)
    args = [d.get(k) for k in ARGS]
    extra = dict(angle0=d.get("angle0"), xprev0=d.get("xprev0"), bprev0=d.get("bprev0"))
    g1 = m3.bwd(*args, dY=dY.cuda(), dhT=dhT.cuda(), **extra)
    g2 = m3.bwd(*args, dY=dY.cuda(), dhT=dhT.cuda(), **extra)
    torch.cuda.synchronize()
    for k in g1:
        assert torch.equal(g1[k], g2[k]), k


def test_bwd_full_siso_workload_one_batch_row():
    # the backward in the launch configuration the benchmark times (b8 L4096 H32
    # P64 N128 bf16, tensor-core chunked kernel), checked on batch row 5: every gradient
    # of its 32 heads, and dB / dC of its one group, which sum over those heads
    from selective_state_space_m3ssd_b200.synth import slice_inputs
    w = WORKLOADS["siso"]
    inp = make_inputs(w)
    gen = torch.Generator().manual_seed(123)
    dY = torch.randn(inp["X"].shape, generator=gen).to(inp["X"].dtype)
    dhT = torch.randn(w.batch, w.nheads, w.dstate, w.headdim, generator=gen) * 0.1
    d = to_dev(inp)
    got = m3.bwd(*(d.get(k) for k in ARGS), dY=dY.cuda(), dhT=dhT.cuda())
    torch.cuda.synchronize()
    bi = 5
    sub = slice_inputs(inp, b=bi)
    ref = oracle.oracle_bwd(**sub, dY=dY[bi:bi + 1], dhT=dhT[bi:bi + 1])
    per_batch = {"dX", "dlogdecay", "dbeta", "dgamma", "dB", "dC", "dtheta", "dh0"}
    for k in per_batch:
        g = np64(got[k][bi:bi + 1])
        assert rel_max_err(g, ref[k]) <= TOL_TC, (k, rel_max_err(g, ref[k]))


def test_bwd_full_siso_workload_fp32_kernel_one_batch_row():
    # the same workload through the fp32 chunked kernel (X one element off the
    # 16-byte grid sends bf16 inputs there), at the fp32 bar
    from selective_state_space_m3ssd_b200.synth import slice_inputs
    w = WORKLOADS["siso"]
    inp = make_inputs(w)
    gen = torch.Generator().manual_seed(321)
    dY = torch.randn(inp["X"].shape, generator=gen).to(inp["X"].dtype)
    dhT = torch.randn(w.batch, w.nheads, w.dstate, w.headdim, generator=gen) * 0.1
    d = to_dev(inp)
    d["X"] = _offset_copy(d["X"])
    got = m3.bwd(*(d.get(k) for k in ARGS), dY=dY.cuda(), dhT=dhT.cuda())
    torch.cuda.synchronize()
    bi = 2
    sub = slice_inputs(inp, b=bi)
    ref = oracle.oracle_bwd(**sub, dY=dY[bi:bi + 1], dhT=dhT[bi:bi + 1])
    for k in ("dX", "dlogdecay", "dbeta", "dgamma", "dB", "dC", "dtheta", "dh0"):
        g = np64(got[k][bi:bi + 1])
        assert rel_max_err(g, ref[k]) <= TOL, (k, rel_max_err(g, ref[k]))


@pytest.mark.parametrize("P,N", [(64, 256), (256, 64)])
def test_bwd_sequential_maximum_state(P, N):
    # the largest states of the sequential backward (N * P = 16384)
    w = WORKLOADS["tiny"].with_(batch=1, seqlen=19, nheads=2, ngroups=1, headdim=P, dstate=N,
                                seed=17 + P)
    inp = with_cache_inputs(make_inputs(w), seed=N)
    dY, dhT = upstream(inp, 90 + P)
    got, ref = run_both(inp, dY, dhT)
    check_all(got, ref)
