"""The Mamba-3 SISO block through the C ABI (m3ssd_block_fwd / m3ssd_block_step)
against the fp64 block oracle on the same seeded bf16 input and weights.

The block's bf16 hand-offs (the in_proj output z, x, B, C, dt, lam, theta, the
normed group vectors of B and C, the scan output y and the gated y * SiLU(z)
that out_proj reads) are rounded to bf16 on both sides (the oracle's ``store``
hook, following the pages' policy that a bf16 op downcasts its output).  With
the fp32 sequential scan in between, the two sides then agree to the final
output rounding (the general-shape cases below show it); the chunked scan adds
its bf16 tensor-core operands.

Bars (the pages state none for the block; derived here):
  - per element, |gpu - oracle| beyond the final bf16 rounding is at most
    2e-2 of the output RMS (the scan's bf16 bar) plus 2^-7 of the element:
    the outputs are heavy tailed (max / RMS reaches 16, from the head bias
    that makes C'.B' about N) and each large element keeps the relative error
    of the bf16 values it was built from -- a hand-off can land one bf16 ulp
    (2^-8) away from the oracle's rounding, and the chunked scan's operands
    carry 2^-9 each;
  - against the unrounded fp64 oracle, the RMS error is at most 8e-3: each
    stage on the path (in_proj output, normed B and C, the scan's bf16
    operands, y, the gated product, the output) adds a relative rounding error
    of RMS 2^-9 / sqrt(3) ~ 1.1e-3, and the stages are not independent (a
    rounded dt or lam shifts the decay of every later state), so the bar takes
    their plain sum over seven stages, 7.9e-3, rather than the root-sum-square.
"""
import numpy as np
import pytest
import torch

import selective_state_space_m3ssd_b200 as m3
from oracle import block as ob
from selective_state_space_m3ssd_b200.synth import BLOCKS, make_block
from tests.gpu_util import rel_close_err, rms_rel_err

pytestmark = pytest.mark.gpu
TOL_ABS, RTOL, TOL_RMS_EXACT = 2e-2, 2.0 ** -7, 8e-3


def bf16_store(a):
    """Round to bf16 (nearest even) and back, as the device stores a hand-off."""
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).double().numpy()

SHAPES = {
    # general sequential path (P, N off the chunked kernel's shape), two groups, ragged L
    "small_g2": dict(batch=2, seqlen=70, d_model=32, nheads=4, headdim=8, dstate=8, ngroups=2),
    # chunked tensor-core path: P = 64, N = 128; L spans 4 chunks and a tail
    "chunked": dict(batch=2, seqlen=200, d_model=64, nheads=2, headdim=64, dstate=128, ngroups=1),
    # one token
    "one_token": dict(batch=3, seqlen=1, d_model=32, nheads=4, headdim=8, dstate=8, ngroups=1),
    # in_proj rows of 75 values (off the 16-byte grid): the GEMM's plain stores and the
    # element-wise gate and prep kernels
    "odd_width": dict(batch=2, seqlen=33, d_model=32, nheads=3, headdim=8, dstate=6, ngroups=1),
}


def _np(w):
    return {k: (v.double().cpu().numpy() if isinstance(v, torch.Tensor) else v)
            for k, v in w.items()}


def setup(name, seed=7):
    s = BLOCKS["small"].with_(seed=seed, **SHAPES[name])
    u, w = make_block(s)
    ud = u.cuda()
    wd = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in w.items()}
    return s, u, w, ud, wd


def check(got, ref):
    got = got.double().cpu().numpy() if isinstance(got, torch.Tensor) else got
    e = rel_close_err(got, ref, RTOL, True)
    assert e <= TOL_ABS, e


@pytest.mark.parametrize("name", sorted(SHAPES))
def test_block_fwd_matches_oracle(name):
    s, u, w, ud, wd = setup(name)
    out = m3.block_fwd(ud, wd)
    torch.cuda.synchronize()
    args = (u.double().numpy(), _np(w), s.nheads, s.headdim, s.dstate, s.ngroups)
    ref, _ = ob.oracle_block_fwd(*args, store=bf16_store)
    check(out, ref)
    exact, _ = ob.oracle_block_fwd(*args)
    assert rms_rel_err(out.double().cpu().numpy(), exact) <= TOL_RMS_EXACT


@pytest.mark.parametrize("name", ["small_g2", "chunked"])
def test_block_prefill_then_steps_match_the_forward(name):
    s, u, w, ud, wd = setup(name, seed=8)
    H, P, N, G = s.nheads, s.headdim, s.dstate, s.ngroups
    ref, ref_cache = ob.oracle_block_fwd(u.double().numpy(), _np(w), H, P, N, G,
                                         store=bf16_store)
    L1 = s.seqlen - 6
    cache = m3.new_block_cache(s.batch, H, P, N, G, "cuda")
    pre = m3.block_fwd(ud[:, :L1].contiguous(), wd, cache_out=cache)
    torch.cuda.synchronize()
    check(pre, ref[:, :L1])
    for t in range(L1, s.seqlen):
        o = m3.block_step(cache, ud[:, t].contiguous(), wd)
        torch.cuda.synchronize()
        check(o, ref[:, t])
    hs = cache["ssm"].double().cpu().numpy()
    assert np.max(np.abs(hs - ref_cache["ssm"])) <= TOL_ABS * np.sqrt(np.mean(ref_cache["ssm"] ** 2))


def test_block_fwd_continues_from_its_own_cache_in_place():
    # cache_in and cache_out the same dict: the second half reads the first
    # half's state and overwrites it with its own
    s, u, w, ud, wd = setup("small_g2", seed=9)
    H, P, N, G = s.nheads, s.headdim, s.dstate, s.ngroups
    ref, _ = ob.oracle_block_fwd(u.double().numpy(), _np(w), H, P, N, G, store=bf16_store)
    cache = m3.new_block_cache(s.batch, H, P, N, G, "cuda")
    m3.block_fwd(ud[:, :33].contiguous(), wd, cache_out=cache)
    tail = m3.block_fwd(ud[:, 33:].contiguous(), wd, cache_in=cache, cache_out=cache)
    torch.cuda.synchronize()
    check(tail, ref[:, 33:])


def test_block_at_model_size_one_batch_row():
    # the block in the configuration the benchmark times (b8 L4096 d_model 1024,
    # H32 P64 N128 G1): batch row 3 against the oracle with the same hand-offs
    s = BLOCKS["model"]
    u, w = make_block(s)
    wd = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in w.items()}
    out = m3.block_fwd(u.cuda(), wd)
    torch.cuda.synchronize()
    bi = 3
    ref, _ = ob.oracle_block_fwd(u[bi:bi + 1].double().numpy(), _np(w), s.nheads, s.headdim,
                                 s.dstate, s.ngroups, store=bf16_store)
    check(out[bi:bi + 1], ref)
