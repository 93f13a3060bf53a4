"""The projection GEMM (m3ssd_gemm_bf16) against an fp64 product of the same
bf16 operands.  Each output may differ from the exact product by its bf16
rounding (half an ulp) plus the fp32 accumulation error, bounded here by
K 2^-23 sum_k |a_k w_k|.  Shapes span ragged M, N and K tails (tiles are
128 x 256 with K slices of 64), a strided and an unaligned output, and the
block's two projections at model size (checked on sampled rows)."""
import ctypes

import numpy as np
import pytest
import torch

import selective_state_space_m3ssd_b200 as m3

pytestmark = pytest.mark.gpu


def bound(A, W, ref):
    A64, W64 = A.double().cpu().numpy(), W.double().cpu().numpy()
    acc = np.abs(A64) @ np.abs(W64).T * (A.shape[1] * 2.0 ** -23)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
    return 0.5 * ulp + acc + 1e-30


def check(D, A, W):
    ref = A.double().cpu().numpy() @ W.double().cpu().numpy().T
    got = D.double().cpu().numpy()
    assert np.all(np.abs(got - ref) <= bound(A, W, ref))


def operands(M, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    A = torch.randn(M, K, generator=g).bfloat16().cuda()
    W = (torch.randn(N, K, generator=g) / K ** 0.5).bfloat16().cuda()
    return A, W


@pytest.mark.parametrize("M,N,K", [(1, 8, 8), (5, 24, 16), (127, 255, 64), (128, 256, 64),
                                   (129, 257, 72), (300, 520, 1032), (1000, 6464 // 8, 200),
                                   (2049, 1024, 136)])
def test_gemm_matches_fp64(M, N, K):
    A, W = operands(M, N, K, M + N + K)
    D = m3.gemm_bf16(A, W)
    torch.cuda.synchronize()
    check(D, A, W)


def test_gemm_strided_and_unaligned_outputs():
    M, N, K = 333, 300, 96
    A, W = operands(M, N, K, 4)
    lib = m3.load()
    big = torch.full((M, N + 13), 7.0, dtype=torch.bfloat16, device="cuda")
    st = lib.m3ssd_gemm_bf16(M, N, K, ctypes.c_void_p(A.data_ptr()), ctypes.c_void_p(W.data_ptr()),
                             ctypes.c_void_p(big.data_ptr()), N + 13, None)
    assert st == m3.OK
    flat = torch.full((M * N + 1,), 7.0, dtype=torch.bfloat16, device="cuda")
    st = lib.m3ssd_gemm_bf16(M, N, K, ctypes.c_void_p(A.data_ptr()), ctypes.c_void_p(W.data_ptr()),
                             ctypes.c_void_p(flat.data_ptr() + 2), N, None)  # 2-byte aligned
    assert st == m3.OK
    torch.cuda.synchronize()
    check(big[:, :N], A, W)
    assert torch.all(big[:, N:] == 7.0)  # the columns past N are not written
    check(flat[1:].view(M, N), A, W)
    assert flat[0].item() == 7.0


def test_gemm_two_half_tiles_ragged():
    """A shape whose 256-row tiles fill the SMs evenly (the two-half instance),
    with ragged M and K, on sampled rows."""
    M, N, K = 4000, 37 * 256, 520
    A, W = operands(M, N, K, 5)
    D = m3.gemm_bf16(A, W)
    torch.cuda.synchronize()
    rows = torch.tensor([0, 127, 128, 255, 256, 2047, 3839, 3840, 3967, 3999]).cuda()
    check(D[rows], A[rows], W)


def test_gemm_block_shapes_sampled():
    """The in_proj (32768 x 6464 x 1024) and out_proj (32768 x 1024 x 2048) shapes
    of the block at model size, on sampled rows."""
    for (M, N, K) in ((32768, 6464, 1024), (32768, 1024, 2048)):
        A, W = operands(M, N, K, 9)
        D = m3.gemm_bf16(A, W)
        torch.cuda.synchronize()
        rows = torch.tensor([0, 1, 127, 128, 4095, 20000, 32767])
        check(D[rows.cuda()], A[rows.cuda()], W)
    assert m3.device_wait_timeouts() == 0
