"""The parity metric itself (CPU): the half-ulp allowance for bf16 outputs is
exactly the rounding torch's RNE conversion makes, and no more."""
import numpy as np
import torch

from tests.gpu_util import bf16_half_ulp, rel_max_err, rel_max_err_out


def test_half_ulp_values():
    np.testing.assert_array_equal(bf16_half_ulp([1.0, 1.5, 2.0, 3.0, 0.75, -8.0]),
                                  [2 ** -8, 2 ** -8, 2 ** -7, 2 ** -7, 2 ** -9, 2 ** -5])


def test_rne_rounding_is_within_the_allowance():
    g = torch.Generator().manual_seed(0)
    x = torch.randn(1 << 16, generator=g, dtype=torch.float64) * torch.exp(
        torch.randn(1 << 16, generator=g, dtype=torch.float64) * 3)
    r = x.to(torch.bfloat16).double().numpy()
    xn = x.numpy()
    assert np.all(np.abs(r - xn) <= bf16_half_ulp(np.maximum(np.abs(r), np.abs(xn))))
    assert rel_max_err_out(r, xn, True) == 0.0
    assert rel_max_err(r, xn) > 0.0


def test_allowance_does_not_hide_real_errors():
    ref = np.linspace(-3, 3, 101)
    bad = ref.copy()
    bad[50] += 0.1  # an arithmetic error far above half an ulp at |ref| ~ 0
    assert rel_max_err_out(bad, ref, True) > 0.05
