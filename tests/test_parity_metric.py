"""The parity metric itself (CPU): the half-ulp allowance for bf16 outputs is
exactly the rounding torch's RNE conversion makes, and no more."""
import numpy as np
import torch

from tests import gpu_util
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


def test_rel_close_err_gives_each_element_its_relative_slack():
    ref = np.array([1.0, -1.0, 100.0, 0.0])
    rms = np.sqrt(np.mean(ref ** 2))
    # errors exactly at the relative slack: nothing left over
    got = ref + 0.01 * np.abs(ref)
    assert gpu_util.rel_close_err(got, ref, 0.01, False) < 1e-15
    # an absolute error on the zero element is measured against the RMS
    got = ref.copy()
    got[3] = 0.5
    assert abs(gpu_util.rel_close_err(got, ref, 0.01, False) - 0.5 / rms) < 1e-15
    # beyond the slack of the large element
    got = ref.copy()
    got[2] = 103.0
    assert abs(gpu_util.rel_close_err(got, ref, 0.01, False) - 2.0 / rms) < 1e-12
