"""CPU checks of the parity bound itself: half an ulp of the stored dtype is
the largest error that rounding to that dtype makes, and it is reached."""

import numpy as np
import torch

from tests import parity_util as pu


def _rounding_ratio(dtype_name, torch_dtype, seed):
    g = torch.Generator().manual_seed(seed)
    src = torch.float32 if torch_dtype == torch.bfloat16 else torch.float64
    x = torch.randn(200000, generator=g, dtype=src) * torch.exp(3 * torch.randn(200000, generator=g, dtype=src))
    # one rounding from the source (fp32 values for bf16, fp64 values for fp32)
    r = x.to(torch_dtype).to(torch.float64)
    x = x.double()
    err = (r - x).abs().numpy()
    return err / pu.half_ulp(x.numpy(), dtype_name)


def test_half_ulp_bounds_and_is_reached_bf16():
    ratio = _rounding_ratio("bf16", torch.bfloat16, 0)
    assert ratio.max() <= 1.0 + 1e-12
    assert ratio.max() > 0.99


def test_half_ulp_bounds_and_is_reached_fp32():
    ratio = _rounding_ratio("fp32", torch.float32, 1)
    assert ratio.max() <= 1.0 + 1e-12
    assert ratio.max() > 0.99


def test_half_ulp_values():
    # bf16 has 8 significant bits: the spacing in [1, 2) is 2^-7, in [4, 8) 2^-5
    np.testing.assert_array_equal(pu.half_ulp(np.array([1.0, 1.99, 4.0, 7.9, -3.0]), "bf16"),
                                  [2.0 ** -8, 2.0 ** -8, 2.0 ** -6, 2.0 ** -6, 2.0 ** -7])
    np.testing.assert_array_equal(pu.half_ulp(np.array([1.0, 0.75]), "fp32"), [2.0 ** -24, 2.0 ** -25])


def test_bound_is_absolute_below_one():
    # at |x| = 0.5 the bound is 0.02 + 2^-9 (half a bf16 ulp there): 0.0219 passes,
    # 0.0221 fails; at |x| = 100 the bf16 store adds half its ulp (0.25)
    want = np.array([0.5, 100.0])
    s = pu.err_stats(torch.tensor([0.5219, 100.0], dtype=torch.float64), want, "bf16")
    assert s["max_ratio"] <= 1.0
    s = pu.err_stats(torch.tensor([0.5221, 100.0], dtype=torch.float64), want, "bf16")
    assert s["max_ratio"] > 1.0
    s = pu.err_stats(torch.tensor([0.5, 100.26], dtype=torch.float64), want, "bf16")
    assert s["max_ratio"] <= 1.0
