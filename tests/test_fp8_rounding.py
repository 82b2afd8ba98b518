"""The e4m3 rounding model the fp8 forward's tolerance rests on (CPU):
round-to-nearest-even to 3 mantissa bits gives a relative error of at most
2^-4 for values >= 2^-6 (the smallest normal) and an absolute error of at
most 2^-10 (half the subnormal spacing 2^-9) below it, and never saturates
for values up to 448.  The kernel's P lies in [0, 2^8] relative to its
running reference (the reference moves when a tile's max exceeds it by more
than 8 in log2 units), so these are the cases that occur."""

import numpy as np
import torch


def test_e4m3_rounding_error_bounds():
    x = torch.cat([torch.exp2(torch.linspace(-14.0, 8.0, 200001)),
                   torch.linspace(0.0, 256.0, 100001)]).double()
    r = x.float().to(torch.float8_e4m3fn).double()
    err = (r - x).abs()
    normal = x >= 2.0 ** -6
    assert float((err[normal] / x[normal]).max()) <= 2.0 ** -4 + 1e-12
    assert float(err[~normal].max()) <= 2.0 ** -10 + 1e-12
    assert float(r.max()) <= 256.0 and torch.isfinite(r).all()


def test_e4m3_holds_the_workload_draws():
    # N(0, 1) draws divided by descale factors down to 0.25 stay below 448,
    # the largest finite e4m3 value, so quantising them never saturates
    g = torch.Generator().manual_seed(0)
    x = torch.randn(1 << 20, generator=g) / 0.25
    assert float(x.abs().max()) < 448.0
    q = x.to(torch.float8_e4m3fn).float()
    assert torch.isfinite(q).all()
    assert np.isclose(float(q.abs().max()), float(x.abs().max()), rtol=2 ** -4)
