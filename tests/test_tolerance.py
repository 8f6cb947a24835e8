"""CPU: the 16-bit output-rounding allowance used by the forward parity checks is a true
bound on round-to-nearest of an fp32 value (what the kernel rounds) into bf16 / fp16."""

import numpy as np
import torch

from tests.parity import half_ulp16


def test_half_ulp_bounds_rounding():
    r = np.random.default_rng(0)
    x = np.concatenate([r.standard_normal(200000) * s for s in (1e-3, 0.1, 1.0, 5.0, 100.0)])
    x = x.astype(np.float32).astype(np.float64)      # the kernel rounds fp32 values
    for dt in (torch.bfloat16, torch.float16):
        rx = torch.from_numpy(x.astype(np.float32)).to(dt).double().numpy()
        assert np.all(np.abs(rx - x) <= half_ulp16(x, dt) * (1 + 1e-12))
        # and it is tight: some values need (almost) the whole allowance
        assert np.max(np.abs(rx - x) / half_ulp16(x, dt)) > 0.99


def test_half_ulp_values():
    assert half_ulp16(np.array([1.0]), torch.bfloat16)[0] == 2.0 ** -8
    assert half_ulp16(np.array([3.9]), torch.bfloat16)[0] == 2.0 ** -7
    assert half_ulp16(np.array([1.0]), torch.float16)[0] == 2.0 ** -11
