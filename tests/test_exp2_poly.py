"""The FMA-pipe exp2 the kernels use for part of their exponentials (csrc/sm100.cuh,
exp2_poly2): its coefficients are the minimax fit that tests/fit_exp2_poly.py reproduces, and
on the GPU its values meet the accuracy include/fa.h claims for fa_selftest_exp2_poly."""

from __future__ import annotations

import os
import re

import numpy as np
import pytest

from tests import fit_exp2_poly as fit_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def kernel_coefficients():
    src = open(os.path.join(ROOT, "exact_attention_111_b200", "csrc", "sm100.cuh")).read()
    body = src[src.index("exp2_poly2"):]
    m = re.search(r"c1\s*=\s*([-+0-9.eE]+)f,\s*c2\s*=\s*([-+0-9.eE]+)f,\s*c3\s*=\s*([-+0-9.eE]+)f", body)
    assert m, "coefficients not found in exp2_poly2"
    return [np.float32(float(x)) for x in m.groups()]


def test_kernel_coefficients_are_the_fit_in_fp32():
    c = fit_mod.fit()
    got = kernel_coefficients()
    for k, (a, b) in enumerate(zip(got, c)):
        assert a == np.float32(b), f"c{k + 1}: kernel {a!r}, fit {np.float32(b)!r}"


def test_fit_error_bound():
    c = fit_mod.fit()
    # 1.013e-4 in exact arithmetic, 1.014e-4 with fp32 Horner evaluation
    assert fit_mod.max_rel_error(c, fp32=False) < 1.02e-4
    assert fit_mod.max_rel_error(c, fp32=True) < 1.02e-4


def test_fit_is_minimax_not_taylor():
    # The Taylor cubic of 2^f at 0 has max relative error ~7.9e-4 on [-1/2, 1/2]; the minimax
    # fit must be several times better (a fit that fell back to Taylor would fail here).
    ln2 = np.log(2.0)
    taylor = [ln2, ln2 ** 2 / 2, ln2 ** 3 / 6]
    assert fit_mod.max_rel_error(taylor, fp32=False) > 5e-4
    assert fit_mod.max_rel_error(fit_mod.fit(), fp32=False) < 0.2 * fit_mod.max_rel_error(taylor, fp32=False)


@pytest.mark.gpu
def test_gpu_exp2_poly_accuracy():
    import torch
    import exact_attention_111_b200 as fa
    from tests import parity as P
    P.ensure_built()
    # dense grid over [-127, 0], the boundary points, and the special values
    grid = np.concatenate([np.linspace(-127.0, 0.0, 2_000_001), np.arange(-127, 1, dtype=np.float64),
                           np.arange(-127, 1, dtype=np.float64) + 0.5, [-np.inf, -200.0, -127.0, -126.0, 0.0]])
    x = torch.tensor(grid, dtype=torch.float32)
    xd = x.cuda()
    y = torch.full_like(xd, float("nan"))
    fa.fa_selftest_exp2_poly(xd, y, x.numel())
    torch.cuda.synchronize()
    yv = y.cpu().numpy().astype(np.float64)
    xv = x.numpy().astype(np.float64)
    ref = np.exp2(xv)
    assert np.all(np.isfinite(yv)) and np.all(yv >= 0)
    normal = xv >= -126.0
    rel = np.abs(yv[normal] / ref[normal] - 1.0)
    assert rel.max() <= 1.1e-4, rel.max()
    sub = (xv > -127.0) & (xv < -126.0)
    assert np.abs(yv[sub] - ref[sub]).max() < 2.0 ** -126
    assert np.all(yv[xv <= -127.0] == 0.0)          # includes -inf and -200
    assert np.all(yv[xv == 0.0] == 1.0)
    # odd length: the last element is paired with 0 internally and still computed
    y3 = torch.zeros(3, device="cuda")
    fa.fa_selftest_exp2_poly(torch.tensor([-1.0, -2.0, -3.0], device="cuda"), y3, 3)
    assert np.allclose(y3.cpu().numpy(), [0.5, 0.25, 0.125], rtol=1.1e-4, atol=0)
