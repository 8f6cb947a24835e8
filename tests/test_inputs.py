"""CPU-only: the seeded input generators (exact_attention_111_b200/inputs.py) follow their
stated recipe."""

from __future__ import annotations

import numpy as np
import torch

from exact_attention_111_b200.inputs import make_inputs, quantize_e4m3, workloads


def test_inputs_are_seeded_bf16_draws():
    a = make_inputs(1, 2, 64, 64, seed=3)
    b = make_inputs(1, 2, 64, 64, seed=3)
    c = make_inputs(1, 2, 64, 64, seed=4)
    for n in ("q", "k", "v", "dout"):
        assert a[n].dtype == torch.bfloat16 and torch.equal(a[n], b[n]) and not torch.equal(a[n], c[n])
    # fp32 N(0, 1) rounded to bf16: the first draw of q equals torch's own fp32 draw, rounded
    g = torch.Generator().manual_seed(3)
    ref = torch.randn((1, 2, 64, 64), generator=g, dtype=torch.float32).to(torch.bfloat16)
    assert torch.equal(a["q"], ref)


def test_k_scale_is_exact():
    x = make_inputs(1, 1, 32, 64, seed=5)
    y = make_inputs(1, 1, 32, 64, seed=5, k_scale=4.0)
    assert torch.equal(y["k"].float(), 4.0 * x["k"].float())


def test_quantize_e4m3_bounds():
    x = make_inputs(1, 2, 256, 128, seed=6, with_dout=False)["v"]
    codes, ds = quantize_e4m3(x)
    assert codes.dtype == torch.float8_e4m3fn
    deq = codes.to(torch.float64).numpy() * ds
    xv = x.to(torch.float64).numpy()
    assert np.abs(codes.to(torch.float32).numpy()).max() <= 448.0
    assert abs(np.abs(codes.to(torch.float32).numpy()).max() - 448.0) < 1e-6   # the largest |x| maps to 448
    # round to nearest: relative error <= 2^-4 in E4M3's normal range (|code| >= 2^-6)
    normal = np.abs(xv / ds) >= 2.0 ** -6
    assert np.all(np.abs(deq - xv)[normal] <= 2.0 ** -4 * np.abs(xv)[normal] + 1e-12)
    assert np.all(np.abs(deq - xv)[~normal] <= 2.0 ** -10 * ds + 1e-12)


def test_workload_names_state_their_sizes():
    for name, w in workloads().items():
        assert f"N{w.N}" in name and f"d{w.d}" in name, name
