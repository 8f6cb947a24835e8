"""GPU parity of the fused forward kernel against the fp64 oracle (through the C ABI)."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from exact_attention_111_b200.inputs import butterfly_blockmask, random_blockmask, workloads
from tests import parity as P

pytestmark = pytest.mark.gpu

SMALL = [
    # (B, H, N, d, causal)
    (1, 1, 128, 64, False),     # one tile: the single-head workload
    (1, 2, 1, 64, False),       # N = 1: O = V
    (1, 2, 1, 128, True),
    (2, 2, 127, 64, True),      # ragged single tile
    (1, 2, 129, 128, False),    # one full tile + 1-row tail
    (1, 2, 256, 64, True),
    (1, 2, 300, 128, True),     # two query tiles in one CTA, ragged
    (2, 1, 1000, 64, False),
    (1, 2, 1000, 128, True),
    (1, 1, 640, 64, False),     # odd number of query tiles (second tile of last CTA empty)
]


@pytest.mark.parametrize("B,H,N,d,causal", SMALL)
def test_forward_small(B, H, N, d, causal):
    inp = P.inputs(B, H, N, d, seed=7 + N + d)
    o, lse, _ = P.gpu_forward(inp, causal, None)
    o_ref, lse_ref = P.oracle_forward(inp, causal, None)
    P.check_forward(o, lse, o_ref, lse_ref, o16_dtype=torch.bfloat16, label=f"N{N} d{d} causal{causal}")


@pytest.mark.parametrize("d", [64, 128])
def test_forward_fp32_output_strict(d):
    """fp32 O: the 1e-2 bound holds with no output-rounding allowance."""
    inp = P.inputs(1, 2, 700, d, seed=11, k_scale=4.0)
    o, lse, _ = P.gpu_forward(inp, True, None, o_fp32=True)
    o_ref, lse_ref = P.oracle_forward(inp, True, None)
    P.check_forward(o, lse, o_ref, lse_ref, o16_dtype=None, label="fp32 O")


@pytest.mark.parametrize("d", [64, 128])
def test_forward_fp16(d):
    inp = P.inputs(2, 2, 333, d, seed=12, dtype=torch.float16)
    o, lse, _ = P.gpu_forward(inp, False, None)
    o_ref, lse_ref = P.oracle_forward(inp, False, None)
    P.check_forward(o, lse, o_ref, lse_ref, o16_dtype=torch.float16, label="fp16")


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_forward_blockmask_and_visits(causal, d):
    N = 1100
    T = (N + 127) // 128
    mask = random_blockmask(T, 0.4, seed=3 + d, keep_diagonal=False)
    mask[3, :] = 0   # a query tile with no key tile at all: O = 0, LSE = -inf
    inp = P.inputs(2, 2, N, d, seed=13)
    o, lse, vl = P.gpu_forward(inp, causal, mask, visit=True)
    o_ref, lse_ref = P.oracle_forward(inp, causal, mask.numpy())
    P.check_forward(o, lse, o_ref, lse_ref, o16_dtype=torch.bfloat16, label="blockmask")
    assert np.array_equal(vl.cpu().numpy(), P.expected_visits(2, 2, N, causal, mask.numpy())), "tile visits differ"


def test_forward_masked_tiles_are_not_read():
    """Only key tile 0 is kept; K/V rows of every other tile are NaN and must never be read."""
    N, d = 1024, 64
    T = N // 128
    mask = torch.zeros((T, T), dtype=torch.uint8)
    mask[:, 0] = 1
    inp = P.inputs(1, 2, N, d, seed=14)
    poisoned = dict(inp)
    for name in ("k", "v"):
        t = inp[name].clone()
        t[:, :, 128:, :] = float("nan")
        poisoned[name] = t
    o, lse, _ = P.gpu_forward(poisoned, False, mask)
    o_ref, lse_ref = P.oracle_forward(inp, False, mask.numpy())
    P.check_forward(o, lse, o_ref, lse_ref, o16_dtype=torch.bfloat16, label="NaN poison")


@pytest.mark.parametrize("name", ["head_N128_d64", "gpt2_B64_H16_N1024_d64", "butterfly_B8_H16_N4096_d64",
                                  "long_B1_H32_N16384_d128_causal_k4", "sweep_B4_H16_N4096_d128",
                                  "sweep_B1_H32_N16384_d64_causal"])
def test_forward_workloads_sampled(name):
    w = workloads()[name]
    inp = P.inputs(w.B, w.H, w.N, w.d, w.seed, k_scale=w.k_scale)
    mask = butterfly_blockmask(w.tiles) if w.butterfly else None
    o, lse, vl = P.gpu_forward(inp, w.causal, mask, visit=w.butterfly)
    heads = P.sample_heads(w.B, w.H, 4 if w.N >= 8192 else 8, seed=w.seed)
    if w.B * w.H <= 8:
        heads = None
    o_ref, lse_ref = P.oracle_forward(inp, w.causal, None if mask is None else mask.numpy(), heads=heads)
    P.check_forward(o, lse, o_ref, lse_ref, heads=heads, o16_dtype=torch.bfloat16, label=name)
    if w.butterfly:
        assert np.array_equal(vl.cpu().numpy(), P.expected_visits(w.B, w.H, w.N, False, mask.numpy()))


def test_forward_long_context_fp32_output_strict():
    """The peaked long-context workload (K scaled by 4, causal, N = 16384, d = 128) with fp32
    O: max |O - O_ref| <= 1e-2 with no output-rounding allowance, on sampled whole heads."""
    w = workloads()["long_B1_H32_N16384_d128_causal_k4"]
    inp = P.inputs(w.B, w.H, w.N, w.d, w.seed, k_scale=w.k_scale)
    o, lse, _ = P.gpu_forward(inp, True, None, o_fp32=True)
    heads = P.sample_heads(w.B, w.H, 4, seed=w.seed + 1)
    o_ref, lse_ref = P.oracle_forward(inp, True, None, heads=heads)
    worst_o, worst_l = P.check_forward(o, lse, o_ref, lse_ref, heads=heads, o16_dtype=None, label="long fp32 O")
    print(f"long-context fp32 O: max |O err| {worst_o:.4g}, max |LSE err| {worst_l:.4g}")


def test_forward_deterministic():
    inp = P.inputs(2, 4, 2000, 128, seed=15)
    o1, l1, _ = P.gpu_forward(inp, True, None)
    o2, l2, _ = P.gpu_forward(inp, True, None)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
