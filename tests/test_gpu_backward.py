"""GPU parity of the backward kernels (bwd_pre, bwd_main, bwd_post) against the fp64 oracle."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from exact_attention_111_b200.inputs import butterfly_blockmask, random_blockmask, workloads
from tests import parity as P

pytestmark = pytest.mark.gpu

SMALL = [
    (1, 1, 128, 64, False),
    (1, 2, 1, 64, False),
    (1, 2, 1, 128, True),
    (2, 2, 127, 64, True),
    (1, 2, 129, 128, False),
    (1, 2, 256, 64, True),
    (1, 2, 300, 128, True),
    (2, 1, 1000, 64, False),
    (1, 2, 1000, 128, True),
    (1, 1, 640, 128, False),
]


def _run(inp, causal, mask, visit=False):
    o, lse, _ = P.gpu_forward(inp, causal, mask)
    dq, dk, dv, vl = P.gpu_backward(inp, o, lse, causal, mask, visit=visit)
    return {"dq": dq, "dk": dk, "dv": dv}, vl


@pytest.mark.parametrize("B,H,N,d,causal", SMALL)
def test_backward_small(B, H, N, d, causal):
    inp = P.inputs(B, H, N, d, seed=21 + N + d)
    got, _ = _run(inp, causal, None)
    ref, _, _ = P.oracle_backward(inp, causal, None)
    P.check_grads(got, ref, label=f"N{N} d{d} causal{causal}")


@pytest.mark.parametrize("d", [64, 128])
def test_backward_fp16(d):
    inp = P.inputs(1, 2, 500, d, seed=22, dtype=torch.float16)
    got, _ = _run(inp, True, None)
    ref, _, _ = P.oracle_backward(inp, True, None)
    P.check_grads(got, ref, label="fp16")


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_backward_blockmask_and_visits(causal, d):
    N = 1100
    T = (N + 127) // 128
    mask = random_blockmask(T, 0.4, seed=5 + d, keep_diagonal=False)
    mask[3, :] = 0     # query tile with no keys: zero gradients for its rows
    mask[:, 5] = 0     # key tile no query uses: dK = dV = 0 there
    inp = P.inputs(2, 2, N, d, seed=23)
    got, vl = _run(inp, causal, mask, visit=True)
    ref, _, _ = P.oracle_backward(inp, causal, mask.numpy())
    P.check_grads(got, ref, label="blockmask")
    assert np.array_equal(vl.cpu().numpy(), P.expected_visits(2, 2, N, causal, mask.numpy()))
    assert torch.count_nonzero(got["dk"][:, :, 5 * 128:6 * 128]) == 0


def test_backward_masked_tiles_are_not_read():
    N, d = 1024, 128
    T = N // 128
    mask = torch.zeros((T, T), dtype=torch.uint8)
    mask[:, 0] = 1
    inp = P.inputs(1, 2, N, d, seed=24)
    o, lse, _ = P.gpu_forward(inp, False, mask)
    poisoned = dict(inp)
    for name in ("k", "v"):
        t = inp[name].clone()
        t[:, :, 128:, :] = float("nan")
        poisoned[name] = t
    dq, dk, dv, _ = P.gpu_backward(poisoned, o, lse, False, mask)
    ref, _, _ = P.oracle_backward(inp, False, mask.numpy())
    # rows >= 128 of dK/dV belong to never-used key tiles: exactly zero
    assert torch.count_nonzero(dk[:, :, 128:]) == 0 and torch.count_nonzero(dv[:, :, 128:]) == 0
    P.check_grads({"dq": dq, "dk": dk, "dv": dv}, ref, label="NaN poison")


@pytest.mark.parametrize("name", ["head_N128_d64", "gpt2_B64_H16_N1024_d64", "butterfly_B8_H16_N4096_d64",
                                  "long_B1_H32_N16384_d128_causal_k4", "sweep_B4_H16_N4096_d128",
                                  "sweep_B1_H32_N16384_d64_causal"])
def test_backward_workloads_sampled(name):
    w = workloads()[name]
    inp = P.inputs(w.B, w.H, w.N, w.d, w.seed, k_scale=w.k_scale)
    mask = butterfly_blockmask(w.tiles) if w.butterfly else None
    got, vl = _run(inp, w.causal, mask, visit=w.butterfly)
    heads = P.sample_heads(w.B, w.H, 4 if w.N >= 8192 else 8, seed=w.seed)
    if w.B * w.H <= 8:
        heads = None
    ref, _, _ = P.oracle_backward(inp, w.causal, None if mask is None else mask.numpy(), heads=heads)
    P.check_grads(got, ref, heads=heads, label=name)
    if w.butterfly:
        assert np.array_equal(vl.cpu().numpy(), P.expected_visits(w.B, w.H, w.N, False, mask.numpy()))
