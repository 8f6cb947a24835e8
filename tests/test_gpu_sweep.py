"""GPU parity over every point of the sequence-length sweep (N = 512 .. 16384, B = 16384/N,
(H, d) in {(32, 64), (16, 128)}, causal and not), forward and backward, at full size: the whole
batch runs on the GPU, a seeded sample of whole heads (always the first and the last) is
compared with the fp64 oracle."""

from __future__ import annotations

import pytest
import torch

from exact_attention_111_b200.inputs import workloads
from tests import parity as P

pytestmark = pytest.mark.gpu

SWEEP = sorted(n for n in workloads() if n.startswith("sweep_"))


@pytest.mark.parametrize("name", SWEEP)
def test_sweep_point_forward_backward(name):
    w = workloads()[name]
    inp = P.inputs(w.B, w.H, w.N, w.d, w.seed, k_scale=w.k_scale)
    o, lse, _ = P.gpu_forward(inp, w.causal, None)
    dq, dk, dv, _ = P.gpu_backward(inp, o, lse, w.causal, None)
    heads = P.sample_heads(w.B, w.H, 2 if w.N >= 8192 else 3, seed=w.seed + w.N)
    ref, o_ref, lse_ref = P.oracle_backward(inp, w.causal, None, heads=heads)
    P.check_forward(o, lse, o_ref, lse_ref, heads=heads, o16_dtype=torch.bfloat16, label=name)
    P.check_grads({"dq": dq, "dk": dk, "dv": dv}, ref, heads=heads, label=name)
