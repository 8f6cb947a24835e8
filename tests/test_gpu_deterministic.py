"""GPU: the deterministic backward (int64 fixed-point dQ accumulation) -- parity with the
fp64 oracle, bitwise repeatability, agreement with the default backward, and the range
error for partials too large for the fixed-point format."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import exact_attention_111_b200 as fa
from exact_attention_111_b200.inputs import random_blockmask, workloads, workload_inputs
from tests import parity as P

pytestmark = pytest.mark.gpu


def _backward(inp, o, lse, causal, mask, deterministic, dtype_code=None):
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "dout"))
    dq, dk, dv = fa.attention_backward(q, k, v, o, lse, do, causal=causal, blockmask=P.to_dev(mask),
                                       deterministic=deterministic)
    fa.fa_check_status()
    torch.cuda.synchronize()
    return {"dq": dq, "dk": dk, "dv": dv}


CASES = [
    # B, H, N, d, causal, mask, dtype
    (1, 1, 128, 64, False, False, torch.bfloat16),
    (2, 2, 127, 64, True, False, torch.bfloat16),
    (1, 2, 129, 128, False, False, torch.bfloat16),
    (2, 1, 1000, 64, False, False, torch.bfloat16),
    (1, 2, 1000, 128, True, False, torch.bfloat16),
    (2, 2, 1100, 64, True, True, torch.bfloat16),
    (1, 2, 900, 128, False, True, torch.bfloat16),
    (1, 2, 500, 64, True, False, torch.float16),
    (1, 2, 500, 128, False, False, torch.float16),
]


@pytest.mark.parametrize("B,H,N,d,causal,use_mask,dtype", CASES)
def test_deterministic_matches_oracle(B, H, N, d, causal, use_mask, dtype):
    P.ensure_built()
    inp = P.inputs(B, H, N, d, seed=5100 + N + d, dtype=dtype)
    T = (N + 127) // 128
    mask = None
    if use_mask:
        mask = random_blockmask(T, 0.5, seed=3, keep_diagonal=False)
        mask[1, :] = 0
    o, lse, _ = P.gpu_forward(inp, causal, mask)
    got = _backward(inp, o, lse, causal, mask, True)
    ref, _, _ = P.oracle_backward(inp, causal, None if mask is None else mask.numpy())
    P.check_grads(got, ref, label=f"deterministic N{N} d{d}")


@pytest.mark.parametrize("d,causal", [(64, False), (128, True)])
def test_deterministic_is_bitwise_repeatable(d, causal):
    """Many heads and key tiles, so the CTAs' finishing order varies between runs."""
    P.ensure_built()
    inp = P.inputs(4, 8, 2048, d, seed=5200 + d)
    o, lse, _ = P.gpu_forward(inp, causal, None)
    first = _backward(inp, o, lse, causal, None, True)
    for _ in range(4):
        again = _backward(inp, o, lse, causal, None, True)
        for n in ("dq", "dk", "dv"):
            assert torch.equal(first[n], again[n]), n
    default = _backward(inp, o, lse, causal, None, False)
    for n in ("dq", "dk", "dv"):
        a, b = first[n].float(), default[n].float()
        # the two modes differ only by the summation of dQ partials: a few 16-bit ulps
        assert (a - b).abs().max().item() <= 2e-3 * b.abs().max().item(), n


def test_deterministic_full_size_default_workload():
    """The 64 x 16 x 1024 x 64 workload: repeatable bits, parity on sampled heads."""
    P.ensure_built()
    w = workloads()["gpt2_B64_H16_N1024_d64"]
    inp = workload_inputs(w)
    o, lse, _ = P.gpu_forward(inp, False, None)
    a = _backward(inp, o, lse, False, None, True)
    b = _backward(inp, o, lse, False, None, True)
    for n in ("dq", "dk", "dv"):
        assert torch.equal(a[n], b[n]), n
    heads = P.sample_heads(w.B, w.H, 4, seed=5300)
    ref, _, _ = P.oracle_backward(inp, False, None, heads=heads)
    P.check_grads(a, ref, heads=heads, label="deterministic full size")


def test_range_error_is_reported_and_cleared():
    """dO and V scaled by 2^12 make dS * K partials far above 2^20: the call reports
    FA_ERR_RANGE through fa_check_status, and the next call is clean again."""
    P.ensure_built()
    inp = P.inputs(1, 2, 256, 64, seed=5400)
    big = dict(inp)
    big["v"] = (inp["v"].float() * 4096).to(torch.bfloat16)
    big["dout"] = (inp["dout"].float() * 4096).to(torch.bfloat16)
    o, lse, _ = P.gpu_forward(big, False, None)
    q, k, v, do = (big[n].cuda() for n in ("q", "k", "v", "dout"))
    fa.attention_backward(q, k, v, o, lse, do, deterministic=True)
    with pytest.raises(fa.FAError) as e:
        fa.fa_check_status()
    assert e.value.code == fa.FA_ERR_RANGE
    fa.fa_check_status()                       # cleared by the read
    o2, lse2, _ = P.gpu_forward(inp, False, None)
    got = _backward(inp, o2, lse2, False, None, True)
    ref, _, _ = P.oracle_backward(inp, False, None)
    P.check_grads(got, ref, label="after range error")
