"""GPU: the backward with each key tile's query range split over several CTAs
(fa_bwd_args.query_splits), against the fp64 oracle and the unsplit backward.

The split ranges add their dK / dV partials in fp32, so the result equals the unsplit one up to
summation order; it is held to the same tolerances against the oracle (tests/parity.py), and
every (query tile, key tile) pair the masks keep is computed exactly once across the ranges
(visit log).  Ranges that hold no kept tile (more splits than steps, causal tails) do nothing."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import exact_attention_111_b200 as fa
import oracle.dropout as od
from exact_attention_111_b200.inputs import random_blockmask, workloads, workload_inputs
from tests import parity as P

pytestmark = pytest.mark.gpu

CASES = [
    # B, H, N, d, causal, mask, S, dtype
    (1, 1, 1000, 64, True, None, 3, torch.bfloat16),
    (1, 2, 640, 128, False, None, 2, torch.bfloat16),
    (2, 1, 2048, 128, True, None, 4, torch.bfloat16),
    (1, 1, 777, 64, False, "random", 5, torch.bfloat16),
    (1, 1, 300, 128, True, None, 7, torch.bfloat16),        # more ranges than steps
    (1, 2, 1100, 64, True, "random", 3, torch.float16),
    (1, 1, 4096, 128, True, None, 3, torch.bfloat16),
]


def _mask(kind, N, seed):
    if kind is None:
        return None
    m = random_blockmask((N + 127) // 128, 0.5, seed)
    return m


@pytest.mark.parametrize("B,H,N,d,causal,mask_kind,S,dtype", CASES)
def test_split_backward_matches_oracle_and_unsplit(B, H, N, d, causal, mask_kind, S, dtype):
    P.ensure_built()
    inp = P.inputs(B, H, N, d, seed=7100 + N + S, dtype=dtype)
    mask = _mask(mask_kind, N, 17)
    o, lse, _ = P.gpu_forward(inp, causal, mask)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "dout"))
    m = P.to_dev(mask)
    T = (N + 127) // 128
    vl = torch.zeros((B, H, T, T), dtype=torch.int32, device="cuda")
    dq, dk, dv = fa.attention_backward(q, k, v, o, lse, do, causal=causal, blockmask=m, query_splits=S, visit_log=vl)
    ref_q, ref_k, ref_v = fa.attention_backward(q, k, v, o, lse, do, causal=causal, blockmask=m)
    fa.fa_check_status()
    torch.cuda.synchronize()
    assert np.array_equal(vl.cpu().numpy(), P.expected_visits(B, H, N, causal, mask))
    ref, _, _ = P.oracle_backward(inp, causal, mask)
    P.check_grads({"dq": dq, "dk": dk, "dv": dv}, ref, label=f"split S={S}")
    for g, r in ((dq, ref_q), (dk, ref_k), (dv, ref_v)):
        scale = r.float().abs().max().item()
        assert (g.float() - r.float()).abs().max().item() <= 2e-2 * scale + 1e-6


def test_split_backward_with_dropout():
    P.ensure_built()
    B, H, N, d, p, seed = 1, 2, 640, 64, 0.2, 4242
    inp = P.inputs(B, H, N, d, seed=7200)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "dout"))
    o, lse = fa.attention_forward(q, k, v, causal=True, dropout_p=p, dropout_seed=seed)
    dq, dk, dv = fa.attention_backward(q, k, v, o, lse, do, causal=True, dropout_p=p, dropout_seed=seed,
                                       query_splits=3)
    fa.fa_check_status()
    rq, rk, rv, _, _ = od.attention_bwd_dropout(inp["q"], inp["k"], inp["v"], inp["dout"], 1.0 / np.sqrt(d), p,
                                                seed, True)
    P.check_grads({"dq": dq, "dk": dk, "dv": dv}, {"dq": rq, "dk": rk, "dv": rv}, label="split + dropout")


def test_split_backward_refuses_deterministic():
    P.ensure_built()
    inp = P.inputs(1, 1, 256, 64, seed=7300)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "dout"))
    o, lse = fa.attention_forward(q, k, v)
    with pytest.raises(fa.FAError):
        fa.attention_backward(q, k, v, o, lse, do, deterministic=True, query_splits=2)


def test_split_backward_full_size_single_causal_head():
    """One causal head of 16384 tokens with the chosen split count (the case the split is for),
    the whole head against the oracle."""
    P.ensure_built()
    w = workloads()["splitkv_B1_H1_N16384_d128_causal"]
    S = fa.fa_bwd_splitq_choose(w.B, w.H, w.N, w.causal, torch.cuda.get_device_properties(0).multi_processor_count)
    assert S >= 2
    inp = workload_inputs(w)
    o, lse, _ = P.gpu_forward(inp, w.causal, None)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "dout"))
    dq, dk, dv = fa.attention_backward(q, k, v, o, lse, do, causal=True, query_splits=S)
    fa.fa_check_status()
    ref, _, _ = P.oracle_backward(inp, True, None)
    P.check_grads({"dq": dq, "dk": dk, "dv": dv}, ref, label=f"full-size split S={S}")
