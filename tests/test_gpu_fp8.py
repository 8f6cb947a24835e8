"""GPU parity of the FP8 (E4M3) forward against the fp64 oracle evaluated on the values
the E4M3 codes stand for (codes * per-tensor dequantisation factor).

Bound (derived in include/fa.h): the kernel's only departure from the exact attention of
those values is rounding 256 P to E4M3 before the P V product -- relative error 2^-4, or
absolute 2^-18 on P below E4M3's normal range -- so elementwise
    |O - O_ref| <= 2^-4 (P |V|)_ic + 2^-18 sum_j |V_jc| + 1e-3
(the 1e-3 covers the fp32 accumulation and exp2), plus half an output ulp for bf16 O.
LSE comes from the unrounded P: 1e-3, as for the 16-bit forward."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import exact_attention_111_b200 as fa
import oracle.attention as ora
from exact_attention_111_b200.inputs import quantize_e4m3, random_blockmask, workloads, workload_inputs
from tests import parity as P

pytestmark = pytest.mark.gpu


def _quantized(inp):
    out = {}
    for n in ("q", "k", "v"):
        codes, ds = quantize_e4m3(inp[n])
        out[n] = (codes, ds, codes.to(torch.float64) * ds)
    return out


def _check(o, lse, qz, causal, mask, heads, o_fp32, label):
    q, k, v = (qz[n][2] for n in ("q", "k", "v"))
    scale = 1.0 / np.sqrt(q.shape[-1])
    og = o.double().cpu().numpy()
    lg = lse.double().cpu().numpy()
    worst = 0.0
    for b, h in heads:
        O, L, Pm = ora.attention_fwd_head(q[b, h].numpy(), k[b, h].numpy(), v[b, h].numpy(), scale, causal,
                                          None if mask is None else mask.numpy(), return_p=True)
        av = np.abs(v[b, h].numpy())
        bound = 2.0 ** -4 * (Pm @ av) + 2.0 ** -18 * av.sum(axis=0)[None, :] + 1e-3
        if not o_fp32:
            bound = bound + P.half_ulp16(np.abs(O) + bound, torch.bfloat16)
        err = np.abs(og[b, h] - O)
        assert np.all(np.isfinite(og[b, h])), label
        assert np.all(err <= bound), f"{label}: O error {err.max():.4g} above its bound at head {(b, h)}"
        neg = np.isneginf(L)
        assert np.array_equal(neg, np.isneginf(lg[b, h])), label
        if (~neg).any():
            assert np.abs(lg[b, h][~neg] - L[~neg]).max() <= P.LSE_TOL, label
        worst = max(worst, float((err / bound).max()))
    return worst


CASES = [
    # B, H, N, causal, mask, o_fp32
    (1, 2, 128, False, False, False),
    (1, 1, 1, False, False, True),
    (2, 2, 300, True, False, False),
    (1, 2, 129, False, False, True),
    (1, 2, 1000, False, False, False),
    (1, 2, 1000, True, False, True),
    (2, 1, 777, False, True, False),
    (1, 2, 1100, True, True, False),
]


@pytest.mark.parametrize("B,H,N,causal,use_mask,o_fp32", CASES)
def test_fp8_forward_within_bound(B, H, N, causal, use_mask, o_fp32):
    P.ensure_built()
    inp = P.inputs(B, H, N, 128, seed=7000 + N)
    qz = _quantized(inp)
    mask = None
    if use_mask:
        mask = random_blockmask((N + 127) // 128, 0.5, seed=8, keep_diagonal=False)
        mask[1, :] = 0
    q8, k8, v8 = (qz[n][0].cuda() for n in ("q", "k", "v"))
    o, lse = fa.attention_forward_fp8(q8, k8, v8, qz["q"][1], qz["k"][1], qz["v"][1], causal=causal,
                                      blockmask=P.to_dev(mask), o_fp32=o_fp32)
    assert fa.fa_last_launch_count() == 2
    fa.fa_check_status()
    torch.cuda.synchronize()
    heads = [(b, h) for b in range(B) for h in range(H)]
    _check(o, lse, qz, causal, mask, heads, o_fp32, f"fp8 N{N} causal{causal}")


def test_fp8_is_deterministic_and_close_to_bf16():
    P.ensure_built()
    inp = P.inputs(1, 4, 2048, 128, seed=7100)
    qz = _quantized(inp)
    q8, k8, v8 = (qz[n][0].cuda() for n in ("q", "k", "v"))
    a = fa.attention_forward_fp8(q8, k8, v8, qz["q"][1], qz["k"][1], qz["v"][1])
    b = fa.attention_forward_fp8(q8, k8, v8, qz["q"][1], qz["k"][1], qz["v"][1])
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_fp8_full_size_sampled_heads():
    """The 4 x 16 x 4096 x 128 sweep point, quantized per tensor; two whole heads checked."""
    P.ensure_built()
    w = workloads()["sweep_B4_H16_N4096_d128"]
    inp = workload_inputs(w, with_dout=False)
    qz = _quantized(inp)
    q8, k8, v8 = (qz[n][0].cuda() for n in ("q", "k", "v"))
    o, lse = fa.attention_forward_fp8(q8, k8, v8, qz["q"][1], qz["k"][1], qz["v"][1])
    fa.fa_check_status()
    torch.cuda.synchronize()
    _check(o, lse, qz, False, None, [(0, 0), (3, 15)], False, "fp8 full size")
