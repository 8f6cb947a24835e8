"""GPU: fused dropout in the forward and backward kernels against the fp64 dropout oracle
(oracle/dropout.py: Philox4x32-10 mask, byte threshold t = round(256 p), scale 256/(256-t)).

O tolerance, elementwise and derived from the arithmetic.  With P~ = P o M (M the keep mask
times s = 256/(256 - t)), the kernel forms O_ic = sum_j r(p_ij s m_ij) V_jc / l_i, where p_ij
is P's unnormalised fp32 value and r() the rounding of the PV operand to 16 bits.  The error
against the exact O_ref = sum_j P~_ij V_jc is at most
  - u * sum_j P~_ij |V_jc| from r() (u = 2^-8 for bf16, 2^-11 for fp16: half an ulp, relative);
  - 1.1e-4 * sum_j P~_ij |V_jc| from each p_ij's exp2 (the FMA-pipe polynomial's bound; the
    special-function unit is far more accurate), and 1.1e-4 * |O| from l_i, the sum of the
    same values;
  - fp32 accumulation in the tensor cores and the final 1/l multiply: a few 2^-24 relative;
so |O_gpu - O_ref| <= (u + 5e-4) * (P~ |V|)_ic + 1e-6, plus half an output ulp for 16-bit O.
(P~ |V|)_ic comes from the oracle's own P and M.  LSE (undropped) and the gradients keep
their tolerances.

The keep decisions are integers and are compared bit-exactly: with V an identity block the
forward's O is P o M itself, and with dO an identity block the backward's dV is (P o M)ᵀ,
so their zero patterns are the masks the kernels drew.  Values are compared within the
forward / backward tolerances."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import exact_attention_111_b200 as fa
import oracle.dropout as od
from exact_attention_111_b200.inputs import random_blockmask, workloads, workload_inputs
from tests import parity as P

pytestmark = pytest.mark.gpu


def _fwd(inp, causal, mask, p, seed):
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o, lse = fa.attention_forward(q, k, v, causal=causal, blockmask=P.to_dev(mask), dropout_p=p, dropout_seed=seed)
    fa.fa_check_status()
    torch.cuda.synchronize()
    return o, lse


def _bwd(inp, o, lse, causal, mask, p, seed, deterministic=False):
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "dout"))
    dq, dk, dv = fa.attention_backward(q, k, v, o, lse, do, causal=causal, blockmask=P.to_dev(mask),
                                       dropout_p=p, dropout_seed=seed, deterministic=deterministic)
    fa.fa_check_status()
    torch.cuda.synchronize()
    return {"dq": dq, "dk": dk, "dv": dv}


@pytest.mark.parametrize("B,H,N", [(2, 2, 256), (1, 3, 384)])
def test_forward_mask_is_bit_exact(B, H, N):
    """V = identity on one 128-key tile (zero elsewhere): O[i, j] = (P o M)[i, 128 kt + j]."""
    P.ensure_built()
    p, seed = 0.3, 0x0123_4567_89AB_CDEF
    base = P.inputs(B, H, N, 128, seed=6000 + N)
    for kt in range(N // 128):
        inp = dict(base)
        v = torch.zeros((B, H, N, 128), dtype=torch.bfloat16)
        v[:, :, 128 * kt:128 * (kt + 1)] = torch.eye(128, dtype=torch.bfloat16)
        inp["v"] = v
        o, _ = _fwd(inp, False, None, p, seed)
        kept = (o.float() != 0).cpu().numpy()
        for b in range(B):
            for h in range(H):
                ref = od.keep_mask(b * H + h, N, N, seed, p)[:, 128 * kt:128 * (kt + 1)]
                assert np.array_equal(kept[b, h], ref), (b, h, kt)


@pytest.mark.parametrize("d", [64, 128])
def test_backward_mask_is_bit_exact(d):
    """dO = identity on query rows off .. off+d-1 (zero elsewhere): dV[j, c] = (P o M)[off + c, j].
    d = 64 runs the four-group layout (32 query columns per group), d = 128 the two-group one."""
    P.ensure_built()
    B, H, N, p, seed = 2, 2, 384, 0.45, 987654321
    inp = P.inputs(B, H, N, d, seed=6100 + d)
    o, lse = _fwd(inp, False, None, p, seed)
    for off in range(0, 128, d):
        do = torch.zeros((B, H, N, d), dtype=torch.bfloat16)
        do[:, :, off:off + d] = torch.eye(d, dtype=torch.bfloat16)
        inp2 = dict(inp)
        inp2["dout"] = do
        g = _bwd(inp2, o, lse, False, None, p, seed)
        kept = (g["dv"].float() != 0).cpu().numpy()         # [B, H, N keys, d query rows]
        for b in range(B):
            for h in range(H):
                ref = od.keep_mask(b * H + h, N, N, seed, p)[off:off + d, :].T
                assert np.array_equal(kept[b, h], ref), (b, h, off)


CASES = [
    # B, H, N, d, causal, mask, p, dtype
    (1, 2, 128, 64, False, False, 0.1, torch.bfloat16),
    (2, 2, 300, 64, True, False, 0.5, torch.bfloat16),
    (1, 2, 1000, 128, False, False, 0.2, torch.bfloat16),
    (1, 2, 1000, 128, True, False, 0.1, torch.bfloat16),
    (2, 1, 777, 64, False, True, 0.3, torch.bfloat16),
    (1, 2, 640, 128, True, True, 0.9, torch.bfloat16),
    (1, 2, 500, 64, True, False, 0.25, torch.float16),
    (1, 1, 129, 128, False, False, 0.6, torch.float16),
]


def dropout_o_bound(inp, causal, mask, p, seed, dtype, heads=None):
    """Elementwise O bound of the module docstring, [B, H, N, d] (NaN on unevaluated heads)."""
    q, k, v = (inp[n].double().numpy() for n in ("q", "k", "v"))
    B, H, N, d = q.shape
    u = 2.0 ** -8 if dtype == torch.bfloat16 else 2.0 ** -11
    bound = np.full(q.shape, np.nan)
    bm = None if mask is None else np.asarray(mask)
    for b, h in (heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]):
        keep = od.keep_mask(b * H + h, N, N, seed, p)
        _, _, Pm, M = od.attention_fwd_head_dropout(q[b, h], k[b, h], v[b, h], 1.0 / np.sqrt(d), keep,
                                                     od.keep_scale(p), causal, bm)
        bound[b, h] = (u + 5e-4) * ((Pm * M) @ np.abs(v[b, h])) + 1e-6
    return bound


def _oracle(inp, causal, mask, p, seed):
    d = inp["q"].shape[-1]
    return od.attention_bwd_dropout(inp["q"], inp["k"], inp["v"], inp["dout"], 1.0 / np.sqrt(d), p, seed, causal,
                                    None if mask is None else mask.numpy())


@pytest.mark.parametrize("B,H,N,d,causal,use_mask,p,dtype", CASES)
def test_dropout_matches_oracle(B, H, N, d, causal, use_mask, p, dtype):
    P.ensure_built()
    seed = 1000 + N + d
    inp = P.inputs(B, H, N, d, seed=6200 + N + d, dtype=dtype)
    mask = None
    if use_mask:
        mask = random_blockmask((N + 127) // 128, 0.5, seed=4, keep_diagonal=False)
        mask[0, :] = 0
    o, lse = _fwd(inp, causal, mask, p, seed)
    dq, dk, dv, o_ref, lse_ref = _oracle(inp, causal, mask, p, seed)
    P.check_forward(o, lse, o_ref, lse_ref, o16_dtype=dtype, label=f"dropout p={p}",
                    o_bound=dropout_o_bound(inp, causal, mask, p, seed, dtype))
    got = _bwd(inp, o, lse, causal, mask, p, seed)
    P.check_grads(got, {"dq": dq, "dk": dk, "dv": dv}, label=f"dropout p={p}")


def test_p_zero_is_the_plain_path_and_seeds_matter():
    P.ensure_built()
    inp = P.inputs(1, 2, 700, 64, seed=6300)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o0, l0 = fa.attention_forward(q, k, v, causal=True)
    o1, l1 = fa.attention_forward(q, k, v, causal=True, dropout_p=0.0, dropout_seed=5)
    a1, _ = fa.attention_forward(q, k, v, causal=True, dropout_p=0.2, dropout_seed=5)
    a2, _ = fa.attention_forward(q, k, v, causal=True, dropout_p=0.2, dropout_seed=5)
    b1, lb = fa.attention_forward(q, k, v, causal=True, dropout_p=0.2, dropout_seed=6)
    torch.cuda.synchronize()
    assert torch.equal(o0, o1) and torch.equal(l0, l1)
    assert torch.equal(a1, a2)                       # same seed: same mask, same bits
    assert not torch.equal(a1, b1)                   # another seed: another mask
    assert torch.equal(lb, l0)                       # LSE is that of the undropped scores


def test_dropout_with_deterministic_backward_repeats_bitwise():
    P.ensure_built()
    inp = P.inputs(2, 4, 2048, 64, seed=6400)
    o, lse = _fwd(inp, False, None, 0.1, 77)
    a = _bwd(inp, o, lse, False, None, 0.1, 77, deterministic=True)
    b = _bwd(inp, o, lse, False, None, 0.1, 77, deterministic=True)
    for n in ("dq", "dk", "dv"):
        assert torch.equal(a[n], b[n]), n


def test_dropout_full_size_sampled_heads():
    P.ensure_built()
    w = workloads()["gpt2_B64_H16_N1024_d64"]
    inp = workload_inputs(w)
    p, seed = 0.1, 2718281828
    o, lse = _fwd(inp, False, None, p, seed)
    got = _bwd(inp, o, lse, False, None, p, seed)
    heads = P.sample_heads(w.B, w.H, 3, seed=6500)
    dq, dk, dv, o_ref, lse_ref = od.attention_bwd_dropout(inp["q"], inp["k"], inp["v"], inp["dout"], w.scale, p,
                                                          seed, heads=heads)
    P.check_forward(o, lse, o_ref, lse_ref, heads=heads, o16_dtype=torch.bfloat16, label="dropout full size",
                    o_bound=dropout_o_bound(inp, False, None, p, seed, torch.bfloat16, heads=heads))
    P.check_grads(got, {"dq": dq, "dk": dk, "dv": dv}, heads=heads, label="dropout full size")
