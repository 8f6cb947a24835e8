"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI binding and
compare with the fp64 oracle on the same seeded inputs.

Tolerances (fixed for every case):
  * O:  max |O_gpu - O_ref| <= 1e-2 outright for fp32 O.  For 16-bit O the kernel's fp32
        value x (within 1e-2 of O_ref) is then rounded to the output type, which moves it by
        at most half an ulp of x; so elementwise |O_gpu - O_ref| <= 1e-2 + half_ulp(|O_ref| + 1e-2).
  * LSE: max |LSE_gpu - LSE_ref| <= 1e-3 (absolute), and -inf exactly where the oracle has -inf.
  * dQ, dK, dV: max |g_gpu - g_ref| <= 2e-2 * max |g_ref|, per tensor.
"""

from __future__ import annotations

import numpy as np
import torch

import exact_attention_111_b200 as fa
from exact_attention_111_b200 import build as fabuild
from exact_attention_111_b200.inputs import make_inputs
import oracle.attention as ora

O_TOL = 1e-2
LSE_TOL = 1e-3
GRAD_TOL = 2e-2

_built = False


def ensure_built():
    global _built
    if not _built:
        fabuild.build()
        fa.lib()
        _built = True


def to_dev(x):
    return None if x is None else x.cuda()


def gpu_forward(inp, causal, mask, o_fp32=False, visit=False, dtype_code=None):
    ensure_built()
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    m = to_dev(mask)
    B, H, N, d = q.shape
    vl = torch.zeros((B, H, (N + 127) // 128, (N + 127) // 128), dtype=torch.int32, device="cuda") if visit else None
    o, lse = fa.attention_forward(q, k, v, causal=causal, blockmask=m, o_fp32=o_fp32, visit_log=vl)
    fa.fa_check_status()
    torch.cuda.synchronize()
    return o, lse, vl


def gpu_backward(inp, o, lse, causal, mask, visit=False):
    ensure_built()
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "dout"))
    m = to_dev(mask)
    B, H, N, d = q.shape
    vl = torch.zeros((B, H, (N + 127) // 128, (N + 127) // 128), dtype=torch.int32, device="cuda") if visit else None
    dq, dk, dv = fa.attention_backward(q, k, v, o, lse, do, causal=causal, blockmask=m, visit_log=vl)
    fa.fa_check_status()
    torch.cuda.synchronize()
    return dq, dk, dv, vl


def half_ulp16(x: np.ndarray, dtype) -> np.ndarray:
    """Half the spacing of 16-bit floats at magnitude |x| (bf16: 8 significand bits,
    fp16: 11)."""
    bits = 8 if dtype == torch.bfloat16 else 11
    a = np.maximum(np.abs(x), 2.0 ** -14)
    return np.exp2(np.floor(np.log2(a)) - bits)


def check_forward(o_gpu, lse_gpu, o_ref, lse_ref, heads=None, o16_dtype=None, label="", o_tol=O_TOL,
                  o_bound=None):
    """Compare on all heads, or on the listed (b, h) heads.  ``o_bound`` (an array shaped like
    O) replaces the uniform 1e-2 O bound by an elementwise one derived from the arithmetic
    (dropout: see tests/test_gpu_dropout.py)."""
    o_gpu = o_gpu.double().cpu().numpy()
    lse_gpu = lse_gpu.double().cpu().numpy()
    sel = heads if heads is not None else [(b, h) for b in range(o_ref.shape[0]) for h in range(o_ref.shape[1])]
    worst_o = worst_l = 0.0
    for b, h in sel:
        og, orf = o_gpu[b, h], o_ref[b, h]
        lg, lr = lse_gpu[b, h], lse_ref[b, h]
        tol = o_tol if o_bound is None else o_bound[b, h]
        floor = half_ulp16(np.abs(orf) + tol, o16_dtype) if o16_dtype is not None else 0.0
        err = np.abs(og - orf)
        assert np.all(np.isfinite(og)), f"{label}: non-finite O at head {(b, h)}"
        assert np.all(err <= tol + floor), (
            f"{label}: O error {err.max():.4g} (head {(b, h)}, allowed {np.max(tol):.3g} + half an output ulp"
            f"{'' if o_bound is None else ', elementwise bound'})")
        neg = np.isneginf(lr)
        assert np.array_equal(neg, np.isneginf(lg)), f"{label}: -inf LSE pattern differs at head {(b, h)}"
        if (~neg).any():
            el = np.abs(lg[~neg] - lr[~neg]).max()
            assert el <= LSE_TOL, f"{label}: LSE error {el:.4g} at head {(b, h)}"
            worst_l = max(worst_l, el)
        worst_o = max(worst_o, err.max())
    return worst_o, worst_l


def check_grads(got, ref, heads=None, label=""):
    """got/ref: dicts name -> tensor/array [B,H,N,d]; per-tensor max-relative check."""
    out = {}
    for name in ("dq", "dk", "dv"):
        g = got[name].double().cpu().numpy()
        r = ref[name]
        sel = heads if heads is not None else [(b, h) for b in range(r.shape[0]) for h in range(r.shape[1])]
        gs = np.stack([g[b, h] for b, h in sel])
        rs = np.stack([r[b, h] for b, h in sel])
        assert np.all(np.isfinite(gs)), f"{label}: non-finite {name}"
        scale = np.abs(rs).max()
        err = np.abs(gs - rs).max()
        bound = GRAD_TOL * scale if scale > 0 else 1e-6
        assert err <= bound, f"{label}: {name} error {err:.4g} > {GRAD_TOL} * max|ref| = {bound:.4g}"
        out[name] = err / scale if scale > 0 else err
    return out


def oracle_forward(inp, causal, mask, heads=None):
    scale = 1.0 / np.sqrt(inp["q"].shape[-1])
    return ora.attention_fwd(inp["q"], inp["k"], inp["v"], scale, causal, mask, heads=heads)


def oracle_backward(inp, causal, mask, heads=None):
    scale = 1.0 / np.sqrt(inp["q"].shape[-1])
    dq, dk, dv, o, lse = ora.attention_bwd(inp["q"], inp["k"], inp["v"], inp["dout"], scale, causal, mask,
                                           heads=heads)
    return {"dq": dq, "dk": dk, "dv": dv}, o, lse


def sample_heads(B, H, n, seed):
    r = np.random.default_rng(seed)
    heads = {(0, 0), (B - 1, H - 1)}
    while len(heads) < min(n, B * H):
        heads.add((int(r.integers(B)), int(r.integers(H))))
    return sorted(heads)


def expected_visits(B, H, N, causal, mask):
    T = (N + 127) // 128
    keep = np.ones((T, T), bool)
    if causal:
        keep &= np.tri(T, T, 0, dtype=bool)
    if mask is not None:
        keep &= np.asarray(mask).astype(bool)
    return np.broadcast_to(keep.astype(np.int32), (B, H, T, T))


def inputs(B, H, N, d, seed, dtype=torch.bfloat16, k_scale=1.0):
    return make_inputs(B, H, N, d, seed, dtype=dtype, k_scale=k_scale)
