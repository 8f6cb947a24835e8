"""GPU: fa_bwd_noalloc, the backward entry point for callers that cannot allocate device
memory at call time (an engine plugin's enqueue step, a host program without a device
allocator, a frozen memory pool).  It must give the same gradients as fa_bwd with a
caller-provided workspace, call after call, although every call reuses one fixed device
array that still holds the previous call's data.

This file is collected last on purpose: it runs after every other test, and also passes
alone in a fresh process."""

from __future__ import annotations

import gc

import numpy as np
import pytest
import torch

import exact_attention_111_b200 as fa
from exact_attention_111_b200.inputs import make_inputs, random_blockmask
from tests import parity as P

pytestmark = pytest.mark.gpu

CASES = [
    # (B, H, N, d, causal, masked, seed): two different shapes, so the second call finds the
    # first call's leftovers in the shared scratch array at other offsets
    (2, 4, 1000, 128, True, False, 31),
    (1, 3, 777, 64, False, True, 32),
]


def _c_call(L, q, k, v, o, lse, do, dq, dk, dv, B, H, N, d, scale, causal, mask, stream):
    return L.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                            do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d, scale,
                            int(causal), None if mask is None else mask.data_ptr(), stream)


def test_noalloc_backward_matches_workspace_backward_on_consecutive_calls():
    P.ensure_built()
    L = fa.lib()
    stream = torch.cuda.current_stream().cuda_stream
    for B, H, N, d, causal, masked, seed in CASES:
        inp = make_inputs(B, H, N, d, seed)
        q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "dout"))
        T = (N + 127) // 128
        mask = random_blockmask(T, 0.5, seed).cuda() if masked else None
        scale = 1.0 / d ** 0.5
        o, lse = fa.attention_forward(q, k, v, causal=causal, blockmask=mask)
        ref = fa.attention_backward(q, k, v, o, lse, do, causal=causal, blockmask=mask)
        got = [torch.full_like(q, float("nan")) for _ in range(3)]
        rc = _c_call(L, q, k, v, o, lse, do, *got, B, H, N, d, scale, causal, mask, stream)
        assert rc == fa.FA_OK, fa.fa_status_string(rc)
        fa.fa_check_status()
        for name, g, r in zip(("dq", "dk", "dv"), got, ref):
            g64, r64 = g.double().cpu().numpy(), r.double().cpu().numpy()
            assert np.all(np.isfinite(g64)), name
            bound = P.GRAD_TOL * np.abs(r64).max()
            assert np.abs(g64 - r64).max() <= bound, f"{name}: {np.abs(g64 - r64).max()} > {bound}"


def test_noalloc_rejects_sizes_beyond_its_scratch():
    P.ensure_built()
    L = fa.lib()
    # 1 x 64 x 16384 x 128 needs ~540 MB of scratch, far beyond the fixed 64 MiB
    assert fa.fa_bwd_workspace_bytes(1, 64, 16384, 128) > (64 << 20)
    t = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    p = t.data_ptr()
    rc = L.fa_bwd_noalloc(p, p, p, p, p, p, p, p, p, 1, 64, 16384, 128, 0.088, 0, None, None)
    assert rc == fa.FA_ERR_WORKSPACE


def test_noalloc_calls_after_the_first_take_no_device_memory():
    """The first call on a device is its set-up (the runtime loads the code holding the fixed
    array, which commits the array, and the array's address is looked up).  Every later call
    must leave the device's free memory exactly as it was: cudaMemGetInfo (torch.cuda.
    mem_get_info) reads the same before and after it, and torch's allocator holds no more
    (it may hold less: tensors of earlier tests can be collected meanwhile)."""
    P.ensure_built()
    L = fa.lib()
    stream = torch.cuda.current_stream().cuda_stream
    B, H, N, d = 1, 2, 640, 64
    inp = make_inputs(B, H, N, d, 41)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "dout"))
    o, lse = fa.attention_forward(q, k, v, causal=False)
    got = [torch.empty_like(q) for _ in range(3)]
    assert _c_call(L, q, k, v, o, lse, do, *got, B, H, N, d, d ** -0.5, False, None, stream) == fa.FA_OK
    fa.fa_check_status()
    gc.collect()
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    for _ in range(2):
        assert _c_call(L, q, k, v, o, lse, do, *got, B, H, N, d, d ** -0.5, False, None, stream) == fa.FA_OK
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, f"free device memory changed by {free0 - free1} bytes"
    assert torch.cuda.memory_allocated() <= alloc0
    fa.fa_check_status()
