"""GPU: no N x N buffer is ever allocated (NeurIPS22 summary, "核心方法": the fused pass keeps
the score and probability tiles on chip, so memory grows linearly in N).

On the long-context workload (B1 H32 N16384 d128, causal, K x4), after one warm-up step has
loaded the library's device code, a forward + backward step through the C ABI changes
neither the device's free memory (cudaMemGetInfo, read through torch.cuda.mem_get_info) nor
torch's peak allocation: the library allocates nothing, and the only scratch is the caller's
backward workspace, whose size is O(B*H*N*d) -- far below even one head's N x N fp32 score
matrix (1 GiB at N = 16384)."""

from __future__ import annotations

import pytest
import torch

import exact_attention_111_b200 as fa
from exact_attention_111_b200.inputs import workloads
from tests import parity as P

pytestmark = pytest.mark.gpu


def test_step_allocates_nothing_and_workspace_is_linear_in_n():
    P.ensure_built()
    w = workloads()["long_B1_H32_N16384_d128_causal_k4"]
    B, H, N, d = w.B, w.H, w.N, w.d
    g = torch.Generator(device="cuda").manual_seed(5)
    q, k, v, do = (torch.randn((B, H, N, d), generator=g, device="cuda").to(torch.bfloat16) for _ in range(4))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    wsb = fa.fa_bwd_workspace_bytes(B, H, N, d)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        fa.fa_fwd(q, k, v, o, lse, B, H, N, d, w.scale, True, None, stream)
        fa.fa_bwd(q, k, v, o, lse, do, dq, dk, dv, B, H, N, d, w.scale, True, None, ws, wsb, stream)

    step()                              # loads the kernels' modules on this device
    fa.fa_check_status()
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats()
    base = torch.cuda.memory_allocated()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(2):
        step()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    fa.fa_check_status()
    assert free1 == free0, f"a step changed free device memory by {free0 - free1} bytes"
    assert torch.cuda.max_memory_allocated() == base
    # the workspace: fp32 dQ accumulator plus two per-row fp32 vectors over whole tiles
    Np = (N + 127) // 128 * 128
    assert wsb == B * H * N * d * 4 + 2 * B * H * Np * 4
    one_head_scores = N * N * 4
    assert wsb < one_head_scores / 3
    assert torch.isfinite(dq.float()).all() and torch.isfinite(o.float()).all()
