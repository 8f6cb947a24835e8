"""GPU parity of the split-KV forward, the forward over a key slice, and the LSE merge,
against the fp64 oracle (attention over a key slice at a key offset, and its merge).

The merge rule (O = sum_s exp(LSE_s - LSE) O_s, LSE = logsumexp_s LSE_s) is the
online-softmax rescaling of FlashAttention-NeurIPS22 "核心方法 / Tiling 与 online softmax"
applied once per slice of the keys."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import exact_attention_111_b200 as fa
import oracle.attention as ora
from exact_attention_111_b200.inputs import random_blockmask, butterfly_blockmask, workloads, workload_inputs
from tests.parity import (O_TOL, LSE_TOL, check_forward, ensure_built, half_ulp16, inputs,
                          oracle_forward, to_dev)

pytestmark = pytest.mark.gpu


def _mask(kind, T, seed):
    if kind is None:
        return None
    if kind == "random":
        return random_blockmask(T, 0.5, seed)
    if kind == "butterfly":
        return butterfly_blockmask(T)
    if kind == "holes":          # whole tile rows without any key: O = 0, LSE = -inf there
        m = random_blockmask(T, 0.5, seed, keep_diagonal=False)
        m[1, :] = 0
        return m
    raise ValueError(kind)


SPLIT_CASES = [
    # B, H, N, d, causal, mask, num_splits
    (1, 2, 1000, 64, False, None, 2),
    (1, 2, 1000, 64, True, None, 3),
    (2, 1, 777, 128, False, None, 4),
    (1, 1, 1500, 128, True, "random", 5),
    (1, 2, 640, 64, False, None, 9),          # more ranges than key tiles: ranges of 1 tile
    (1, 1, 2048, 64, False, "holes", 4),
    (1, 1, 4096, 64, False, "butterfly", 8),
    (2, 2, 300, 128, True, None, 64),
    (1, 1, 129, 64, False, None, 2),          # second range holds one key
]


@pytest.mark.parametrize("B,H,N,d,causal,mask_kind,S", SPLIT_CASES)
def test_splitkv_matches_oracle(B, H, N, d, causal, mask_kind, S):
    ensure_built()
    inp = inputs(B, H, N, d, seed=4000 + N + S)
    T = (N + 127) // 128
    mask = _mask(mask_kind, T, 7)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o, lse, used = fa.attention_forward_splitkv(q, k, v, causal=causal, blockmask=to_dev(mask), num_splits=S)
    sp = -(-T // S)
    assert fa.fa_last_launch_count() == (2 if S > 1 else 1) and used == S
    fa.fa_check_status()
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle_forward(inp, causal, mask)
    check_forward(o, lse, o_ref, lse_ref, o16_dtype=torch.bfloat16, label=f"splitkv S={S} ({sp} tiles/range)")


def test_splitkv_one_range_is_the_plain_forward():
    ensure_built()
    inp = inputs(1, 2, 1000, 64, seed=4100)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o1, l1, _ = fa.attention_forward_splitkv(q, k, v, causal=True, num_splits=1)
    assert fa.fa_last_launch_count() == 1
    o2, l2 = fa.attention_forward(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_splitkv_is_deterministic():
    ensure_built()
    inp = inputs(1, 1, 3000, 128, seed=4101)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    a = fa.attention_forward_splitkv(q, k, v, num_splits=6)
    b = fa.attention_forward_splitkv(q, k, v, num_splits=6)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


PARTIAL_CASES = [
    # B, H, N, Nk, key_offset, d, causal, mask
    (1, 2, 1000, 384, 256, 64, False, None),
    (1, 2, 1000, 384, 256, 64, True, None),
    (2, 1, 900, 260, 640, 128, True, "random"),     # ragged last slice at the sequence end
    (1, 1, 1024, 128, 896, 64, True, None),         # one key tile: rows before it see nothing
    (1, 1, 640, 512, 128, 128, False, "holes"),
    (1, 2, 300, 1000, 0, 64, False, None),          # cross-attention: more keys than queries
    (1, 1, 200, 77, 4096, 128, False, None),        # no mask: the offset is free
]


@pytest.mark.parametrize("B,H,N,Nk,off,d,causal,mask_kind", PARTIAL_CASES)
def test_partial_matches_oracle(B, H, N, Nk, off, d, causal, mask_kind):
    ensure_built()
    T = (N + 127) // 128
    mask = _mask(mask_kind, T, 9)
    qin = inputs(B, H, N, d, seed=4200 + N)
    if causal or mask is not None:
        full = inputs(B, H, N, d, seed=4300 + N)
        k = full["k"][:, :, off:off + Nk].contiguous()
        v = full["v"][:, :, off:off + Nk].contiguous()
    else:
        kv = inputs(B, H, Nk, d, seed=4300 + Nk)
        k, v = kv["k"], kv["v"]
    o, lse = fa.attention_forward_partial(qin["q"].cuda(), k.cuda(), v.cuda(), key_offset=off, causal=causal,
                                          blockmask=to_dev(mask))
    fa.fa_check_status()
    torch.cuda.synchronize()
    o_ref, lse_ref = ora.attention_fwd_partial(qin["q"], k, v, 1.0 / np.sqrt(d), causal, mask, key_offset=off)
    check_forward(o, lse, o_ref, lse_ref, o16_dtype=None, label=f"partial Nk={Nk} off={off}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("out", [torch.bfloat16, torch.float16, torch.float32])
def test_merge_matches_oracle(d, out):
    ensure_built()
    g = torch.Generator().manual_seed(4400 + d)
    S, B, H, N = 5, 2, 3, 301
    o_parts = torch.randn((S, B, H, N, d), generator=g)
    lse_parts = torch.randn((S, B, H, N), generator=g) * 4 + 10
    drop = torch.rand((S, B, H, N), generator=g) < 0.3
    lse_parts[drop] = -float("inf")
    o_parts[drop] = 0.0
    lse_parts[:, 0, 0, :7] = -float("inf")           # rows no part saw a key for
    o_parts[:, 0, 0, :7] = 0.0
    dev_o = [o_parts[s].cuda().contiguous() for s in range(S)]
    dev_l = [lse_parts[s].cuda().contiguous() for s in range(S)]
    o, lse = fa.lse_merge(dev_o, dev_l, out_dtype=out)
    assert fa.fa_last_launch_count() == 1
    torch.cuda.synchronize()
    o_ref, lse_ref = ora.lse_merge(o_parts.double().numpy(), lse_parts.double().numpy())
    og = o.double().cpu().numpy()
    lg = lse.double().cpu().numpy()
    # fp32 arithmetic on O(1) values: 1e-5, plus half an output ulp for 16-bit outputs
    floor = half_ulp16(np.abs(o_ref) + 1e-5, out) if out != torch.float32 else 0.0
    assert np.all(np.abs(og - o_ref) <= 1e-5 + floor)
    neg = np.isneginf(lse_ref)
    assert np.array_equal(neg, np.isneginf(lg))
    assert np.abs(lg[~neg] - lse_ref[~neg]).max() <= 1e-5
    assert np.all(og[0, 0, :7] == 0.0)


@pytest.mark.parametrize("R,causal,mask_kind", [(2, False, None), (3, True, None), (4, True, "random"),
                                                (5, False, "butterfly")])
def test_sharded_partials_merge_to_full_attention(R, causal, mask_kind):
    """A sequence sharded over R key shards (each its own tensor at its key offset) gives,
    after the merge, full attention over the whole sequence -- the exchange of a
    sequence-sharded forward, run here one shard after another on one GPU."""
    ensure_built()
    B, H, N, d = 1, 2, 2000, 64
    T = (N + 127) // 128
    mask = _mask(mask_kind, T, 11)
    inp = inputs(B, H, N, d, seed=4500 + R)
    q = inp["q"].cuda()
    cuts = [(r * T // R) * 128 for r in range(R)] + [N]    # R non-empty tile-aligned shards
    parts = []
    for r in range(R):
        a, b = cuts[r], cuts[r + 1]
        k = inp["k"][:, :, a:b].contiguous().cuda()
        v = inp["v"][:, :, a:b].contiguous().cuda()
        parts.append(fa.attention_forward_partial(q, k, v, key_offset=a, causal=causal, blockmask=to_dev(mask)))
    o, lse = fa.lse_merge([p[0] for p in parts], [p[1] for p in parts])
    fa.fa_check_status()
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle_forward(inp, causal, mask)
    check_forward(o, lse, o_ref, lse_ref, o16_dtype=torch.bfloat16, label=f"{R} shards")


@pytest.mark.parametrize("name", ["splitkv_B1_H1_N16384_d128", "splitkv_B1_H1_N16384_d128_causal"])
def test_splitkv_full_size_sampled_rows(name):
    """The full workload with the split count chosen for this GPU; the oracle evaluates a
    seeded sample of whole query rows (each row's O and LSE depend only on that row's
    query, so a row sample is exact), always including the first and last rows."""
    ensure_built()
    w = workloads()[name]
    inp = workload_inputs(w, with_dout=False)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o, lse, S = fa.attention_forward_splitkv(q, k, v, causal=w.causal)
    assert S == fa.fa_splitkv_choose(w.B, w.H, w.N, w.causal,
                                     torch.cuda.get_device_properties(0).multi_processor_count)
    assert S > 1, "the workload is meant to exercise several key ranges"
    fa.fa_check_status()
    torch.cuda.synchronize()
    r = np.random.default_rng(4600)
    rows = np.unique(np.concatenate([[0, 127, 128, w.N - 1], r.integers(0, w.N, 200)]))
    o_ref, lse_ref = ora.attention_fwd_rows(inp["q"][0, 0].double().numpy(), inp["k"][0, 0].double().numpy(),
                                            inp["v"][0, 0].double().numpy(), w.scale, w.causal, rows)
    og = o[0, 0, rows].double().cpu().numpy()
    lg = lse[0, 0, rows].double().cpu().numpy()
    assert np.all(np.abs(og - o_ref) <= O_TOL + half_ulp16(np.abs(o_ref) + O_TOL, torch.bfloat16))
    assert np.abs(lg - lse_ref).max() <= LSE_TOL
