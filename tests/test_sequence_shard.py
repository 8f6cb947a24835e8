"""CPU (gloo): the exchange of the sequence-sharded forward -- shard bounds, key offsets,
the all-gather of partial results and their merge -- run on world-size 2, 3 and 5 CPU ranks
with the oracle's slice attention and merge standing in for the kernels (no GPU here).
The kernels themselves are checked on the GPU by tests/test_gpu_splitkv.py."""

from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from exact_attention_111_b200.sequence_shard import shard_bounds


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_shard_bounds():
    assert shard_bounds(2000, 2) == [0, 1024, 2000]
    assert shard_bounds(2000, 5) == [0, 384, 768, 1152, 1536, 2000]
    assert shard_bounds(100, 3) == [0, 0, 0, 100]          # one tile: the first ranks hold nothing
    for N in (1, 127, 128, 129, 1000, 16384):
        for world in (1, 2, 3, 8, 13):
            b = shard_bounds(N, world)
            assert b[0] == 0 and b[-1] == N and all(x <= y for x, y in zip(b, b[1:]))
            assert all(x % 128 == 0 for x in b[:-1])
            sizes = [y - x for x, y in zip(b, b[1:])]
            assert max(sizes) - min(s for s in sizes) <= 128 + (N % 128 and 128)


def _oracle_partial(q, k, v, key_offset, causal, blockmask, scale):
    import oracle
    s = (1.0 / q.shape[-1] ** 0.5) if scale is None else scale
    o, l = oracle.attention_fwd_partial(q, k, v, s, causal, blockmask, key_offset=key_offset)
    return torch.from_numpy(o), torch.from_numpy(l)


def _oracle_merge(o_parts, lse_parts, out_dtype=None):
    import oracle
    o, l = oracle.lse_merge(np.stack([p.numpy() for p in o_parts]), np.stack([p.numpy() for p in lse_parts]))
    return torch.from_numpy(o), torch.from_numpy(l)


def _worker(rank, world, port, N, causal, use_mask, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from exact_attention_111_b200.inputs import make_inputs, random_blockmask
        from exact_attention_111_b200.sequence_shard import sequence_sharded_forward
        d = 16
        x = make_inputs(1, 2, N, d, 77, with_dout=False)          # the same sequence on every rank
        mask = random_blockmask(-(-N // 128), 0.6, 5) if use_mask else None
        b = shard_bounds(N, world)
        q = x["q"].double()
        k = x["k"][:, :, b[rank]:b[rank + 1]].double().contiguous()
        v = x["v"][:, :, b[rank]:b[rank + 1]].double().contiguous()
        o, lse = sequence_sharded_forward(q, k, v, causal=causal, blockmask=mask,
                                          partial=lambda *a, **kw: _oracle_partial(*a, **kw),
                                          merge=_oracle_merge)
        out_q.put((rank, o.numpy(), lse.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,N,causal,use_mask", [(2, 700, False, False), (3, 700, True, False),
                                                     (5, 700, True, True), (3, 200, True, False)])
def test_sharded_forward_equals_full_attention(world, N, causal, use_mask):
    """(3, 200): two tiles over three ranks, so rank 0 holds no keys at all."""
    import oracle
    from exact_attention_111_b200.inputs import make_inputs, random_blockmask
    port = _free_port()
    ctx = mp.get_context("spawn")
    out_q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, N, causal, use_mask, out_q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [out_q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x = make_inputs(1, 2, N, 16, 77, with_dout=False)
    mask = random_blockmask(-(-N // 128), 0.6, 5) if use_mask else None
    o_ref, lse_ref = oracle.attention_fwd(x["q"], x["k"], x["v"], 0.25, causal, mask)
    for rank, o, lse in res:
        fin = np.isfinite(lse_ref)
        assert np.array_equal(np.isfinite(lse), fin), rank
        assert np.max(np.abs(lse[fin] - lse_ref[fin])) < 1e-12, rank
        assert np.max(np.abs(o - o_ref)) < 1e-12, rank
