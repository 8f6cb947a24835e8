"""Sequence-sharded forward: one head's keys spread over the ranks of a process group.

Every rank holds all query rows and one contiguous, tile-aligned shard of the keys and
values (``shard_bounds``).  Each rank computes attention of every query over its own keys
only (``fa_fwd_partial``: fp32 O and LSE of its slice), the ranks exchange those partial
results, and each rank combines them with ``fa_lse_merge``:
    LSE = ln sum_r exp(LSE_r),   O = sum_r exp(LSE_r - LSE) O_r,
the online-softmax rescaling (FlashAttention-NeurIPS22 summary, "核心方法 / Tiling 与
online softmax") applied once per shard.  The NeurIPS22 summary leaves multi-GPU
sequence parallelism to future work ("设计取舍", "局限与 Future Work"); this is its exchange
step.

The exchange is an all-gather of the fp32 partials over the group's backend (NCCL on GPUs):
world x B*H*N*(4d + 4) bytes arrive at every rank.  The merge kernel reads its parts
through plain pointers, so a peer-memory variant (each rank reading the others' partials
over NVLink instead of gathering copies) needs no kernel change.
"""

from __future__ import annotations

TILE = 128


def shard_bounds(N: int, world: int) -> list[int]:
    """Key rows of each rank: rank r owns [bounds[r], bounds[r + 1]), tile-aligned, in order.
    Shards differ by at most one 128-row tile; with more ranks than tiles some are empty."""
    T = (N + TILE - 1) // TILE
    return [min(N, (r * T // world) * TILE) for r in range(world)] + [N]


def sequence_sharded_forward(q, k_shard, v_shard, causal=False, blockmask=None, scale=None, group=None,
                             partial=None, merge=None):
    """q: [B, H, N, d] (all query rows, identical on every rank); k_shard, v_shard: this rank's
    keys, rows shard_bounds(N, world)[rank] ..[rank + 1] of the sequence.  Returns (O, LSE)
    of attention over the whole sequence, on every rank.

    ``partial`` / ``merge`` default to the CUDA entry points (attention_forward_partial,
    lse_merge); they are parameters so that the exchange logic can also run on CPU ranks."""
    import torch
    import torch.distributed as dist

    from . import attention_forward_partial, lse_merge

    partial = attention_forward_partial if partial is None else partial
    merge = lse_merge if merge is None else merge
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, H, N, d = q.shape
    bounds = shard_bounds(N, world)
    nk = bounds[rank + 1] - bounds[rank]
    if k_shard.shape[2] != nk or v_shard.shape[2] != nk:
        raise ValueError(f"rank {rank} must hold key rows [{bounds[rank]}, {bounds[rank + 1]})")
    if nk > 0:
        o_part, lse_part = partial(q, k_shard, v_shard, key_offset=bounds[rank], causal=causal,
                                   blockmask=blockmask, scale=scale)
    else:  # no keys here: a part that every row ignores, in the partials' type (fp32 for 16-bit q)
        pt = torch.promote_types(q.dtype, torch.float32)
        o_part = torch.zeros((B, H, N, d), dtype=pt, device=q.device)
        lse_part = torch.full((B, H, N), float("-inf"), dtype=pt, device=q.device)
    o_all = [torch.empty_like(o_part) for _ in range(world)]
    lse_all = [torch.empty_like(lse_part) for _ in range(world)]
    dist.all_gather(o_all, o_part.contiguous(), group=group)
    dist.all_gather(lse_all, lse_part.contiguous(), group=group)
    return merge(o_all, lse_all, out_dtype=q.dtype)
