"""Seeded synthetic inputs shared by the kernels' tests, the benchmark and the oracle checks.

This module holds no attention arithmetic: it only draws random tensors and builds the
fixed tile mask used by the block-sparse workload.  Both the CUDA path and the fp64
oracle consume exactly the bits produced here.

Recipe (one rule for every workload):
  * a CPU ``torch.Generator`` seeded with ``seed`` draws fp32 N(0, 1) values in the order
    q, k, v, dO; each is rounded to nearest even into the compute dtype (bf16 or fp16);
  * the long-context workload multiplies K by 4 after rounding (exact in bf16/fp16, it is a
    power of two), which makes the softmax rows peaked;
  * the block-sparse workload uses the butterfly tile mask below, shared by all heads.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

TILE = 128  # side of one block-mask tile, in rows/keys


@dataclass(frozen=True)
class Workload:
    """One attention problem shape: [B, H, N, d] tensors plus masking options."""

    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool = False
    k_scale: float = 1.0
    butterfly: bool = False
    seed: int = 0
    fwd_splits: int | None = None   # None: plain forward; 0: split-KV, count chosen; n: n ranges
    extra: dict = field(default_factory=dict, compare=False)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def tiles(self) -> int:
        return (self.N + TILE - 1) // TILE


def workloads() -> dict[str, Workload]:
    """The workload families, named by what they are and their sizes: the single head, the
    GPT-2-shaped batch, the sequence-length sweep, the long peaked-causal context, the
    butterfly block-sparse batch, and one long head too few query tiles to fill the GPU
    (the split-KV forward's case)."""
    w: dict[str, Workload] = {}
    w["head_N128_d64"] = Workload("head_N128_d64", 1, 1, 128, 64, seed=1001)
    w["gpt2_B64_H16_N1024_d64"] = Workload("gpt2_B64_H16_N1024_d64", 64, 16, 1024, 64, seed=1002)
    for N in (512, 1024, 2048, 4096, 8192, 16384):
        B = 16384 // N
        for H, d in ((32, 64), (16, 128)):
            for causal in (False, True):
                name = f"sweep_B{B}_H{H}_N{N}_d{d}{'_causal' if causal else ''}"
                w[name] = Workload(name, B, H, N, d, causal=causal, seed=1003)
    w["long_B1_H32_N16384_d128_causal_k4"] = Workload(
        "long_B1_H32_N16384_d128_causal_k4", 1, 32, 16384, 128, causal=True, k_scale=4.0, seed=1004)
    w["butterfly_B8_H16_N4096_d64"] = Workload(
        "butterfly_B8_H16_N4096_d64", 8, 16, 4096, 64, butterfly=True, seed=1005)
    for causal in (False, True):
        name = f"splitkv_B1_H1_N16384_d128{'_causal' if causal else ''}"
        w[name] = Workload(name, 1, 1, 16384, 128, causal=causal, seed=1006, fwd_splits=0)
    return w


def butterfly_blockmask(T: int) -> torch.Tensor:
    """uint8 [T, T] tile mask: tile (i, j) kept iff i == j, i XOR j is a power of two,
    or the tile lies in the first tile row or column."""
    i = torch.arange(T).view(T, 1)
    j = torch.arange(T).view(1, T)
    x = i ^ j
    pow2 = (x > 0) & ((x & (x - 1)) == 0)
    keep = (i == j) | pow2 | (i == 0) | (j == 0)
    return keep.to(torch.uint8)


def random_blockmask(T: int, density: float, seed: int, keep_diagonal: bool = True) -> torch.Tensor:
    """uint8 [T, T] random tile mask (edge-case tests)."""
    g = torch.Generator().manual_seed(seed)
    m = (torch.rand((T, T), generator=g) < density)
    if keep_diagonal:
        m |= torch.eye(T, dtype=torch.bool)
    return m.to(torch.uint8)


def make_inputs(B: int, H: int, N: int, d: int, seed: int, dtype=torch.bfloat16,
                k_scale: float = 1.0, with_dout: bool = True) -> dict[str, torch.Tensor]:
    """CPU tensors q, k, v (and dout) of shape [B, H, N, d] in ``dtype``."""
    g = torch.Generator().manual_seed(seed)
    shape = (B, H, N, d)
    out = {}
    for name in ("q", "k", "v") + (("dout",) if with_dout else ()):
        out[name] = torch.randn(shape, generator=g, dtype=torch.float32).to(dtype)
    if k_scale != 1.0:
        out["k"] = (out["k"].float() * k_scale).to(dtype)
    return out


def workload_inputs(w: Workload, dtype=torch.bfloat16, with_dout: bool = True) -> dict[str, torch.Tensor]:
    x = make_inputs(w.B, w.H, w.N, w.d, w.seed, dtype=dtype, k_scale=w.k_scale, with_dout=with_dout)
    x["blockmask"] = butterfly_blockmask(w.tiles) if w.butterfly else None
    return x


def attention_flops(B: int, H: int, N: int, d: int, causal: bool, backward: bool) -> float:
    """Workload FLOP count used for TFLOP/s: 4*B*H*N^2*d for the forward pass, 2.5x that
    for the backward pass, both halved under causal masking."""
    f = 4.0 * B * H * N * N * d
    if backward:
        f *= 3.5
    if causal:
        f *= 0.5
    return f


def quantize_e4m3(x: torch.Tensor):
    """Per-tensor E4M3 codes of x: descale = max|x| / 448 and codes = E4M3(x / descale)
    (round to nearest even, torch.float8_e4m3fn).  Returns (codes, descale); the values
    the codes stand for are codes * descale."""
    amax = float(x.float().abs().max())
    descale = amax / 448.0 if amax > 0 else 1.0
    codes = (x.float() / descale).to(torch.float8_e4m3fn)
    return codes, descale
