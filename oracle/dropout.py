"""fp64 CPU oracle for attention with dropout -- TEST INFRASTRUCTURE, not part of the product.

Same rules as ``attention.py``: only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU legs may import it, and it shares no code with the CUDA path.

The pages fuse dropout into the attention kernel and regenerate its mask in the backward
pass from the saved random-generator state instead of storing it (FlashAttention-NeurIPS22
summary, "核心方法 / Kernel fusion" and "Backward recomputation").  They fix neither the
generator nor the mask layout; the readings taken here:

  * generator: Philox4x32-10, the counter-based generator of Salmon, Moraes, Dror and
    Shaw, "Parallel random numbers: as easy as 1, 2, 3" (SC'11): a 128-bit counter and a
    64-bit key, ten rounds of two 32x32->64-bit products with the constants below, the key
    bumped by two Weyl constants between rounds;
  * key = (seed mod 2^32, seed div 2^32); counter = (j div 16, i, b*H + h, 0) for query
    row i and key j of head (b, h), so one call covers 16 consecutive keys of one row;
  * byte k (0..15) of the call's 128 output bits, little-endian within each 32-bit word,
    decides key 16*(j div 16) + k: dropped iff byte < t with t = floor(256 p + 1/2), so the
    dropout probability p is applied in steps of 1/256, and kept entries are scaled by
    256 / (256 - t) (so E[mask] = 1 exactly);
  * forward: O = (P o M) V with M = keep * 256/(256 - t); the row statistics (max, exp-sum,
    LSE) are those of the undropped P, which the backward needs;
  * backward (textbook calculus on L = sum(dO o O)):
        dV = (P o M)ᵀ dO,   dP = (dO Vᵀ) o M,   D_i = sum_j P_ij dP_ij = sum_c dO_ic O_ic,
        dS = P o (dP - D),  dQ = scale * dS K,  dK = scale * dSᵀ Q.
"""

from __future__ import annotations

import numpy as np

from .attention import _keep_matrix, softmax_rows, _as64

PHILOX_M0, PHILOX_M1 = 0xD2511F53, 0xCD9E8D57     # round multipliers
PHILOX_W0, PHILOX_W1 = 0x9E3779B9, 0xBB67AE85     # key increments (Weyl sequence)
_MASK32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(ctr, key):
    """ctr: uint32 array [..., 4]; key: (k0, k1).  Returns uint32 [..., 4]."""
    c = [np.asarray(ctr, np.uint64)[..., t] for t in range(4)]
    k0, k1 = np.uint64(key[0]), np.uint64(key[1])
    for r in range(10):
        if r > 0:
            k0 = (k0 + np.uint64(PHILOX_W0)) & _MASK32
            k1 = (k1 + np.uint64(PHILOX_W1)) & _MASK32
        p0 = np.uint64(PHILOX_M0) * c[0]
        p1 = np.uint64(PHILOX_M1) * c[2]
        c = [(p1 >> np.uint64(32)) ^ c[1] ^ k0, p1 & _MASK32, (p0 >> np.uint64(32)) ^ c[3] ^ k1, p0 & _MASK32]
    return np.stack(c, axis=-1).astype(np.uint32)


def drop_threshold(p: float) -> int:
    """Byte threshold t: an entry is dropped iff its random byte < t."""
    if not (0.0 <= p < 1.0):
        raise ValueError("dropout probability must be in [0, 1)")
    return min(255, int(np.floor(256.0 * p + 0.5)))


def keep_mask(bh: int, N: int, Nk: int, seed: int, p: float) -> np.ndarray:
    """Boolean [N, Nk]: True where score (i, j) of head index bh = b*H + h is kept."""
    t = drop_threshold(p)
    nb = (Nk + 15) // 16
    i, jb = np.meshgrid(np.arange(N, dtype=np.uint64), np.arange(nb, dtype=np.uint64), indexing="ij")
    ctr = np.stack([jb, i, np.full_like(i, bh), np.zeros_like(i)], axis=-1)
    words = philox4x32_10(ctr, (seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF))   # [N, nb, 4]
    # bytes in key order: word w holds keys 4w .. 4w+3 of the block, least significant byte first
    by = np.stack([(words >> np.uint32(8 * s)) & np.uint32(0xFF) for s in range(4)], axis=-1)   # [N, nb, 4, 4]
    by = by.reshape(N, nb * 16)
    return by[:, :Nk] >= t


def keep_scale(p: float) -> float:
    return 256.0 / (256 - drop_threshold(p))


def attention_fwd_head_dropout(q, k, v, scale: float, keep, drop_scale: float, causal: bool = False,
                               blockmask=None, tile: int = 128):
    """One head with a given keep mask [N, N]: returns (O, LSE, P, M)."""
    q, k, v = (np.asarray(x, np.float64) for x in (q, k, v))
    N = q.shape[0]
    S = scale * (q @ k.T)
    km = _keep_matrix(N, causal, blockmask, tile)
    if km is not None:
        S = np.where(km, S, -np.inf)
    P, _, _, lse = softmax_rows(S)
    M = np.where(keep, drop_scale, 0.0)
    return (P * M) @ v, lse, P, M


def attention_bwd_head_dropout(q, k, v, dout, scale: float, keep, drop_scale: float, causal: bool = False,
                               blockmask=None, tile: int = 128):
    """Returns (dQ, dK, dV, O, LSE) of L = sum(dout o O) for the dropout forward above."""
    q, k, v, dout = (np.asarray(x, np.float64) for x in (q, k, v, dout))
    O, lse, P, M = attention_fwd_head_dropout(q, k, v, scale, keep, drop_scale, causal, blockmask, tile)
    dV = (P * M).T @ dout
    dP = (dout @ v.T) * M
    D = (P * dP).sum(axis=1)
    dS = P * (dP - D[:, None])
    return scale * (dS @ k), scale * (dS.T @ q), dV, O, lse


def attention_fwd_dropout(q, k, v, scale: float, p: float, seed: int, causal: bool = False, blockmask=None,
                          heads=None):
    """Batched [B, H, N, d]: (O, LSE) with the Philox mask of every (b, h); others NaN."""
    q, k, v = _as64(q), _as64(k), _as64(v)
    B, H, N, _ = q.shape
    bm = None if blockmask is None else _as64(blockmask)
    O = np.full(q.shape, np.nan)
    L = np.full((B, H, N), np.nan)
    ds = keep_scale(p)
    for b, h in (heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]):
        keep = keep_mask(b * H + h, N, N, seed, p)
        O[b, h], L[b, h], _, _ = attention_fwd_head_dropout(q[b, h], k[b, h], v[b, h], scale, keep, ds, causal, bm)
    return O, L


def attention_bwd_dropout(q, k, v, dout, scale: float, p: float, seed: int, causal: bool = False, blockmask=None,
                          heads=None):
    """Batched: (dQ, dK, dV, O, LSE); unevaluated heads are NaN."""
    q, k, v, dout = _as64(q), _as64(k), _as64(v), _as64(dout)
    B, H, N, d = q.shape
    bm = None if blockmask is None else _as64(blockmask)
    out = [np.full(q.shape, np.nan) for _ in range(4)] + [np.full((B, H, N), np.nan)]
    ds = keep_scale(p)
    for b, h in (heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]):
        keep = keep_mask(b * H + h, N, N, seed, p)
        r = attention_bwd_head_dropout(q[b, h], k[b, h], v[b, h], dout[b, h], scale, keep, ds, causal, bm)
        for t in range(5):
            out[t][b, h] = r[t]
    return tuple(out)
