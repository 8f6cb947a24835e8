"""fp64 CPU oracle for exact attention -- TEST INFRASTRUCTURE, not part of the product.

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py`` (its cpu_baseline leg and its
``--impl reference`` arm) may import this module.  It shares no code with the CUDA path:
no kernels, headers, helpers or constants.  It is plain numpy in float64.

What it computes
----------------
The method on the pages (FlashAttention-NeurIPS22 summary, sections "问题与动机" and
"核心方法"; FlashAttention-2 wiki, section "背景") claims to compute *exactly* the standard
attention output, only with fewer HBM accesses.  The oracle therefore writes out the
standard, materialised form (FlashAttention-NeurIPS22, "问题与动机": S = Q Kᵀ and
P = softmax(S) are both built as N x N matrices):

    S   = scale * Q Kᵀ                          (N x N, per (b, h) head)
    S_ij = -inf where the mask drops (i, j)
    m_i = max_j S_ij,  l_i = sum_j exp(S_ij - m_i)
    P   = exp(S - m) / l                        (rows sum to 1)
    O   = P V
    LSE_i = m_i + ln l_i                        (the saved softmax normalisation factor,
                                                 "核心方法 / Backward recomputation")

Backward: the closed-form gradient of softmax followed by two matrix products (textbook
calculus -- the pages name backward recomputation but print no formula):

    dV = Pᵀ dO,   dP = dO Vᵀ,   D_i = sum_j P_ij dP_ij,
    dS = P o (dP - D),   dQ = scale * dS K,   dK = scale * dSᵀ Q

Readings of points the pages leave open:
  * scale: the pages write softmax(QKᵀ)V with no scale; a caller-supplied ``scale``
    multiplies QKᵀ (1/sqrt(d) in every workload).
  * causal: key j is visible to query i iff j <= i (top-left aligned, equal lengths).
  * block mask: uint8 [T, T] over 128 x 128 tiles, shared by all heads; a zero tile drops
    every score in it ("核心方法 / Block-sparse 扩展": zero blocks are skipped).
  * a row with no visible key has O = 0, LSE = -inf and zero gradients.
  * a slice of the keys (one split of a split-KV forward, or one GPU's shard of a
    sequence-sharded one): key row j of the slice is key position key_offset + j, and
    causal and the block mask use that position.  Results over disjoint slices combine
    exactly by ``lse_merge`` (the online-softmax rescaling of "核心方法 / Tiling 与 online
    softmax", applied once per slice).

Also here, for the oracle's own self-test only: ``attention_fwd_head_tiled`` -- the
blockwise online-softmax recurrence of "核心方法 / Tiling 与 online softmax" (running row
max m and exp-sum l merged block by block), used to check that the tiled method reaches
the direct definition.  The CUDA path never calls anything here.
"""

from __future__ import annotations

import numpy as np

TILE = 128


def _keep_matrix(N: int, causal: bool, blockmask, tile: int = TILE, Nk: int | None = None,
                 key_offset: int = 0) -> np.ndarray | None:
    """Boolean [N, Nk]: True where score (i, j) takes part in the softmax; None = all.

    Key row j sits at position ``key_offset + j`` of the query sequence (0 and Nk = N for
    self-attention); causal and the block mask compare positions, not row indices."""
    Nk = N if Nk is None else Nk
    keep = None
    pos = key_offset + np.arange(Nk)
    if causal:
        keep = pos[None, :] <= np.arange(N)[:, None]
    if blockmask is not None:
        bm = np.asarray(blockmask).astype(bool)
        bk = bm[(np.arange(N) // tile)[:, None], (pos // tile)[None, :]]
        keep = bk if keep is None else (keep & bk)
    return keep


def softmax_rows(S: np.ndarray):
    """Row softmax of S (which may hold -inf).  Returns P, m, l, LSE."""
    m = S.max(axis=1)
    m_ref = np.where(np.isfinite(m), m, 0.0)
    E = np.exp(S - m_ref[:, None])
    l = E.sum(axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        P = np.where(l[:, None] > 0, E / np.where(l > 0, l, 1.0)[:, None], 0.0)
        lse = np.where(l > 0, m_ref + np.log(np.where(l > 0, l, 1.0)), -np.inf)
    return P, m, l, lse


def attention_fwd_head(q, k, v, scale: float, causal: bool = False, blockmask=None,
                       return_p: bool = False, tile: int = TILE, key_offset: int = 0):
    """One head: q is [N, d], k and v are [Nk, d] float64 (Nk = N for self-attention).
    Returns (O [N, d], LSE [N]) (and P).  ``tile`` is the block-mask tile side (128 for the
    product; small in oracle self-tests); ``key_offset`` places key row 0 in the query
    sequence (a slice of the keys: one split or one shard)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    N = q.shape[0]
    S = scale * (q @ k.T)
    keep = _keep_matrix(N, causal, blockmask, tile, k.shape[0], key_offset)
    if keep is not None:
        S = np.where(keep, S, -np.inf)
    P, _, _, lse = softmax_rows(S)
    O = P @ v
    if return_p:
        return O, lse, P
    return O, lse


def lse_merge(o_parts, lse_parts):
    """Combine attention results computed over disjoint key subsets of the same rows.

    o_parts [S, ..., d] are each normalised over their own keys with log-sum-exp
    lse_parts [S, ...].  Over the union of the keys the row sum of exp is the sum of the
    parts' sums, so LSE = ln sum_s exp(LSE_s) and O = sum_s exp(LSE_s - LSE) O_s -- the same
    rescaling that merges two blocks' running (m, l) statistics in the online softmax
    (FlashAttention-NeurIPS22 summary, "核心方法 / Tiling 与 online softmax").  Rows where
    every part saw no key stay O = 0, LSE = -inf."""
    o_parts = np.asarray(o_parts, np.float64)
    lse_parts = np.asarray(lse_parts, np.float64)
    m = lse_parts.max(axis=0)
    m_ref = np.where(np.isfinite(m), m, 0.0)
    w = np.exp(lse_parts - m_ref[None])               # 0 for parts that saw no key
    tot = w.sum(axis=0)
    with np.errstate(divide="ignore", invalid="ignore"):
        lse = np.where(tot > 0, m_ref + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
        frac = np.where(tot[None] > 0, w / np.where(tot > 0, tot, 1.0)[None], 0.0)
    O = (frac[..., None] * o_parts).sum(axis=0)
    return O, lse


def attention_bwd_head(q, k, v, dout, scale: float, causal: bool = False, blockmask=None,
                       tile: int = TILE):
    """One head: returns (dQ, dK, dV, O, LSE) for upstream gradient ``dout`` [N, d]."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    dout = np.asarray(dout, np.float64)
    O, lse, P = attention_fwd_head(q, k, v, scale, causal, blockmask, return_p=True, tile=tile)
    dV = P.T @ dout
    dP = dout @ v.T
    D = (P * dP).sum(axis=1)
    dS = P * (dP - D[:, None])
    dQ = scale * (dS @ k)
    dK = scale * (dS.T @ q)
    return dQ, dK, dV, O, lse


def attention_fwd_head_tiled(q, k, v, scale: float, causal: bool = False, blockmask=None,
                             block_rows: int = 128, block_cols: int = 128, tile: int = TILE):
    """Self-test only: the blockwise online-softmax recurrence, in fp64.

    For each block of query rows, walk the key/value blocks keeping a running row max m
    and exp-sum l; when m grows, rescale l and the output accumulator by exp(m_old - m_new).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    N, d = q.shape
    keep = _keep_matrix(N, causal, blockmask, tile)
    O = np.zeros((N, v.shape[1]))
    lse = np.full(N, -np.inf)
    for r0 in range(0, N, block_rows):
        r1 = min(N, r0 + block_rows)
        m = np.full(r1 - r0, -np.inf)
        l = np.zeros(r1 - r0)
        acc = np.zeros((r1 - r0, v.shape[1]))
        for c0 in range(0, N, block_cols):
            c1 = min(N, c0 + block_cols)
            s = scale * (q[r0:r1] @ k[c0:c1].T)
            if keep is not None:
                s = np.where(keep[r0:r1, c0:c1], s, -np.inf)
            m_new = np.maximum(m, s.max(axis=1))
            ref = np.where(np.isfinite(m_new), m_new, 0.0)
            alpha = np.exp(np.where(np.isfinite(m), m, -np.inf) - ref)
            p = np.exp(s - ref[:, None])
            l = alpha * l + p.sum(axis=1)
            acc = alpha[:, None] * acc + p @ v[c0:c1]
            m = m_new
        ok = l > 0
        O[r0:r1][ok] = acc[ok] / l[ok][:, None]
        lse[r0:r1][ok] = m[ok] + np.log(l[ok])
    return O, lse


# ---------------------------------------------------------------------------------------
# Batched wrappers over [B, H, N, d] arrays (a loop over heads; heads are independent).
# ---------------------------------------------------------------------------------------

def _as64(x):
    if hasattr(x, "detach"):  # torch tensor -> exact fp64 copy
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, np.float64)


def attention_fwd(q, k, v, scale: float, causal: bool = False, blockmask=None, heads=None):
    """q, k, v: [B, H, N, d].  ``heads``: optional list of (b, h) to evaluate (others are
    left as NaN).  Returns (O [B,H,N,d], LSE [B,H,N]) as float64."""
    q, k, v = _as64(q), _as64(k), _as64(v)
    B, H, N, _ = q.shape
    bm = None if blockmask is None else _as64(blockmask)
    O = np.full(q.shape[:3] + (v.shape[3],), np.nan)
    L = np.full((B, H, N), np.nan)
    for b, h in (heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]):
        O[b, h], L[b, h] = attention_fwd_head(q[b, h], k[b, h], v[b, h], scale, causal, bm)
    return O, L


def attention_bwd(q, k, v, dout, scale: float, causal: bool = False, blockmask=None, heads=None):
    """Returns (dQ, dK, dV, O, LSE) as float64 arrays; unevaluated heads are NaN."""
    q, k, v, dout = _as64(q), _as64(k), _as64(v), _as64(dout)
    B, H, N, d = q.shape
    bm = None if blockmask is None else _as64(blockmask)
    dQ = np.full(q.shape, np.nan)
    dK = np.full(k.shape, np.nan)
    dV = np.full(v.shape, np.nan)
    O = np.full(q.shape[:3] + (v.shape[3],), np.nan)
    L = np.full((B, H, N), np.nan)
    for b, h in (heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]):
        dQ[b, h], dK[b, h], dV[b, h], O[b, h], L[b, h] = attention_bwd_head(
            q[b, h], k[b, h], v[b, h], dout[b, h], scale, causal, bm)
    return dQ, dK, dV, O, L


def attention_fwd_partial(q, k, v, scale: float, causal: bool = False, blockmask=None,
                          key_offset: int = 0, heads=None):
    """q: [B, H, N, d]; k, v: [B, H, Nk, d], key row 0 at position ``key_offset``.
    Attention of every query row over these keys only: (O [B,H,N,d], LSE [B,H,N]) as
    float64; unevaluated heads are NaN."""
    q, k, v = _as64(q), _as64(k), _as64(v)
    B, H, N, _ = q.shape
    bm = None if blockmask is None else _as64(blockmask)
    O = np.full(q.shape[:3] + (v.shape[3],), np.nan)
    L = np.full((B, H, N), np.nan)
    for b, h in (heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]):
        O[b, h], L[b, h] = attention_fwd_head(q[b, h], k[b, h], v[b, h], scale, causal, bm,
                                              key_offset=key_offset)
    return O, L


def attention_fwd_rows(q, k, v, scale: float, causal: bool, rows):
    """One head, only the query rows ``rows`` (no block mask): (O [len(rows), d], LSE).
    A row's output depends only on its own query and the keys it sees, so evaluating a
    sample of rows is exact -- used to check full-size problems whose N x N matrices do not
    fit in memory."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    rows = np.asarray(rows)
    S = scale * (q[rows] @ k.T)
    if causal:
        S = np.where(np.arange(k.shape[0])[None, :] <= rows[:, None], S, -np.inf)
    P, _, _, lse = softmax_rows(S)
    return P @ v, lse
