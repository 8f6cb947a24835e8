"""Checks that pin the fp64 oracle to facts fixed by the mathematics, not by itself.

Each ``pin_*`` takes the oracle's per-head functions (so a test can hand in a deliberately
broken copy) and raises AssertionError when a fact fails.  The facts:

  * rows of P sum to 1 (FlashAttention-NeurIPS22, "问题与动机": P = softmax(S));
  * one key: O = V and LSE = S_00; its gradients are dV = dO, dQ = dK = 0;
  * softmax is invariant to a per-row shift of S, which moves LSE by the same amount;
  * a constant V gives a constant O;
  * Q = 0: P is uniform over the visible keys, LSE = ln(#visible), O = their mean
    (with causal masking, row i averages V_0..V_i);
  * causal row 0 sees only key 0: O_0 = V_0;
  * the blockwise online-softmax recurrence ("核心方法 / Tiling 与 online softmax")
    reaches the direct formula for several block shapes and ragged tails;
  * analytic gradients agree with central finite differences of L = sum(dO o O);
  * D_i = sum_j P_ij dP_ij equals sum_c dO_ic O_ic;
  * fp64 torch scaled_dot_product_attention (+ autograd) agrees on small shapes;
  * a hand-derived two-key example (tests/golden/closed_forms.json);
  * a slice of the keys placed at a key offset (one split or one shard) matches a
    brute-force double loop over explicit query and key positions;
  * merging the results of disjoint key slices reaches the direct formula over all keys,
    and the merge has closed forms: one part is the identity, two equal parts add ln 2 to
    LSE, a part that saw no key contributes nothing, and LSEs ln 1 and ln 3 weigh the parts
    1/4 and 3/4 (also at LSE near 1000, where exp itself overflows).
"""

from __future__ import annotations

import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def pin_rows_sum_to_one(fwd):
    r = _rng(1)
    N, d = 37, 8
    q, k, v = r.standard_normal((3, N, d))
    for causal in (False, True):
        bm = np.array([[1, 0, 1], [0, 1, 0], [1, 1, 0]], np.uint8)
        for mask in (None, bm):
            _, _, P = fwd(q, k, v, 0.3, causal, mask, return_p=True, tile=16)
            s = P.sum(axis=1)
            assert np.all(np.abs(s - 1.0) < 1e-12), f"row sums {s.min()}..{s.max()}"
            assert np.all(P >= 0)


def pin_fully_masked_row(fwd, bwd):
    r = _rng(2)
    N, d = 20, 4
    q, k, v, do = r.standard_normal((4, N, d))
    # tile row 1 (rows 8..15) keeps only tile column 2, which causal masking then removes
    bm = np.array([[1, 0, 0], [0, 0, 1], [1, 1, 1]], np.uint8)
    O, lse = fwd(q, k, v, 0.5, True, bm, tile=8)
    assert np.all(O[8:16] == 0.0) and np.all(np.isneginf(lse[8:16]))
    assert np.all(np.isfinite(O[:8])) and np.all(np.isfinite(lse[16:]))
    dq, dk, dv, _, _ = bwd(q, k, v, do, 0.5, True, bm, tile=8)
    assert np.all(dq[8:16] == 0.0)
    assert np.all(np.isfinite(dq)) and np.all(np.isfinite(dk)) and np.all(np.isfinite(dv))


def pin_single_key(fwd, bwd):
    r = _rng(3)
    d = 5
    q, k, v, do = r.standard_normal((4, 1, d))
    scale = 0.7
    O, lse = fwd(q, k, v, scale, False, None)
    assert np.allclose(O, v, rtol=0, atol=1e-15)
    assert abs(lse[0] - scale * float(q[0] @ k[0])) < 1e-14
    dq, dk, dv, _, _ = bwd(q, k, v, do, scale, False, None)
    assert np.allclose(dv, do, rtol=0, atol=1e-15)
    assert np.max(np.abs(dq)) < 1e-15 and np.max(np.abs(dk)) < 1e-15


def pin_shift_invariance(fwd):
    """Append a column c_i/scale to Q and a column of ones to K: S_ij += c_i exactly."""
    r = _rng(4)
    N, d = 29, 6
    q, k, v = r.standard_normal((3, N, d))
    scale = 0.25
    c = 3.0 * r.standard_normal(N)
    qa = np.concatenate([q, (c / scale)[:, None]], axis=1)
    ka = np.concatenate([k, np.ones((N, 1))], axis=1)
    for causal in (False, True):
        O0, l0 = fwd(q, k, v, scale, causal, None)
        O1, l1 = fwd(qa, ka, v, scale, causal, None)
        assert np.max(np.abs(O1 - O0)) < 1e-12
        assert np.max(np.abs(l1 - (l0 + c))) < 1e-12


def pin_constant_v(fwd):
    r = _rng(5)
    N, d = 23, 4
    q, k = r.standard_normal((2, N, d))
    row = r.standard_normal(d)
    v = np.tile(row, (N, 1))
    for causal in (False, True):
        O, _ = fwd(q, k, v, 0.9, causal, None)
        assert np.max(np.abs(O - row[None, :])) < 1e-13


def pin_zero_query_closed_form(fwd):
    r = _rng(6)
    N, d = 19, 3
    k, v = r.standard_normal((2, N, d))
    q = np.zeros((N, d))
    O, lse = fwd(q, k, v, 1.3, False, None)
    assert np.max(np.abs(lse - math.log(N))) < 1e-14
    assert np.max(np.abs(O - v.mean(axis=0)[None, :])) < 1e-14
    O, lse = fwd(q, k, v, 1.3, True, None)
    for i in range(N):
        assert abs(lse[i] - math.log(i + 1)) < 1e-14
        assert np.max(np.abs(O[i] - v[: i + 1].mean(axis=0))) < 1e-14


def pin_causal_row0(fwd):
    r = _rng(7)
    N, d = 17, 4
    q, k, v = r.standard_normal((3, N, d))
    O, lse = fwd(q, k, v, 0.5, True, None)
    assert np.max(np.abs(O[0] - v[0])) < 1e-15
    assert abs(lse[0] - 0.5 * float(q[0] @ k[0])) < 1e-14


def pin_tiled_equals_direct(fwd, tiled):
    r = _rng(8)
    for N, br, bc in ((64, 16, 16), (200, 16, 128), (300, 128, 128), (257, 64, 32)):
        d = 8
        q, k, v = r.standard_normal((3, N, d))
        q *= 2.0  # peaked rows exercise the rescaling branch
        T = (N + 31) // 32
        bm = (r.random((T, T)) < 0.5).astype(np.uint8)
        np.fill_diagonal(bm, 1)
        for causal in (False, True):
            for mask in (None, bm):
                O0, l0 = fwd(q, k, v, 0.4, causal, mask, tile=32)
                O1, l1 = tiled(q, k, v, 0.4, causal, mask, block_rows=br, block_cols=bc, tile=32)
                fin = np.isfinite(l0)
                assert np.array_equal(fin, np.isfinite(l1))
                assert np.max(np.abs(O0 - O1)) < 1e-12
                assert np.max(np.abs(l0[fin] - l1[fin])) < 1e-12


def pin_finite_differences(bwd, fwd):
    r = _rng(9)
    h = 1e-6
    bm = np.array([[1, 0], [1, 1]], np.uint8)
    for N, d, causal, mask in ((5, 3, False, None), (7, 4, True, None), (8, 2, False, bm),
                               (6, 3, True, bm)):
        q, k, v, do = r.standard_normal((4, N, d))
        scale = 0.8
        dq, dk, dv, _, _ = bwd(q, k, v, do, scale, causal, mask, tile=4)

        def loss(qq, kk, vv):
            O, _ = fwd(qq, kk, vv, scale, causal, mask, tile=4)
            return float((do * O).sum())

        for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
            num = np.zeros_like(x)
            for idx in np.ndindex(*x.shape):
                plus = {"q": q, "k": k, "v": v}
                minus = {"q": q, "k": k, "v": v}
                plus[name] = x.copy()
                minus[name] = x.copy()
                plus[name][idx] += h
                minus[name][idx] -= h
                num[idx] = (loss(plus["q"], plus["k"], plus["v"]) -
                            loss(minus["q"], minus["k"], minus["v"])) / (2 * h)
            err = np.max(np.abs(num - g)) / max(1e-12, np.max(np.abs(g)))
            assert err < 1e-6, f"d{name}: finite-difference relative error {err:.3g}"


def pin_d_identity(fwd):
    r = _rng(10)
    N, d = 31, 5
    q, k, v, do = r.standard_normal((4, N, d))
    for causal in (False, True):
        O, _, P = fwd(q, k, v, 0.6, causal, None, return_p=True)
        dP = do @ v.T
        assert np.max(np.abs((P * dP).sum(axis=1) - (do * O).sum(axis=1))) < 1e-12


def pin_torch_sdpa(fwd, bwd):
    import torch
    import torch.nn.functional as F

    r = _rng(11)
    for N, d, causal, use_mask in ((16, 8, False, False), (33, 16, True, False),
                                   (40, 8, False, True), (48, 4, True, True)):
        q, k, v, do = r.standard_normal((4, N, d))
        scale = 1.0 / math.sqrt(d)
        T = (N + 7) // 8
        bm = (r.random((T, T)) < 0.6).astype(np.uint8)
        np.fill_diagonal(bm, 1)
        mask = bm if use_mask else None
        tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
        attn_mask = None
        if use_mask:
            t = torch.arange(N) // 8
            keep = torch.tensor(bm, dtype=torch.bool)[t[:, None], t[None, :]]
            if causal:
                keep &= torch.ones(N, N, dtype=torch.bool).tril()
            attn_mask = keep
        to = F.scaled_dot_product_attention(tq[None], tk[None], tv[None], attn_mask=attn_mask,
                                            is_causal=causal and not use_mask, scale=scale)[0]
        to.backward(torch.tensor(do))
        O, _ = fwd(q, k, v, scale, causal, mask, tile=8)
        dq, dk, dv, _, _ = bwd(q, k, v, do, scale, causal, mask, tile=8)
        assert np.max(np.abs(O - to.detach().numpy())) < 1e-10
        for a, b in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
            assert np.max(np.abs(a - b.numpy())) < 1e-10


def pin_golden_closed_forms(fwd, bwd):
    with open(os.path.join(GOLDEN, "closed_forms.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        q, k, v = (np.array(c[x], np.float64) for x in ("q", "k", "v"))
        O, lse = fwd(q, k, v, c["scale"], c["causal"], None)
        assert np.max(np.abs(O - np.array(c["O"]))) < 1e-12, c["name"]
        assert np.max(np.abs(lse - np.array([eval_ln(x) for x in c["LSE"]]))) < 1e-12, c["name"]
        if "dout" in c:
            do = np.array(c["dout"], np.float64)
            dq, dk, dv, _, _ = bwd(q, k, v, do, c["scale"], c["causal"], None)
            for key, got in (("dQ", dq), ("dK", dk), ("dV", dv)):
                assert np.max(np.abs(got - np.array(c[key]))) < 1e-12, (c["name"], key)


def eval_ln(x):
    """Golden LSE values are written as numbers or as 'ln(a)' strings."""
    if isinstance(x, str) and x.startswith("ln(") and x.endswith(")"):
        return math.log(float(x[3:-1]))
    return float(x)


ALL_FWD_PINS = (pin_rows_sum_to_one, pin_shift_invariance, pin_constant_v,
                pin_zero_query_closed_form, pin_causal_row0, pin_d_identity)


def _brute_slice(q, k, v, scale, causal, bm, tile, key_offset):
    """Pure-Python double loop: row i sees key row j iff position key_offset + j passes."""
    N, Nk = len(q), len(k)
    O = [[0.0] * len(v[0]) for _ in range(N)]
    L = [-math.inf] * N
    for i in range(N):
        sc = []
        for j in range(Nk):
            pos = key_offset + j
            if causal and pos > i:
                continue
            if bm is not None and not bm[i // tile][pos // tile]:
                continue
            sc.append((j, scale * sum(float(a) * float(b) for a, b in zip(q[i], k[j]))))
        if not sc:
            continue
        m = max(x for _, x in sc)
        tot = sum(math.exp(x - m) for _, x in sc)
        L[i] = m + math.log(tot)
        for j, x in sc:
            w = math.exp(x - m) / tot
            for c in range(len(v[0])):
                O[i][c] += w * float(v[j][c])
    return np.array(O), np.array(L)


def pin_key_slice_brute_force(fwd):
    r = _rng(11)
    N, d, tile = 13, 3, 4
    q = r.standard_normal((N, d))
    bm = np.array([[1, 1, 0, 1], [0, 1, 1, 1], [1, 0, 1, 0], [1, 1, 1, 1]], np.uint8)
    for key_offset, Nk in ((0, 13), (4, 5), (8, 5), (12, 1), (4, 9)):
        k, v = r.standard_normal((2, Nk, d))
        for causal in (False, True):
            for mask in (None, bm):
                O, lse = fwd(q, k, v, 0.7, causal, mask, tile=tile, key_offset=key_offset)
                Ob, Lb = _brute_slice(q, k, v, 0.7, causal, mask, tile, key_offset)
                fin = np.isfinite(Lb)
                assert np.array_equal(np.isfinite(lse), fin), (key_offset, causal)
                assert np.max(np.abs(lse[fin] - Lb[fin]), initial=0.0) < 1e-12, (key_offset, causal)
                assert np.max(np.abs(O - Ob)) < 1e-12, (key_offset, causal)


def pin_merge_partition(fwd, merge):
    """Partials over a partition of the keys, merged, equal attention over all keys."""
    r = _rng(12)
    N, d, tile = 23, 5, 4
    q, k, v = r.standard_normal((3, N, d))
    bm = (r.random((6, 6)) < 0.6).astype(np.uint8)
    bm[3, :] = 0                                   # tile row 3: no visible key at all
    for cuts in ((0, 23), (0, 8, 23), (0, 4, 12, 16, 23), (0, 20, 23)):
        for causal in (False, True):
            for mask in (None, bm):
                Of, Lf = fwd(q, k, v, 0.4, causal, mask, tile=tile)
                parts = [fwd(q, k[a:b], v[a:b], 0.4, causal, mask, tile=tile, key_offset=a)
                         for a, b in zip(cuts[:-1], cuts[1:])]
                O, L = merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
                fin = np.isfinite(Lf)
                assert np.array_equal(np.isfinite(L), fin), (cuts, causal)
                assert np.max(np.abs(L[fin] - Lf[fin]), initial=0.0) < 1e-12, (cuts, causal)
                assert np.max(np.abs(O - Of)) < 1e-12, (cuts, causal)


def pin_merge_closed_forms(merge):
    r = _rng(13)
    o1, o2 = r.standard_normal((2, 6, 4))
    l1 = r.standard_normal(6)
    # one part: identity
    O, L = merge(o1[None], l1[None])
    assert np.max(np.abs(O - o1)) < 1e-15 and np.max(np.abs(L - l1)) < 1e-15
    # two equal parts: same O, LSE + ln 2
    O, L = merge(np.stack([o1, o1]), np.stack([l1, l1]))
    assert np.max(np.abs(O - o1)) < 1e-14 and np.max(np.abs(L - (l1 + math.log(2.0)))) < 1e-14
    # a part that saw no key (LSE = -inf) contributes nothing, whatever its O holds
    ninf = np.full(6, -np.inf)
    O, L = merge(np.stack([o1, o2]), np.stack([l1, ninf]))
    assert np.max(np.abs(O - o1)) < 1e-15 and np.max(np.abs(L - l1)) < 1e-15
    # no part saw a key: O = 0, LSE = -inf
    O, L = merge(np.stack([o1, o2]), np.stack([ninf, ninf]))
    assert np.all(O == 0.0) and np.all(np.isneginf(L))
    # LSE ln 1 and ln 3 (then both shifted to ~1000): weights 1/4 and 3/4, LSE ln 4 (+shift)
    for shift in (0.0, 1000.0):
        la, lb = np.full(6, shift), np.full(6, shift + math.log(3.0))
        O, L = merge(np.stack([o1, o2]), np.stack([la, lb]))
        # (at 1000 the inputs carry ulp(1000) ~ 1e-13 of representation error)
        assert np.max(np.abs(O - (0.25 * o1 + 0.75 * o2))) < 1e-12, shift
        assert np.max(np.abs(L - (shift + math.log(4.0)))) < 1e-12, shift
