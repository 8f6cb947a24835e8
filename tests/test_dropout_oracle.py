"""CPU-only: pins of the dropout oracle (oracle/dropout.py) to facts outside itself.

  * Philox4x32-10 reproduces the generator's published known-answer vectors
    (tests/golden/philox4x32_10_kat.json);
  * the keep mask follows the stated layout, checked element by element from single
    generator calls (byte k of call (j div 16, i, bh, 0) decides key 16*(j div 16) + k);
  * p = 0 keeps everything at scale 1: the dropout forward is then plain attention;
  * the kept fraction matches (256 - t)/256 within a binomial bound, for several p;
  * the dropout output is unbiased: its mean over many seeds approaches plain attention;
  * the dropout backward agrees with central finite differences of L = sum(dO o O) for a
    fixed mask, and D = sum_j P_ij dP_ij equals sum_c dO_ic O_ic;
  * planted mistakes in the mask layout, the rescaling and the backward each fail a pin.
"""

from __future__ import annotations

import json
import math
import os

import numpy as np
import pytest

import oracle
import oracle.dropout as od
import oracle.attention as ora

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def pin_philox_kat(philox):
    with open(os.path.join(GOLDEN, "philox4x32_10_kat.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        ctr = np.array([[int(x, 16) for x in c["ctr"]]], np.uint32)
        key = tuple(int(x, 16) for x in c["key"])
        got = philox(ctr, key)[0]
        assert [int(x) for x in got] == [int(x, 16) for x in c["out"]], c


def pin_mask_layout(mask_fn):
    seed, p = 0x1234_5678_9ABC_DEF0, 0.3
    t = od.drop_threshold(p)
    m = mask_fn(5, 40, 70, seed, p)
    for i, j in ((0, 0), (0, 15), (0, 16), (3, 33), (39, 69), (17, 47), (22, 5)):
        words = od.philox4x32_10(np.array([[j // 16, i, 5, 0]], np.uint32), (seed & 0xFFFFFFFF, seed >> 32))[0]
        k = j % 16
        byte = (int(words[k // 4]) >> (8 * (k % 4))) & 0xFF
        assert bool(m[i, j]) == (byte >= t), (i, j)


def pin_p_zero_is_plain(fwd_dropout):
    r = np.random.default_rng(31)
    q, k, v = r.standard_normal((3, 37, 8))
    keep = od.keep_mask(0, 37, 37, 99, 0.0)
    assert keep.all() and od.keep_scale(0.0) == 1.0
    for causal in (False, True):
        O, L, _, _ = fwd_dropout(q, k, v, 0.3, keep, 1.0, causal)
        O0, L0 = ora.attention_fwd_head(q, k, v, 0.3, causal)
        assert np.max(np.abs(O - O0)) < 1e-14 and np.max(np.abs(L - L0)) < 1e-14


def pin_keep_rate(mask_fn):
    for p in (0.1, 0.25, 0.5, 0.9):
        m = mask_fn(7, 512, 1024, 2024, p)
        q = (256 - od.drop_threshold(p)) / 256
        n = m.size
        assert abs(m.mean() - q) < 5 * math.sqrt(q * (1 - q) / n), p


def pin_unbiased(fwd_dropout, scale_fn=od.keep_scale):
    r = np.random.default_rng(32)
    N, d, p = 6, 3, 0.4
    q, k, v = r.standard_normal((3, N, d))
    O0, _ = ora.attention_fwd_head(q, k, v, 0.5)
    outs = np.stack([fwd_dropout(q, k, v, 0.5, od.keep_mask(0, N, N, s, p), scale_fn(p))[0] for s in range(3000)])
    se = outs.std(axis=0) / math.sqrt(len(outs))
    assert np.all(np.abs(outs.mean(axis=0) - O0) < 5 * se + 1e-12)


def pin_finite_differences(bwd_dropout, fwd_dropout):
    r = np.random.default_rng(33)
    N, d, h = 7, 4, 1e-6
    q, k, v, do = r.standard_normal((4, N, d))
    keep = od.keep_mask(2, N, N, 77, 0.3)
    ds = od.keep_scale(0.3)
    for causal in (False, True):
        dq, dk, dv, _, _ = bwd_dropout(q, k, v, do, 0.6, keep, ds, causal)
        for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
            num = np.zeros_like(x)
            for idx in np.ndindex(*x.shape):
                xp, xm = x.copy(), x.copy()
                xp[idx] += h
                xm[idx] -= h
                args = {"q": q, "k": k, "v": v}
                args[name] = xp
                lp = (fwd_dropout(args["q"], args["k"], args["v"], 0.6, keep, ds, causal)[0] * do).sum()
                args[name] = xm
                lm = (fwd_dropout(args["q"], args["k"], args["v"], 0.6, keep, ds, causal)[0] * do).sum()
                num[idx] = (lp - lm) / (2 * h)
            assert np.max(np.abs(num - g)) < 1e-6 * max(1.0, np.abs(g).max()), (name, causal)


def test_philox_known_answers():
    pin_philox_kat(od.philox4x32_10)


def test_mask_layout():
    pin_mask_layout(od.keep_mask)


def test_p_zero_is_plain_attention():
    pin_p_zero_is_plain(od.attention_fwd_head_dropout)


def test_keep_rate():
    pin_keep_rate(od.keep_mask)


def test_unbiased_over_seeds():
    pin_unbiased(od.attention_fwd_head_dropout)


def test_finite_differences():
    pin_finite_differences(od.attention_bwd_head_dropout, od.attention_fwd_head_dropout)


def test_d_identity_with_dropout():
    r = np.random.default_rng(34)
    q, k, v, do = r.standard_normal((4, 20, 5))
    keep = od.keep_mask(1, 20, 20, 5, 0.5)
    O, _, P, M = od.attention_fwd_head_dropout(q, k, v, 0.4, keep, od.keep_scale(0.5))
    dP = (do @ v.T) * M
    assert np.max(np.abs((P * dP).sum(1) - (do * O).sum(1))) < 1e-12


def test_threshold_rule():
    assert od.drop_threshold(0.0) == 0 and od.drop_threshold(0.1) == 26 and od.drop_threshold(0.5) == 128
    assert od.drop_threshold(0.999) == 255
    with pytest.raises(ValueError):
        od.drop_threshold(1.0)


def test_batched_wrappers_use_head_index():
    from exact_attention_111_b200.inputs import make_inputs
    x = make_inputs(2, 2, 40, 8, 3)
    O, L = od.attention_fwd_dropout(x["q"], x["k"], x["v"], 0.35, 0.2, 11)
    for b in range(2):
        for h in range(2):
            keep = od.keep_mask(b * 2 + h, 40, 40, 11, 0.2)
            o, l, _, _ = od.attention_fwd_head_dropout(x["q"][b, h].double().numpy(), x["k"][b, h].double().numpy(),
                                                       x["v"][b, h].double().numpy(), 0.35, keep, od.keep_scale(0.2))
            assert np.max(np.abs(O[b, h] - o)) < 1e-13


# ----------------------------------------------------------------------------------------
# planted mistakes
# ----------------------------------------------------------------------------------------

def _fails(fn):
    try:
        fn()
    except AssertionError:
        return True
    return False


def test_planted_mask_transposed_is_caught():
    bad = lambda bh, N, Nk, seed, p: od.keep_mask(bh, Nk, N, seed, p).T
    assert _fails(lambda: pin_mask_layout(bad))


def test_planted_byte_order_is_caught():
    def bad(bh, N, Nk, seed, p):
        m = od.keep_mask(bh, N, (Nk + 15) // 16 * 16, seed, p)
        return m.reshape(N, -1, 4, 4)[:, :, :, ::-1].reshape(N, -1)[:, :Nk]
    assert _fails(lambda: pin_mask_layout(bad))


def test_planted_missing_rescale_is_caught():
    assert _fails(lambda: pin_unbiased(od.attention_fwd_head_dropout, scale_fn=lambda p: 1.0))


@pytest.mark.parametrize("kind", ["dp_unmasked", "dv_undropped", "ds_dropped_p"])
def test_planted_backward_mistake_is_caught(kind):
    def bwd(q, k, v, dout, scale, keep, ds, causal=False, blockmask=None, tile=128):
        O, lse, P, M = od.attention_fwd_head_dropout(q, k, v, scale, keep, ds, causal, blockmask, tile)
        dV = (P.T @ dout) if kind == "dv_undropped" else ((P * M).T @ dout)
        dP = (dout @ np.asarray(v).T) if kind == "dp_unmasked" else ((dout @ np.asarray(v).T) * M)
        D = (P * dP).sum(axis=1)
        Pu = P * M if kind == "ds_dropped_p" else P
        dS = Pu * (dP - D[:, None])
        return scale * (dS @ k), scale * (dS.T @ q), dV, O, lse
    assert _fails(lambda: pin_finite_differences(bwd, od.attention_fwd_head_dropout))
