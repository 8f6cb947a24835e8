"""CPU-only: the fp64 oracle against the facts that pin it (see oracle_pins.py), the
butterfly tile mask against a brute-force count, and planted mistakes that the pins catch."""

from __future__ import annotations

import numpy as np
import pytest

import oracle.attention as ora
from exact_attention_111_b200.inputs import butterfly_blockmask, attention_flops
from tests import oracle_pins as pins

fwd, bwd, tiled = ora.attention_fwd_head, ora.attention_bwd_head, ora.attention_fwd_head_tiled


def test_rows_sum_to_one():
    pins.pin_rows_sum_to_one(fwd)


def test_fully_masked_row():
    pins.pin_fully_masked_row(fwd, bwd)


def test_single_key():
    pins.pin_single_key(fwd, bwd)


def test_shift_invariance():
    pins.pin_shift_invariance(fwd)


def test_constant_v():
    pins.pin_constant_v(fwd)


def test_zero_query_closed_form():
    pins.pin_zero_query_closed_form(fwd)


def test_causal_row0():
    pins.pin_causal_row0(fwd)


def test_tiled_recurrence_equals_direct():
    pins.pin_tiled_equals_direct(fwd, tiled)


def test_finite_differences():
    pins.pin_finite_differences(bwd, fwd)


def test_d_identity():
    pins.pin_d_identity(fwd)


def test_torch_sdpa_fp64():
    pins.pin_torch_sdpa(fwd, bwd)


def test_golden_closed_forms():
    pins.pin_golden_closed_forms(fwd, bwd)


def test_key_slice_brute_force():
    pins.pin_key_slice_brute_force(fwd)


def test_merge_partition_equals_direct():
    pins.pin_merge_partition(fwd, ora.lse_merge)


def test_merge_closed_forms():
    pins.pin_merge_closed_forms(ora.lse_merge)


def test_row_sample_matches_whole_head():
    r = np.random.default_rng(21)
    q, k, v = r.standard_normal((3, 50, 6))
    rows = np.array([0, 3, 17, 49])
    for causal in (False, True):
        O, L = fwd(q, k, v, 0.4, causal)
        Os, Ls = ora.attention_fwd_rows(q, k, v, 0.4, causal, rows)
        assert np.max(np.abs(Os - O[rows])) < 1e-13 and np.max(np.abs(Ls - L[rows])) < 1e-13


def test_batched_wrappers_match_heads():
    r = np.random.default_rng(12)
    q, k, v, do = r.standard_normal((4, 2, 3, 40, 8))
    O, L = ora.attention_fwd(q, k, v, 0.3, True)
    dq, dk, dv, O2, L2 = ora.attention_bwd(q, k, v, do, 0.3, True, heads=[(1, 2)])
    o12, l12 = fwd(q[1, 2], k[1, 2], v[1, 2], 0.3, True)
    assert np.array_equal(O[1, 2], o12) and np.array_equal(L[1, 2], l12)
    assert np.array_equal(O2[1, 2], o12)
    assert np.isnan(dq[0, 0]).all()  # unevaluated head


# --------------------------------------------------------------------------------------
# Butterfly tile mask: brute-force count on T = 32 tiles (244 kept, 6..32 per row).
# --------------------------------------------------------------------------------------

def _butterfly_brute(T):
    keep = np.zeros((T, T), np.uint8)
    for i in range(T):
        for j in range(T):
            x = i ^ j
            if i == j or bin(x).count("1") == 1 or i == 0 or j == 0:
                keep[i, j] = 1
    return keep


def test_butterfly_mask_brute_force():
    for T in (1, 2, 7, 32, 33):
        assert np.array_equal(butterfly_blockmask(T).numpy(), _butterfly_brute(T))
    m = butterfly_blockmask(32).numpy()
    assert int(m.sum()) == 244
    per_row = m.sum(axis=1)
    assert per_row.min() == 6 and per_row.max() == 32
    assert np.array_equal(m, m.T)


def test_flop_formula():
    # 4*B*H*N^2*d forward; the 64x16x1024x64 shape gives 274.9 GFLOP forward.
    assert abs(attention_flops(64, 16, 1024, 64, False, False) - 274.877906944e9) < 1
    assert attention_flops(1, 1, 128, 64, False, True) == 3.5 * 4 * 128 * 128 * 64
    assert attention_flops(1, 1, 128, 64, True, True) == 0.5 * 3.5 * 4 * 128 * 128 * 64


# --------------------------------------------------------------------------------------
# Planted mistakes: each broken copy of the oracle must fail at least one pin.
# --------------------------------------------------------------------------------------

def _mut_fwd(kind):
    def f(q, k, v, scale, causal=False, blockmask=None, return_p=False, tile=128):
        q = np.asarray(q, np.float64)
        k = np.asarray(k, np.float64)
        v = np.asarray(v, np.float64)
        N = q.shape[0]
        s = 1.0 if kind == "drop_scale" else scale
        S = s * (q @ k.T)
        keep = ora._keep_matrix(N, causal, blockmask, tile)
        if kind == "causal_transposed" and keep is not None and causal:
            keep = keep.T.copy()
        if keep is not None:
            S = np.where(keep, S, -np.inf)
        P, m, l, lse = ora.softmax_rows(S)
        if kind == "lse_no_max":
            lse = np.log(np.where(l > 0, l, 1.0))
        if kind == "p_unnormalised":
            P = P * l[:, None]
        O = (P.T @ v) if kind == "p_transposed" else (P @ v)
        if return_p:
            return O, lse, P
        return O, lse
    return f


def _mut_bwd(kind):
    def b(q, k, v, dout, scale, causal=False, blockmask=None, tile=128):
        O, lse, P = fwd(q, k, v, scale, causal, blockmask, return_p=True, tile=tile)
        dout = np.asarray(dout, np.float64)
        dV = (P @ dout) if kind == "dv_untransposed" else (P.T @ dout)
        dP = dout @ np.asarray(v).T
        D = (P * dP).sum(axis=1)
        dS = P * (dP + D[:, None]) if kind == "d_sign" else P * (dP - D[:, None])
        dQ = scale * (dS @ k)
        dK = (scale * (dS @ q)) if kind == "dk_untransposed" else (scale * (dS.T @ q))
        if kind == "dq_no_scale":
            dQ = dS @ k
        return dQ, dK, dV, O, lse
    return b


def _fails(fn):
    try:
        fn()
    except AssertionError:
        return True
    return False


@pytest.mark.parametrize("kind", ["drop_scale", "causal_transposed", "lse_no_max",
                                  "p_unnormalised", "p_transposed"])
def test_planted_forward_mistake_is_caught(kind):
    f = _mut_fwd(kind)
    checks = [lambda: pins.pin_rows_sum_to_one(f), lambda: pins.pin_shift_invariance(f),
              lambda: pins.pin_constant_v(f), lambda: pins.pin_zero_query_closed_form(f),
              lambda: pins.pin_causal_row0(f), lambda: pins.pin_golden_closed_forms(f, bwd),
              lambda: pins.pin_torch_sdpa(f, bwd), lambda: pins.pin_single_key(f, bwd)]
    assert any(_fails(c) for c in checks), f"no pin caught the planted mistake {kind}"


@pytest.mark.parametrize("kind", ["dv_untransposed", "d_sign", "dk_untransposed", "dq_no_scale"])
def test_planted_backward_mistake_is_caught(kind):
    b = _mut_bwd(kind)
    checks = [lambda: pins.pin_finite_differences(b, fwd), lambda: pins.pin_golden_closed_forms(fwd, b),
              lambda: pins.pin_torch_sdpa(fwd, b), lambda: pins.pin_single_key(fwd, b)]
    assert any(_fails(c) for c in checks), f"no pin caught the planted mistake {kind}"


def _mut_slice_fwd(kind):
    """Forward over a key slice with the offset mishandled."""
    def f(q, k, v, scale, causal=False, blockmask=None, return_p=False, tile=128, key_offset=0):
        off = {"offset_ignored": 0, "offset_negated": -key_offset}.get(kind, key_offset)
        return fwd(q, k, v, scale, causal, blockmask, return_p=return_p, tile=tile, key_offset=off)
    return f


def _mut_merge(kind):
    def m(o_parts, lse_parts):
        o_parts = np.asarray(o_parts, np.float64)
        lse_parts = np.asarray(lse_parts, np.float64)
        if kind == "no_max_shift":
            w = np.exp(lse_parts)
        else:
            mx = lse_parts.max(axis=0)
            ref = np.where(np.isfinite(mx), mx, 0.0)
            w = np.exp(ref[None] - lse_parts) if kind == "weight_sign" else np.exp(lse_parts - ref[None])
        tot = w.sum(axis=0)
        with np.errstate(divide="ignore", invalid="ignore"):
            lse = np.log(tot) if kind == "no_max_shift" else np.where(tot > 0, np.log(tot) + ref, -np.inf)
            frac = w if kind == "unnormalised" else w / tot[None]
        if kind == "lse_mean":
            lse = lse_parts.mean(axis=0)
        O = (np.nan_to_num(frac)[..., None] * o_parts).sum(axis=0)
        return O, lse
    return m


@pytest.mark.parametrize("kind", ["offset_ignored", "offset_negated"])
def test_planted_key_offset_mistake_is_caught(kind):
    f = _mut_slice_fwd(kind)
    checks = [lambda: pins.pin_key_slice_brute_force(f), lambda: pins.pin_merge_partition(f, ora.lse_merge)]
    assert any(_fails(c) for c in checks), f"no pin caught the planted mistake {kind}"


@pytest.mark.parametrize("kind", ["no_max_shift", "weight_sign", "unnormalised", "lse_mean"])
def test_planted_merge_mistake_is_caught(kind):
    m = _mut_merge(kind)
    checks = [lambda: pins.pin_merge_partition(fwd, m), lambda: pins.pin_merge_closed_forms(m)]
    assert any(_fails(c) for c in checks), f"no pin caught the planted mistake {kind}"
