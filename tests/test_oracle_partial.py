"""Pins of the key-range partial attention and of the merge of partial results
(oracle/partial.py), CPU only.

The merge is the online-softmax update of "FlashAttention (TR)", section
"Çevrimiçi Softmax Hesaplama", applied to whole key ranges; what fixes it is
that merging the partials of any split of the keys gives back the full
attention (the definition), which these tests check, together with a
pure-Python brute force of a partial and closed forms of the merge.
"""
import math

import numpy as np
import pytest

from oracle import attention_fp64, attention_partial_fp64, merge_partials_fp64
from synthetic import bf16_bits, make_qkv

CASES = [
    # B, Hq, Hkv, Nq, Nkv, d, causal
    (1, 2, 2, 37, 37, 16, True),
    (2, 4, 2, 20, 50, 8, True),     # Nq < Nkv: bottom-right (a cache before the rows)
    (1, 2, 1, 45, 30, 8, True),     # Nq > Nkv: rows that see no key
    (1, 2, 2, 33, 70, 16, False),
]


def _bits(case, seed):
    B, Hq, Hkv, Nq, Nkv, d, _ = case
    q, k, v = make_qkv(B, Hq, Hkv, Nq, Nkv, d, seed=seed)
    return bf16_bits(q), bf16_bits(k), bf16_bits(v)


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_full_range_is_the_definition(case):
    q, k, v = _bits(case, 11)
    causal, d = case[6], case[5]
    O, L = attention_partial_fp64(q, k, v, 0, case[4], causal, 1 / math.sqrt(d))
    Or, Lr = attention_fp64(q, k, v, causal, 1 / math.sqrt(d))
    assert np.array_equal(np.isinf(L), np.isinf(Lr))
    fin = np.isfinite(Lr)
    assert np.abs(L[fin] - Lr[fin]).max() < 1e-12
    assert np.abs(O - Or).max() < 1e-12


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
@pytest.mark.parametrize("n_parts", [2, 3, 5])
def test_merged_splits_equal_full_attention(case, n_parts):
    """Any split of the keys (empty ranges and ranges some rows cannot see
    included) merges back to the full result."""
    q, k, v = _bits(case, 12 + n_parts)
    Nkv, d, causal = case[4], case[5], case[6]
    rng = np.random.default_rng(n_parts * 100 + Nkv)
    cuts = np.sort(rng.integers(0, Nkv + 1, size=n_parts - 1))
    bounds = [0, *cuts.tolist(), Nkv]
    parts = [attention_partial_fp64(q, k, v, lo, hi, causal, 1 / math.sqrt(d))
             for lo, hi in zip(bounds[:-1], bounds[1:])]
    O, L = merge_partials_fp64(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    Or, Lr = attention_fp64(q, k, v, causal, 1 / math.sqrt(d))
    assert np.array_equal(np.isinf(L), np.isinf(Lr))
    fin = np.isfinite(Lr)
    assert np.abs(L[fin] - Lr[fin]).max() < 1e-12
    assert np.abs(O - Or).max() < 1e-12


def test_partial_brute_force_tiny():
    """Pure-Python loops over the keys of the range, global causal mask."""
    case = (1, 2, 1, 6, 9, 4, True)
    q, k, v = _bits(case, 21)
    from oracle import widen_bf16
    qf, kf, vf = widen_bf16(q), widen_bf16(k), widen_bf16(v)
    scale = 0.4
    for lo, hi in [(0, 9), (2, 6), (5, 9), (7, 8), (4, 4)]:
        O, L = attention_partial_fp64(q, k, v, lo, hi, True, scale)
        for h in range(2):
            for i in range(6):
                keys = [j for j in range(lo, hi) if j <= i + (9 - 6)]
                if not keys:
                    assert L[0, h, i] == -math.inf and not O[0, h, i].any()
                    continue
                s = [scale * math.fsum(qf[0, h, i, c] * kf[0, 0, j, c] for c in range(4))
                     for j in keys]
                mx = max(s)
                e = [math.exp(x - mx) for x in s]
                tot = math.fsum(e)
                assert abs(L[0, h, i] - (mx + math.log(tot))) < 1e-13
                for c in range(4):
                    oc = math.fsum(ei * vf[0, 0, j, c] for ei, j in zip(e, keys)) / tot
                    assert abs(O[0, h, i, c] - oc) < 1e-13


def test_merge_closed_forms():
    rng = np.random.default_rng(5)
    o = rng.standard_normal((3, 4, 8))
    lse = rng.standard_normal((3, 4))
    # one part: itself
    O1, L1 = merge_partials_fp64(o[:1], lse[:1])
    assert np.allclose(O1, o[0], rtol=0, atol=1e-15) and np.allclose(L1, lse[0], rtol=0, atol=1e-15)
    # two equal parts: same O, LSE + ln 2
    O2, L2 = merge_partials_fp64(np.stack([o[0], o[0]]), np.stack([lse[0], lse[0]]))
    assert np.abs(O2 - o[0]).max() < 1e-15 and np.abs(L2 - (lse[0] + math.log(2))).max() < 1e-15
    # a part that saw no key carries no weight
    lse_m = lse.copy()
    lse_m[1] = -np.inf
    Om, Lm = merge_partials_fp64(o, lse_m)
    Or, Lr = merge_partials_fp64(o[[0, 2]], lse[[0, 2]])
    assert np.abs(Om - Or).max() < 1e-15 and np.abs(Lm - Lr).max() < 1e-15
    # no part saw a key: O = 0, LSE = -inf
    Oz, Lz = merge_partials_fp64(o, np.full((3, 4), -np.inf))
    assert not Oz.any() and np.all(Lz == -np.inf)
    # weights: exp(LSE_s - LSE), summing to one
    Ow, Lw = merge_partials_fp64(o, lse)
    w = np.exp(lse - Lw)
    assert np.abs(w.sum(axis=0) - 1).max() < 1e-14
    assert np.abs(Ow - (w[..., None] * o).sum(axis=0)).max() < 1e-14


def test_merge_order_and_grouping():
    rng = np.random.default_rng(9)
    o = rng.standard_normal((4, 3, 5, 6))
    lse = 3 * rng.standard_normal((4, 3, 5))
    O, L = merge_partials_fp64(o, lse)
    perm = [2, 0, 3, 1]
    Op, Lp = merge_partials_fp64(o[perm], lse[perm])
    assert np.abs(O - Op).max() < 1e-14 and np.abs(L - Lp).max() < 1e-14
    Oa, La = merge_partials_fp64(o[:2], lse[:2])
    Ob, Lb = merge_partials_fp64(o[2:], lse[2:])
    Og, Lg = merge_partials_fp64(np.stack([Oa, Ob]), np.stack([La, Lb]))
    assert np.abs(O - Og).max() < 1e-14 and np.abs(L - Lg).max() < 1e-14
