"""Pins for the fp64 CPU oracle (CPU only).

Each pin ties the oracle to something other than itself:
  * brute force: a pure-Python loop with math.fsum on tiny inputs;
  * a library special case: torch SDPA in float64;
  * invariants the pages state: exactness of tiling + online softmax
    ("FlashAttention (TR)", "Çevrimiçi Softmax Hesaplama"), shift invariance
    under K mean smoothing ("Makale Bülteni — SageAttention", "İddia ve
    Gerçeklik"), rows of P summing to one, permutation equivariance, GQA as MHA
    on repeated K/V;
  * closed forms (Q = 0, V = 1, causal row 0, a dominant key);
  * planted mistakes: a wrong oracle must fail at least one pin.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as oatt
from synthetic import bf16_bits, make_qkv, WORKLOADS, make_workload

RNG_CASES = [
    # B, Hq, Hkv, Nq, Nkv, d, causal
    (1, 2, 2, 7, 7, 4, False),
    (1, 2, 2, 16, 16, 8, True),
    (1, 2, 1, 5, 11, 8, False),
    (2, 4, 2, 9, 9, 6, True),
    (1, 2, 2, 1, 1, 4, True),
    (1, 1, 1, 3, 13, 8, False),
]


def _bits(B, Hq, Hkv, Nq, Nkv, d, seed=5, dist="normal"):
    q, k, v = make_qkv(B, Hq, Hkv, Nq, Nkv, d, seed, dist)
    return bf16_bits(q), bf16_bits(k), bf16_bits(v)


def brute_force(qb, kb, vb, causal, scale):
    """Pure-Python loops, math.fsum, no numpy arithmetic."""
    B, Hq, Nq, d = qb.shape
    Hkv, Nkv = kb.shape[1], kb.shape[2]
    q = oracle.widen_bf16(qb).tolist()
    k = oracle.widen_bf16(kb).tolist()
    v = oracle.widen_bf16(vb).tolist()
    O = [[[[0.0] * d for _ in range(Nq)] for _ in range(Hq)] for _ in range(B)]
    L = [[[0.0] * Nq for _ in range(Hq)] for _ in range(B)]
    g = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            hk = h // g
            for i in range(Nq):
                vis = [j for j in range(Nkv) if (not causal or j <= i)]
                s = [scale * math.fsum(q[b][h][i][c] * k[b][hk][j][c] for c in range(d)) for j in vis]
                m = max(s)
                e = [math.exp(x - m) for x in s]
                l = math.fsum(e)
                for c in range(d):
                    O[b][h][i][c] = math.fsum(e[t] * v[b][hk][j][c] for t, j in enumerate(vis)) / l
                L[b][h][i] = m + math.log(l)
    return np.array(O), np.array(L)


@pytest.mark.parametrize("case", RNG_CASES)
def test_brute_force(case):
    B, Hq, Hkv, Nq, Nkv, d, causal = case
    qb, kb, vb = _bits(*case[:6], seed=11 + Nq)
    scale = 1.0 / math.sqrt(d)
    O, L = oracle.attention_fp64(qb, kb, vb, causal, scale)
    Ob, Lb = brute_force(qb, kb, vb, causal, scale)
    assert np.max(np.abs(O - Ob)) < 1e-13
    assert np.max(np.abs(L - Lb)) < 1e-13


def _sdpa64(qb, kb, vb, causal, scale):
    q = torch.from_numpy(oracle.widen_bf16(qb))
    k = torch.from_numpy(oracle.widen_bf16(kb))
    v = torch.from_numpy(oracle.widen_bf16(vb))
    g = q.shape[1] // k.shape[1]
    k = k.repeat_interleave(g, dim=1)
    v = v.repeat_interleave(g, dim=1)
    return torch.nn.functional.scaled_dot_product_attention(
        q, k, v, is_causal=causal, scale=scale).numpy()


@pytest.mark.parametrize("shape", [
    (1, 2, 2, 256, 256, 64, False),
    (1, 4, 4, 300, 300, 128, True),
    (2, 8, 2, 129, 129, 64, True),
    (1, 4, 1, 200, 77, 128, False),
])
def test_sdpa_float64(shape):
    qb, kb, vb = _bits(*shape[:6], seed=3)
    scale = 1.0 / math.sqrt(shape[5])
    O, _ = oracle.attention_fp64(qb, kb, vb, shape[6], scale)
    ref = _sdpa64(qb, kb, vb, shape[6], scale)
    assert np.max(np.abs(O - ref)) < 1e-12


def test_tiny_workload_matches_sdpa():
    w = WORKLOADS["tiny_256_d64"]
    q, k, v = make_workload(w)
    qb, kb, vb = bf16_bits(q), bf16_bits(k), bf16_bits(v)
    O, _ = oracle.attention_fp64(qb, kb, vb, w.causal, w.scale)
    assert np.max(np.abs(O - _sdpa64(qb, kb, vb, w.causal, w.scale))) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_p_rows_sum_to_one_and_lse_consistency(causal):
    qb, kb, vb = _bits(1, 2, 2, 64, 64, 16, seed=9)
    scale = 0.25
    O, L, P = oracle.attention_fp64(qb, kb, vb, causal, scale, return_p=True)
    assert np.max(np.abs(P.sum(-1) - 1.0)) < 1e-12
    q = oracle.widen_bf16(qb)
    k = oracle.widen_bf16(kb)
    for h in range(2):
        S = oatt.score_matrix_fp64(q[0, h], k[0, h], scale, causal)
        # exp(S - LSE) reproduces P
        assert np.max(np.abs(np.exp(S - L[0, h][:, None]) - P[0, h])) < 1e-12
        # LSE is the log of the sum of exponentials (fsum, per row)
        for i in range(0, 64, 7):
            ref = math.log(math.fsum(math.exp(x) for x in S[i] if x != -np.inf))
            assert abs(L[0, h, i] - ref) < 1e-12
    if causal:
        assert np.all(P[0, :, np.triu_indices(64, 1)[0], np.triu_indices(64, 1)[1]] == 0.0)


def online_softmax_blocks(S, V, block):
    """Blockwise running max / running sum recurrence (test-only restatement of
    the online softmax description): returns (O, LSE) for one head."""
    N = S.shape[1]
    m = np.full(S.shape[0], -np.inf)
    l = np.zeros(S.shape[0])
    acc = np.zeros((S.shape[0], V.shape[1]))
    for j0 in range(0, N, block):
        Sb = S[:, j0:j0 + block]
        m_new = np.maximum(m, Sb.max(axis=1))
        m_safe = np.where(np.isinf(m_new), 0.0, m_new)
        alpha = np.exp(m - m_safe)
        Pb = np.exp(Sb - m_safe[:, None])
        l = alpha * l + Pb.sum(axis=1)
        acc = alpha[:, None] * acc + Pb @ V[j0:j0 + block]
        m = m_new
    return acc / l[:, None], m + np.log(l)


@pytest.mark.parametrize("causal", [False, True])
def test_online_softmax_equals_one_shot(causal):
    qb, kb, vb = _bits(1, 2, 2, 300, 300, 32, seed=21)
    scale = 1 / math.sqrt(32)
    O, L = oracle.attention_fp64(qb, kb, vb, causal, scale)
    q, k, v = (oracle.widen_bf16(x) for x in (qb, kb, vb))
    for h in range(2):
        S = oatt.score_matrix_fp64(q[0, h], k[0, h], scale, causal)
        for block in (128, 64, 7):
            Ob, Lb = online_softmax_blocks(S, v[0, h], block)
            assert np.max(np.abs(Ob - O[0, h])) < 1e-12
            assert np.max(np.abs(Lb - L[0, h])) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_shift_invariance_k_mean_smoothing(causal):
    qb, kb, vb = _bits(1, 4, 2, 96, 96, 16, seed=31, dist="outlier_k")
    scale = 0.25
    O, L = oracle.attention_fp64(qb, kb, vb, causal, scale)
    q, k, v = (oracle.widen_bf16(x) for x in (qb, kb, vb))
    kbar = k.mean(axis=2, keepdims=True)
    O2, L2 = oracle.attention_f64(q, k - kbar, v, causal, scale)
    assert np.max(np.abs(O2 - O)) < 1e-12
    qk = np.einsum("bhnd,bhd->bhn", q, np.repeat(kbar[:, :, 0, :], 2, axis=1))
    assert np.max(np.abs(L2 - (L - scale * qk))) < 1e-10


def test_permutation_equivariance():
    qb, kb, vb = _bits(1, 2, 2, 40, 57, 8, seed=41)
    perm = np.random.default_rng(0).permutation(57)
    O, L = oracle.attention_fp64(qb, kb, vb, False, 0.3)
    O2, L2 = oracle.attention_fp64(qb, kb[:, :, perm], vb[:, :, perm], False, 0.3)
    assert np.max(np.abs(O - O2)) < 1e-12 and np.max(np.abs(L - L2)) < 1e-12


def test_gqa_is_mha_on_repeated_kv():
    qb, kb, vb = _bits(2, 8, 2, 33, 33, 8, seed=51)
    for causal in (False, True):
        O, L = oracle.attention_fp64(qb, kb, vb, causal, 0.35)
        O2, L2 = oracle.attention_fp64(qb, np.repeat(kb, 4, axis=1), np.repeat(vb, 4, axis=1), causal, 0.35)
        assert np.array_equal(O, O2) and np.array_equal(L, L2)


def test_closed_forms():
    qb, kb, vb = _bits(1, 2, 2, 20, 20, 8, seed=61)
    v = oracle.widen_bf16(vb)
    zeros = np.zeros_like(qb)
    # Q = 0: uniform weights over the visible keys
    for causal in (False, True):
        O, L = oracle.attention_fp64(zeros, kb, vb, causal, 0.5)
        for i in range(20):
            nvis = i + 1 if causal else 20
            assert np.allclose(O[0, :, i], v[0, :, :nvis].mean(axis=1), atol=1e-14, rtol=0)
            assert abs(L[0, 0, i] - math.log(nvis)) < 1e-14
    # V = 1: output is exactly one
    ones = np.full_like(vb, 0x3F80)   # bf16 1.0
    O, _ = oracle.attention_fp64(qb, kb, ones, True, 0.5)
    assert np.max(np.abs(O - 1.0)) < 1e-14
    # causal row 0 sees only key 0: O_0 = V_0, LSE_0 = scale * q_0 . k_0
    O, L = oracle.attention_fp64(qb, kb, vb, True, 0.5)
    q, k = oracle.widen_bf16(qb), oracle.widen_bf16(kb)
    assert np.array_equal(O[0, :, 0], v[0, :, 0])
    assert np.allclose(L[0, :, 0], 0.5 * np.einsum("hd,hd->h", q[0, :, 0], k[0, :, 0]), atol=1e-14, rtol=0)
    # one dominant key under a huge scale -> that key's V row
    O, _ = oracle.attention_fp64(qb, kb, vb, False, 1e4)
    S = np.einsum("hid,hjd->hij", q[0], k[0])
    arg = S.argmax(-1)
    for h in range(2):
        assert np.allclose(O[0, h], v[0, h][arg[h]], atol=1e-9, rtol=0)


def test_rows_subset_matches_full():
    w = WORKLOADS["tiny_256_d64"]
    qb, kb, vb = _bits(1, 2, 2, 256, 256, 64, seed=71)
    rows = np.array([[[0, 3, 100, 255]] * 2])
    for causal in (False, True):
        O, L = oracle.attention_fp64(qb, kb, vb, causal, w.scale)
        Os, Ls = oracle.attention_fp64(qb, kb, vb, causal, w.scale, rows=rows)
        assert np.array_equal(Os, O[:, :, rows[0, 0]]) and np.array_equal(Ls, L[:, :, rows[0, 0]])


# ----------------------------------------------------------------------------
# Planted mistakes: each mutant of the oracle must fail at least one pin.
# ----------------------------------------------------------------------------
def _pin_suite(att):
    """Small pin suite run against an oracle callable; returns a list of bools."""
    res = []
    for case in [(1, 2, 2, 9, 9, 4, True), (1, 4, 2, 6, 10, 4, False)]:
        qb, kb, vb = _bits(*case[:6], seed=101)
        O, L = att(qb, kb, vb, case[6], 0.4)
        Ob, Lb = brute_force(qb, kb, vb, case[6], 0.4)
        res.append(np.max(np.abs(O - Ob)) < 1e-12 and np.max(np.abs(L - Lb)) < 1e-12)
    qb, kb, vb = _bits(1, 2, 2, 8, 8, 4, seed=102)
    O, L = att(qb, kb, vb, True, 0.4)
    res.append(np.array_equal(O[0, :, 0], oracle.widen_bf16(vb)[0, :, 0]))
    return res


def test_pin_suite_passes_on_oracle():
    assert all(_pin_suite(oracle.attention_fp64))


@pytest.mark.parametrize("mutant", ["dropped_scale", "strict_causal", "gqa_modulo",
                                    "lse_without_max", "transposed_v", "no_max_shift_sign"])
def test_planted_mistakes_are_caught(monkeypatch, mutant):
    if mutant == "dropped_scale":
        orig = oatt.score_matrix_fp64
        monkeypatch.setattr(oatt, "score_matrix_fp64",
                            lambda q, k, scale, causal, rows=None: orig(q, k, 1.0, causal, rows))
    elif mutant == "strict_causal":
        def bad(q, k, scale, causal, rows=None):
            idx = np.arange(q.shape[0]) if rows is None else rows
            S = scale * (q[idx] @ k.T)
            if causal:
                S = np.where(np.arange(k.shape[0])[None, :] < idx[:, None], S, -np.inf)
                S[:, 0] = np.where(idx == 0, scale * (q[idx] @ k.T)[:, 0], S[:, 0])
            return S
        monkeypatch.setattr(oatt, "score_matrix_fp64", bad)
    elif mutant == "gqa_modulo":
        monkeypatch.setattr(oatt, "_kv_head", lambda h, Hq, Hkv: h % Hkv)
    elif mutant == "lse_without_max":
        orig = oatt.attention_f64

        def bad(*a, **kw):
            O, L = orig(*a, **kw)
            return O, np.log(np.exp(L) * 0.5 + 0.5)
        monkeypatch.setattr(oatt, "attention_f64", bad)
    elif mutant == "transposed_v":
        orig = oatt.attention_f64

        def bad(q, k, v, *a, **kw):
            vv = np.asarray(v)
            vflip = vv[:, :, ::-1, :].copy()
            return orig(q, k, vflip, *a, **kw)
        monkeypatch.setattr(oatt, "attention_f64", bad)
    elif mutant == "no_max_shift_sign":
        orig = oatt.score_matrix_fp64
        monkeypatch.setattr(oatt, "score_matrix_fp64",
                            lambda q, k, scale, causal, rows=None: -orig(q, k, scale, causal, rows)
                            if not causal else orig(-q, k, scale, causal, rows))
    assert not all(_pin_suite(oatt.attention_fp64))
