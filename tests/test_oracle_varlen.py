"""Pins for bottom-right causal alignment (Nq != Nkv) and packed variable-length
sequences in the oracle (CPU only)."""
import math

import numpy as np
import pytest
import torch

import oracle
from synthetic import bf16_bits, make_qkv


def _bits(B, Hq, Hkv, Nq, Nkv, d, seed):
    q, k, v = make_qkv(B, Hq, Hkv, Nq, Nkv, d, seed)
    return bf16_bits(q), bf16_bits(k), bf16_bits(v)


def brute(qb, kb, vb, scale):
    """Pure-Python loops, key j visible to query i iff j <= i + (Nkv - Nq)."""
    B, Hq, Nq, d = qb.shape
    Hkv, Nkv = kb.shape[1], kb.shape[2]
    q, k, v = (oracle.widen_bf16(x).tolist() for x in (qb, kb, vb))
    O = np.zeros((B, Hq, Nq, d))
    L = np.full((B, Hq, Nq), -np.inf)
    for b in range(B):
        for h in range(Hq):
            hk = h // (Hq // Hkv)
            for i in range(Nq):
                vis = [j for j in range(Nkv) if j <= i + Nkv - Nq]
                if not vis:
                    continue
                s = [scale * math.fsum(q[b][h][i][c] * k[b][hk][j][c] for c in range(d)) for j in vis]
                m = max(s)
                e = [math.exp(x - m) for x in s]
                l = math.fsum(e)
                for c in range(d):
                    O[b, h, i, c] = math.fsum(e[t] * v[b][hk][j][c] for t, j in enumerate(vis)) / l
                L[b, h, i] = m + math.log(l)
    return O, L


@pytest.mark.parametrize("Nq,Nkv", [(5, 9), (9, 9), (9, 5), (1, 7), (12, 3)])
def test_bottom_right_causal_brute_force(Nq, Nkv):
    qb, kb, vb = _bits(1, 4, 2, Nq, Nkv, 6, seed=Nq * 31 + Nkv)
    O, L = oracle.attention_fp64(qb, kb, vb, True, 0.4)
    Ob, Lb = brute(qb, kb, vb, 0.4)
    assert np.max(np.abs(O - Ob)) < 1e-13
    assert np.array_equal(np.isinf(L), np.isinf(Lb))
    fin = np.isfinite(L)
    assert np.max(np.abs(L[fin] - Lb[fin])) < 1e-13


def test_rows_without_keys_are_zero_with_minus_inf_lse():
    qb, kb, vb = _bits(1, 2, 2, 10, 4, 8, seed=3)
    O, L = oracle.attention_fp64(qb, kb, vb, True, 0.3)
    # rows 0..5 see no key (j <= i - 6)
    assert np.all(O[:, :, :6] == 0.0) and np.all(np.isneginf(L[:, :, :6]))
    assert np.all(np.isfinite(L[:, :, 6:]))


def test_prefill_with_cache_equals_tail_of_full_causal():
    # the last Lq queries of a causal problem over N tokens, against all N keys,
    # are a bottom-right causal problem with Nq = Lq, Nkv = N
    qb, kb, vb = _bits(2, 4, 2, 300, 300, 16, seed=11)
    O, L = oracle.attention_fp64(qb, kb, vb, True, 0.25)
    for lq in (1, 77, 128, 300):
        Ot, Lt = oracle.attention_fp64(qb[:, :, -lq:], kb, vb, True, 0.25)
        assert np.max(np.abs(Ot - O[:, :, -lq:])) < 1e-13
        assert np.max(np.abs(Lt - L[:, :, -lq:])) < 1e-12


def test_bottom_right_matches_sdpa_with_explicit_mask():
    qb, kb, vb = _bits(1, 2, 2, 70, 200, 32, seed=5)
    O, _ = oracle.attention_fp64(qb, kb, vb, True, 0.2)
    q, k, v = (torch.from_numpy(oracle.widen_bf16(x)) for x in (qb, kb, vb))
    mask = torch.arange(200)[None, :] <= torch.arange(70)[:, None] + 130
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=0.2)
    assert np.max(np.abs(O - ref.numpy())) < 1e-12


def _packed(lens_q, lens_k, Hq, Hkv, d, seed):
    g = torch.Generator().manual_seed(seed)
    tq, tk = sum(lens_q), sum(lens_k)
    q = torch.randn((tq, Hq, d), generator=g).to(torch.bfloat16)
    k = torch.randn((tk, Hkv, d), generator=g).to(torch.bfloat16)
    v = torch.randn((tk, Hkv, d), generator=g).to(torch.bfloat16)
    cq = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    ck = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    return bf16_bits(q), bf16_bits(k), bf16_bits(v), cq, ck


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_equals_block_diagonal_dense(causal):
    lens_q, lens_k = [5, 17, 1, 40], [9, 17, 3, 40]
    qb, kb, vb, cq, ck = _packed(lens_q, lens_k, 4, 2, 8, seed=7)
    O, L = oracle.attention_varlen_fp64(qb, kb, vb, cq, ck, causal, 0.35)
    # one dense problem over the concatenation with a block-diagonal mask
    q, k, v = (torch.from_numpy(oracle.widen_bf16(x)).permute(1, 0, 2) for x in (qb, kb, vb))
    k = k.repeat_interleave(2, dim=0)
    v = v.repeat_interleave(2, dim=0)
    tq, tk = cq[-1], ck[-1]
    mask = torch.zeros((tq, tk), dtype=torch.bool)
    for s in range(len(lens_q)):
        for i in range(cq[s], cq[s + 1]):
            for j in range(ck[s], ck[s + 1]):
                if not causal or (j - ck[s]) <= (i - cq[s]) + lens_k[s] - lens_q[s]:
                    mask[i, j] = True
    S = 0.35 * torch.einsum("hid,hjd->hij", q, k)
    S = S.masked_fill(~mask, -float("inf"))
    P = torch.softmax(S, dim=-1)
    ref = torch.einsum("hij,hjd->hid", P, v).permute(1, 0, 2).numpy()
    assert np.max(np.abs(O - ref)) < 1e-12
    lref = torch.logsumexp(S, dim=-1).numpy()
    assert np.max(np.abs(L - lref)) < 1e-12


def test_varlen_equal_lengths_equals_batched():
    B, N, Hq, Hkv, d = 3, 33, 4, 2, 8
    qb, kb, vb = _bits(B, Hq, Hkv, N, N, d, seed=9)
    O, L = oracle.attention_fp64(qb, kb, vb, True, 0.3)
    cu = np.arange(0, (B + 1) * N, N, dtype=np.int32)
    pack = lambda x: np.ascontiguousarray(x.transpose(0, 2, 1, 3).reshape(B * N, x.shape[1], d))  # noqa: E731
    Ov, Lv = oracle.attention_varlen_fp64(pack(qb), pack(kb), pack(vb), cu, cu, True, 0.3)
    assert np.array_equal(Ov, O.transpose(0, 2, 1, 3).reshape(B * N, Hq, d))
    assert np.array_equal(Lv, L.transpose(1, 0, 2).reshape(Hq, B * N))
