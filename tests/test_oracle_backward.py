"""Pins for the fp64 backward oracle (CPU only): torch autograd in float64 on
the same definition (a library special case), central finite differences of
a scalar loss (brute force), and the identity rowsum(P * dP) = rowsum(dO * O)
the kernels rely on."""
import math

import numpy as np
import pytest
import torch

import oracle
from synthetic import bf16_bits, make_qkv


def _inputs(B, Hq, Hkv, Nq, Nkv, d, seed):
    q, k, v = make_qkv(B, Hq, Hkv, Nq, Nkv, d, seed)
    g = torch.Generator().manual_seed(seed + 1)
    do = torch.randn((B, Hq, Nq, d), generator=g).to(torch.bfloat16)
    return bf16_bits(q), bf16_bits(k), bf16_bits(v), bf16_bits(do)


def _autograd(qb, kb, vb, dob, causal, scale):
    q, k, v, do = (torch.from_numpy(oracle.widen_bf16(x)).requires_grad_(True) for x in (qb, kb, vb, dob))
    g = q.shape[1] // k.shape[1]
    Nq, Nkv = q.shape[2], k.shape[2]
    mask = None
    if causal:
        mask = torch.arange(Nkv)[None, :] <= torch.arange(Nq)[:, None] + (Nkv - Nq)
    o = torch.nn.functional.scaled_dot_product_attention(
        q, k.repeat_interleave(g, dim=1), v.repeat_interleave(g, dim=1), attn_mask=mask, scale=scale)
    o.backward(do.detach())
    return q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


@pytest.mark.parametrize("shape,causal", [
    ((1, 2, 2, 33, 33, 16), False), ((2, 4, 2, 40, 40, 8), True), ((1, 4, 1, 17, 60, 16), True),
    ((1, 2, 2, 64, 20, 8), False),
])
def test_backward_matches_torch_autograd(shape, causal):
    qb, kb, vb, dob = _inputs(*shape, seed=sum(shape))
    scale = 1 / math.sqrt(shape[-1])
    dQ, dK, dV = oracle.attention_bwd_fp64(qb, kb, vb, dob, causal, scale)
    rq, rk, rv = _autograd(qb, kb, vb, dob, causal, scale)
    for a, r in ((dQ, rq), (dK, rk), (dV, rv)):
        assert np.max(np.abs(a - r)) < 1e-11


def test_backward_finite_differences():
    qb, kb, vb, dob = _inputs(1, 2, 1, 6, 7, 4, seed=5)
    scale = 0.4
    dQ, dK, dV = oracle.attention_bwd_fp64(qb, kb, vb, dob, True, scale)
    q, k, v, do = (oracle.widen_bf16(x) for x in (qb, kb, vb, dob))

    def loss(q_, k_, v_):
        O, _ = oracle.attention_f64(q_, k_, v_, True, scale)
        return float((O * do).sum())
    eps = 1e-6
    for x, g in ((q, dQ), (k, dK), (v, dV)):
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = [xp if x is a else a for a in (q, k, v)]
            args_m = [xm if x is a else a for a in (q, k, v)]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - g[idx]) < 1e-7


def test_delta_identity():
    qb, kb, vb, dob = _inputs(1, 2, 2, 50, 50, 16, seed=9)
    O, _, P = oracle.attention_fp64(qb, kb, vb, True, 0.25, return_p=True)
    do = oracle.widen_bf16(dob)
    v = oracle.widen_bf16(vb)
    dP = np.einsum("bhid,bhjd->bhij", do, v)
    assert np.max(np.abs((P * dP).sum(-1) - (do * O).sum(-1))) < 1e-12


@pytest.mark.parametrize("block_rows", [7, 16, 1000])
def test_row_blocked_head_matches_whole_matrix(block_rows):
    qb, kb, vb, dob = _inputs(1, 2, 1, 45, 60, 16, seed=12)
    scale = 0.3
    dQ, dK, dV = oracle.attention_bwd_fp64(qb, kb, vb, dob, True, scale)
    w = oracle.widen_bf16
    gK = np.zeros_like(dK[0, 0])
    gV = np.zeros_like(dV[0, 0])
    for h in range(2):
        q, do = w(qb[0, h]), w(dob[0, h])
        k, v = w(kb[0, 0]), w(vb[0, 0])
        hq, hk, hv = oracle.backward.attention_bwd_head(q, k, v, do, True, scale, block_rows)
        assert np.max(np.abs(hq - dQ[0, h])) < 1e-13
        gK += hk
        gV += hv
        # the blocks' O and LSE are the forward's
        O, L = oracle.attention_f64(q[None, None], k[None, None], v[None, None], True, scale)
        for blk in oracle.backward.attention_bwd_head_blocks(q, k, v, do, True, scale, block_rows):
            assert np.max(np.abs(blk["O"] - O[0, 0, blk["i0"]:blk["i1"]])) < 1e-13
            assert np.max(np.abs(blk["LSE"] - L[0, 0, blk["i0"]:blk["i1"]])) < 1e-13
    assert np.max(np.abs(gK - dK[0, 0])) < 1e-13 and np.max(np.abs(gV - dV[0, 0])) < 1e-13


def _packed(lens_q, lens_k, Hq, Hkv, d, seed):
    g = torch.Generator().manual_seed(seed)
    tq, tk = sum(lens_q), sum(lens_k)
    q = torch.randn((tq, Hq, d), generator=g).to(torch.bfloat16)
    k = torch.randn((tk, Hkv, d), generator=g).to(torch.bfloat16)
    v = torch.randn((tk, Hkv, d), generator=g).to(torch.bfloat16)
    do = torch.randn((tq, Hq, d), generator=g).to(torch.bfloat16)
    cq = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int64)
    ck = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int64)
    return bf16_bits(q), bf16_bits(k), bf16_bits(v), bf16_bits(do), cq, ck


def test_varlen_backward_equal_lengths_is_dense_backward():
    B, H, N, d = 3, 2, 20, 8
    qb, kb, vb, dob = _inputs(B, H, H, N, N, d, seed=40)
    dQ, dK, dV = oracle.attention_bwd_fp64(qb, kb, vb, dob, True, 0.3)
    pack = lambda x: np.ascontiguousarray(x.transpose(0, 2, 1, 3).reshape(B * N, H, d))  # noqa: E731
    cu = np.arange(0, (B + 1) * N, N)
    gq, gk, gv = oracle.backward.attention_varlen_bwd_fp64(pack(qb), pack(kb), pack(vb), pack(dob),
                                                           cu, cu, True, 0.3)
    assert np.array_equal(gq, pack(dQ)) and np.array_equal(gk, pack(dK)) and np.array_equal(gv, pack(dV))


def test_varlen_backward_finite_differences():
    """Central differences of <O, dO> through the packed forward oracle, with
    unequal lengths, a prefix of keys (cache) and an empty key set."""
    qb, kb, vb, dob, cq, ck = _packed([3, 2, 4], [5, 0, 4], 2, 1, 4, seed=41)
    scale = 0.5
    dQ, dK, dV = oracle.backward.attention_varlen_bwd_fp64(qb, kb, vb, dob, cq, ck, True, scale)
    w = oracle.widen_bf16
    q, k, v, do = w(qb), w(kb), w(vb), w(dob)

    def loss(q_, k_, v_):
        # <O, dO> with O from the definition on float64 inputs, sequence by
        # sequence (the packed forward oracle takes bf16 bits, which a
        # perturbed input is not)
        total = 0.0
        for s in range(len(cq) - 1):
            a, b, c, e = cq[s], cq[s + 1], ck[s], ck[s + 1]
            if b == a:
                continue
            t = lambda x, i, j: x[i:j].transpose(1, 0, 2)[None]  # noqa: E731
            O, _ = oracle.attention_f64(t(q_, a, b), t(k_, c, e), t(v_, c, e), True, scale)
            total += float((O[0].transpose(1, 0, 2) * do[a:b]).sum())
        return total
    eps = 1e-6
    for x, g in ((q, dQ), (k, dK), (v, dV)):
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            fd = (loss(*[xp if x is a else a for a in (q, k, v)]) -
                  loss(*[xm if x is a else a for a in (q, k, v)])) / (2 * eps)
            assert abs(fd - g[idx]) < 1e-7
