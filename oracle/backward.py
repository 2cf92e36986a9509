"""Attention backward in fp64 from the derivative of the definition (test
infrastructure).

The glossary page "FlashAttention" (aisaas-seo) says the backward pass
recomputes the few cheap intermediates instead of storing them; the gradients
themselves follow from differentiating O = softmax(scale * Q K^T) V (the
definition on "FlashAttention (TR)", "Standart Attention Mekanizmasının
Sorunları"). For one (batch, head), with P the softmax probabilities:

    dV  = P^T dO
    dP  = dO V^T
    dS  = P * (dP - rowsum(P * dP))        (softmax Jacobian, row by row)
    dQ  = scale * dS K
    dK  = scale * dS^T Q

GQA: a kv head's dK and dV are the sums over the query heads of its group.
Masked positions have P = 0 and hence dS = 0. Everything in float64 on the
exact bf16 inputs.
"""
from __future__ import annotations

import numpy as np

from .attention import _kv_head, score_matrix_fp64, widen_bf16


def attention_bwd_fp64(q_bits, k_bits, v_bits, do_bits, causal: bool, scale: float):
    """q_bits, do_bits: uint16 [B, Hq, Nq, d]; k_bits, v_bits: uint16 [B, Hkv, Nkv, d].
    Returns (dQ [B, Hq, Nq, d], dK [B, Hkv, Nkv, d], dV [B, Hkv, Nkv, d]) float64."""
    B, Hq, Nq, d = q_bits.shape
    Hkv, Nkv = k_bits.shape[1], k_bits.shape[2]
    dQ = np.zeros((B, Hq, Nq, d))
    dK = np.zeros((B, Hkv, Nkv, d))
    dV = np.zeros((B, Hkv, Nkv, d))
    for b in range(B):
        for h in range(Hq):
            hk = _kv_head(h, Hq, Hkv)
            q = widen_bf16(q_bits[b, h])
            k = widen_bf16(k_bits[b, hk])
            v = widen_bf16(v_bits[b, hk])
            do = widen_bf16(do_bits[b, h])
            S = score_matrix_fp64(q, k, scale, causal)
            m = S.max(axis=1)
            empty = np.isinf(m)
            E = np.exp(S - np.where(empty, 0.0, m)[:, None])
            l = E.sum(axis=1)
            P = np.where(empty[:, None], 0.0, E / np.where(empty, 1.0, l)[:, None])
            dV[b, hk] += P.T @ do
            dP = do @ v.T
            dS = P * (dP - (P * dP).sum(axis=1, keepdims=True))
            dQ[b, h] = scale * (dS @ k)
            dK[b, hk] += scale * (dS.T @ q)
    return dQ, dK, dV


def attention_bwd_head_blocks(q, k, v, do, causal: bool, scale: float, block_rows: int = 2048):
    """One (batch, query head) of the same computation on float64 arrays
    q, do [Nq, d] and k, v [Nkv, d], walked over blocks of query rows so that
    long sequences fit in memory. Every row of a block is complete (all of its
    keys), so each yielded quantity is exact for its rows:

        dict(i0, i1, S (scaled, masked -inf), P, O, LSE, D, dP, dS)

    The gradients of the head are then dQ[i0:i1] = scale * dS K and the sums
    over blocks of scale * dS^T Q[i0:i1] (dK) and P^T dO[i0:i1] (dV)."""
    Nq, Nkv = q.shape[0], k.shape[0]
    off = Nkv - Nq
    for i0 in range(0, Nq, block_rows):
        i1 = min(Nq, i0 + block_rows)
        S = (q[i0:i1] @ k.T) * scale
        if causal:
            rows = np.arange(i0, i1)[:, None]
            S = np.where(np.arange(Nkv)[None, :] <= rows + off, S, -np.inf)
        m = S.max(axis=1)
        empty = np.isinf(m)
        E = np.exp(S - np.where(empty, 0.0, m)[:, None])
        l = E.sum(axis=1)
        P = np.where(empty[:, None], 0.0, E / np.where(empty, 1.0, l)[:, None])
        lse = np.where(empty, -np.inf, m + np.log(np.where(empty, 1.0, l)))
        O = P @ v
        D = (do[i0:i1] * O).sum(axis=1)
        dP = do[i0:i1] @ v.T
        dS = P * (dP - D[:, None])
        yield dict(i0=i0, i1=i1, S=S, P=P, O=O, LSE=lse, D=D, dP=dP, dS=dS)


def attention_bwd_head(q, k, v, do, causal: bool, scale: float, block_rows: int = 2048):
    """dQ [Nq, d], dK, dV [Nkv, d] of one head from attention_bwd_head_blocks."""
    dQ = np.zeros_like(q)
    dK = np.zeros_like(k)
    dV = np.zeros_like(v)
    for blk in attention_bwd_head_blocks(q, k, v, do, causal, scale, block_rows):
        i0, i1 = blk["i0"], blk["i1"]
        dQ[i0:i1] = scale * (blk["dS"] @ k)
        dK += scale * (blk["dS"].T @ q[i0:i1])
        dV += blk["P"].T @ do[i0:i1]
    return dQ, dK, dV


def attention_varlen_bwd_fp64(q_bits, k_bits, v_bits, do_bits, cu_q, cu_k, causal: bool,
                              scale: float):
    """Backward of attention_varlen_fp64: packed sequences q, do [total_q, Hq, d],
    k, v [total_k, Hkv, d] (uint16 bf16 bits), sequence s owning query rows
    cu_q[s]:cu_q[s+1] and key rows cu_k[s]:cu_k[s+1]; each sequence is the
    dense backward on its own rows (causal mask bottom-right per sequence).
    Returns float64 (dQ, dK, dV) in the packed layouts."""
    total_q, Hq, d = q_bits.shape
    total_k, Hkv, _ = k_bits.shape
    dQ = np.zeros((total_q, Hq, d))
    dK = np.zeros((total_k, Hkv, d))
    dV = np.zeros((total_k, Hkv, d))
    for s in range(len(cu_q) - 1):
        q0, q1, k0, k1 = int(cu_q[s]), int(cu_q[s + 1]), int(cu_k[s]), int(cu_k[s + 1])
        if q1 == q0 or k1 == k0:
            continue  # no query or no key: every gradient of the sequence is 0
        seq = lambda x, a, b: np.ascontiguousarray(x[a:b].transpose(1, 0, 2))[None]  # noqa: E731
        gq, gk, gv = attention_bwd_fp64(seq(q_bits, q0, q1), seq(k_bits, k0, k1), seq(v_bits, k0, k1),
                                        seq(do_bits, q0, q1), causal, scale)
        dQ[q0:q1] = gq[0].transpose(1, 0, 2)
        dK[k0:k1] = gk[0].transpose(1, 0, 2)
        dV[k0:k1] = gv[0].transpose(1, 0, 2)
    return dQ, dK, dV
