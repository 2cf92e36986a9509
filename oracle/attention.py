"""Exact attention forward in fp64, materialising S and P (test infrastructure).

Follows the definition on "FlashAttention (TR)" (systems-analysis.info),
section "Standart Attention Mekanizmasının Sorunları":
    Attention(Q, K, V) = softmax(Q K^T / sqrt(d_k)) V
computed the naive way the same section describes (the full S = Q K^T matrix
is formed, here one (batch, head) at a time). The fused method reaches this
same result exactly ("FlashAttention" glossary page: exact, not an
approximation, mathematically identical to the naive implementation), so the
oracle is the plain definition and nothing else.

Readings of points the pages leave open (each is listed in the design notes):
  * GQA: query head h reads kv head floor(h / (Hq / Hkv)) (contiguous groups;
    the pages only name MQA, "FlashAttention-2 (2023)" section).
  * Causal: key j is visible to query i iff j <= i + (Nkv - Nq) (aligned to
    the bottom right, so the last query sees every key: a prefill whose first
    Nkv - Nq keys are a cache). For Nq == Nkv this is j <= i. A row that sees
    no key (possible only when Nq > Nkv) has O = 0 and LSE = -inf.
  * scale is an explicit argument (1/sqrt(d) by default in the binding).
  * LSE_i = ln sum_j exp(scale * S_raw_ij) over visible j, natural log,
    scale included.

Everything is float64: the bf16 inputs are widened exactly (bf16 bits << 16
give the float32 bits, float32 -> float64 is exact).
"""
from __future__ import annotations

import numpy as np


def widen_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact float64 values."""
    bits = np.asarray(bits)
    if bits.dtype != np.uint16:
        raise TypeError("expected uint16 bf16 bit patterns")
    f32 = (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return f32.astype(np.float64)


def _kv_head(h: int, Hq: int, Hkv: int) -> int:
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    return h // (Hq // Hkv)


def score_matrix_fp64(q: np.ndarray, k: np.ndarray, scale: float, causal: bool,
                      rows: np.ndarray | None = None) -> np.ndarray:
    """S = scale * Q K^T for one head (fp64), with -inf at masked positions.

    q: [Nq, d] float64, k: [Nkv, d] float64; ``rows`` selects query rows (their
    absolute indices are used by the causal mask).
    """
    Nq = q.shape[0]
    Nkv = k.shape[0]
    idx = np.arange(Nq) if rows is None else np.asarray(rows)
    S = scale * (q[idx] @ k.T)
    if causal:
        j = np.arange(Nkv)
        S = np.where(j[None, :] <= idx[:, None] + (Nkv - Nq), S, -np.inf)
    return S


def attention_fp64(q_bits: np.ndarray, k_bits: np.ndarray, v_bits: np.ndarray,
                   causal: bool, scale: float, rows: np.ndarray | None = None,
                   return_p: bool = False):
    """Exact attention forward on bf16 inputs.

    q_bits: uint16 [B, Hq, Nq, d]; k_bits, v_bits: uint16 [B, Hkv, Nkv, d]
    (bf16 bit patterns, as produced by ``synthetic.bf16_bits``).
    rows: optional int array [B, Hq, R] of query rows to evaluate.

    Returns (O, LSE) as float64: O [B, Hq, R, d], LSE [B, Hq, R] (R = Nq when
    rows is None); with return_p=True also P [B, Hq, R, Nkv].
    """
    for a in (q_bits, k_bits, v_bits):
        if np.asarray(a).dtype != np.uint16:
            raise TypeError("expected uint16 bf16 bit patterns")
    return attention_f64(q_bits, k_bits, v_bits, causal, scale, rows, return_p,
                         _widen=widen_bf16)


def attention_f64(q, k, v, causal: bool, scale: float, rows=None, return_p: bool = False,
                  _widen=None):
    """Same definition on float64 arrays ([B, H, N, d]); used by the pins that
    need inputs which are not bf16 values (e.g. mean-smoothed K)."""
    widen = _widen if _widen is not None else (lambda a: np.asarray(a, dtype=np.float64))
    B, Hq, Nq, d = q.shape
    Bk, Hkv, Nkv, dk = k.shape
    if (Bk, dk) != (B, d) or v.shape != k.shape:
        raise ValueError("shape mismatch between Q and K/V")
    R = Nq if rows is None else rows.shape[-1]
    O = np.empty((B, Hq, R, d), dtype=np.float64)
    L = np.empty((B, Hq, R), dtype=np.float64)
    Ps = np.empty((B, Hq, R, Nkv), dtype=np.float64) if return_p else None
    for b in range(B):
        for h in range(Hq):
            hk = _kv_head(h, Hq, Hkv)
            qh = widen(q[b, h])
            kh = widen(k[b, hk])
            vh = widen(v[b, hk])
            r = None if rows is None else rows[b, h]
            S = score_matrix_fp64(qh, kh, scale, causal, r)
            m = S.max(axis=1) if S.shape[1] else np.full(S.shape[0], -np.inf)
            empty = np.isinf(m)                    # rows that see no key
            m_safe = np.where(empty, 0.0, m)
            E = np.exp(S - m_safe[:, None])        # exp(-inf) = 0 at masked keys
            l = E.sum(axis=1)
            with np.errstate(invalid="ignore", divide="ignore"):
                P = np.where(empty[:, None], 0.0, E / np.where(empty, 1.0, l)[:, None])
                L[b, h] = np.where(empty, -np.inf, m_safe + np.log(l))
            O[b, h] = P @ vh
            if return_p:
                Ps[b, h] = P
    if return_p:
        return O, L, Ps
    return O, L


def attention_varlen_fp64(q_bits, k_bits, v_bits, cu_seqlens_q, cu_seqlens_k, causal: bool,
                          scale: float):
    """Packed variable-length attention: q_bits uint16 [total_q, Hq, d], k/v
    [total_k, Hkv, d]; sequence s owns query rows cu_seqlens_q[s]:cu_seqlens_q[s+1]
    and key rows cu_seqlens_k[s]:cu_seqlens_k[s+1], and attends only within
    itself (causal masks are per sequence, bottom-right aligned).

    Returns O float64 [total_q, Hq, d] and LSE float64 [Hq, total_q].
    """
    total_q, Hq, d = q_bits.shape
    O = np.zeros((total_q, Hq, d))
    L = np.full((Hq, total_q), -np.inf)
    for s in range(len(cu_seqlens_q) - 1):
        q0, q1 = int(cu_seqlens_q[s]), int(cu_seqlens_q[s + 1])
        k0, k1 = int(cu_seqlens_k[s]), int(cu_seqlens_k[s + 1])
        if q1 == q0:
            continue
        qs = np.ascontiguousarray(q_bits[q0:q1].transpose(1, 0, 2))[None]
        ks = np.ascontiguousarray(k_bits[k0:k1].transpose(1, 0, 2))[None]
        vs = np.ascontiguousarray(v_bits[k0:k1].transpose(1, 0, 2))[None]
        Os, Ls = attention_fp64(qs, ks, vs, causal, scale)
        O[q0:q1] = Os[0].transpose(1, 0, 2)
        L[:, q0:q1] = Ls[0]
    return O, L
