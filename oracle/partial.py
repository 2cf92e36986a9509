"""Attention over a range of keys, and the exact merge of such partial results
(test infrastructure).

"FlashAttention (TR)" (systems-analysis.info), section "Çevrimiçi Softmax
Hesaplama": the softmax is computed piece by piece, keeping the running
maximum and the running sum of exponentials and updating both as each new
block of keys is processed, and the result is the exact one. Applied to whole
key ranges instead of single tiles, the same update combines independent
partial results: attention of the query rows over keys [lo_s, hi_s) gives a
normalised O_s and LSE_s = ln sum_{j in range s} exp(S_ij), and over the
union of the ranges

    LSE = ln sum_s exp(LSE_s),      O = sum_s exp(LSE_s - LSE) * O_s.

(The "FlashAttention-2 (2023)" section credits its speed-up to better
parallelism and work partitioning; splitting the keys is one such partition.)

Readings (listed in the design notes):
  * A key range is a slice [kv_lo, kv_hi) of the full key sequence of length
    Nkv; the causal mask stays the global one (key j visible to query i iff
    j <= i + (Nkv - Nq), bottom-right aligned), so a range may hold no
    visible key for some rows. Such a row's partial is O_s = 0,
    LSE_s = -inf, and it carries zero weight in the merge.
  * A row with LSE_s = -inf in every part merges to O = 0, LSE = -inf, as
    the full attention gives for a row that sees no key.
"""
from __future__ import annotations

import numpy as np

from .attention import _kv_head, score_matrix_fp64, widen_bf16


def attention_partial_fp64(q_bits, k_bits, v_bits, kv_lo: int, kv_hi: int, causal: bool,
                           scale: float):
    """Exact attention of every query row over keys [kv_lo, kv_hi) only.

    q_bits uint16 [B, Hq, Nq, d]; k_bits, v_bits uint16 [B, Hkv, Nkv, d] (the
    full key sequence). Returns O float64 [B, Hq, Nq, d] (normalised over the
    range) and LSE float64 [B, Hq, Nq] (ln of the sum over the range).
    """
    B, Hq, Nq, d = q_bits.shape
    _, Hkv, Nkv, _ = k_bits.shape
    if not 0 <= kv_lo <= kv_hi <= Nkv:
        raise ValueError("key range outside [0, Nkv]")
    O = np.zeros((B, Hq, Nq, d))
    L = np.full((B, Hq, Nq), -np.inf)
    for b in range(B):
        for h in range(Hq):
            hk = _kv_head(h, Hq, Hkv)
            # the global mask first, then the range's columns
            S = score_matrix_fp64(widen_bf16(q_bits[b, h]), widen_bf16(k_bits[b, hk]), scale,
                                  causal)[:, kv_lo:kv_hi]
            vh = widen_bf16(v_bits[b, hk])[kv_lo:kv_hi]
            m = S.max(axis=1) if S.shape[1] else np.full(Nq, -np.inf)
            seen = np.isfinite(m)
            if not seen.any():
                continue
            E = np.exp(S[seen] - m[seen][:, None])
            l = E.sum(axis=1)
            O[b, h, seen] = (E / l[:, None]) @ vh
            L[b, h, seen] = m[seen] + np.log(l)
    return O, L


def merge_partials_fp64(o_parts, lse_parts):
    """Merge partial results over disjoint key ranges.

    o_parts float [S, ..., d], lse_parts float [S, ...] (natural-log LSE, -inf
    for a row that saw no key in that part). Returns (O [..., d], LSE [...])
    in float64.
    """
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    if o_parts.shape[:-1] != lse_parts.shape:
        raise ValueError("o_parts must be lse_parts' shape plus a trailing d")
    m = lse_parts.max(axis=0)
    seen = np.isfinite(m)
    m_safe = np.where(seen, m, 0.0)
    w = np.exp(lse_parts - m_safe)               # 0 for the -inf parts
    total = w.sum(axis=0)
    with np.errstate(divide="ignore"):
        lse = np.where(seen, m_safe + np.log(np.where(seen, total, 1.0)), -np.inf)
    weight = np.where(seen, w / np.where(seen, total, 1.0), 0.0)
    o = (weight[..., None] * o_parts).sum(axis=0)
    return o, lse
