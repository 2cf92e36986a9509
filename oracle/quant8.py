"""SageAttention-style 8-bit steps, written out plainly (test infrastructure).

Follows "Makale Bülteni — SageAttention" (cmlonder.com), section
"İddia ve Gerçeklik: SageAttention": attention is two GEMMs (Q K^T, then P V);
the first runs on INT8 after K is mean-centred ("smoothing"), which the
shift-invariance of softmax makes lossless; the second runs on FP8 because P
already lies in [0, 1]; accumulation is in higher precision.

The granularities are the ones the 8-bit workload fixes: one fp32 scale per
128-token block for Q and for smoothed K, one fp32 scale per (kv head,
channel) for V, P encoded as e4m3 after multiplying by 448.

Readings of points the page leaves open (each listed in the design notes):
  * K mean: over all Nkv tokens per (batch, kv head, channel), computed in
    float64 and rounded once to float32 (so the value is unique).
  * INT8: scale = fp32(amax / 127) (amax = 0 -> scale 1), code =
    round-half-even(fp32(x / scale)) clamped to [-127, 127]. All of this in
    float32, the precision the kernel takes the same decision in.
  * FP8: e4m3fn (bias 7, 3 mantissa bits, max 448, no infinities), round to
    nearest even, saturating at +-448. V scale = fp32(amax_channel / 448).
  * Smoothing shifts every score of query row i by -scale * q_i . kbar, so the
    true LSE is the smoothed one plus scale * q_i . kbar.
"""
from __future__ import annotations

import numpy as np

from .attention import widen_bf16, _kv_head

E4M3_MAX = 448.0
INT8_MAX = 127
BLOCK = 128


# --------------------------------------------------------------------------
# FP8 e4m3 (fn variant) encode / decode, from the format definition.
# --------------------------------------------------------------------------
def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """e4m3fn byte -> float64. 0x7F / 0xFF are NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return sign * val


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """float -> e4m3fn byte, round to nearest even, saturate to +-448.

    Works in float64 on the (exactly widened) input. The quantum of the binade
    containing |x| is 2^(e-3) for normal numbers (e >= -6) and 2^-9 below.
    """
    x = np.asarray(x, dtype=np.float64)
    sign = np.signbit(x)
    a = np.abs(x)
    nan = np.isnan(a)
    a = np.where(nan, 0.0, a)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    # guard floor(log2) against rounding at exact powers of two
    e = np.where(np.exp2(e) > a, e - 1, e)
    e = np.where(np.exp2(e + 1) <= a, e + 1, e)
    e = np.maximum(e, -6.0)
    quantum = np.exp2(e - 3.0)
    r = np.rint(a / quantum) * quantum          # np.rint: round half to even
    r = np.minimum(r, E4M3_MAX)                 # saturate
    # re-encode the (representable) magnitude r
    with np.errstate(divide="ignore"):
        er = np.floor(np.log2(np.where(r > 0, r, 1.0)))
    er = np.where(np.exp2(er) > r, er - 1, er)
    er = np.where(np.exp2(er + 1) <= r, er + 1, er)
    normal = r >= 2.0 ** -6
    exp_field = np.where(normal, er + 7.0, 0.0)
    man_field = np.where(normal, r / np.exp2(er) * 8.0 - 8.0, r / 2.0 ** -9)
    code = (exp_field.astype(np.int64) << 3) | np.rint(man_field).astype(np.int64)
    code = np.where(sign, code | 0x80, code)
    code = np.where(nan, 0x7F, code)
    return code.astype(np.uint8)


# --------------------------------------------------------------------------
# Prepass steps
# --------------------------------------------------------------------------
def k_channel_mean(k_bits: np.ndarray) -> np.ndarray:
    """kbar[b, hkv, c] = mean over tokens of K[b, hkv, :, c] (fp64, rounded to fp32)."""
    return widen_bf16(k_bits).mean(axis=2).astype(np.float32)


def smooth_k(k_bits: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """K' = K - kbar, one float32 subtraction per element."""
    kf = widen_bf16(k_bits).astype(np.float32)
    return (kf - kbar[:, :, None, :]).astype(np.float32)


def quant_int8_blocks(x: np.ndarray, block: int = BLOCK):
    """Per-(b, h, 128-token block) symmetric INT8 quantisation in float32.

    x: float32 [B, H, N, d]. Returns (codes int8 [B, H, N, d],
    scales float32 [B, H, ceil(N / block)]).
    """
    x = np.asarray(x, dtype=np.float32)
    B, H, N, d = x.shape
    nb = -(-N // block)
    codes = np.empty((B, H, N, d), dtype=np.int8)
    scales = np.empty((B, H, nb), dtype=np.float32)
    for i in range(nb):
        blk = x[:, :, i * block:(i + 1) * block, :]
        amax = np.abs(blk).max(axis=(2, 3)).astype(np.float32)
        s = np.where(amax > 0, amax / np.float32(INT8_MAX), np.float32(1.0)).astype(np.float32)
        q = np.rint(blk / s[:, :, None, None]).astype(np.float32)
        codes[:, :, i * block:(i + 1) * block, :] = np.clip(q, -INT8_MAX, INT8_MAX).astype(np.int8)
        scales[:, :, i] = s
    return codes, scales


def quant_e4m3_blocks(x: np.ndarray, block: int = BLOCK):
    """Per-(b, h, 128-token block) FP8 e4m3 quantisation in float32 (block-wise
    dynamic scaling in the FlashAttention-3 manner: scale = fp32(amax / 448),
    amax = 0 -> 1; code = e4m3(fp32(x / scale))).

    Returns (codes uint8 [B, H, N, d], scales float32 [B, H, ceil(N / block)]).
    """
    x = np.asarray(x, dtype=np.float32)
    B, H, N, d = x.shape
    nb = -(-N // block)
    codes = np.empty((B, H, N, d), dtype=np.uint8)
    scales = np.empty((B, H, nb), dtype=np.float32)
    for i in range(nb):
        blk = x[:, :, i * block:(i + 1) * block, :]
        amax = np.abs(blk).max(axis=(2, 3)).astype(np.float32)
        s = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
        codes[:, :, i * block:(i + 1) * block, :] = e4m3_encode((blk / s[:, :, None, None]).astype(np.float32))
        scales[:, :, i] = s
    return codes, scales


def quant_v_fp8(v_bits: np.ndarray):
    """Per-(b, hkv, channel) FP8 e4m3 quantisation of V.

    Returns (codes uint8 [B, Hkv, N, d], scales float32 [B, Hkv, d]).
    """
    vf = widen_bf16(v_bits).astype(np.float32)
    amax = np.abs(vf).max(axis=2).astype(np.float32)
    s = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    scaled = (vf / s[:, :, None, :]).astype(np.float32)
    return e4m3_encode(scaled), s


def q_dot_kbar(q_bits: np.ndarray, kbar: np.ndarray, Hkv: int) -> np.ndarray:
    """qk[b, hq, i] = q_i . kbar[b, hkv(hq)] in float64."""
    q = widen_bf16(q_bits)
    B, Hq, N, d = q.shape
    out = np.empty((B, Hq, N))
    for h in range(Hq):
        out[:, h] = np.einsum("bnd,bd->bn", q[:, h], kbar[:, _kv_head(h, Hq, Hkv)].astype(np.float64))
    return out


# --------------------------------------------------------------------------
# One-shot quantised attention built from the steps above
# --------------------------------------------------------------------------
def quantised_operands(q_bits, k_bits, v_bits, qk_format: str = "int8"):
    """The operands each 8-bit method feeds its two GEMMs, from the steps above.

    qk_format "int8": SageAttention's INT8 Q and mean-smoothed K (one scale per
    128-token block), with qk = q . kbar to undo the smoothing in LSE.
    qk_format "fp8" : e4m3 Q and K with one scale per 128-token block and no
    smoothing (block-wise dynamic scaling in the FlashAttention-3 manner); qk = 0.
    Both: V as e4m3 with one scale per (batch, kv head, channel).

    Returns a dict of float64 arrays: qd [B,Hq,Nq,d] and kd [B,Hkv,Nkv,d] (the
    dequantised Q and K), vd (dequantised V), qk [B,Hq,Nq], and the raw codes
    and scales (q8, sq, k8, sk, v8, sv).
    """
    B, Hq, Nq, d = q_bits.shape
    Hkv, Nkv = k_bits.shape[1], k_bits.shape[2]
    v8, sv = quant_v_fp8(v_bits)
    if qk_format == "int8":
        kbar = k_channel_mean(k_bits)
        q8, sq = quant_int8_blocks(widen_bf16(q_bits).astype(np.float32))
        k8, sk = quant_int8_blocks(smooth_k(k_bits, kbar))
        qd = q8.astype(np.float64) * np.repeat(sq, BLOCK, axis=2)[:, :, :Nq, None].astype(np.float64)
        kd = k8.astype(np.float64) * np.repeat(sk, BLOCK, axis=2)[:, :, :Nkv, None].astype(np.float64)
        qk = q_dot_kbar(q_bits, kbar, Hkv)
    elif qk_format == "fp8":
        q8, sq = quant_e4m3_blocks(widen_bf16(q_bits).astype(np.float32))
        k8, sk = quant_e4m3_blocks(widen_bf16(k_bits).astype(np.float32))
        qd = e4m3_decode(q8) * np.repeat(sq, BLOCK, axis=2)[:, :, :Nq, None].astype(np.float64)
        kd = e4m3_decode(k8) * np.repeat(sk, BLOCK, axis=2)[:, :, :Nkv, None].astype(np.float64)
        qk = np.zeros((B, Hq, Nq))
    else:
        raise ValueError("qk_format must be 'int8' or 'fp8'")
    vd = e4m3_decode(v8) * sv[:, :, None, :].astype(np.float64)
    return {"qd": qd, "kd": kd, "vd": vd, "qk": qk, "q8": q8, "sq": sq, "k8": k8, "sk": sk,
            "v8": v8, "sv": sv}


def _one_shot(ops, v_exact, causal: bool, scale: float, rows, quantise_pv: bool,
              p_scale: float):
    """softmax of the dequantised scores, then P V, one (batch, query head) at a
    time. With quantise_pv, P is encoded as e4m3(p * p_scale) with p relative to
    the exact row maximum and V is the dequantised e4m3 V; without it, P and V
    are exact (only the scores carry the 8-bit error)."""
    qd, kd = ops["qd"], ops["kd"]
    B, Hq, Nq, d = qd.shape
    Hkv, Nkv = kd.shape[1], kd.shape[2]
    R = Nq if rows is None else rows.shape[-1]
    O = np.empty((B, Hq, R, d))
    L = np.empty((B, Hq, R))
    for b in range(B):
        for h in range(Hq):
            hk = _kv_head(h, Hq, Hkv)
            idx = np.arange(Nq) if rows is None else rows[b, h]
            S = scale * (qd[b, h, idx] @ kd[b, hk].T)
            if causal:   # bottom-right aligned, as the exact definition
                S = np.where(np.arange(Nkv)[None, :] <= idx[:, None] + (Nkv - Nq), S, -np.inf)
            m = S.max(axis=1)
            empty = np.isinf(m)                     # rows that see no key
            m = np.where(empty, 0.0, m)
            E = np.exp(S - m[:, None])
            l = E.sum(axis=1)
            ls = np.where(empty, 1.0, l)
            if quantise_pv:
                P8 = e4m3_decode(e4m3_encode((E * p_scale).astype(np.float32)))
                O[b, h] = (P8 @ ops["vd"][b, hk]) / (p_scale * ls[:, None])
            else:
                O[b, h] = (E @ v_exact[b, hk]) / ls[:, None]
            with np.errstate(divide="ignore"):
                L[b, h] = np.where(empty, -np.inf, m + np.log(ls) + scale * ops["qk"][b, h, idx])
            O[b, h][empty] = 0.0
    return O, L


def sage8_attention_fp64(q_bits, k_bits, v_bits, causal: bool, scale: float, rows=None,
                         p_scale: float = E4M3_MAX):
    """Quantised attention with every quantised operand taken from the steps
    above and every other operation in float64; P is encoded as
    e4m3(p * p_scale) relative to the exact row maximum (p_scale = 448: the
    largest weight encodes to the e4m3 maximum). Returns (O, LSE) float64 like
    ``attention_fp64`` (causal mask bottom-right aligned; a row that sees no
    key gets O = 0, LSE = -inf).

    This is the 8-bit method's own result without online rescaling; the GPU's
    8-bit path encodes P relative to a running (lagging) maximum, so the two
    agree only within the quantisation error, not bit for bit.
    """
    ops = quantised_operands(q_bits, k_bits, v_bits, "int8")
    return _one_shot(ops, None, causal, scale, rows, True, p_scale)


def fp8qk_attention_fp64(q_bits, k_bits, v_bits, causal: bool, scale: float, rows=None,
                         p_scale: float = E4M3_MAX):
    """The FP8-Q K^T variant as a one-shot computation: e4m3 Q and K with one
    scale per 128-token block and no smoothing, P and V as in
    ``sage8_attention_fp64`` (P encoded relative to the exact row maximum)."""
    ops = quantised_operands(q_bits, k_bits, v_bits, "fp8")
    return _one_shot(ops, None, causal, scale, rows, True, p_scale)


def quantised_scores_attention_fp64(q_bits, k_bits, v_bits, causal: bool, scale: float,
                                    qk_format: str = "int8", rows=None):
    """The exact softmax of an 8-bit method's dequantised scores, applied to the
    exact V: everything of the method except the e4m3 rounding of P and V.

    Returns (O_q, LSE_q, A) float64, where A = sum_j P_q[i, j] |V[j, c]| (the
    P_q-weighted magnitudes that bound the effect of rounding P and V
    elementwise). Used to split an 8-bit result's error into the part the
    scores carry (computed here exactly) and the part P and V rounding adds
    (bounded elementwise).
    """
    ops = quantised_operands(q_bits, k_bits, v_bits, qk_format)
    vx = widen_bf16(v_bits)
    O, L = _one_shot(ops, vx, causal, scale, rows, False, E4M3_MAX)
    A, _ = _one_shot(ops, np.abs(vx), causal, scale, rows, False, E4M3_MAX)
    return O, L, A
