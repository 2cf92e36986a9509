"""Pins for the 8-bit (SageAttention-style) oracle steps (CPU only).

The encoders are pinned to the number formats' definitions and to torch's own
float8_e4m3fn casts; the INT8 block quantiser to its error bound and special
cases; the smoothing step to the shift invariance the SageAttention page
states; the one-shot quantised attention to the exact oracle within the 8-bit
tolerance.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import quant8 as q8
from synthetic import bf16_bits, make_qkv


def test_e4m3_decode_matches_torch_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = q8.e4m3_decode(codes)
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(mine))
    assert np.array_equal(ref[~nan], mine[~nan])


def test_e4m3_roundtrip_every_finite_code():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    back = q8.e4m3_encode(q8.e4m3_decode(codes).astype(np.float32))
    # +0 and -0 both decode to zero; the sign bit is kept
    assert np.array_equal(back, codes)


def test_e4m3_encode_matches_torch_cast_in_range():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.normal(size=20000) * s for s in (1e-3, 0.05, 1.0, 30.0, 150.0)])
    x = np.clip(x, -448, 448).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q8.e4m3_encode(x), ref)


def test_e4m3_ties_to_even_and_saturation():
    # 1 + 1/16 lies halfway between 1.0 (mantissa 0) and 1.125 (mantissa 1): even -> 1.0
    assert q8.e4m3_decode(q8.e4m3_encode(np.float32(1.0625))) == 1.0
    # 1 + 3/16 lies halfway between 1.125 (odd) and 1.25 (even) -> 1.25
    assert q8.e4m3_decode(q8.e4m3_encode(np.float32(1.1875))) == 1.25
    assert q8.e4m3_decode(q8.e4m3_encode(np.float32(1e6))) == 448.0
    assert q8.e4m3_decode(q8.e4m3_encode(np.float32(-500.0))) == -448.0
    # smallest subnormal 2^-9 and half of it (a tie -> even -> 0)
    assert q8.e4m3_decode(q8.e4m3_encode(np.float32(2.0 ** -9))) == 2.0 ** -9
    assert q8.e4m3_decode(q8.e4m3_encode(np.float32(2.0 ** -10))) == 0.0


def test_int8_block_quantisation_bounds():
    rng = np.random.default_rng(1)
    x = (rng.normal(size=(2, 3, 300, 16)) * rng.uniform(0.1, 20, size=(2, 3, 1, 1))).astype(np.float32)
    x[1, 2, 128:256] = 0.0                              # an all-zero block
    codes, s = q8.quant_int8_blocks(x)
    assert codes.dtype == np.int8 and s.shape == (2, 3, 3)
    assert np.all(np.abs(codes.astype(np.int32)) <= 127)
    assert s[1, 2, 1] == 1.0 and np.all(codes[1, 2, 128:256] == 0)
    for b in range(2):
        for h in range(3):
            for i in range(3):
                blk = x[b, h, i * 128:(i + 1) * 128]
                c = codes[b, h, i * 128:(i + 1) * 128].astype(np.float64)
                if np.abs(blk).max() == 0:
                    continue
                # the largest magnitude maps to +-127
                assert np.abs(c).max() == 127
                err = np.abs(c * float(s[b, h, i]) - blk.astype(np.float64)).max()
                assert err <= 0.5 * float(s[b, h, i]) * (1 + 1e-6)


def test_k_mean_and_smoothing_shift_invariance():
    q, k, v = make_qkv(1, 2, 2, 64, 64, 8, seed=7, dist="outlier_k")
    qb, kb, vb = bf16_bits(q), bf16_bits(k), bf16_bits(v)
    kbar = q8.k_channel_mean(kb)
    assert np.allclose(kbar, oracle.widen_bf16(kb).mean(axis=2), rtol=1e-7, atol=1e-7)
    ks = q8.smooth_k(kb, kbar)
    assert np.abs(ks.astype(np.float64).mean(axis=2)).max() < 1e-5
    O, L = oracle.attention_fp64(qb, kb, vb, True, 0.3)
    O2, L2 = oracle.attention_f64(oracle.widen_bf16(qb), ks.astype(np.float64), oracle.widen_bf16(vb), True, 0.3)
    # kbar and K' are float32 (the precision the prepass stores); the exact
    # fp64 identity is pinned in test_oracle.py, here it holds to the size of
    # those float32 roundings (|dS| ~ scale * |q| * 2^-24 * |K|)
    assert np.max(np.abs(O - O2)) < 1e-6
    qk = q8.q_dot_kbar(qb, kbar, 2)
    assert np.max(np.abs(L2 + 0.3 * qk - L)) < 1e-5


def test_v_fp8_quantisation_error_bound():
    _, _, v = make_qkv(1, 1, 2, 8, 200, 16, seed=8)
    vb = bf16_bits(v)
    codes, s = q8.quant_v_fp8(vb)
    deq = q8.e4m3_decode(codes) * s[:, :, None, :]
    vf = oracle.widen_bf16(vb)
    # e4m3 relative spacing is 2^-3; half of it bounds RNE error (normal range)
    assert np.all(np.abs(deq - vf) <= np.abs(vf) * 2.0 ** -4 + s[:, :, None, :] * 2.0 ** -10)
    # the per-channel absolute maximum encodes to exactly 448 * scale
    assert np.allclose(np.abs(deq).max(axis=2), np.abs(vf).max(axis=2), rtol=1e-6, atol=0)


@pytest.mark.parametrize("dist", ["normal", "outlier_k"])
def test_sage8_one_shot_within_8bit_tolerance(dist):
    q, k, v = make_qkv(1, 2, 2, 256, 256, 64, seed=9, dist=dist)
    qb, kb, vb = bf16_bits(q), bf16_bits(k), bf16_bits(v)
    scale = 1 / math.sqrt(64)
    O, L = oracle.attention_fp64(qb, kb, vb, True, scale)
    O8, L8 = q8.sage8_attention_fp64(qb, kb, vb, True, scale)
    cos = (O * O8).sum() / math.sqrt((O * O).sum() * (O8 * O8).sum())
    assert cos >= 0.999
    # A causal row with few visible keys averages few e4m3-rounded V elements,
    # whose relative error reaches 2^-4; the 5e-2 bound holds once a row sees
    # enough keys for those errors to average out (>= 128 here) ...
    assert np.max(np.abs(O - O8)[:, :, 127:]) <= 5e-2
    # ... and every row stays within the e4m3 bound on its own V elements.
    vmax = np.abs(oracle.widen_bf16(vb)).max()
    assert np.max(np.abs(O - O8)) <= vmax * 2.0 ** -4 * 1.5
    assert np.max(np.abs(L - L8)) <= 5e-2


def test_e4m3_block_quantisation_bounds():
    rng = np.random.default_rng(2)
    x = (rng.normal(size=(1, 2, 200, 32)) * rng.uniform(0.1, 30, size=(1, 2, 1, 1))).astype(np.float32)
    x[0, 1, :128] = 0.0
    codes, s = q8.quant_e4m3_blocks(x)
    assert s[0, 1, 0] == 1.0 and np.all(codes[0, 1, :128] == 0)
    deq = q8.e4m3_decode(codes) * np.repeat(s, 128, axis=2)[:, :, :200, None]
    for h in range(2):
        for i in range(2):
            blk = x[0, h, i * 128:(i + 1) * 128]
            if np.abs(blk).max() == 0:
                continue
            # the block maximum encodes to exactly 448 * scale
            assert np.isclose(np.abs(deq[0, h, i * 128:(i + 1) * 128]).max(), np.abs(blk).max(), rtol=1e-6)
            # relative error <= 2^-4 in the normal range, plus the subnormal quantum
            err = np.abs(deq[0, h, i * 128:(i + 1) * 128] - blk)
            assert np.all(err <= np.abs(blk) * 2.0 ** -4 + float(s[0, h, i]) * 2.0 ** -10)


def test_smoothing_beats_unsmoothed_fp8_on_outlier_channels():
    # the SageAttention page's claim: outlier channels in K break a plain
    # 8-bit Q K^T; mean-centring K first makes the INT8 product accurate
    q, k, v = make_qkv(1, 2, 2, 512, 512, 128, seed=9, dist="outlier_k")
    qb, kb, vb = bf16_bits(q), bf16_bits(k), bf16_bits(v)
    sc = 1 / math.sqrt(128)
    O, L = oracle.attention_fp64(qb, kb, vb, True, sc)
    Os, Ls = q8.sage8_attention_fp64(qb, kb, vb, True, sc)
    Of, Lf = q8.fp8qk_attention_fp64(qb, kb, vb, True, sc)
    cos = lambda a: (O * a).sum() / math.sqrt((O * O).sum() * (a * a).sum())  # noqa: E731
    assert cos(Os) >= 0.999 > cos(Of)
    assert np.abs(L - Ls).max() * 5 < np.abs(L - Lf).max()
