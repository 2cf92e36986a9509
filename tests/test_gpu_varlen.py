"""GPU parity for causal attention with Nq != Nkv (mask aligned to the bottom
right) and for packed variable-length sequences, against the fp64 oracle.

Same tolerances as the dense bf16 path (max |dO| <= 1e-2, mean <= 1e-3,
|dLSE| <= 1e-3); rows that see no key must give O = 0 and LSE = -inf exactly.
"""
import math

import numpy as np
import pytest
import torch

import exact_attention_134_b200 as attn
import oracle
from synthetic import bf16_bits, make_qkv

pytestmark = pytest.mark.gpu

MAX_TOL, MEAN_TOL, LSE_TOL = 1e-2, 1e-3, 1e-3


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    attn.lib()


def _check(og, lg, O, L, packed=False):
    """O-like arrays [..., rows, d] (dense) or [rows, H, d] (packed); LSE
    [..., rows] (dense) or [H, rows] (packed)."""
    og = og.astype(np.float64)
    lg = lg.astype(np.float64)
    empty = np.isneginf(L)
    assert np.array_equal(np.isneginf(lg), empty)
    empty_o = empty.T if packed else empty  # the row mask in O's layout
    assert np.all(og[empty_o] == 0.0)
    fin = ~empty_o
    d = np.abs(og - O)[fin]
    if d.size:
        assert d.max() <= MAX_TOL and d.mean() <= MEAN_TOL, (d.max(), d.mean())
        assert np.abs(lg[~empty] - L[~empty]).max() <= LSE_TOL


@pytest.mark.parametrize("shape", [
    (1, 4, 2, 100, 333, 128), (1, 2, 2, 300, 1000, 64), (2, 4, 4, 513, 1537, 128),
    (1, 2, 2, 1, 700, 128), (1, 2, 2, 300, 100, 128), (1, 4, 1, 257, 129, 64),
    (1, 2, 2, 500, 130, 256), (1, 4, 2, 100, 333, 256),
])
def test_causal_bottom_right_dense(shape):
    B, Hq, Hkv, Nq, Nkv, d = shape
    q, k, v = make_qkv(B, Hq, Hkv, Nq, Nkv, d, seed=sum(shape))
    o, lse = attn.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True)
    assert attn.get_status()[0] == 0
    O, L = oracle.attention_fp64(bf16_bits(q), bf16_bits(k), bf16_bits(v), True, 1 / math.sqrt(d))
    _check(o.cpu().float().numpy(), lse.cpu().numpy(), O, L)


def test_prefill_with_cache_matches_tail_of_full_causal():
    q, k, v = make_qkv(1, 4, 2, 1024, 1024, 128, seed=41)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o_full, l_full = attn.attn_fwd(qc, kc, vc, causal=True)
    o_tail, l_tail = attn.attn_fwd(qc[:, :, -300:].contiguous(), kc, vc, causal=True)
    # same keys, same visible sets; rows are computed by different tiles, so
    # they agree to the kernel's rounding, not bit for bit
    assert (o_tail.float() - o_full[:, :, -300:].float()).abs().max().item() <= 2e-2
    assert (l_tail - l_full[:, :, -300:]).abs().max().item() <= 1e-3


def _packed(lens_q, lens_k, Hq, Hkv, d, seed):
    g = torch.Generator().manual_seed(seed)
    tq, tk = sum(lens_q), sum(lens_k)
    q = torch.randn((tq, Hq, d), generator=g).to(torch.bfloat16)
    k = torch.randn((tk, Hkv, d), generator=g).to(torch.bfloat16)
    v = torch.randn((tk, Hkv, d), generator=g).to(torch.bfloat16)
    cq = torch.tensor(np.concatenate([[0], np.cumsum(lens_q)]), dtype=torch.int32)
    ck = torch.tensor(np.concatenate([[0], np.cumsum(lens_k)]), dtype=torch.int32)
    return q, k, v, cq, ck


VARLEN = [
    ([1, 17, 128, 129, 300, 1000], None, 4, 2, 128, True),
    ([1, 17, 128, 129, 300, 1000], None, 4, 2, 64, False),
    ([64, 200, 513], [1000, 200, 700], 8, 2, 128, True),     # prefill with a cache
    ([300, 50, 5], [100, 0, 5], 2, 2, 128, True),            # Lq > Lk, an empty key set
    ([700, 0, 33], [700, 40, 33], 4, 4, 64, True),           # an empty query sequence
    ([129, 64, 300], [129, 500, 300], 4, 2, 96, True),       # head dim 96
    ([1, 17, 128, 129, 300], None, 4, 2, 256, True),         # head dim 256
    ([64, 200, 513], [1000, 200, 700], 4, 2, 256, True),     # head dim 256, prefill with a cache
    ([300, 50, 5], [100, 0, 5], 2, 2, 256, True),            # head dim 256, Lq > Lk, an empty key set
    ([700, 0, 33], [700, 40, 33], 2, 2, 256, False),         # head dim 256, an empty query sequence
    # one long prompt among many tiny and empty ones: work items map to units
    # across sequence boundaries, with empty items between them
    ([700] + [0, 1, 2, 3, 5, 1, 0, 4] * 5 + [257], None, 4, 2, 128, True),
    ([3, 0, 300] + [1, 0, 2] * 6 + [129], None, 2, 1, 256, True),
]


@pytest.mark.parametrize("case", VARLEN, ids=range(len(VARLEN)))
def test_varlen_matches_oracle(case):
    lens_q, lens_k, Hq, Hkv, d, causal = case
    lens_k = lens_k or lens_q
    q, k, v, cq, ck = _packed(lens_q, lens_k, Hq, Hkv, d, seed=len(lens_q) + d)
    o, lse = attn.attn_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), cq.cuda(), ck.cuda(), max(lens_q),
                                  causal=causal)
    assert attn.get_status()[0] == 0
    O, L = oracle.attention_varlen_fp64(bf16_bits(q), bf16_bits(k), bf16_bits(v), cq.numpy(),
                                        ck.numpy(), causal, 1 / math.sqrt(d))
    _check(o.cpu().float().numpy(), lse.cpu().numpy(), O, L, packed=True)


@pytest.mark.parametrize("d", [128, 256])
def test_varlen_equal_lengths_is_bit_identical_to_dense(d):
    B, H, N = 3, 4, 300
    q, k, v = make_qkv(B, H, H, N, N, d, seed=8)
    o_d, l_d = attn.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True)
    pack = lambda x: x.permute(0, 2, 1, 3).reshape(B * N, H, d).contiguous().cuda()  # noqa: E731
    cu = torch.arange(0, (B + 1) * N, N, dtype=torch.int32).cuda()
    o_v, l_v = attn.attn_fwd_varlen(pack(q), pack(k), pack(v), cu, cu, N, causal=True)
    assert torch.equal(o_v, o_d.permute(0, 2, 1, 3).reshape(B * N, H, d))
    assert torch.equal(l_v, l_d.permute(1, 0, 2).reshape(H, B * N))


@pytest.mark.parametrize("d", [64, 256])
def test_varlen_writes_only_its_rows(d):
    lens = [100, 0, 37]
    q, k, v, cq, ck = _packed(lens, lens, 2, 2, d, seed=3)
    pad = 4096
    obuf = torch.full((q.numel() + 2 * pad,), 9.0, dtype=torch.bfloat16, device="cuda")
    o = obuf[pad:pad + q.numel()].view(q.shape)
    attn.attn_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), cq.cuda(), ck.cuda(), 100, causal=True, out=o)
    torch.cuda.synchronize()
    assert torch.all(obuf[:pad] == 9.0) and torch.all(obuf[-pad:] == 9.0)
    assert torch.all(o != 9.0)


def test_q8_causal_bottom_right():
    B, Hq, Hkv, Nq, Nkv, d = 1, 4, 2, 256, 900, 128
    q, k, v = make_qkv(B, Hq, Hkv, Nq, Nkv, d, seed=77, dist="outlier_k")
    o, lse = attn.attn_fwd_q8(q.cuda(), k.cuda(), v.cuda(), causal=True)
    assert attn.get_status()[0] == 0
    O, L = oracle.attention_fp64(bf16_bits(q), bf16_bits(k), bf16_bits(v), True, 1 / math.sqrt(d))
    og = o.cpu().float().numpy().astype(np.float64)
    cos = (og * O).sum() / math.sqrt((og * og).sum() * (O * O).sum())
    assert cos >= 0.999
    # every row sees >= 645 keys here, so the 5e-2 bound applies to all
    assert np.abs(og - O).max() <= 5e-2
    assert np.abs(lse.cpu().numpy() - L).max() <= 5e-2
