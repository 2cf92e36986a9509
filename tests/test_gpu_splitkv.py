"""GPU parity of the key-range partials (attn_fwd_partial), their merge
(attn_merge_partials) and the split-key forward (attn_fwd_splitkv) against the
fp64 oracle (oracle.partial, oracle.attention).

Tolerances: the partials and the split-key forward carry the bf16 path's
(max |dO| <= 1e-2, mean |dO| <= 1e-3, max |dLSE| <= 1e-3; P is rounded to
bf16 for the P V product either way). The merge kernel alone works on fp32
inputs in fp32 and rounds O to bf16 once: |dO| <= 2^-8 |O| + 1e-5 (one bf16
rounding plus fp32 sums over a few parts), |dLSE| <= 1e-5 (1 + |LSE|).
A row with no visible key must give exactly O = 0 and LSE = -inf.
"""
import math

import numpy as np
import pytest
import torch

import exact_attention_134_b200 as attn
import oracle
from synthetic import bf16_bits, make_qkv, sample_rows

pytestmark = pytest.mark.gpu

MAX_TOL, MEAN_TOL, LSE_TOL = 1e-2, 1e-3, 1e-3


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    attn.lib()


def _status_ok():
    st, where = attn.get_status()
    assert st == 0, f"device status {st} at {where:#x}"


def _check(o, lse, O, L):
    o = o.float().cpu().numpy().astype(np.float64)
    lse = lse.cpu().numpy().astype(np.float64)
    empty = np.isinf(L)
    assert np.array_equal(np.isinf(lse), empty) and np.all(lse[empty] < 0)
    assert not o[empty].any()
    d = np.abs(o - O)
    dl = np.abs(lse[~empty] - L[~empty])
    assert d.max() <= MAX_TOL and d.mean() <= MEAN_TOL, (d.max(), d.mean())
    assert dl.size == 0 or dl.max() <= LSE_TOL, dl.max()


PARTIAL = [
    # B, Hq, Hkv, Nq, keys before the range, keys in it, keys after it, d, causal
    (1, 2, 2, 300, 0, 300, 0, 128, True),       # the whole sequence: attn_fwd's mask
    (1, 4, 2, 200, 150, 333, 500, 128, True),   # a middle range: many rows see none of it
    (2, 2, 1, 129, 64, 700, 0, 64, True),       # the last range of a prefill with a cache
    (1, 2, 2, 77, 1000, 260, 37, 96, True),
    (1, 4, 4, 256, 256, 512, 256, 128, False),
    (1, 4, 2, 100, 300, 500, 200, 128, True),   # head pairs (Nq <= 128, even group)
]


@pytest.mark.parametrize("num_splits", [1, 3])
@pytest.mark.parametrize("case", PARTIAL, ids=[str(c) for c in PARTIAL])
def test_partial_matches_oracle(case, num_splits):
    """num_splits = 1: one launch (attn_fwd_partial); 3: the range's keys in
    up to three sub-ranges merged on the device (attn_fwd_partial_splitkv)."""
    B, Hq, Hkv, Nq, lo, n, tail, d, causal = case
    q, k, v = make_qkv(B, Hq, Hkv, Nq, lo + n + tail, d, seed=sum(case))
    scale = 1 / math.sqrt(d)
    ks, vs = k[:, :, lo:lo + n].contiguous(), v[:, :, lo:lo + n].contiguous()
    o, lse = attn.attn_fwd_partial(q.cuda(), ks.cuda(), vs.cuda(), causal=causal, kv_tail=tail,
                                   num_splits=num_splits)
    _status_ok()
    assert o.dtype == torch.float32
    O, L = oracle.attention_partial_fp64(bf16_bits(q), bf16_bits(k), bf16_bits(v), lo, lo + n,
                                         causal, scale)
    _check(o, lse, O, L)


@pytest.mark.parametrize("d", [64, 96, 128, 256])
def test_merge_kernel_matches_oracle_merge(d):
    g = torch.Generator().manual_seed(d)
    S, B, Hq, Nq = 5, 2, 3, 77
    o_parts = torch.randn((S, B, Hq, Nq, d), generator=g)
    lse_parts = 4 * torch.randn((S, B, Hq, Nq), generator=g)
    lse_parts[1, :, :, ::3] = -math.inf                  # parts that saw no key
    lse_parts[:, 1, 2, 5:9] = -math.inf                  # rows that saw no key at all
    o_parts[:, 1, 2, 5:9] = 0
    o, lse = attn.merge_partials(o_parts.cuda(), lse_parts.cuda())
    _status_ok()
    O, L = oracle.merge_partials_fp64(o_parts.double().numpy(), lse_parts.double().numpy())
    og = o.float().cpu().numpy().astype(np.float64)
    lg = lse.cpu().numpy().astype(np.float64)
    empty = np.isinf(L)
    assert empty.sum() == 4 * 1 and np.array_equal(np.isinf(lg), empty)
    assert not og[empty].any()
    assert np.all(np.abs(og - O) <= 2.0 ** -8 * np.abs(O) + 1e-5)
    assert np.all(np.abs(lg[~empty] - L[~empty]) <= 1e-5 * (1 + np.abs(L[~empty])))


SPLIT = [
    # B, Hq, Hkv, Nq, Nkv, d, causal, num_splits (0 = automatic)
    (1, 4, 2, 128, 4096, 128, True, 0),
    (1, 4, 2, 100, 3000, 128, False, 3),
    (2, 8, 1, 37, 2000, 64, True, 7),
    (1, 2, 2, 300, 1000, 96, True, 2),
    (1, 2, 2, 513, 513, 128, True, 4),      # square causal: ranges past a row's diagonal
    (1, 2, 2, 1, 777, 128, True, 0),         # one query row (decode)
    (1, 4, 2, 64, 1500, 96, True, 3),        # head pairs, d = 96
]


@pytest.mark.parametrize("case", SPLIT, ids=[str(c) for c in SPLIT])
def test_splitkv_matches_oracle(case):
    B, Hq, Hkv, Nq, Nkv, d, causal, S = case
    q, k, v = make_qkv(B, Hq, Hkv, Nq, Nkv, d, seed=sum(case[:6]))
    assert attn.splitkv_num_splits(B, Hq, Hkv, Nq, Nkv, d, S) > 1
    o, lse = attn.attn_fwd_splitkv(q.cuda(), k.cuda(), v.cuda(), causal=causal, num_splits=S)
    _status_ok()
    assert o.dtype == torch.bfloat16
    O, L = oracle.attention_fp64(bf16_bits(q), bf16_bits(k), bf16_bits(v), causal, 1 / math.sqrt(d))
    _check(o, lse, O, L)


def test_splitkv_one_range_is_attn_fwd():
    q, k, v = make_qkv(1, 4, 2, 300, 700, 128, seed=5)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o1, l1 = attn.attn_fwd_splitkv(qc, kc, vc, causal=True, num_splits=1)
    o2, l2 = attn.attn_fwd(qc, kc, vc, causal=True)
    _status_ok()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_two_shards_merged_match_oracle():
    """The key-sharded forward on one GPU: two ranges computed as separate
    partials (the first with the second's keys as its causal tail), stacked
    as an all-gather would, merged."""
    B, Hq, Hkv, Nq, Nkv, d = 1, 4, 2, 256, 1500, 128
    q, k, v = make_qkv(B, Hq, Hkv, Nq, Nkv, d, seed=77)
    from exact_attention_134_b200.kv_shard import shard_bounds
    parts = []
    for r in range(2):
        lo, hi = shard_bounds(Nkv, 2, r)
        parts.append(attn.attn_fwd_partial(q.cuda(), k[:, :, lo:hi].contiguous().cuda(),
                                           v[:, :, lo:hi].contiguous().cuda(), causal=True,
                                           kv_tail=Nkv - hi))
    o, lse = attn.merge_partials(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]))
    _status_ok()
    O, L = oracle.attention_fp64(bf16_bits(q), bf16_bits(k), bf16_bits(v), True, 1 / math.sqrt(d))
    _check(o, lse, O, L)


def test_splitkv_long_cache_sampled_rows():
    """The bench's long-cache shape (B=1, Hq=32, Hkv=8, 128 query rows, 128k
    keys, d=128, automatic ranges), checked on 8 sampled rows per head."""
    from synthetic import Workload
    w = Workload("kvcache", 1, 32, 8, 128, 131072, 128, False, 1010)
    q, k, v = make_qkv(w.B, w.Hq, w.Hkv, w.Nq, w.Nkv, w.d, w.seed)
    o, lse = attn.attn_fwd_splitkv(q.cuda(), k.cuda(), v.cuda(), causal=False)
    _status_ok()
    rows = sample_rows(w, 8)
    O, L = oracle.attention_fp64(bf16_bits(q), bf16_bits(k), bf16_bits(v), False, w.scale, rows=rows)
    og = np.take_along_axis(o.float().cpu().numpy().astype(np.float64), rows[..., None], axis=2)
    lg = np.take_along_axis(lse.cpu().numpy().astype(np.float64), rows, axis=2)
    d = np.abs(og - O)
    assert d.max() <= MAX_TOL and d.mean() <= MEAN_TOL and np.abs(lg - L).max() <= LSE_TOL


def test_packed_merge_equals_stacked_merge():
    """merge_partials_packed over parts packed as one all-gather lays them out
    (O then LSE per part, padded) is bit-identical to merge_partials over the
    same parts stacked, with a part that has -inf rows."""
    B, Hq, Hkv, Nq, Nkv, d = 1, 4, 2, 400, 900, 128  # rows 0..99 see none of the last range
    q, k, v = make_qkv(B, Hq, Hkv, Nq, Nkv, d, seed=13)
    from exact_attention_134_b200.kv_shard import shard_bounds
    parts = []
    for r in range(3):
        lo, hi = shard_bounds(Nkv, 3, r)
        parts.append(attn.attn_fwd_partial(q.cuda(), k[:, :, lo:hi].contiguous().cuda(),
                                           v[:, :, lo:hi].contiguous().cuda(), causal=True,
                                           kv_tail=Nkv - hi))
    o_st, l_st = attn.merge_partials(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]))
    rows = B * Hq * Nq
    stride = attn.partial_packed_floats(B, Hq, Nq, d)
    assert stride % 4 == 0 and stride >= rows * (d + 1)
    packed = torch.full((3, stride), float("nan"), dtype=torch.float32, device="cuda")
    for i, (o, l) in enumerate(parts):
        packed[i, :rows * d] = o.reshape(-1)
        packed[i, rows * d:rows * d + rows] = l.reshape(-1)
    o_pk, l_pk = attn.merge_partials_packed(packed, B, Hq, Nq, d)
    _status_ok()
    assert torch.isinf(parts[2][1]).any()
    assert torch.equal(o_pk, o_st) and torch.equal(l_pk, l_st)


def test_partial_split_long_range_sampled_rows():
    """Two halves of the long-cache shape's keys (causal, the first half with the
    second as its tail), each an automatically split partial (many sub-ranges
    merged on the device in fp32), then merged: 8 sampled rows per head
    against the full oracle."""
    from synthetic import Workload
    w = Workload("kvcache_causal", 1, 32, 8, 128, 131072, 128, True, 1011)
    q, k, v = make_qkv(w.B, w.Hq, w.Hkv, w.Nq, w.Nkv, w.d, w.seed)
    qc = q.cuda()
    half = w.Nkv // 2
    assert attn.splitkv_num_splits(w.B, w.Hq, w.Hkv, w.Nq, half, w.d) > 1
    parts = [attn.attn_fwd_partial(qc, k[:, :, lo:lo + half].contiguous().cuda(),
                                   v[:, :, lo:lo + half].contiguous().cuda(), causal=True,
                                   kv_tail=w.Nkv - lo - half)
             for lo in (0, half)]
    o, lse = attn.merge_partials(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]))
    _status_ok()
    rows = sample_rows(w, 8)
    O, L = oracle.attention_fp64(bf16_bits(q), bf16_bits(k), bf16_bits(v), True, w.scale, rows=rows)
    og = np.take_along_axis(o.float().cpu().numpy().astype(np.float64), rows[..., None], axis=2)
    lg = np.take_along_axis(lse.cpu().numpy().astype(np.float64), rows, axis=2)
    d = np.abs(og - O)
    assert d.max() <= MAX_TOL and d.mean() <= MEAN_TOL and np.abs(lg - L).max() <= LSE_TOL


def test_kv_sharded_module_single_rank_nccl():
    """kv_shard.attention_kv_sharded through its default path (attn_fwd_partial,
    an NCCL all-gather, merge_partials) in a one-rank process group: the
    product code of the key-sharded forward on the GPU; its multi-rank host
    logic is tested with gloo ranks on the CPU."""
    import socket
    import torch.distributed as dist
    from exact_attention_134_b200.kv_shard import attention_kv_sharded
    if dist.is_initialized():
        pytest.skip("a process group already exists")
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device("cuda:0"))
    try:
        B, Hq, Hkv, Nq, Nkv, d = 1, 4, 2, 200, 900, 128
        q, k, v = make_qkv(B, Hq, Hkv, Nq, Nkv, d, seed=91)
        o, lse = attention_kv_sharded(q.cuda(), k.cuda(), v.cuda(), Nkv, causal=True)
        _status_ok()
        O, L = oracle.attention_fp64(bf16_bits(q), bf16_bits(k), bf16_bits(v), True, 1 / math.sqrt(d))
        _check(o, lse, O, L)
    finally:
        dist.destroy_process_group()
