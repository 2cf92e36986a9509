"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Tolerances (bf16 path, N(0,1)-scale inputs): max |dO| <= 1e-2, mean |dO| <=
1e-3, max |dLSE| <= 1e-3, element by element against the oracle on the same
seeded bf16 inputs. Small shapes are compared on every output; the large
workloads on a seeded subset of query rows per (batch, head) that always
includes the first and last row.
"""
import math

import numpy as np
import pytest
import torch

import exact_attention_134_b200 as attn
import oracle
from synthetic import WORKLOADS, bf16_bits, make_qkv, sample_rows

pytestmark = pytest.mark.gpu

MAX_TOL, MEAN_TOL, LSE_TOL = 1e-2, 1e-3, 1e-3


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    attn.lib()


def _run(q, k, v, causal, scale=None):
    o, lse = attn.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, scale=scale)
    st, where = attn.get_status()
    assert st == 0, f"device status {st} at {where:#x}"
    return o.cpu(), lse.cpu()


def _compare(o, lse, O, L, rows=None):
    og = o.float().numpy().astype(np.float64)
    lg = lse.numpy().astype(np.float64)
    if rows is not None:
        og = np.take_along_axis(og, rows[..., None], axis=2)
        lg = np.take_along_axis(lg, rows, axis=2)
    assert np.all(np.isfinite(og)) and np.all(np.isfinite(lg))
    d = np.abs(og - O)
    dl = np.abs(lg - L)
    return d.max(), d.mean(), dl.max()


def _check(B, Hq, Hkv, Nq, Nkv, d, causal, seed, dist="normal", n_rows=None):
    q, k, v = make_qkv(B, Hq, Hkv, Nq, Nkv, d, seed, dist)
    scale = 1.0 / math.sqrt(d)
    o, lse = _run(q, k, v, causal)
    rows = None
    if n_rows:
        from synthetic import Workload
        rows = sample_rows(Workload("t", B, Hq, Hkv, Nq, Nkv, d, causal, seed), n_rows)
    O, L = oracle.attention_fp64(bf16_bits(q), bf16_bits(k), bf16_bits(v), causal, scale, rows=rows)
    mx, mean, dl = _compare(o, lse, O, L, rows)
    assert mx <= MAX_TOL and mean <= MEAN_TOL and dl <= LSE_TOL, (mx, mean, dl)
    return mx, mean, dl


@pytest.mark.slow
@pytest.mark.parametrize("name", ["outlier_8k_causal", "outlier_8k_full"])
def test_large_workloads_every_row(name):
    """Every row of every (batch, head) of the 8k outlier workloads against the
    fp64 oracle (one (batch, head) per worker process)."""
    from tests.oracle_pool import attention_fp64_parallel
    w = WORKLOADS[name]
    q, k, v = make_qkv(w.B, w.Hq, w.Hkv, w.Nq, w.Nkv, w.d, w.seed, w.dist)
    o, lse = _run(q, k, v, w.causal)
    O, L = attention_fp64_parallel(bf16_bits(q), bf16_bits(k), bf16_bits(v), w.causal, w.scale)
    mx, mean, dl = _compare(o, lse, O, L)
    assert mx <= MAX_TOL and mean <= MEAN_TOL and dl <= LSE_TOL, (mx, mean, dl)


SMALL = [
    # B, Hq, Hkv, Nq, Nkv, d, causal
    (1, 2, 2, 256, 256, 64, False),
    (1, 2, 2, 256, 256, 128, True),
    (1, 1, 1, 1, 1, 64, False),
    (1, 1, 1, 1, 1, 128, True),
    (1, 2, 2, 17, 17, 128, True),
    (1, 2, 1, 127, 127, 64, True),
    (2, 2, 2, 129, 129, 128, False),
    (1, 4, 2, 255, 255, 128, True),
    (1, 4, 4, 257, 257, 64, True),
    (1, 2, 2, 300, 300, 128, False),
    (1, 8, 1, 513, 513, 128, True),
    (2, 8, 2, 1000, 1000, 64, True),
    (1, 4, 2, 100, 333, 128, False),
    (2, 4, 1, 512, 64, 64, False),
    (1, 2, 2, 640, 1900, 128, False),
    # Nq <= 128 with an even GQA group: two query heads per CTA
    (2, 8, 2, 128, 1000, 128, True),
    (1, 4, 2, 1, 513, 64, False),
    (1, 6, 3, 77, 77, 96, True),
    (1, 8, 1, 100, 300, 64, True),
    (1, 16, 2, 1024, 1024, 128, True),
    # head dim 96: three 32-column boxes per row
    (1, 2, 2, 256, 256, 96, False),
    (1, 4, 2, 300, 300, 96, True),
    (2, 8, 1, 513, 513, 96, True),
    (1, 2, 2, 100, 777, 96, False),
    (1, 2, 2, 200, 650, 96, True),
    # head dim 256: one query tile per CTA, Q held in TMEM, 64-key K/V tiles
    (1, 2, 2, 256, 256, 256, False),
    (1, 1, 1, 1, 1, 256, True),
    (1, 4, 2, 300, 300, 256, True),
    (2, 2, 1, 129, 700, 256, False),
    (1, 4, 4, 1000, 1000, 256, True),
    (1, 2, 2, 64, 65, 256, True),
]


@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "x".join(map(str, s)))
def test_small_shapes(shape):
    _check(*shape, seed=sum(shape) + 17)


def test_tiny_workload():
    w = WORKLOADS["tiny_256_d64"]
    _check(w.B, w.Hq, w.Hkv, w.Nq, w.Nkv, w.d, w.causal, w.seed)


def test_causal_2k_workload():
    w = WORKLOADS["causal_2k_d128"]
    _check(w.B, w.Hq, w.Hkv, w.Nq, w.Nkv, w.d, w.causal, w.seed)


@pytest.mark.parametrize("name", ["outlier_8k_causal", "outlier_8k_full", "gqa_32k_d128", "gqa_32k_d64",
                                  "d256_8k_causal"])
def test_large_workloads_sampled_rows(name):
    w = WORKLOADS[name]
    _check(w.B, w.Hq, w.Hkv, w.Nq, w.Nkv, w.d, w.causal, w.seed, w.dist, n_rows=w.oracle_rows)


def test_causal_row_zero_is_v0_bit_exact():
    q, k, v = make_qkv(1, 4, 2, 384, 384, 128, seed=5)
    o, lse = _run(q, k, v, True)
    g = 2
    for h in range(4):
        assert torch.equal(o[0, h, 0], v[0, h // g, 0])
    ql, kl = q.double(), k.double()
    ref = torch.einsum("hd,hd->h", ql[0, :, 0], kl[0, [0, 0, 1, 1], 0]) / math.sqrt(128)
    assert torch.max(torch.abs(lse[0, :, 0].double() - ref)) < 1e-4


def test_deterministic():
    q, k, v = make_qkv(1, 4, 4, 700, 700, 128, seed=6)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o1, l1 = attn.attn_fwd(qc, kc, vc, causal=True)
    o2, l2 = attn.attn_fwd(qc, kc, vc, causal=True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("path,d,causal,N", [
    ("fwd", 64, False, 200), ("fwd", 96, True, 333), ("fwd", 128, True, 300), ("fwd", 256, True, 130),
    ("fwd_pair", 128, True, 100), ("q8", 128, True, 300), ("fp8", 64, False, 257),
    ("partial_split", 128, True, 100),
])
def test_no_writes_outside_outputs(path, d, causal, N):
    """Canary values around O and LSE stay untouched, and every element of O
    and LSE is written, for each output epilogue (TMA box store, row stores at
    d = 96 and 256, head pairs, 8-bit, split-key partial in fp32)."""
    B, Hq, Hkv = 1, 4, 2
    Nkv = 2000 if path == "partial_split" else N
    q, k, v = make_qkv(B, Hq, Hkv, N, Nkv, d, seed=8 + d + N)
    pad = 4096
    odt = torch.float32 if path == "partial_split" else torch.bfloat16
    n_o, n_l = B * Hq * N * d, B * Hq * N
    obuf = torch.full((n_o + 2 * pad,), 7.0, dtype=odt, device="cuda")
    lbuf = torch.full((n_l + 2 * pad,), 7.0, dtype=torch.float32, device="cuda")
    o = obuf[pad:pad + n_o].view(B, Hq, N, d)
    lse = lbuf[pad:pad + n_l].view(B, Hq, N)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    if path in ("fwd", "fwd_pair"):
        attn.attn_fwd(qc, kc, vc, causal=causal, out=o, lse=lse)
    elif path in ("q8", "fp8"):
        attn.attn_fwd_q8(qc, kc, vc, causal=causal, out=o, lse=lse,
                         qk_format="int8" if path == "q8" else "fp8")
    else:
        attn.attn_fwd_partial(qc, kc, vc, causal=causal, kv_tail=50, out=o, lse=lse, num_splits=4)
    torch.cuda.synchronize()
    assert attn.get_status()[0] == 0
    assert torch.all(obuf[:pad] == 7.0) and torch.all(obuf[-pad:] == 7.0)
    assert torch.all(lbuf[:pad] == 7.0) and torch.all(lbuf[-pad:] == 7.0)
    assert not torch.any(o == 7.0) and not torch.any(lse == 7.0)


def test_non_default_scale_and_stream():
    # scale 0.3 (3.4x 1/sqrt(128)) makes rows peaky: a few keys dominate, so the
    # bf16 rounding of P (relative error up to 2^-8 per weight) no longer
    # averages out. The bound per output is that rounding applied to every
    # term, 2^-8 * sum_j P_ij |V_jc|, plus half a bf16 ulp for rounding O.
    q, k, v = make_qkv(1, 2, 2, 333, 333, 128, seed=9)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o, lse = attn.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True, scale=0.3)
    s.synchronize()
    O, L, P = oracle.attention_fp64(bf16_bits(q), bf16_bits(k), bf16_bits(v), True, 0.3, return_p=True)
    og = o.cpu().float().numpy().astype(np.float64)
    vabs = np.abs(oracle.widen_bf16(bf16_bits(v)))
    p_bound = 2.0 ** -8 * np.einsum("bhij,bhjc->bhic", P, vabs)
    half_ulp = 2.0 ** (np.floor(np.log2(np.abs(O) + p_bound + 1e-30)) - 8)
    assert np.all(np.abs(og - O) <= p_bound + half_ulp + 1e-4)
    assert np.abs(og - O).mean() <= MEAN_TOL
    assert np.abs(lse.cpu().numpy() - L).max() <= LSE_TOL


def test_host_buffer_entry_point():
    q, k, v = make_qkv(2, 4, 2, 300, 300, 64, seed=10)
    o, lse = attn.attn_fwd_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), causal=True)
    O, L = oracle.attention_fp64(bf16_bits(q), bf16_bits(k), bf16_bits(v), True, 1 / 8)
    mx, mean, dl = _compare(o, lse, O, L)
    assert mx <= MAX_TOL and mean <= MEAN_TOL and dl <= LSE_TOL


def test_host_entry_pipelined_chunks_match_device_entry():
    """attn_fwd_host splits the work into chunks of kv-head groups (8 here,
    GQA 4:1, two batch entries) and must give exactly attn_fwd's result."""
    q, k, v = make_qkv(2, 16, 4, 700, 700, 128, seed=12)
    o_h, l_h = attn.attn_fwd_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), causal=True)
    o_d, l_d = attn.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True)
    assert torch.equal(o_h, o_d.cpu()) and torch.equal(l_h, l_d.cpu())
    q1, k1, v1 = make_qkv(1, 3, 1, 129, 300, 256, seed=13)  # one group: one chunk, d = 256
    o_h, l_h = attn.attn_fwd_host(q1.pin_memory(), k1.pin_memory(), v1.pin_memory(), causal=False)
    o_d, l_d = attn.attn_fwd(q1.cuda(), k1.cuda(), v1.cuda(), causal=False)
    assert torch.equal(o_h, o_d.cpu()) and torch.equal(l_h, l_d.cpu())
