"""GPU parity of the attention backward (attn_bwd) against the fp64 oracle.

Tolerance, derived from the kernel's arithmetic (u = 2^-8 is the unit
roundoff of bf16, whose significand has 8 bits; g_n = n * 2^-24 bounds an fp32
sum of n terms):
  * P is recomputed in fp32 from the given LSE; its relative error per row is
    eP_i = |LSE_given - LSE|_i + g_d * scale * max_j |q_i|.|k_j| + 2^-21.
  * D_i is summed in fp32 from the given bf16 O:
    eD_i = sum_c |dO_ic| |O_given - O|_ic + g_d * sum_c |dO_ic O_given,ic|.
  * dP = dO V^T in fp32: edP_ij = g_d * (|dO| |V|^T)_ij.
  * dS is rounded to bf16 once: per element its error is at most
    E_ij = (1 + u) P_ij (eP_i |dP_ij - D_i| + edP_ij + eD_i) + u |dS_ij|.
  * dV takes bf16(P):   e_dV = ((u + (1 + u) eP + g_Nq) P)^T |dO|,
    dK, dQ take bf16(dS): e_dK = scale (E^T |Q| + g_Nq |dS|^T |Q|),
                          e_dQ = scale (E |K| + g_Nkv |dS| |K|),
  and each output is rounded to bf16 once more: the bound is
  (1 + u) e + u |exact| + 1e-6.
The bounds are checked element by element; each test also checks that the
bound is far below the gradients themselves (it is not vacuous).
"""
import math

import numpy as np
import pytest
import torch

import exact_attention_134_b200 as attn
import oracle
from oracle.backward import attention_bwd_head_blocks
from synthetic import WORKLOADS, bf16_bits, make_dout, make_qkv, make_workload, sample_rows

pytestmark = pytest.mark.gpu

U = 2.0 ** -8  # bf16 unit roundoff


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    attn.lib()


def _f64(t):
    return t.detach().cpu().to(torch.float64).numpy()


class HeadRef:
    """Exact gradients and error bounds of one (batch, query head), optionally
    restricted to some query rows (dQ) and key rows (dK, dV)."""

    def __init__(self, q, k, v, do, o_in, lse_in, causal, scale, q_rows=None, kv_rows=None,
                 block_rows=2048):
        Nq, d = q.shape
        Nkv = k.shape[0]
        self.q_rows = np.arange(Nq) if q_rows is None else np.asarray(q_rows)
        self.kv_rows = np.arange(Nkv) if kv_rows is None else np.asarray(kv_rows)
        gd, gq, gk = d * 2.0 ** -24, Nq * 2.0 ** -24, Nkv * 2.0 ** -24
        kr = self.kv_rows
        self.dQ = np.zeros((len(self.q_rows), d))
        self.bQ = np.zeros((len(self.q_rows), d))
        self.dK = np.zeros((len(kr), d))
        self.bK = np.zeros((len(kr), d))
        self.dV = np.zeros((len(kr), d))
        self.bV = np.zeros((len(kr), d))
        aK, aV, aQ, aDO = np.abs(k), np.abs(v), np.abs(q), np.abs(do)
        pos = {int(r): n for n, r in enumerate(self.q_rows)}
        for blk in attention_bwd_head_blocks(q, k, v, do, causal, scale, block_rows):
            i0, i1 = blk["i0"], blk["i1"]
            P, dS, dP, D, L = blk["P"], blk["dS"], blk["dP"], blk["D"], blk["LSE"]
            fin = ~np.isinf(L)
            lse_err = np.zeros_like(L)
            lse_err[fin] = np.abs(lse_in[i0:i1][fin] - L[fin])
            eP = lse_err + gd * scale * (aQ[i0:i1] @ aK.T).max(axis=1) + 2.0 ** -21
            eD = (aDO[i0:i1] * np.abs(o_in[i0:i1] - blk["O"])).sum(1) + \
                gd * np.abs(do[i0:i1] * o_in[i0:i1]).sum(1)
            edP = gd * (aDO[i0:i1] @ aV.T)
            E = (1 + U) * P * (eP[:, None] * np.abs(dP - D[:, None]) + edP + eD[:, None]) + U * np.abs(dS)
            sel = [n for n in range(i0, i1) if n in pos]
            if sel:
                loc = np.asarray(sel) - i0
                dst = [pos[n] for n in sel]
                self.dQ[dst] = scale * (dS[loc] @ k)
                self.bQ[dst] = scale * (E[loc] @ aK + gk * (np.abs(dS[loc]) @ aK))
            self.dK += scale * (dS[:, kr].T @ q[i0:i1])
            self.bK += scale * (E[:, kr].T @ aQ[i0:i1] + gq * (np.abs(dS[:, kr]).T @ aQ[i0:i1]))
            self.dV += P[:, kr].T @ do[i0:i1]
            self.bV += ((U + (1 + U) * eP[:, None] + gq) * P[:, kr]).T @ aDO[i0:i1]
        self.bQ = (1 + U) * self.bQ + U * np.abs(self.dQ) + 1e-6


def _check(name, got, exp, bound, vacuous=0.05):
    err = np.abs(got - exp)
    worst = float((err / bound).max())
    assert np.all(err <= bound), f"{name}: max err/bound {worst:.3f}, max err {err.max():.3e}"
    # the bound itself must be small next to the gradient (not vacuous); a
    # gradient that is exactly 0 (e.g. a query seeing one key: P = 1, dS = 0)
    # has nothing to compare with
    if np.abs(exp).max() >= 1e-3:
        assert bound.max() <= vacuous * np.abs(exp).max(), (name, bound.max(), np.abs(exp).max())
    return worst


def _run_and_check(q, k, v, do, causal, scale, o_in, lse_in, heads=None, q_rows=None, kv_rows=None,
                   dq=None, dk=None, dv=None, vacuous=0.05):
    """q.. bf16 CPU tensors; o_in / lse_in the O and LSE given to the backward
    (CPU). Runs attn_bwd unless dq/dk/dv are given, then checks the listed
    (b, query head) pairs (all by default)."""
    B, Hq, Nq, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    if dq is None:
        dq, dk, dv = attn.attn_bwd(q.cuda(), k.cuda(), v.cuda(), o_in.cuda(), lse_in.cuda(), do.cuda(),
                                   causal=causal, scale=scale)
        assert attn.get_status()[0] == 0
    dq, dk, dv = _f64(dq), _f64(dk), _f64(dv)
    qf, kf, vf, dof, of = _f64(q), _f64(k), _f64(v), _f64(do), _f64(o_in)
    lf = lse_in.cpu().numpy().astype(np.float64)
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(Hq)]
    worst = 0.0
    kv_acc = {}
    for b, h in heads:
        hk = h // G
        ref = HeadRef(qf[b, h], kf[b, hk], vf[b, hk], dof[b, h], of[b, h], lf[b, h], causal, scale,
                      None if q_rows is None else q_rows[b, h], kv_rows)
        worst = max(worst, _check("dQ", dq[b, h][ref.q_rows], ref.dQ, ref.bQ, vacuous))
        acc = kv_acc.setdefault((b, hk), [0, 0, 0, 0, 0, ref.kv_rows])
        acc[0] = acc[0] + ref.dK
        acc[1] = acc[1] + ref.bK
        acc[2] = acc[2] + ref.dV
        acc[3] = acc[3] + ref.bV
        acc[4] += 1
    for (b, hk), (eK, bK, eV, bV, n, rows) in kv_acc.items():
        if n != G:
            continue  # dK/dV of a kv head are checked only when all its query heads were
        bK = (1 + U) * bK + U * np.abs(eK) + 1e-6
        bV = (1 + U) * bV + U * np.abs(eV) + 1e-6
        worst = max(worst, _check("dK", dk[b, hk][rows], eK, bK, vacuous))
        worst = max(worst, _check("dV", dv[b, hk][rows], eV, bV, vacuous))
    return worst


def _oracle_forward(q, k, v, causal, scale):
    O, L = oracle.attention_fp64(bf16_bits(q), bf16_bits(k), bf16_bits(v), causal, scale)
    return torch.from_numpy(O).to(torch.bfloat16), torch.from_numpy(L).to(torch.float32)


SHAPES = [
    # B, Hq, Hkv, Nq, Nkv, d, causal
    (1, 2, 2, 384, 384, 128, True),      # three full blocks
    (1, 4, 2, 300, 300, 64, False),      # ragged, GQA 2:1
    (2, 4, 1, 200, 700, 128, True),      # Nq < Nkv (a cache), GQA 4:1
    (1, 2, 2, 500, 130, 128, True),      # Nq > Nkv: rows that see no key
    (1, 2, 2, 1, 257, 64, False),        # one query row
    (1, 2, 2, 1000, 1000, 128, True),
    (1, 2, 2, 129, 129, 64, True),       # one row / key past a block
    (1, 2, 2, 300, 300, 96, True),       # d = 96: three 32-column boxes, 64-byte swizzle
    (2, 4, 2, 200, 450, 96, False),      # d = 96, GQA 2:1, Nq < Nkv
]


@pytest.mark.parametrize("shape", SHAPES, ids=[str(s) for s in SHAPES])
def test_bwd_matches_oracle(shape):
    B, Hq, Hkv, Nq, Nkv, d, causal = shape
    q, k, v = make_qkv(B, Hq, Hkv, Nq, Nkv, d, seed=sum(shape))
    do = make_dout(B, Hq, Nq, d, seed=sum(shape))
    scale = 1 / math.sqrt(d)
    o_in, lse_in = _oracle_forward(q, k, v, causal, scale)
    _run_and_check(q, k, v, do, causal, scale, o_in, lse_in)


def test_bwd_outlier_keys_and_scale():
    # Every row of dS sums to zero, so K's large per-channel offsets cancel in
    # the exact dQ = scale dS K, but the bf16 rounding residue of dS does not
    # cancel and is multiplied by them: the bound reaches ~26% of max |dQ|
    # here, and the guard against an empty bound is relaxed to 30%.
    q, k, v = make_qkv(1, 2, 2, 256, 256, 128, seed=5, dist="outlier_k")
    do = make_dout(1, 2, 256, 128, seed=5)
    o_in, lse_in = _oracle_forward(q, k, v, True, 0.05)
    _run_and_check(q, k, v, do, True, 0.05, o_in, lse_in, vacuous=0.3)


def test_bwd_after_gpu_forward():
    """Forward then backward on the GPU, as a training step runs them; the
    bound takes the forward's own O and LSE errors into account."""
    q, k, v = make_qkv(1, 4, 2, 1000, 1000, 128, seed=21)
    do = make_dout(1, 4, 1000, 128, seed=21)
    o, lse = attn.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True)
    _run_and_check(q, k, v, do, True, 1 / math.sqrt(128), o.cpu(), lse.cpu())


def test_bwd_repeatable_and_writes_only_outputs():
    q, k, v = make_qkv(1, 4, 2, 300, 500, 128, seed=3)
    do = make_dout(1, 4, 300, 128, seed=3)
    qc, kc, vc, dc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = attn.attn_fwd(qc, kc, vc, causal=True)
    pad = 4096
    bufs = [torch.full((t.numel() + 2 * pad,), 7.0, dtype=torch.bfloat16, device="cuda") for t in (qc, kc, vc)]
    outs = [b[pad:pad + t.numel()].view(t.shape) for b, t in zip(bufs, (qc, kc, vc))]
    dq1, dk1, dv1 = attn.attn_bwd(qc, kc, vc, o, lse, dc, causal=True, dq=outs[0], dk=outs[1], dv=outs[2])
    torch.cuda.synchronize()
    for b in bufs:
        assert torch.all(b[:pad] == 7.0) and torch.all(b[-pad:] == 7.0)
    dq2, dk2, dv2 = attn.attn_bwd(qc, kc, vc, o, lse, dc, causal=True)
    # dK, dV: fixed summation order; dQ: fp32 atomics in any order, then bf16,
    # so two runs may round to neighbouring bf16 values (one ulp <= 2u |x|)
    assert torch.equal(dk1, dk2) and torch.equal(dv1, dv2)
    assert ((dq1.float() - dq2.float()).abs() <= 2 * U * dq2.float().abs() + 1e-6).all()


def test_bwd_full_size_sampled():
    """The backward at the benchmark's size (outlier channels, 8k causal,
    B=2, H=32, d=128), after the GPU forward, checked on two heads: 64 sampled
    query rows (dQ) and 64 sampled key rows (dK, dV) each. The keys carry
    outlier channels, hence the relaxed guard (see the test above)."""
    w = WORKLOADS["outlier_8k_causal"]
    q, k, v = make_workload(w)
    do = make_dout(w.B, w.Hq, w.Nq, w.d, w.seed)
    qc, kc, vc, dc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = attn.attn_fwd(qc, kc, vc, causal=w.causal)
    dq, dk, dv = attn.attn_bwd(qc, kc, vc, o, lse, dc, causal=w.causal)
    assert attn.get_status()[0] == 0
    rows = sample_rows(w)
    kv_rows = sample_rows(w, seed_offset=91)[0, 0]
    heads = [(0, 0), (1, w.Hq - 1)]
    # only the two heads are compared: slice everything to them
    sl = lambda t: torch.stack([t[b, h] for b, h in heads])[:, None]  # noqa: E731
    worst = _run_and_check(sl(q), sl(k), sl(v), sl(do), w.causal, w.scale, sl(o.cpu()), sl(lse.cpu()),
                           q_rows=np.stack([rows[b, h] for b, h in heads])[:, None], kv_rows=kv_rows,
                           dq=sl(dq.cpu()), dk=sl(dk.cpu()), dv=sl(dv.cpu()), vacuous=0.3)
    assert worst <= 1.0


def test_autograd_function_matches_torch_fp32():
    """attention() as a torch.autograd.Function: gradients of a scalar loss
    through it against torch's own autograd of the fp32 definition."""
    B, Hq, Hkv, N, d = 1, 4, 2, 300, 128
    q, k, v = make_qkv(B, Hq, Hkv, N, N, d, seed=31)
    qc, kc, vc = (t.cuda().requires_grad_() for t in (q, k, v))
    o = attn.attention(qc, kc, vc, causal=True)
    w = make_dout(B, Hq, N, d, seed=31).cuda()
    (o.float() * w.float()).sum().backward()
    qf, kf, vf = (t.cuda().float().requires_grad_() for t in (q, k, v))
    mask = torch.ones(N, N, dtype=torch.bool, device="cuda").tril()
    of = torch.nn.functional.scaled_dot_product_attention(
        qf, kf.repeat_interleave(2, 1), vf.repeat_interleave(2, 1), attn_mask=mask)
    (of * w.float()).sum().backward()
    for a, r in ((qc.grad, qf.grad), (kc.grad, kf.grad), (vc.grad, vf.grad)):
        assert a.dtype == torch.bfloat16 and a.shape == r.shape
        assert (a.float() - r).abs().max().item() <= 2e-2 * r.abs().max().item()


def _packed_case(lens_q, lens_k, Hq, Hkv, d, seed):
    g = torch.Generator().manual_seed(seed)
    tq, tk = sum(lens_q), sum(lens_k)
    q = torch.randn((tq, Hq, d), generator=g).to(torch.bfloat16)
    k = torch.randn((tk, Hkv, d), generator=g).to(torch.bfloat16)
    v = torch.randn((tk, Hkv, d), generator=g).to(torch.bfloat16)
    do = torch.randn((tq, Hq, d), generator=g).to(torch.bfloat16)
    cq = torch.tensor(np.concatenate([[0], np.cumsum(lens_q)]), dtype=torch.int32)
    ck = torch.tensor(np.concatenate([[0], np.cumsum(lens_k)]), dtype=torch.int32)
    return q, k, v, do, cq, ck


VARLEN_BWD = [
    ([1, 17, 128, 129, 300], None, 4, 2, 128, True),
    ([1, 17, 128, 129, 300], None, 2, 2, 64, False),
    ([64, 200, 513], [1000, 200, 700], 4, 2, 128, True),    # prefill with a cache
    ([300, 50, 5], [100, 0, 5], 2, 2, 128, True),           # Lq > Lk, an empty key set
    ([100, 0, 37], [100, 40, 37], 2, 1, 128, True),         # an empty query sequence
    ([1, 17, 128, 129, 300], [40, 17, 200, 129, 300], 4, 2, 96, True),  # d = 96
]


@pytest.mark.parametrize("case", VARLEN_BWD, ids=range(len(VARLEN_BWD)))
def test_varlen_bwd_matches_oracle(case):
    """Each sequence checked as a dense problem with the element-wise bound;
    rows of a sequence without keys give dQ = 0, keys no query sees dK = dV = 0."""
    lens_q, lens_k, Hq, Hkv, d, causal = case
    lens_k = lens_k or lens_q
    q, k, v, do, cq, ck = _packed_case(lens_q, lens_k, Hq, Hkv, d, seed=sum(lens_q) + d)
    scale = 1 / math.sqrt(d)
    O, L = oracle.attention_varlen_fp64(bf16_bits(q), bf16_bits(k), bf16_bits(v), cq.numpy(), ck.numpy(),
                                        causal, scale)
    o_in = torch.from_numpy(O).to(torch.bfloat16)
    lse_in = torch.from_numpy(L).to(torch.float32)
    dq, dk, dv = attn.attn_bwd_varlen(q.cuda(), k.cuda(), v.cuda(), o_in.cuda(), lse_in.cuda(), do.cuda(),
                                      cq.cuda(), ck.cuda(), max(lens_q), max(lens_k), causal=causal)
    assert attn.get_status()[0] == 0
    dq, dk, dv = dq.cpu(), dk.cpu(), dv.cpu()
    seq = lambda x, a, b: x[a:b].permute(1, 0, 2).unsqueeze(0).contiguous()  # noqa: E731
    for s in range(len(lens_q)):
        a, b, c, e = int(cq[s]), int(cq[s + 1]), int(ck[s]), int(ck[s + 1])
        if b == a or e == c:
            # no query or no key: every gradient of the sequence is exactly 0
            assert torch.all(dq[a:b] == 0) and torch.all(dk[c:e] == 0) and torch.all(dv[c:e] == 0)
            continue
        _run_and_check(seq(q, a, b), seq(k, c, e), seq(v, c, e), seq(do, a, b), causal, scale,
                       seq(o_in, a, b), lse_in[:, a:b].unsqueeze(0).contiguous(),
                       dq=seq(dq, a, b), dk=seq(dk, c, e), dv=seq(dv, c, e))


def test_varlen_bwd_equal_lengths_matches_dense():
    B, H, N, d = 3, 4, 300, 128
    q, k, v = make_qkv(B, H, H, N, N, d, seed=8)
    do = make_dout(B, H, N, d, seed=8)
    qc, kc, vc, dc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = attn.attn_fwd(qc, kc, vc, causal=True)
    gq, gk, gv = attn.attn_bwd(qc, kc, vc, o, lse, dc, causal=True)
    pack = lambda x: x.permute(0, 2, 1, 3).reshape(B * N, H, d).contiguous()  # noqa: E731
    cu = torch.arange(0, (B + 1) * N, N, dtype=torch.int32).cuda()
    lse_p = lse.permute(1, 0, 2).reshape(H, B * N).contiguous()
    vq, vk, vv = attn.attn_bwd_varlen(pack(qc), pack(kc), pack(vc), pack(o), lse_p, pack(dc), cu, cu, N, N,
                                      causal=True)
    # dK, dV: same sums in the same order; dQ: fp32 reductions in any order
    assert torch.equal(vk, pack(gk)) and torch.equal(vv, pack(gv))
    assert ((vq.float() - pack(gq).float()).abs() <= 2 * U * pack(gq).float().abs() + 1e-6).all()


def test_autograd_varlen_matches_dense_autograd_per_sequence():
    lens = [130, 7, 300]
    q, k, v, w, cq, _ = _packed_case(lens, lens, 4, 2, 128, seed=77)
    qc, kc, vc = (t.cuda().requires_grad_() for t in (q, k, v))
    o = attn.attention_varlen(qc, kc, vc, cq.cuda(), cq.cuda(), max(lens), max(lens), causal=True)
    (o.float() * w.cuda().float()).sum().backward()
    for s in range(len(lens)):
        a, b = int(cq[s]), int(cq[s + 1])
        seq = lambda x: x[a:b].permute(1, 0, 2).unsqueeze(0).contiguous().cuda().requires_grad_()  # noqa: E731
        qs, ks, vs = seq(q), seq(k), seq(v)
        od = attn.attention(qs, ks, vs, causal=True)
        (od.float() * w[a:b].permute(1, 0, 2).unsqueeze(0).cuda().float()).sum().backward()
        back = lambda g: g[0].permute(1, 0, 2)  # noqa: E731
        assert torch.equal(kc.grad[a:b], back(ks.grad)) and torch.equal(vc.grad[a:b], back(vs.grad))
        assert ((qc.grad[a:b].float() - back(qs.grad).float()).abs()
                <= 2 * U * back(qs.grad).float().abs() + 1e-6).all()
