"""C-ABI checks that need no GPU: the library builds and loads, exports every
entry point include/attn.h declares, and rejects bad arguments before it
touches CUDA (no compute call is made here)."""
import ctypes
import os
import re

import pytest

import exact_attention_134_b200 as attn
from exact_attention_134_b200 import build as attn_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"ATTN_API\s+[\w\s\*]+?\b(attn_\w+)\s*\(", text))
    return names


@pytest.fixture(scope="module")
def lib():
    attn_build.build()
    return attn.lib()


def test_every_declared_symbol_is_exported(lib):
    names = _declared_symbols()
    assert "attn_fwd" in names and len(names) >= 8
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_strings(lib):
    assert attn.version() >= 100
    assert lib.attn_status_string(0) == b"ATTN_OK"
    assert lib.attn_status_string(5) == b"ATTN_ERR_TIMEOUT"
    assert lib.attn_status_string(99) == b"ATTN_ERR_UNKNOWN"


P = 0x10000  # a fake, 16-byte-aligned "device pointer": never dereferenced on these paths


def _fwd(lib, q=P, k=P, v=P, o=P, lse=P, B=1, Hq=2, Hkv=2, Nq=128, Nkv=128, d=128, causal=0, scale=0.125):
    return lib.attn_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, d, causal, scale, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), 1), (dict(lse=0), 1), (dict(B=0), 1), (dict(Nq=0), 1), (dict(Nkv=-1), 1),
    (dict(Hq=3, Hkv=2), 1), (dict(scale=0.0), 1), (dict(scale=float("nan")), 1),
    (dict(scale=float("inf")), 1), (dict(scale=-1.0), 1), (dict(causal=2), 1),
    (dict(d=80), 2), (dict(d=512), 2), (dict(d=32), 2), (dict(B=70000), 2),
    (dict(q=P + 2), 3), (dict(o=P + 8), 3), (dict(lse=P + 4), 3),
])
def test_argument_validation(lib, kw, code):
    assert _fwd(lib, **kw) == code


def test_host_entry_rejects_bad_workspace(lib):
    need = lib.attn_fwd_host_buffer_size(1, 2, 2, 128, 128, 64)
    assert need >= 2 * (2 * 128 * 64 * 2) + 2 * 128 * 64 * 2 + 2 * 128 * 4
    args = [P, P, P, P, P, 1, 2, 2, 128, 128, 64, 0, 0.125]
    assert lib.attn_fwd_host(*args, None, need, None) == 6
    assert lib.attn_fwd_host(*args, P + 1, need, None) == 6
    assert lib.attn_fwd_host(*args, P, need - 1, None) == 6
    assert lib.attn_fwd_host_buffer_size(0, 2, 2, 128, 128, 64) == 0


def test_timeout_setter(lib):
    assert lib.attn_set_timeout_ms(0) == 1
    assert lib.attn_set_timeout_ms(1000) == 0


def test_binding_requires_cuda_tensors():
    import torch
    q = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        attn.attn_fwd(q, q, q)


def test_q8_entry_validation(lib):
    need = lib.attn_fwd_q8_workspace_size(1, 2, 2, 300, 300, 128)
    off = (ctypes.c_size_t * 11)()
    assert lib.attn_q8_workspace_offsets(1, 2, 2, 300, 300, 128, off) == 0
    assert off[10] == need and list(off) == sorted(off)
    assert all(o % 256 == 0 for o in off)
    # q8 / k8 / v8 hold one byte per element, then the fp32 scales
    assert off[1] - off[0] >= 2 * 300 * 128 and off[3] - off[2] >= 2 * 300 * 128
    args = [P, P, P, P, P, 1, 2, 2, 300, 300, 128, 0, 0.125]
    assert lib.attn_fwd_q8(*args, None, need, None) == 6
    assert lib.attn_fwd_q8(*args, P + 8, need, None) == 6
    assert lib.attn_fwd_q8(*args, P, need - 1, None) == 6
    assert lib.attn_fwd_q8(P, P, P, P, P, 1, 2, 2, 300, 300, 96, 0, 0.125, P, need, None) == 2
    assert lib.attn_fwd_fp8(P, P, P, P, P, 1, 2, 2, 300, 300, 96, 0, 0.125, P, need, None) == 2
    assert lib.attn_fwd_q8(P, P, P, P, P, 1, 2, 2, 300, 300, 256, 0, 0.125, P, need, None) == 2
    assert lib.attn_q8_prepass(P, P, P, 1, 2, 2, 300, 300, 128, None, need, None) == 6
    assert lib.attn_q8_workspace_offsets(0, 2, 2, 300, 300, 128, off) == 1


def test_varlen_entry_validation(lib):
    def call(cq=P, ck=P, n=2, mq=64, tq=100, tk=120, Hq=4, Hkv=2, d=128, causal=1, scale=0.1, q=P):
        return lib.attn_fwd_varlen(q, P, P, P, P, cq, ck, n, mq, tq, tk, Hq, Hkv, d, causal, scale, None)
    assert call(cq=None) == 1 and call(ck=None) == 1
    assert call(n=0) == 1 and call(mq=0) == 1 and call(tq=0) == 1 and call(Hq=3) == 1
    assert call(scale=float("nan")) == 1 and call(causal=3) == 1
    assert call(d=80) == 2 and call(d=512) == 2 and call(n=70000) == 2  # d = 256 is supported
    assert call(q=P + 2) == 3 and call(cq=P + 2) == 3


def test_bwd_entry_validation(lib):
    need = lib.attn_bwd_workspace_size(2, 4, 2, 300, 500, 128)
    # fp32 dQ accumulator over 384 padded rows, then LSE_2 and D, 256-byte aligned
    rows = 2 * 4 * 384
    assert need >= 4 * rows * 128 + 8 * rows and need % 256 == 0
    assert lib.attn_bwd_workspace_size(0, 4, 2, 300, 500, 128) == 0

    def call(dq=P, ws=P, nbytes=need, d=128, Hq=4, B=2, causal=1, scale=0.1, dout=P):
        return lib.attn_bwd(P, P, P, P, P, dout, dq, P, P, B, Hq, 2, 300, 500, d, causal, scale,
                            ws, nbytes, None)
    assert call(dq=None) == 1 and call(dout=None) == 1 and call(Hq=3) == 1
    assert call(causal=2) == 1 and call(scale=-1.0) == 1
    assert call(d=80) == 2 and call(d=256) == 2 and call(B=70000) == 2
    assert call(dq=P + 4) == 3
    assert call(ws=None) == 6 and call(ws=P + 8) == 6 and call(nbytes=need - 1) == 6


def test_bwd_varlen_entry_validation(lib):
    need = lib.attn_bwd_varlen_workspace_size(3, 4, 300, 128)
    assert need > 4 * 3 * 4 * 384 * 128 and lib.attn_bwd_varlen_workspace_size(0, 4, 300, 128) == 0

    def call(cq=P, ws=P, nbytes=need, d=128, n=3, mq=300, mk=300, causal=1, q=P):
        return lib.attn_bwd_varlen(q, P, P, P, P, P, P, P, P, cq, P, n, mq, mk, 700, 700, 4, 2, d,
                                   causal, 0.1, ws, nbytes, None)
    assert call(cq=None) == 1 and call(n=0) == 1 and call(mq=0) == 1 and call(mk=0) == 1
    assert call(causal=5) == 1 and call(d=80) == 2 and call(n=70000) == 2
    assert call(q=P + 2) == 3 and call(cq=P + 2) == 3
    assert call(ws=None) == 6 and call(nbytes=need - 1) == 6


def test_partial_and_merge_entry_validation(lib):
    def partial(q=P, o=P, lse=P, d=128, tail=0, Nkv=500):
        return lib.attn_fwd_partial(q, P, P, o, lse, 1, 4, 2, 300, Nkv, d, 1, 0.1, tail, None)
    assert partial(o=None) == 1 and partial(lse=None) == 1 and partial(tail=-1) == 1
    assert partial(Nkv=0) == 1 and partial(Nkv=2 ** 31 - 10, tail=20) == 1
    assert partial(d=256) == 2 and partial(d=80) == 2
    assert partial(q=P + 2) == 3 and partial(o=P + 4) == 3

    def merge(op=P, lp=P, n=3, d=128, o=P, lse=P, B=2):
        return lib.attn_merge_partials(op, lp, n, B, 4, 300, d, o, lse, None)
    assert merge(op=None) == 1 and merge(o=None) == 1 and merge(n=0) == 1 and merge(B=0) == 1
    assert merge(d=80) == 2 and merge(d=512) == 2
    assert merge(lp=P + 4) == 3 and merge(o=P + 8) == 3


def test_splitkv_plan_and_validation(lib):
    # the automatic choice fills one wave of CTAs (at most 148 here: without a
    # GPU the library assumes 148 SMs) with ranges of at least two key tiles
    n = attn.splitkv_num_splits
    assert n(1, 32, 8, 128, 131072, 128) == 9     # head pairs: 16 CTAs -> 9 ranges
    assert n(1, 32, 32, 128, 131072, 128) == 4    # one head per CTA: 32 CTAs -> 4 ranges
    assert n(2, 32, 32, 8192, 8192, 128) == 1     # already > 148 CTAs
    assert n(1, 1, 1, 16, 1 << 20, 128) == 64     # capped at 64 ranges
    assert n(1, 2, 2, 10, 300, 128) == 1          # 3 tiles: ranges of >= 2
    assert n(1, 2, 2, 10, 1000, 128, 5) == 4      # 8 tiles in ranges of 2
    assert n(1, 2, 2, 10, 1000, 128, 100) == 8    # at most one range per tile
    assert n(0, 2, 2, 10, 1000, 128) == 0 and n(1, 3, 2, 10, 1000, 128) == 0
    need = lib.attn_fwd_splitkv_workspace_size(1, 32, 8, 128, 131072, 128, 0)
    assert need >= 9 * 32 * 128 * (128 + 1) * 4 and need % 256 == 0
    assert lib.attn_fwd_splitkv_workspace_size(2, 32, 32, 8192, 8192, 128, 0) == 0  # one range

    def call(ws=P, nbytes=need, d=128, B=1, S=0):
        return lib.attn_fwd_splitkv(P, P, P, P, P, B, 32, 8, 128, 131072, d, 0, 0.1, S, ws,
                                    nbytes, None)
    assert call(ws=None) == 6 and call(ws=P + 8) == 6 and call(nbytes=need - 1) == 6
    assert call(d=256) == 2 and call(B=20000, S=64) == 2

    # the split partial of a key range: same plan and workspace, plus kv_tail
    def pcall(ws=P, nbytes=need, d=128, tail=0, o=P):
        return lib.attn_fwd_partial_splitkv(P, P, P, o, P, 1, 32, 8, 128, 131072, d, 1, 0.1, tail, 0,
                                            ws, nbytes, None)
    assert pcall(ws=None) == 6 and pcall(nbytes=need - 1) == 6
    assert pcall(tail=-1) == 1 and pcall(o=None) == 1 and pcall(d=256) == 2
