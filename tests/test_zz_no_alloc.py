"""The allocation-free 8-bit entry point, attn_fwd_q8_noalloc.

It exists for callers that cannot allocate device memory — code handed only
its input and output buffers (a plugin inside another framework's inference
engine, for example) or a program that must not call cudaMalloc while it
serves. Its scratch is a fixed 32 MiB static device array inside the library.
This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import exact_attention_134_b200 as attn
from synthetic import make_qkv

P = 0x10000  # fake, aligned pointer for the checks that never reach the GPU


def _entry():
    lib = attn.lib()
    fn = lib.attn_fwd_q8_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 7 + [ctypes.c_float, ctypes.c_void_p]
    cap = lib.attn_fwd_q8_static_scratch_bytes
    cap.restype = ctypes.c_size_t
    cap.argtypes = []
    return fn, int(cap())


def test_noalloc_rejects_problems_beyond_its_scratch():
    fn, cap = _entry()
    assert cap == 32 << 20
    # 2 x 32 heads x 8192 tokens x 128 channels needs ~192 MiB of scratch
    assert fn(P, P, P, P, P, 2, 32, 32, 8192, 8192, 128, 1, 0.088, None) == 6
    # invalid arguments are still reported as such
    assert fn(P, P, P, P, P, 1, 3, 2, 128, 128, 128, 0, 0.088, None) == 1
    assert fn(0, P, P, P, P, 1, 2, 2, 128, 128, 128, 0, 0.088, None) == 1


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    fn, cap = _entry()
    cases = [((1, 8, 2, 1024, 1024, 128), True, 11), ((2, 4, 4, 700, 700, 64), False, 12)]
    for shape, causal, seed in cases:  # two calls in a row, different shapes, shared scratch
        B, Hq, Hkv, Nq, Nkv, d = shape
        assert attn.q8_workspace_size(*shape) <= cap
        q, k, v = (t.cuda() for t in make_qkv(*shape, seed, "outlier_k"))
        o_ref, l_ref = attn.attn_fwd_q8(q, k, v, causal=causal)
        o = torch.empty_like(q)
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device="cuda")
        st = fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                B, Hq, Hkv, Nq, Nkv, d, int(causal), 1.0 / math.sqrt(d),
                torch.cuda.current_stream().cuda_stream)
        assert st == 0
        status, where = attn.get_status()
        assert status == 0, (status, where)
        a = o.float().cpu().numpy().astype(np.float64)
        b = o_ref.float().cpu().numpy().astype(np.float64)
        cos = (a * b).sum() / math.sqrt((a * a).sum() * (b * b).sum())
        assert cos >= 0.999 and np.abs(a - b).max() <= 5e-2
        assert (lse - l_ref).abs().max().item() <= 5e-2
        # same kernels on the same inputs: the results are in fact identical
        assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)
