"""Failure detection on the GPU without a fault: a bounded wait that nothing
completes must end by its budget, record ATTN_ERR_TIMEOUT in the device status
word, and leave the context usable for the next attention call."""
import math
import time

import numpy as np
import pytest
import torch

import exact_attention_134_b200 as attn
import oracle
from synthetic import bf16_bits, make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    attn.lib()
    attn.get_status()  # start from a clean status word


def test_wait_times_out_and_reports_status():
    t0 = time.perf_counter()
    attn.selftest_wait_timeout(50_000)  # 50 ms
    status, where = attn.get_status()
    elapsed = time.perf_counter() - t0
    assert status == 5 and where == 0xF00, (status, where)
    assert 0.04 <= elapsed < 5.0, elapsed
    assert attn.get_status() == (0, 0)  # read clears it


def test_context_usable_after_timeout():
    attn.selftest_wait_timeout(20_000)
    assert attn.get_status()[0] == 5
    q, k, v = make_qkv(1, 2, 2, 200, 200, 128, seed=4)
    o, lse = attn.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True)
    assert attn.get_status() == (0, 0)
    O, L = oracle.attention_fp64(bf16_bits(q), bf16_bits(k), bf16_bits(v), True, 1 / math.sqrt(128))
    assert np.abs(o.float().cpu().numpy() - O).max() <= 1e-2


def test_bad_budget_rejected():
    with pytest.raises(attn.AttnError):
        attn.selftest_wait_timeout(0)
