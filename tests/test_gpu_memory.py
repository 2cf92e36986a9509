"""The forward allocates no device memory: with O and LSE supplied, an
attn_fwd call leaves the device's free memory and torch's allocator exactly
as they were ("FlashAttention (TR)", "İşlemlerin Tek Bir CUDA Çekirdeğinde
Birleştirilmesi": only the final result is written to HBM — there is no
N x N score matrix, nor any other temporary, in device memory)."""
import pytest
import torch

import exact_attention_134_b200 as attn
from synthetic import make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    attn.lib()


@pytest.mark.parametrize("causal", [False, True])
def test_fwd_allocates_no_device_memory(causal):
    # N = 8192: an N x N fp32 score matrix for the two heads would be 512 MiB
    B, H, N, d = 1, 2, 8192, 128
    q, k, v = (t.cuda() for t in make_qkv(B, H, H, N, N, d, seed=77))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    attn.attn_fwd(q, k, v, causal=causal, out=o, lse=lse)  # first call: module load, per-device set-up
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0, reserved0 = torch.cuda.memory_allocated(), torch.cuda.memory_reserved()
    for _ in range(3):
        attn.attn_fwd(q, k, v, causal=causal, out=o, lse=lse)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert attn.get_status()[0] == 0
    assert free1 == free0
    assert torch.cuda.memory_allocated() == alloc0 and torch.cuda.memory_reserved() == reserved0
