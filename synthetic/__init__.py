"""Seeded synthetic inputs for the exact-attention forward.

This module is the ONE piece shared by the CUDA path's tests/bench and the CPU
oracle. It holds none of the method's arithmetic: it only draws random numbers
and rounds them to bf16. Every workload below stands in for the model-level
workloads the FlashAttention / SageAttention pages measure on (BERT, GPT-2,
Long-Range Arena, video diffusion), which are not available here.

Recipe (same for every workload; the backward's dO: see ``make_dout``):
  * ``torch.Generator('cpu').manual_seed(seed)``;
  * fp32 ``randn`` draws in the order Q, K, V, then any extras;
  * the "outlier K" distribution adds a per-(kv head, channel) offset b that is
    shared across batch and tokens: per head, exactly round(0.1 * d) channels
    (drawn without replacement with ``randperm``) get b ~ 10 * N(0,1), all
    other channels get b ~ N(0,1);
  * each tensor is rounded to bf16 (round-to-nearest-even) once; the GPU and
    the oracle consume the identical bf16 bits.

Tensors are returned on the CPU as contiguous bf16 ``[B, H, N, d]``.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nkv: int
    d: int
    causal: bool
    seed: int
    dist: str = "normal"          # "normal" | "outlier_k"
    path: str = "bf16"            # "bf16" | "q8" (8-bit mainloop) | "splitkv" (split keys)
    oracle_rows: int = 0          # 0 = every query row; else rows sampled per (b, hq)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def flops(self) -> float:
        """4*B*Hq*Nq*Nkv*d, halved for causal (the N^2/2 convention)."""
        f = 4.0 * self.B * self.Hq * self.Nq * self.Nkv * self.d
        return f / 2.0 if self.causal else f

    @property
    def min_hbm_bytes(self) -> int:
        """Read Q, K, V once and write O (bf16) plus LSE (fp32)."""
        qo = self.B * self.Hq * self.Nq * self.d
        kv = self.B * self.Hkv * self.Nkv * self.d
        return 2 * (qo + 2 * kv + qo) + 4 * self.B * self.Hq * self.Nq


# The five workloads (tiny; causal 2k; outlier-channel 8k causal and not;
# long-context GQA 32k at d=128 and d=64; the 8-bit variant on two input sets).
WORKLOADS = {
    "tiny_256_d64": Workload("tiny_256_d64", 1, 2, 2, 256, 256, 64, False, 1001),
    "causal_2k_d128": Workload("causal_2k_d128", 4, 16, 16, 2048, 2048, 128, True, 1002),
    "outlier_8k_causal": Workload("outlier_8k_causal", 2, 32, 32, 8192, 8192, 128, True, 1003,
                                  dist="outlier_k", oracle_rows=64),
    "outlier_8k_full": Workload("outlier_8k_full", 2, 32, 32, 8192, 8192, 128, False, 1003,
                                dist="outlier_k", oracle_rows=64),
    "gqa_32k_d128": Workload("gqa_32k_d128", 1, 32, 8, 32768, 32768, 128, True, 1004,
                             oracle_rows=64),
    "gqa_32k_d64": Workload("gqa_32k_d64", 1, 64, 8, 32768, 32768, 64, True, 1005,
                            oracle_rows=64),
    "q8_8k_outlier": Workload("q8_8k_outlier", 2, 32, 32, 8192, 8192, 128, True, 1003,
                              dist="outlier_k", path="q8", oracle_rows=64),
    "q8_8k_normal": Workload("q8_8k_normal", 2, 32, 32, 8192, 8192, 128, True, 1006,
                             path="q8", oracle_rows=64),
    # head dim 256 (the largest the FlashAttention-2 section names), 8k causal
    "d256_8k_causal": Workload("d256_8k_causal", 1, 16, 16, 8192, 8192, 256, True, 1008,
                               oracle_rows=64),
    # 128 new query rows against a 128k-key cache (GQA 32/8): too few CTAs for
    # the row-parallel forward; the same inputs through the split-key forward
    "kvcache_128k_q128": Workload("kvcache_128k_q128", 1, 32, 8, 128, 131072, 128, False, 1010,
                                  oracle_rows=8),
    "kvcache_128k_q128_splitkv": Workload("kvcache_128k_q128_splitkv", 1, 32, 8, 128, 131072, 128,
                                          False, 1010, path="splitkv", oracle_rows=8),
}


def _bf16(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.bfloat16).contiguous()


def make_qkv(B: int, Hq: int, Hkv: int, Nq: int, Nkv: int, d: int, seed: int,
             dist: str = "normal"):
    """Draw Q, K, V as bf16 CPU tensors following the module recipe."""
    g = torch.Generator("cpu").manual_seed(seed)
    q = torch.randn((B, Hq, Nq, d), generator=g, dtype=torch.float32)
    k = torch.randn((B, Hkv, Nkv, d), generator=g, dtype=torch.float32)
    v = torch.randn((B, Hkv, Nkv, d), generator=g, dtype=torch.float32)
    if dist == "outlier_k":
        n_big = int(round(0.1 * d))
        offs = torch.randn((Hkv, d), generator=g, dtype=torch.float32)
        for h in range(Hkv):
            big = torch.randperm(d, generator=g)[:n_big]
            offs[h, big] *= 10.0
        k = k + offs[None, :, None, :]
    elif dist != "normal":
        raise ValueError(f"unknown distribution {dist!r}")
    return _bf16(q), _bf16(k), _bf16(v)


def make_workload(w: Workload):
    return make_qkv(w.B, w.Hq, w.Hkv, w.Nq, w.Nkv, w.d, w.seed, w.dist)


def make_dout(B: int, Hq: int, Nq: int, d: int, seed: int) -> torch.Tensor:
    """The upstream gradient dO for a backward pass: fp32 ``randn`` from its
    own generator seeded with ``seed + 500``, rounded to bf16 [B, Hq, Nq, d]."""
    g = torch.Generator("cpu").manual_seed(seed + 500)
    return _bf16(torch.randn((B, Hq, Nq, d), generator=g, dtype=torch.float32))


def sample_rows(w: Workload, n_rows: int | None = None, seed_offset: int = 77):
    """Seeded query-row subset per (b, hq) without replacement, sorted.

    Returns an int64 array [B, Hq, R]. Always contains row 0 and row Nq-1 so the
    first (single-key under a causal mask) and last rows are exercised.
    """
    R = n_rows if n_rows is not None else w.oracle_rows
    R = min(R, w.Nq)
    g = torch.Generator("cpu").manual_seed(w.seed + seed_offset)
    out = np.empty((w.B, w.Hq, R), dtype=np.int64)
    for b in range(w.B):
        for h in range(w.Hq):
            if R == w.Nq:
                out[b, h] = np.arange(w.Nq)
                continue
            perm = torch.randperm(w.Nq - 2, generator=g)[: R - 2].numpy() + 1
            rows = np.concatenate([[0, w.Nq - 1], perm])
            out[b, h] = np.sort(rows)
    return out


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """The raw bf16 bit patterns of a CPU tensor, as a uint16 numpy array."""
    assert t.dtype == torch.bfloat16 and t.device.type == "cpu"
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


@dataclasses.dataclass(frozen=True)
class VarlenWorkload:
    """A batch of prompts of different lengths, packed without padding."""
    name: str
    num_seqs: int
    min_len: int
    max_len: int
    Hq: int
    Hkv: int
    d: int
    causal: bool
    seed: int

    def lengths(self) -> list[int]:
        """Seeded log-uniform lengths in [min_len, max_len]."""
        g = torch.Generator("cpu").manual_seed(self.seed)
        u = torch.rand(self.num_seqs, generator=g, dtype=torch.float64)
        lo, hi = math.log(self.min_len), math.log(self.max_len)
        return [int(round(math.exp(lo + float(x) * (hi - lo)))) for x in u]

    @property
    def flops(self) -> float:
        f = sum(4.0 * self.Hq * L * L * self.d for L in self.lengths())
        return f / 2.0 if self.causal else f


VARLEN_WORKLOADS = {
    "varlen_prefill_mixed": VarlenWorkload("varlen_prefill_mixed", 16, 256, 8192, 32, 8, 128, True, 1007),
}


def make_varlen(w: VarlenWorkload):
    """Packed q [total, Hq, d], k, v [total, Hkv, d] (bf16, CPU) and int32
    cu_seqlens [num_seqs + 1] (the same offsets for queries and keys)."""
    lens = w.lengths()
    total = sum(lens)
    g = torch.Generator("cpu").manual_seed(w.seed + 1)
    q = torch.randn((total, w.Hq, w.d), generator=g, dtype=torch.float32)
    k = torch.randn((total, w.Hkv, w.d), generator=g, dtype=torch.float32)
    v = torch.randn((total, w.Hkv, w.d), generator=g, dtype=torch.float32)
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32)
    return _bf16(q), _bf16(k), _bf16(v), cu


def make_varlen_dout(w: VarlenWorkload) -> torch.Tensor:
    """dO for the packed workload: fp32 ``randn`` [total, Hq, d] from a
    generator seeded with ``seed + 500``, rounded to bf16."""
    total = sum(w.lengths())
    g = torch.Generator("cpu").manual_seed(w.seed + 500)
    return _bf16(torch.randn((total, w.Hq, w.d), generator=g, dtype=torch.float32))
