"""Writes the golden fixtures in this folder. Calls only ``oracle/`` (and the
seeded generator for its inputs); run from the repository root:

    python tests/golden/make_golden.py

The pages print no worked example with numbers, so the fixtures are the
oracle's own values for small seeded inputs, kept to catch any later change to
the oracle's arithmetic (a change must then cite the passage that justifies
it). Definition followed: "FlashAttention (TR)" (systems-analysis.info),
section "Standart Attention Mekanizmasının Sorunları".
"""
import json
import math
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from synthetic import bf16_bits, make_qkv  # noqa: E402

CASES = [
    # name, B, Hq, Hkv, Nq, Nkv, d, causal, seed
    ("mha_noncausal", 1, 2, 2, 12, 12, 8, False, 424242),
    ("gqa_causal", 1, 4, 2, 10, 10, 8, True, 434343),
    ("cross_ragged", 1, 2, 1, 5, 9, 16, False, 444444),
]


def main():
    out = {"citation": "FlashAttention (TR) — Standart Attention Mekanizmasının Sorunları "
                       "(Attention(Q,K,V) = softmax(QK^T/sqrt(d_k)) V)",
           "generator": "synthetic.make_qkv (seeded torch CPU randn -> bf16)",
           "cases": []}
    for name, B, Hq, Hkv, Nq, Nkv, d, causal, seed in CASES:
        q, k, v = make_qkv(B, Hq, Hkv, Nq, Nkv, d, seed)
        scale = 1.0 / math.sqrt(d)
        O, L = oracle.attention_fp64(bf16_bits(q), bf16_bits(k), bf16_bits(v), causal, scale)
        out["cases"].append({"name": name, "B": B, "Hq": Hq, "Hkv": Hkv, "Nq": Nq, "Nkv": Nkv,
                             "d": d, "causal": causal, "seed": seed, "scale": scale,
                             "O": O.tolist(), "LSE": L.tolist()})
    with open(os.path.join(HERE, "oracle_small_cases.json"), "w") as f:
        json.dump(out, f, indent=0)


if __name__ == "__main__":
    main()
