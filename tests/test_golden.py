"""The oracle reproduces its committed fixtures, and a hand-derived example."""
import json
import math
import os

import numpy as np

import oracle
from synthetic import bf16_bits, make_qkv

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_oracle_reproduces_fixtures():
    with open(os.path.join(HERE, "oracle_small_cases.json")) as f:
        data = json.load(f)
    for c in data["cases"]:
        q, k, v = make_qkv(c["B"], c["Hq"], c["Hkv"], c["Nq"], c["Nkv"], c["d"], c["seed"])
        O, L = oracle.attention_fp64(bf16_bits(q), bf16_bits(k), bf16_bits(v), c["causal"], c["scale"])
        assert np.max(np.abs(O - np.array(c["O"]))) < 1e-14
        assert np.max(np.abs(L - np.array(c["LSE"]))) < 1e-14


def test_hand_worked_two_key_example():
    # q = (1, 0), keys (1, 0) and (0, 1), values (1, 2) and (3, 4), scale 1:
    # scores (1, 0) -> weights (e, 1)/(e + 1); O = (e*(1,2) + (3,4))/(e+1);
    # LSE = ln(e + 1). All values are exact in bf16.
    def bits(a):
        import torch
        return bf16_bits(torch.tensor(a, dtype=torch.float32).to(torch.bfloat16).reshape(1, 1, -1, 2))
    O, L = oracle.attention_fp64(bits([[1, 0]]), bits([[1, 0], [0, 1]]), bits([[1, 2], [3, 4]]), False, 1.0)
    e = math.e
    assert np.allclose(O[0, 0, 0], [(e * 1 + 3) / (e + 1), (e * 2 + 4) / (e + 1)], atol=1e-15, rtol=0)
    assert abs(L[0, 0, 0] - math.log(e + 1)) < 1e-15
