"""Writes tests/golden/q8_error_by_keys.json: the error of the 8-bit method itself
(the oracle's one-shot quantised attention, every operation but the quantisation
in fp64, P encoded against the exact row maximum) against the exact oracle, on
every row of the two full-size 8-bit workloads, as the maximum |dO| per band of
visible keys. It calls only oracle/ and the input generator; it takes about half
an hour on 8 host cores.

    python tests/golden/q8_error_by_keys.py [workers]
"""
import json
import multiprocessing as mp
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
EDGES = [1, 64, 128, 144, 160, 192, 256, 384, 512, 1024, 8193]


def _head(args):
    import oracle
    from oracle import quant8
    qh, kh, vh, causal, scale = args
    O, _ = oracle.attention_fp64(qh, kh, vh, causal, scale)
    O8, _ = quant8.sage8_attention_fp64(qh, kh, vh, causal, scale)
    e = np.abs(O8 - O)[0, 0].max(axis=1)
    n = np.arange(e.shape[0]) + 1          # causal, Nq == Nkv: row i sees i + 1 keys
    return [float(e[(n >= lo) & (n < hi)].max()) for lo, hi in zip(EDGES[:-1], EDGES[1:])]


def main():
    from synthetic import WORKLOADS, bf16_bits, make_qkv
    workers = int(sys.argv[1]) if len(sys.argv) > 1 else len(os.sched_getaffinity(0))
    for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS"):
        os.environ[var] = "1"
    out = {"description": "max |O_method - O_exact| over rows whose number of visible keys lies in "
                          "[lo, hi), one-shot 8-bit oracle vs exact fp64 oracle, every row",
           "bands": [[lo, hi] for lo, hi in zip(EDGES[:-1], EDGES[1:])]}
    for name in ("q8_8k_outlier", "q8_8k_normal"):
        w = WORKLOADS[name]
        q, k, v = make_qkv(w.B, w.Hq, w.Hkv, w.Nq, w.Nkv, w.d, w.seed, w.dist)
        qb, kb, vb = bf16_bits(q), bf16_bits(k), bf16_bits(v)
        jobs = [(qb[b:b + 1, h:h + 1], kb[b:b + 1, h:h + 1], vb[b:b + 1, h:h + 1], w.causal, w.scale)
                for b in range(w.B) for h in range(w.Hq)]
        with mp.get_context("spawn").Pool(workers) as pool:
            res = np.array(pool.map(_head, jobs, chunksize=1))
        out[name] = [round(float(x), 4) for x in res.max(axis=0)]
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "q8_error_by_keys.json"), "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
