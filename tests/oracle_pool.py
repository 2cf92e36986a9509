"""Runs the fp64 oracle over many (batch, head) pairs in parallel worker
processes (test infrastructure, like oracle/ itself).

The workers are started with the 'spawn' method (a process forked after the
CUDA context exists can hang) and each uses one BLAS thread, so that the
per-head evaluations, not one matrix product at a time, share the host
cores. Each (batch, query head) is evaluated on its own slice of Q and the
slice of K, V its kv head reads; the oracle's quantities are all per (batch,
kv head), so slicing changes nothing but the summation order inside a matrix
product (results agree with the whole-tensor call to ~1e-15).
"""
from __future__ import annotations

import multiprocessing as mp
import os

import numpy as np

_THREAD_VARS = ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")


def _exact_head(args):
    import oracle
    qh, kh, vh, causal, scale, rows = args
    return oracle.attention_fp64(qh, kh, vh, causal, scale, rows=rows)


def _quantised_head(args):
    from oracle import quant8
    qh, kh, vh, causal, scale, rows, qk_format = args
    return quant8.quantised_scores_attention_fp64(qh, kh, vh, causal, scale, qk_format, rows=rows)


def _run(fn, jobs, workers):
    saved = {k: os.environ.get(k) for k in _THREAD_VARS}
    try:
        for k in _THREAD_VARS:
            os.environ[k] = "1"
        with mp.get_context("spawn").Pool(workers) as pool:
            return pool.map(fn, jobs, chunksize=1)
    finally:
        for k, val in saved.items():
            if val is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = val


def _jobs(qb, kb, vb, rows, extra):
    B, Hq = qb.shape[:2]
    Hkv = kb.shape[1]
    g = Hq // Hkv
    out = []
    for b in range(B):
        for h in range(Hq):
            r = None if rows is None else rows[b:b + 1, h:h + 1]
            out.append((qb[b:b + 1, h:h + 1], kb[b:b + 1, h // g:h // g + 1], vb[b:b + 1, h // g:h // g + 1])
                       + extra(r))
    return out


def _stack(results, B, Hq):
    parts = list(zip(*results))
    return tuple(np.concatenate(p, axis=1).reshape((B, Hq) + p[0].shape[2:]) for p in parts)


def workers_default() -> int:
    return max(1, min(32, len(os.sched_getaffinity(0))))


def attention_fp64_parallel(qb, kb, vb, causal, scale, rows=None, workers=None):
    """oracle.attention_fp64, one (batch, query head) per task."""
    B, Hq = qb.shape[:2]
    jobs = _jobs(qb, kb, vb, rows, lambda r: (causal, scale, r))
    return _stack(_run(_exact_head, jobs, workers or workers_default()), B, Hq)


def quantised_scores_attention_fp64_parallel(qb, kb, vb, causal, scale, qk_format="int8", rows=None,
                                             workers=None):
    """oracle.quant8.quantised_scores_attention_fp64, one (batch, query head)
    per task (for Hq == Hkv: the quantisation blocks are per head)."""
    B, Hq = qb.shape[:2]
    if kb.shape[1] != Hq:
        raise ValueError("per-head slicing of the 8-bit quantisation needs Hq == Hkv")
    jobs = _jobs(qb, kb, vb, rows, lambda r: (causal, scale, r, qk_format))
    return _stack(_run(_quantised_head, jobs, workers or workers_default()), B, Hq)
