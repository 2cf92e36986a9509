"""Multi-rank host logic of bench.py on CPU with gloo (world_size 2).

The forward shards into independent (batch, head) units, so ranks exchange no
data: each rank owns its own batch (its own seed), barriers bracket the timed
region and the reported time is the max over ranks. This checks that plumbing
without a GPU.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    import bench
    from synthetic import WORKLOADS
    w_size, r, _ = bench._dist_setup()
    import torch.distributed as dist
    assert dist.get_backend() == "gloo" and w_size == world and r == rank
    bench._barrier(w_size)
    t = bench._max_over_ranks(10.0 + rank, w_size)          # rank 1 is the slowest
    w = bench.rank_workload(WORKLOADS["tiny_256_d64"], rank)
    seeds = [None] * world
    dist.all_gather_object(seeds, w.seed)
    out[rank] = (t, seeds, bench.aggregate_tflops(w.flops, w_size, t))
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_gloo():
    if torch.cuda.is_available():
        pytest.skip("CPU/gloo test")
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    from synthetic import WORKLOADS
    flops = WORKLOADS["tiny_256_d64"].flops
    for r in range(world):
        t, seeds, agg = res[r]
        assert t == 11.0                                    # max over ranks
        assert seeds == [1001, 2001]                        # independent batch per rank
        assert abs(agg - 2 * flops / 11e-3 / 1e12) < 1e-12  # all ranks' work / slowest time


def test_reference_arm_other_ranks_do_nothing(capsys, monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        workload = "tiny_256_d64"
        steps = 1
        warmup = 0
    bench.run_reference(A())
    assert capsys.readouterr().out == ""


def test_reference_arm_rank0_json(capsys, monkeypatch):
    import json
    import bench
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")

    class A:
        workload = "tiny_256_d64"
        steps = 2
        warmup = 0
    bench.run_reference(A())
    line = json.loads(capsys.readouterr().out.strip())
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["config"]["workload"] == "tiny_256_d64"


# ---------------------------------------------------------------- key-sharded forward

def test_shard_bounds_cover_the_keys_in_rank_order():
    from exact_attention_134_b200.kv_shard import shard_bounds
    for n in (1, 7, 128, 1000, 8193):
        for world in (1, 2, 3, 8):
            b = [shard_bounds(n, world, r) for r in range(world)]
            assert b[0][0] == 0 and b[-1][1] == n
            assert all(b[r][1] == b[r + 1][0] for r in range(world - 1))
            sizes = [hi - lo for lo, hi in b]
            assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)


def _oracle_partial(q, k, v, causal, scale, kv_tail):
    """The partial a rank computes, from the oracle: its keys padded with
    kv_tail dummy keys after them (they only move the causal alignment)."""
    import numpy as np
    from oracle import attention_partial_fp64
    from synthetic import bf16_bits
    pad = torch.zeros((k.shape[0], k.shape[1], kv_tail, k.shape[3]), dtype=k.dtype)
    kb, vb = bf16_bits(torch.cat([k, pad], 2)), bf16_bits(torch.cat([v, pad], 2))
    o, lse = attention_partial_fp64(bf16_bits(q), kb, vb, 0, k.shape[2], causal, scale)
    return torch.from_numpy(np.ascontiguousarray(o)), torch.from_numpy(np.ascontiguousarray(lse))


def _oracle_merge(o_all, lse_all):
    from oracle import merge_partials_fp64
    o, lse = merge_partials_fp64(o_all.numpy(), lse_all.numpy())
    return torch.from_numpy(o), torch.from_numpy(lse)


def _kv_worker(rank, world, port, causal, out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import torch.distributed as dist
    from exact_attention_134_b200.kv_shard import attention_kv_sharded, shard_bounds
    from synthetic import make_qkv
    dist.init_process_group("gloo", rank=rank, world_size=world)
    n_keys = 301
    q, k, v = make_qkv(1, 4, 2, 40, n_keys, 16, seed=31)   # every rank draws the same tensors
    lo, hi = shard_bounds(n_keys, world, rank)
    o, lse = attention_kv_sharded(q, k[:, :, lo:hi].contiguous(), v[:, :, lo:hi].contiguous(),
                                  n_keys, causal=causal, scale=0.25,
                                  partial_fn=_oracle_partial, merge_fn=_oracle_merge)
    out[rank] = (o.numpy(), lse.numpy())
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("causal", [False, True])
def test_kv_sharded_three_ranks_gloo(causal):
    """Three gloo ranks, each holding a third of the keys: the gathered and
    merged partials equal the full attention on every rank (the exchange's
    order, the ranges and the causal tails are what is checked)."""
    if torch.cuda.is_available():
        pytest.skip("CPU/gloo test")
    import numpy as np
    from oracle import attention_fp64
    from synthetic import bf16_bits, make_qkv
    world = 3
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_kv_worker, args=(r, world, port, causal, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    q, k, v = make_qkv(1, 4, 2, 40, 301, 16, seed=31)
    O, L = attention_fp64(bf16_bits(q), bf16_bits(k), bf16_bits(v), causal, 0.25)
    for r in range(world):
        o, lse = res[r]
        assert np.abs(o - O).max() < 1e-12 and np.abs(lse - L).max() < 1e-12


def _kv_errors_worker(port, out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import torch.distributed as dist
    from exact_attention_134_b200.kv_shard import attention_kv_sharded
    dist.init_process_group("gloo", rank=0, world_size=1)
    q = torch.zeros(1, 2, 4, 8)
    k = torch.zeros(1, 2, 5, 8)
    msgs = []
    for n_keys, kk in ((6, k), (0, k[:, :, :0])):
        try:
            attention_kv_sharded(q, kk, kk, n_keys, partial_fn=lambda *a, **kw: None,
                                 merge_fn=lambda *a: None)
            msgs.append("no error")
        except ValueError as e:
            msgs.append(str(e))
    out[0] = msgs
    dist.destroy_process_group()


def test_kv_sharded_rejects_wrong_shards():
    """A rank whose K/V do not hold exactly its range, or a key count below the
    number of ranks, is refused before any kernel or exchange runs."""
    if torch.cuda.is_available():
        pytest.skip("CPU/gloo test")
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        p = ctx.Process(target=_kv_errors_worker, args=(_free_port(), out))
        p.start()
        p.join(120)
        assert p.exitcode == 0
        msgs = out[0]
    assert "must hold keys [0, 6) of 6" in msgs[0]
    assert "at least one key" in msgs[1]


def _bench_kv_worker(rank, world, port, causal, out):
    """bench.py --shard kv's host logic on gloo: this rank's shard from
    bench.kv_shard_inputs, the exchange and merge of kv_shard, oracle partials."""
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import torch.distributed as dist
    import bench
    from exact_attention_134_b200.kv_shard import attention_kv_sharded
    from synthetic import Workload
    dist.init_process_group("gloo", rank=rank, world_size=world)
    w = Workload("kv_test", 1, 4, 2, 48, 333, 16, causal, 77)
    q, ks, vs, n_keys = bench.kv_shard_inputs(w, world, rank)
    o, lse = attention_kv_sharded(q, ks, vs, n_keys, causal=causal, scale=0.25,
                                  partial_fn=_oracle_partial, merge_fn=_oracle_merge)
    shards = [None] * world
    dist.all_gather_object(shards, ks.float().numpy())
    out[rank] = (o.numpy(), lse.numpy(), shards)
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("causal", [False, True])
def test_bench_kv_shard_two_ranks_gloo(causal):
    """Two gloo ranks run bench.py --shard kv's per-rank inputs through the
    key-sharded exchange: the shards tile the keys in rank order and every
    rank's merged result equals the full attention."""
    import numpy as np
    import oracle
    from synthetic import Workload, bf16_bits, make_qkv
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_bench_kv_worker, args=(r, world, port, causal, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(180)
            assert p.exitcode == 0
        res = dict(out)
    w = Workload("kv_test", 1, 4, 2, 48, 333, 16, causal, 77)
    q, k, v = make_qkv(w.B, w.Hq, w.Hkv, w.Nq, w.Nkv, w.d, w.seed, w.dist)
    full_k = k.float().numpy()
    assert np.array_equal(np.concatenate(res[0][2], axis=2), full_k)
    O, L = oracle.attention_fp64(bf16_bits(q), bf16_bits(k), bf16_bits(v), causal, 0.25)
    for r in range(world):
        o, lse, _ = res[r]
        assert np.allclose(o, O, rtol=1e-12, atol=1e-12) and np.allclose(lse, L, rtol=1e-12, atol=1e-12)


def test_reference_arm_config_is_the_gpu_arms():
    import bench
    from synthetic import WORKLOADS
    for name in ("outlier_8k_causal", "tiny_256_d64"):
        w = WORKLOADS[name]
        cfg = bench.workload_config(w, bench.l2_mode_of(w))
        assert set(cfg) >= {"workload", "scale", "l2", "per_rank"}
    assert bench.l2_mode_of(WORKLOADS["outlier_8k_causal"]) == "inputs_larger_than_l2"
    assert bench.l2_mode_of(WORKLOADS["tiny_256_d64"]) == "l2_flushed_between_steps"
