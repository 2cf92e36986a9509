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
