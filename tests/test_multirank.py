"""The multi-GPU form of the benchmark, on CPU: world_size-2 `gloo` ranks on
127.0.0.1 run the host logic bench.py uses under torchrun.  Each rank attends
over its own batch (distinct seeds, weak scaling, no data-path collective),
the job time is the max over ranks, the job rate counts every rank's units,
and the reference arm runs on rank 0 only."""
import json
import math
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import attn_inputs as gen
    import bench
    import oracle

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    # per-rank work: a small attention problem of its own, solved by the oracle
    cfg = dict(B=1, Hq=2, Hkv=1, N=40, d=16, causal=True, dtype="bf16")
    qb, kb, vb = bench.make_inputs(cfg, seed=bench.rank_seed(rank))
    o, _ = oracle.attn_fwd(*(gen.bf16_bits_to_f64(x) for x in (qb, kb, vb)), True, 0.25)
    # per-rank "times": the job time is the slowest rank's
    local = [10.0 + 5.0 * rank, 30.0 - 7.0 * rank]
    reduced = bench.max_over_ranks(local, "cpu", world)
    rate = bench.job_throughput(bench.flops(cfg), 4, world, reduced[0])
    dist.barrier()
    dist.destroy_process_group()
    np.save(os.path.join(out_dir, f"o{rank}.npy"), o)
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
        json.dump({"reduced": reduced, "rate": rate}, f)


def test_two_gloo_ranks(tmp_path):
    import torch.multiprocessing as mp
    world, port = 2, _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world, start_method="spawn", join=True)
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(world)]
    # every rank sees the same element-wise max over ranks
    assert res[0]["reduced"] == res[1]["reduced"] == [15.0, 30.0]
    # whole-job rate: both ranks' units over the slowest rank's time
    flops = 4.0 * 1 * 2 * 40 * 40 * 16 / 2
    assert math.isclose(res[0]["rate"], flops * 4 * world / 15e-3)
    # independent batches: the ranks' problems (and results) differ
    o0, o1 = (np.load(tmp_path / f"o{r}.npy") for r in range(world))
    assert o0.shape == o1.shape and not np.allclose(o0, o1)


def test_reference_arm_runs_on_rank0_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    args = type("A", (), dict(steps=1, warmup=0, gpus=2, cpu_seconds=1.0))()
    assert bench.run_reference(args, bench.workloads()["tiny"], "tiny") == 0
    assert capsys.readouterr().out == ""
