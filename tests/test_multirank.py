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


def _shard_worker(rank, world, port, out_dir):
    """One rank of a call split by (batch, key/value head) units: it computes its
    rectangles (the oracle stands in for the GPU here) and the pieces are
    gathered to rank 0 over gloo, which reassembles the whole output."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import attn_inputs as gen
    import exact_attention_140_b200 as ea
    import oracle

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    B, Hq, Hkv, N, d = 3, 6, 3, 24, 8
    g = Hq // Hkv
    q, k, v = (gen.bf16_bits_to_f64(x) for x in gen.qkv_bf16(B, Hq, Hkv, N, N, d, seed=91))
    pieces = []
    for (b0, b1, g0, g1) in ea.attn_shard_units(B, Hkv, world, rank):
        o, lse = oracle.attn_fwd(q[b0:b1, :, g0 * g:g1 * g], k[b0:b1, :, g0:g1], v[b0:b1, :, g0:g1], True, 0.3)
        pieces.append(((b0, b1, g0, g1), o, lse))
    gathered = [None] * world
    dist.all_gather_object(gathered, pieces)
    dist.barrier()
    dist.destroy_process_group()
    if rank == 0:
        o_all = np.full((B, N, Hq, d), np.nan)
        lse_all = np.full((B, Hq, N), np.nan)
        for rank_pieces in gathered:
            for (b0, b1, g0, g1), o, lse in rank_pieces:
                assert np.all(np.isnan(o_all[b0:b1, :, g0 * g:g1 * g]))  # no unit computed twice
                o_all[b0:b1, :, g0 * g:g1 * g] = o
                lse_all[b0:b1, g0 * g:g1 * g] = lse
        o_ref, lse_ref = oracle.attn_fwd(q, k, v, True, 0.3)
        np.save(os.path.join(out_dir, "o_all.npy"), o_all)
        np.save(os.path.join(out_dir, "o_ref.npy"), o_ref)
        np.save(os.path.join(out_dir, "lse_all.npy"), lse_all)
        np.save(os.path.join(out_dir, "lse_ref.npy"), lse_ref)


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_call_reassembles_on_gloo_ranks(tmp_path, world):
    import torch.multiprocessing as mp
    port = _free_port()
    mp.start_processes(_shard_worker, args=(world, port, str(tmp_path)), nprocs=world, start_method="spawn",
                       join=True)
    o_all, o_ref = np.load(tmp_path / "o_all.npy"), np.load(tmp_path / "o_ref.npy")
    lse_all, lse_ref = np.load(tmp_path / "lse_all.npy"), np.load(tmp_path / "lse_ref.npy")
    assert not np.isnan(o_all).any()  # every unit computed by some rank
    assert np.array_equal(o_all, o_ref) and np.array_equal(lse_all, lse_ref)
