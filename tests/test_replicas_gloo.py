"""The multi-process (replica) plumbing of bench.py on CPU: two ranks over gloo.

The decode step has no exchange between GPUs, so N GPUs run N independent
replicas; what crosses ranks is only the timing (the slowest rank's time is the
job's).  These tests run that host logic with world size 2 on the gloo backend."""
import argparse
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_path):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        cpu = torch.device("cpu")
        # each rank brings its own time; all get the slowest
        slowest = bench.max_over_ranks(1.5 + rank, world, cpu)
        job = bench.job_us_per_step(slowest, world)
        # replicas draw different inputs (seeded by rank)
        prob = bench.make_workload("qwen3_stack_64x2", cpu, seed_offset=rank)
        qsum = float(prob.q.float().sum())
        sums = [None] * world
        dist.all_gather_object(sums, qsum)
        # the reference arm runs on rank 0 only; other ranks return at once
        args = argparse.Namespace(workload="qwen3_stack_64x2", steps=1, warmup=0)
        ref = bench.run_reference(args, rank, world) if rank != 0 else None
        with open(f"{out_path}.{rank}", "w") as f:
            f.write(repr((slowest, job, sums, ref)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_distinct_inputs(tmp_path):
    world = 2
    out = str(tmp_path / "res")
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world,
                       start_method="spawn", join=True)
    res = [eval(open(f"{out}.{r}").read()) for r in range(world)]
    for slowest, job, sums, ref in res:
        assert slowest == 2.5                       # max over ranks
        assert job == pytest.approx(2.5e3 / world)  # µs per decode step of the job
        assert sums[0] != sums[1]                   # each replica has its own inputs
        assert ref is None
    assert res[0][2] == res[1][2]


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, 1, torch.device("cpu")) == 3.25
    assert bench.job_us_per_step(3.25, 1) == pytest.approx(3250.0)


def test_step_spread_uses_nearest_rank():
    sys.path.insert(0, ROOT)
    import bench
    xs = sorted([5.0, 1.0, 2.0, 3.0, 4.0, 6.0, 7.0, 8.0, 9.0, 10.0])
    assert (bench.nearest_rank(xs, 0.1), bench.nearest_rank(xs, 0.5),
            bench.nearest_rank(xs, 0.9)) == (1.0, 5.0, 9.0)
    assert bench.nearest_rank([3.0], 0.9) == 3.0


def test_union_rows_counts_each_group_row_once():
    """The roofline's algorithmic bytes: n_b rows for a group with a retrieval
    head, the size of the union of the heads' sets otherwise (sets end at their
    first -1), counted here by brute force over Python sets."""
    sys.path.insert(0, ROOT)
    import bench
    from types import SimpleNamespace
    g = torch.Generator().manual_seed(7)
    L, B, Hq, Hkv, d, N, k = 3, 2, 8, 2, 64, 40, 12
    G = Hq // Hkv
    seqlens = torch.tensor([40, 23], dtype=torch.int32)
    kb = [12, 6]
    roles = torch.zeros(L, Hq, dtype=torch.uint8)
    roles[0] = 1
    roles[1, 5] = 1                      # layer 1: group 1 dense, group 0 sparse-only
    idx = torch.full((L, B, Hq, k), -1, dtype=torch.int32)
    for l in range(L):
        for b in range(B):
            for h in range(Hq):
                # some sets end early at their first -1, one holds more than k_b
                m = kb[b] - (h % 3) if h != 6 else min(k, int(seqlens[b]))
                pos = torch.randperm(int(seqlens[b]), generator=g)[:m].sort().values
                idx[l, b, h, :m] = pos.int()
    prob = SimpleNamespace(shape=(L, B, Hq, Hkv, d, N), roles=roles, seqlens=seqlens,
                           meta={"kb": kb})
    union, literal, dense = bench.union_rows(prob, idx)
    for l in range(L):
        want_u = want_l = 0
        for b in range(B):
            n = int(seqlens[b])
            for grp in range(Hkv):
                hs = range(grp * G, grp * G + G)
                if any(int(roles[l, h]) for h in hs):
                    want_u += n
                    want_l += n
                else:
                    rows = set()
                    for h in hs:
                        for x in idx[l - 1, b, h].tolist():
                            if x < 0:
                                break
                            rows.add(x)
                    want_u += len(rows)
                    want_l += kb[b]
        assert union[l] == want_u and literal[l] == want_l
        assert dense[l] == Hkv * int(seqlens.sum())


@pytest.mark.parametrize("block", [0, 32])
def test_reference_arm_on_rank0_prints_the_contract_keys(block):
    sys.path.insert(0, ROOT)
    import bench
    args = argparse.Namespace(workload="qwen3_stack_256x2", steps=2, warmup=0, block=block)
    res = bench.run_reference(args, 0, 1)
    assert res["impl"] == "reference" and res["value"] > 0 and not res["higher_is_better"]
    assert res["e2e"]["value"] == res["value"] and res["cpu_baseline"]["kind"] == "oracle"
    assert res["config"]["select"] == ("argsTopK" if block == 0 else "blocks of 32")
    assert "all 2 layers" in res["cpu_baseline"]["sample"]


def test_cpu_baseline_leg_runs_on_host_tensors():
    sys.path.insert(0, ROOT)
    import bench
    prob = bench.make_workload("qwen3_stack_256x3", torch.device("cpu"))
    cb = bench.cpu_baseline(prob, block=32, single_layers=2)
    assert cb["kind"] == "oracle" and cb["value"] > 0 and cb["cores"] >= 1
    assert "all 3 layers" in cb["sample"] and cb["cpu_model"]
    assert cb["single_thread"]["cores"] == 1 and "layers 0..1" in cb["single_thread"]["sample"]
