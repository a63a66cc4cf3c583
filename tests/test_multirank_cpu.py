"""The N > 1 host path of bench.py, as two gloo ranks on the CPU.

Each rank runs the whole workload on its own seeded inputs (weak scaling), the
timings are reduced to the slowest rank, and the value is all ranks' work over that
time.  The reference arm runs on rank 0 only.  No GPU is involved.
"""
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


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    from quantized_attention_fine_b200 import workloads as wl
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        # per-rank inputs: same shapes, different seeds
        w = wl.custom("mr", 1, 2, 160, 160, 64, True, recipe="llm")
        wr = bench.rank_workload(w, rank)
        q, _, _ = wl.generate(wr)
        # rank r reports (10 + r, 3 - r) ms: the reduction must give (10 + world - 1, 3)
        got = bench.max_over_ranks([10.0 + rank, 3.0 - rank])
        # the reference arm does its work on rank 0 only; other ranks return at once
        class _A:
            steps, warmup, cpu_seconds = 1, 0, 0.01
        ref_rc = bench.reference_arm(_A(), w) if rank != 0 else 0
        torch.save({"seed": wr.seed, "q_sum": float(q.float().sum()), "max": got, "ref_rc": ref_rc},
                   os.path.join(out_dir, "rank%d.pt" % rank))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    r = [torch.load(os.path.join(tmp_path, "rank%d.pt" % i)) for i in range(world)]
    assert r[0]["seed"] != r[1]["seed"] and r[0]["q_sum"] != r[1]["q_sum"]
    for x in r:
        assert x["max"] == [11.0, 3.0]
    assert r[1]["ref_rc"] == 0


def test_whole_job_value_is_all_ranks_work_over_slowest_time():
    sys.path.insert(0, ROOT)
    import bench
    # 2 ranks x 8.80 TOPs per step in 10 ms (the slower rank) = 1760 TOPS
    assert bench.whole_job_tops(2, 8.8e12, 10.0) == pytest.approx(1760.0)
    assert bench.whole_job_tops(1, 8.8e12, 10.0) == pytest.approx(880.0)
