"""The N > 1 host path of bench.py, as two gloo ranks on the CPU.

Each rank computes a disjoint slice of one seeded global problem, split by heads
(weak: one batch block per rank; strong: the workload's key/value head groups split
into contiguous ranges).  The oracle run on each rank's slice, put back together,
equals the oracle run on the whole global problem bit for bit, with every head
computed exactly once.  The timings are reduced to the slowest rank, and the value is
all ranks' work over that time.  The reference arm runs on rank 0 only.  No GPU is
involved.
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


def _strong_workload():
    from quantized_attention_fine_b200 import workloads as wl
    # 4 query heads over 2 key/value heads: a rank takes one key/value head group
    return wl.custom("mr_gqa", 1, 4, 150, 200, 64, True, recipe="llm", H_kv=2, seed=777)


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    from quantized_attention_fine_b200 import workloads as wl
    from datetime import timedelta
    global _STRONG
    _STRONG = _strong_workload()
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
        # this rank's slice of the global problem, through the oracle
        import oracle
        slices = {}
        for scaling, wg in (("weak", w), ("strong", _STRONG)):
            sub, qs, ks, vs = bench.rank_inputs(wg, world, rank, scaling)
            o = oracle.sage_attention(*(x.double().numpy() for x in (qs, ks, vs)), causal=wg.causal)
            slices[scaling] = (sub.B, sub.H, sub.Hk, torch.from_numpy(o))
        torch.save({"seed": wr.seed, "q_sum": float(q.float().sum()), "max": got, "ref_rc": ref_rc,
                    "slices": slices}, os.path.join(out_dir, "rank%d.pt" % rank))
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
    # the slices tile the global problem: concatenated, they equal the oracle on the
    # whole global problem, and together they cover each head once
    sys.path.insert(0, ROOT)
    import numpy as np
    import bench
    import oracle
    from quantized_attention_fine_b200 import workloads as wl
    w = wl.custom("mr", 1, 2, 160, 160, 64, True, recipe="llm")
    gq, gk, gv = bench.global_inputs(w, world, "weak")
    assert gq.shape[0] == world * w.B
    full = oracle.sage_attention(*(x.double().numpy() for x in (gq, gk, gv)), causal=True)
    got = np.concatenate([x["slices"]["weak"][3].numpy() for x in r], axis=0)
    assert np.array_equal(got, full)
    ws_ = _strong_workload()
    gq, gk, gv = bench.global_inputs(ws_, world, "strong")
    full = oracle.sage_attention(*(x.double().numpy() for x in (gq, gk, gv)), causal=True)
    heads = [x["slices"]["strong"] for x in r]
    assert [(b, h, hk) for b, h, hk, _ in heads] == [(1, 2, 1)] * world   # 2 query heads over 1 kv head each
    got = np.concatenate([o.numpy() for _, _, _, o in heads], axis=1)
    assert got.shape == full.shape and np.array_equal(got, full)


def test_unit_range_covers_every_unit_once():
    sys.path.insert(0, ROOT)
    import bench
    for n, world in ((32, 1), (32, 2), (32, 8), (96, 4), (8, 8)):
        seen = [u for r in range(world) for u in range(*bench.unit_range(n, world, r))]
        assert seen == list(range(n))
    with pytest.raises(ValueError):
        bench.unit_range(32, 3, 0)


def test_whole_job_value_is_all_ranks_work_over_slowest_time():
    sys.path.insert(0, ROOT)
    import bench
    # 2 ranks x 8.80 TOPs per step in 10 ms (the slower rank) = 1760 TOPS
    assert bench.whole_job_tops(2, 8.8e12, 10.0) == pytest.approx(1760.0)
    assert bench.whole_job_tops(1, 8.8e12, 10.0) == pytest.approx(880.0)
