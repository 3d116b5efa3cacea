"""The multi-rank host logic of bench.py with two gloo ranks on CPU.

The decode path needs no data collective. Each rank decodes its own batch
(weak scaling), and the only cross-rank step is combining timings: the job's
time is the slowest rank's, and its throughput counts the bytes of all ranks.
"""

import json
import os
import socket
from datetime import timedelta

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=timedelta(seconds=60))
    try:
        import bench
        from pkv_inputs import make_case
        from pkv_inputs.workloads import WORKLOADS
        # per-rank timings: rank 1 is slower on the first entry, rank 0 on the second
        got = bench.max_over_ranks([1.0 + rank, 5.0 - rank], torch.device("cpu"))
        seed = bench.rank_seed(WORKLOADS["tiny_f32"]["seed"], rank)
        case = make_case("tiny_f32", seed=seed)
        res = {"rank": rank, "max": got, "seed": seed,
               "q0": float(case.q.flatten()[0]),
               "gbs": bench.whole_job_gbs(4_000_000_000, world, got[0])}
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump(res, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_combine_timings_and_decode_different_batches(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    r = [json.load(open(tmp_path / f"r{i}.json")) for i in range(world)]
    for x in r:
        assert x["max"] == [2.0, 5.0]            # element-wise max over the ranks
        assert abs(x["gbs"] - 4.0) < 1e-12        # 2 ranks x 4 GB / 2 s
    assert r[0]["seed"] != r[1]["seed"]           # weak scaling: one batch per rank
    assert r[0]["q0"] != r[1]["q0"]


def test_single_process_needs_no_collective():
    import bench
    assert not dist.is_initialized()
    assert bench.max_over_ranks([3.0, 1.0], torch.device("cpu")) == [3.0, 1.0]
    assert bench.whole_job_gbs(2_000_000_000, 1, 1.0) == 2.0


def test_reference_arm_only_on_rank_zero():
    import bench

    class A:
        steps, warmup, workload, num_seqs, gpus = 1, 0, "tiny_f32", None, 2

    assert bench.run_reference(A(), rank=1, world=2) is None
