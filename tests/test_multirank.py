"""Multi-process (gloo, world size 2, CPU) checks of the benchmark's rank
logic: independent per-rank inputs (weak scaling, no data-path collective),
the max-over-ranks step time, and the whole-job aggregate."""
import json
import os
import socket
import tempfile

import numpy as np
import pytest


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank), VSA_BENCH_BACKEND="gloo")
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    import workloads as W
    w_world, w_rank, _ = bench.dist_init()
    res = {"world": w_world, "rank": w_rank}
    # every rank contributes a different step time; all must see the maximum
    res["max_ms"] = bench.max_over_ranks(10.0 + 5.0 * rank, w_world)
    bench.barrier(w_world)
    wr = bench.rank_workload(W.tiny(), rank)
    res["seeds"] = list(wr.seeds)
    res["first_q_value"] = int(W.head_tensor(wr, "q", 0, 0)[0, 0])
    res["value"] = bench.aggregate_tflops(2.0e12, w_world, res["max_ms"])
    import torch.distributed as dist
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
        json.dump(res, f)


def test_two_ranks_weak_scaling_logic():
    import torch.multiprocessing as mp
    world = 2
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_worker, args=(world, _free_port(), d), nprocs=world, join=True,
                           start_method="spawn")
        r = [json.load(open(os.path.join(d, f"r{i}.json"))) for i in range(world)]
    assert [x["rank"] for x in r] == [0, 1] and all(x["world"] == 2 for x in r)
    assert all(x["max_ms"] == 15.0 for x in r)
    # ranks draw different inputs (their own batch element) of the same shape
    assert r[0]["seeds"] != r[1]["seeds"]
    assert r[0]["first_q_value"] != r[1]["first_q_value"]
    # 2 ranks x 2 TFLOP per step / 15 ms
    assert abs(r[0]["value"] - 2 * 2.0 / 0.015) < 1e-9


def test_single_rank_helpers():
    import bench
    import workloads as W
    w = W.svg_wan720p()
    assert bench.rank_workload(w, 0).seeds == w.seeds
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.aggregate_tflops(7.48e12, 1, 10.0) == pytest.approx(748.0)
