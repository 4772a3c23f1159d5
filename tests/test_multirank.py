"""Multi-process (gloo, world size 2, CPU) checks of the benchmark's rank
logic: the head split (each rank's contiguous head range, its inputs equal to
those heads' inputs in the whole workload, and the per-rank outputs
reassembled in rank order equal to the whole workload's), independent
per-rank inputs of the batch split (weak scaling, no data-path collective),
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


def _head_worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank), VSA_BENCH_BACKEND="gloo")
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import torch
    import torch.distributed as dist
    import bench
    import oracle
    import workloads as W
    bench.dist_init()
    w = W.tiny_routing()                       # 4 heads, B = 2, structured q/k draws
    ws = bench.rank_shard(w, rank, world, "heads")
    lo, hi = bench.head_range(w.heads, rank, world)
    q, k, v = (W.full_tensor(ws, x) for x in "qkv")
    o = np.zeros((w.B, ws.heads, w.N, w.D))
    for b in range(w.B):
        for h in range(ws.heads):
            o[b, h], _ = oracle.attention_rows(ws.specs[h], (w.T, w.H, w.W), w.unit, w.D, w.scale,
                                               q[b, h], k[b, h], v[b, h], np.arange(w.N), 2)
    parts = [torch.zeros_like(torch.from_numpy(o)) for _ in range(world)]
    dist.all_gather(parts, torch.from_numpy(o))
    total = bench.sum_over_ranks(float(ws.heads), world)
    dist.destroy_process_group()
    if rank == 0:
        np.save(os.path.join(out_dir, "o.npy"), torch.cat(parts, dim=1).numpy())
    with open(os.path.join(out_dir, f"h{rank}.json"), "w") as f:
        json.dump({"range": [lo, hi], "heads": ws.heads, "offset": ws.head_offset, "total": total}, f)


def test_two_ranks_head_split_reassembles_the_whole_workload():
    import torch.multiprocessing as mp
    import oracle
    import workloads as W
    world = 2
    w = W.tiny_routing()
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_head_worker, args=(world, _free_port(), d), nprocs=world, join=True,
                           start_method="spawn")
        r = [json.load(open(os.path.join(d, f"h{i}.json"))) for i in range(world)]
        o_ranks = np.load(os.path.join(d, "o.npy"))
    assert [x["range"] for x in r] == [[0, 2], [2, 4]]
    assert [x["offset"] for x in r] == [0, 2] and all(x["total"] == 4 for x in r)
    q, k, v = (W.full_tensor(w, x) for x in "qkv")
    for b in range(w.B):
        for h in range(w.heads):
            o, _ = oracle.attention_rows(w.specs[h], (w.T, w.H, w.W), w.unit, w.D, w.scale,
                                         q[b, h], k[b, h], v[b, h], np.arange(w.N), 2)
            assert (o_ranks[b, h] == o).all(), (b, h)


def test_head_ranges_cover_every_head_once():
    import bench
    for heads in (1, 10, 24, 40):
        for world in range(1, min(heads, 8) + 1):
            rs = [bench.head_range(heads, r, world) for r in range(world)]
            assert rs[0][0] == 0 and rs[-1][1] == heads
            assert all(a[1] == b[0] for a, b in zip(rs, rs[1:]))
            assert all(hi > lo for lo, hi in rs)
    with pytest.raises(ValueError):
        bench.head_range(4, 0, 8)
