"""The head-sharded exchange definition of the oracle against a real
collective: world_size 2 and 4 gloo ranks on the CPU run all_to_all on their
sequence shards and must end up with exactly the oracle's head-local data
("Sparse VideoGen: accelerating video diffusion attention on TPU",
"performing layout transformation on local heads")."""
import os
import socket

import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.timeout(300)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, B, Hh, N, D, q):
    import torch
    import torch.distributed as dist
    try:
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        g = np.random.Generator(np.random.PCG64(3))
        x = g.standard_normal((B, Hh, N, D)).astype(np.float32)
        shards, head_local = oracle.ulysses_exchange(x, world)
        off = oracle.shard_offsets(N, world)
        hpr = Hh // world
        mine = torch.from_numpy(shards[rank])                      # [B, n_r, Hh, D]
        # to every rank g: this shard's rows of g's heads
        send = [mine[:, :, g * hpr:(g + 1) * hpr].reshape(-1) for g in range(world)]
        rsz = [B * (off[r + 1] - off[r]) * hpr * D for r in range(world)]
        recv = torch.empty(sum(rsz))
        dist.all_to_all_single(recv, torch.cat(send), output_split_sizes=rsz,
                               input_split_sizes=[t.numel() for t in send])
        parts = torch.split(recv, rsz)
        got = torch.cat([parts[r].reshape(B, off[r + 1] - off[r], hpr, D) for r in range(world)], dim=1)
        got = got.permute(0, 2, 1, 3).numpy()                      # [B, hpr, N, D]
        ok = np.array_equal(got, head_local[rank])
        q.put((rank, ok))
        dist.destroy_process_group()
    except Exception as e:  # pragma: no cover - reported to the parent
        q.put((rank, repr(e)))


@pytest.mark.parametrize("world,N", [(2, 37), (4, 30)])
def test_exchange_definition_matches_gloo_all_to_all(world, N):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, 2, 2 * world, N, 8, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    assert all(v is True for v in res.values()), res
