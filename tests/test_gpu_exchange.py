"""GPU: the head-sharded exchange kernels, with every rank's buffers on one
GPU (the kernels only store; a rank's peer pointers are here plain local
pointers).  Each emulated rank scatters its sequence shard into the owners'
slot-ordered buffers; they must equal, bit for bit, the oracle's exchange
followed by each head's slot order (padding zero).  Attention per rank and
the inverse exchange must give, bit for bit, the single-plan path's output
cut into sequence shards."""
import numpy as np
import pytest

import oracle
import workloads as W
from _helpers import torch_bf16

pytestmark = pytest.mark.gpu

S = W.mask_spec


def _specs(hpr, world):
    pool = [S("spatial", 1, rt=1), S("temporal", 1, rh=2, rw=3, layout=1), S("full"),
            S("temporal", 0, rh=1, rw=2), S("spatial", 0, rt=0), S("temporal", 1, rh=1, rw=1, layout=1),
            S("full", 0, layout=1), S("stripe", 1, Tw=1, To=0, Ts=2, Sw=5, So=1, Ss=11)]
    return [pool[i % len(pool)] for i in range(hpr * world)]


@pytest.mark.parametrize("world,grid,D,B", [(2, (4, 9, 11), 128, 2), (4, (3, 16, 20), 64, 1),
                                            (8, (2, 8, 16), 128, 1)])
def test_exchange_emulated_ranks(world, grid, D, B):
    import torch
    import block_sparse_attention_mask_b200 as vsa
    hpr = 2
    specs = _specs(hpr, world)
    Hh = hpr * world
    unit, qt, kt = (1, 8, 8), 128, 128
    T, H, Wd = grid
    N = T * H * Wd
    g = np.random.Generator(np.random.PCG64(5))
    full = {x: W.bf16_bits_from_f32(g.standard_normal((B, Hh, N, D), dtype=np.float32)) for x in "qkv"}
    plans = [vsa.Plan(specs[r * hpr:(r + 1) * hpr], grid, unit, qt, kt) for r in range(world)]
    n_slots = plans[0].n_slots
    layout = torch.tensor([s["layout"] for s in specs], dtype=torch.int32, device="cuda")
    perms = [oracle.tile_major_order(grid, unit, n_slots, layout=s["layout"]) for s in specs]

    tiled = {}
    for x in "qkv":
        shards, head_local = oracle.ulysses_exchange(full[x], world)
        dst = [torch.full((B, hpr, n_slots, D), 7.0, dtype=torch.bfloat16, device="cuda") for _ in range(world)]
        for r in range(world):
            vsa.vsa_ulysses_permute(plans[r].handle, torch_bf16(shards[r]), B, D, r, world, layout, dst)
        torch.cuda.synchronize()
        for r in range(world):
            want = oracle.layout_gather(head_local[r], perms[r * hpr:(r + 1) * hpr])
            got = dst[r].cpu().view(torch.int16).numpy().view(np.uint16)
            assert np.array_equal(got, want), f"{x}: rank {r} buffer"
        tiled[x] = dst

    outs = [torch.full((B, oracle.shard_offsets(N, world)[r + 1] - oracle.shard_offsets(N, world)[r], Hh, D),
                       7.0, dtype=torch.bfloat16, device="cuda") for r in range(world)]
    for r in range(world):
        o_r, _ = vsa.sparse_attn_fwd(plans[r], tiled["q"][r], tiled["k"][r], tiled["v"][r])
        vsa.vsa_ulysses_unpermute(plans[r].handle, o_r, B, D, r, world, layout, outs)
    torch.cuda.synchronize()
    for p in plans:
        p.check()

    plan_all = vsa.Plan(specs, grid, unit, qt, kt)
    o_all, _ = vsa.attention(plan_all, *(torch_bf16(full[x]) for x in "qkv"))
    torch.cuda.synchronize()
    o_all = o_all.cpu().view(torch.int16).numpy().view(np.uint16)
    want_shards, _ = oracle.ulysses_exchange(o_all, world)
    for r in range(world):
        got = outs[r].cpu().view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(got, want_shards[r]), f"output shard {r}"
    for p in plans + [plan_all]:
        p.close()


def test_exchange_rejects_bad_arguments():
    import torch
    import block_sparse_attention_mask_b200 as vsa
    plan = vsa.Plan([S("full")] * 2, (2, 8, 8), (1, 8, 8), 128, 128)
    x = torch.zeros((1, 64, 4, 128), dtype=torch.bfloat16, device="cuda")
    lay = torch.zeros(4, dtype=torch.int32, device="cuda")
    dst = [torch.zeros((1, 2, plan.n_slots, 128), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    for rank, world in ((2, 2), (-1, 2), (0, 9), (0, 0)):
        with pytest.raises(vsa.VsaError):
            vsa.vsa_ulysses_permute(plan.handle, x, 1, 128, rank, world, lay, dst)
    with pytest.raises(vsa.VsaError):
        vsa.vsa_ulysses_permute(plan.handle, x, 1, 96, 0, 2, lay, dst)
    with pytest.raises(vsa.VsaError):
        vsa.vsa_ulysses_unpermute(plan.handle, x, 1, 128, 0, 2, lay, [dst[0], 0])
    plan.close()
