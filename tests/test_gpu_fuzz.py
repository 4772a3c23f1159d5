"""GPU: randomised grids, units, tile shapes and mask parameters (seeded).
Every tile map must equal the oracle's bit for bit; on a subset the attention
output of sampled rows must be within the tolerance of the oracle."""
import numpy as np
import pytest

import oracle
import workloads as W
from _helpers import TOL_MAX, TOL_MEAN, torch_bf16

pytestmark = pytest.mark.gpu

S = W.mask_spec


def _random_spec(g, T, H, Wd):
    kind = ["full", "spatial", "temporal", "sta", "stripe"][int(g.integers(0, 5))]
    sink = int(g.integers(0, 2))
    if kind == "full":
        spec = S("full", sink, layout=int(g.integers(0, 2)), tile_round=int(g.integers(0, 2)))
    elif kind == "spatial":
        spec = S("spatial", sink, rt=int(g.integers(0, T + 1)), tile_round=int(g.integers(0, 2)))
    elif kind == "temporal":
        spec = S("temporal", sink, rh=int(g.integers(0, H + 1)), rw=int(g.integers(0, Wd + 1)),
                 layout=int(g.integers(0, 2)), tile_round=int(g.integers(0, 2)))
    elif kind == "sta":
        spec = S("sta", sink, kt=int(g.integers(1, 4)), kh=int(g.integers(1, 4)), kw=int(g.integers(1, 4)))
    else:
        spec = S("stripe", sink, Tw=int(g.integers(1, 3)), To=int(g.integers(0, 3)), Ts=int(g.integers(1, 5)),
                 Sw=int(g.integers(1, 2 * H * Wd + 1)), So=int(g.integers(0, H * Wd)),
                 Ss=int(g.integers(1, 2 * H * Wd + 1)))
    return spec


def _cases(n, seed):
    import block_sparse_attention_mask_b200 as vsa
    g = np.random.Generator(np.random.PCG64(seed))
    out = []
    while len(out) < n:
        T, H, Wd = int(g.integers(1, 6)), int(g.integers(1, 20)), int(g.integers(1, 24))
        unit = (int(g.integers(1, 3)), int(g.integers(1, 9)), int(2 ** g.integers(0, 5)))
        qt, kt = int(g.choice([64, 128, 256])), int(g.choice([64, 128]))
        specs = [_random_spec(g, T, H, Wd) for _ in range(int(g.integers(1, 4)))]
        try:
            vsa.vsa_layout_info(len(specs), (T, H, Wd), unit, qt, kt)
        except vsa.VsaError:
            continue                                  # tile shape that does not fit the unit
        out.append(((T, H, Wd), unit, qt, kt, specs))
    return out


CASES = _cases(150, 2024)


@pytest.mark.parametrize("i", range(len(CASES)))
def test_random_tile_maps_and_rows(i):
    import torch
    import block_sparse_attention_mask_b200 as vsa
    grid, unit, qt, kt, specs = CASES[i]
    plan = vsa.Plan(specs, grid, unit, qt, kt)
    gmap = plan.tile_map()
    for h, spec in enumerate(specs):
        fn = oracle.rounded_tile_map if spec["tile_round"] else oracle.tile_map
        ref = fn(spec, grid, unit, plan.n_slots, qt, kt)
        assert np.array_equal(gmap[h], ref), f"case {i} head {h}: {spec}"
    if i % 3 == 0:
        D = 64 if i % 2 else 128
        N = int(np.prod(grid))
        g = np.random.Generator(np.random.PCG64(i))
        x = [W.bf16_bits_from_f32(g.standard_normal((1, len(specs), N, D), dtype=np.float32)) for _ in range(3)]
        o, _ = vsa.attention(plan, *(torch_bf16(t) for t in x), scale=D ** -0.5)
        torch.cuda.synchronize()
        plan.check()
        o = o.float().cpu().numpy()
        rows = np.unique(np.linspace(0, N - 1, min(N, 24)).astype(np.int64))
        for h, spec in enumerate(specs):
            if spec["tile_round"]:
                ref, _ = oracle.attention_rows_rounded(spec, grid, unit, plan.n_slots, qt, kt, D, D ** -0.5,
                                                       x[0][0, h], x[1][0, h], x[2][0, h], rows)
            else:
                ref, _ = oracle.attention_rows(spec, grid, unit, D, D ** -0.5, x[0][0, h], x[1][0, h], x[2][0, h],
                                               rows)
            err = np.abs(o[0, h][rows] - ref)
            assert err.max() <= TOL_MAX and err.mean() <= TOL_MEAN, (i, h, spec, err.max(), err.mean())
    plan.close()


def _route_cases(n, seed):
    g = np.random.Generator(np.random.PCG64(seed))
    out = []
    for _ in range(n):
        T, H, Wd = int(g.integers(1, 6)), int(g.integers(1, 12)), int(g.integers(1, 20))
        heads = int(g.integers(1, 4))
        sp = [S("spatial", int(g.integers(0, 2)), rt=int(g.integers(0, T))) for _ in range(heads)]
        tm = [S("temporal", int(g.integers(0, 2)), rh=int(g.integers(0, H)), rw=int(g.integers(0, Wd)),
                layout=int(g.integers(0, 2))) for _ in range(heads)]
        structure = tuple(["", "frame", "position"][int(g.integers(0, 3))] for _ in range(heads))
        out.append(((T, H, Wd), heads, int(g.choice([64, 128])), int(g.integers(1, 3)), sp, tm, structure,
                    float(g.uniform(0.02, 1.0))))
    return out


ROUTE_CASES = _route_cases(40, 77)


@pytest.mark.parametrize("i", range(len(ROUTE_CASES)))
def test_random_routing(i):
    import torch
    import block_sparse_attention_mask_b200 as vsa
    grid, heads, D, B, sp, tm, structure, frac = ROUTE_CASES[i]
    T, H, Wd = grid
    w = W.Workload(f"route_fuzz_{i}", B, T, H, Wd, heads, D, (1, 8, 16), 128, 128, tuple(sp),
                   structure=structure, structure_amp=6.0, route_specs=tuple(zip(sp, tm)))
    x = [W.full_tensor(w, c) for c in "qkv"]
    rows = W.route_rows(w.N, frac, seed=i)
    plan = vsa.Plan(list(sp), grid, w.unit, 128, 128)
    plan.set_route_candidates(sp, tm)
    err, flags = vsa.svg_route(plan, *(torch_bf16(t) for t in x),
                               torch.as_tensor(rows.astype(np.int32)).cuda(), scale=w.scale)
    torch.cuda.synchronize()
    plan.check()
    err_g, flags_g = err.cpu().numpy().astype(np.float64), flags.cpu().numpy()
    err_o, flags_o = oracle.svg_route(sp, tm, grid, D, w.scale, *x, rows)
    eps = 5e-3
    tol = 2.0 * np.sqrt(err_o) * eps + eps * eps
    assert np.all(np.abs(err_g - err_o) <= tol), (i, err_g, err_o)
    assert np.array_equal(flags_g, (err_g[:, 1] < err_g[:, 0]).astype(flags_g.dtype))
    decisive = np.abs(err_o[:, 0] - err_o[:, 1]) > tol[:, 0] + tol[:, 1]
    assert np.array_equal(flags_g[decisive], flags_o[decisive]), (i, flags_g, flags_o)
    plan.close()


@pytest.mark.parametrize("seed", range(12))
def test_random_exchange(seed):
    import torch
    import block_sparse_attention_mask_b200 as vsa
    g = np.random.Generator(np.random.PCG64(1000 + seed))
    world = int(g.integers(1, 9))
    hpr = int(g.integers(1, 3))
    grid = (int(g.integers(1, 5)), int(g.integers(1, 17)), int(g.integers(1, 21)))
    N = int(np.prod(grid))
    if N < world:
        grid = (world, grid[1], grid[2])
        N = int(np.prod(grid))
    D, B = int(g.choice([64, 128])), int(g.integers(1, 3))
    specs = [_random_spec(g, *grid) for _ in range(world * hpr)]
    unit = (1, 8, 8)
    plans = [vsa.Plan(specs[r * hpr:(r + 1) * hpr], grid, unit, 128, 128) for r in range(world)]
    n_slots = plans[0].n_slots
    layout = torch.tensor([s["layout"] for s in specs], dtype=torch.int32, device="cuda")
    perms = [oracle.tile_major_order(grid, unit, n_slots, layout=s["layout"]) for s in specs]
    x = W.bf16_bits_from_f32(g.standard_normal((B, world * hpr, N, D), dtype=np.float32))
    shards, head_local = oracle.ulysses_exchange(x, world)
    dst = [torch.full((B, hpr, n_slots, D), 3.0, dtype=torch.bfloat16, device="cuda") for _ in range(world)]
    for r in range(world):
        vsa.vsa_ulysses_permute(plans[r].handle, torch_bf16(shards[r]), B, D, r, world, layout, dst)
    torch.cuda.synchronize()
    for r in range(world):
        want = oracle.layout_gather(head_local[r], perms[r * hpr:(r + 1) * hpr])
        assert np.array_equal(dst[r].cpu().view(torch.int16).numpy().view(np.uint16), want), (seed, r)
    off = oracle.shard_offsets(N, world)
    outs = [torch.full((B, off[r + 1] - off[r], world * hpr, D), 3.0, dtype=torch.bfloat16, device="cuda")
            for r in range(world)]
    for r in range(world):
        vsa.vsa_ulysses_unpermute(plans[r].handle, dst[r], B, D, r, world, layout, outs)
    torch.cuda.synchronize()
    # the round trip returns every shard unchanged
    for r in range(world):
        assert np.array_equal(outs[r].cpu().view(torch.int16).numpy().view(np.uint16), shards[r]), (seed, r)
    for p in plans:
        p.close()
