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
