"""GPU parity on small grids: every row, every tile, every head.

Grids span several tiles, include ragged tails (slots past the padded grid),
partial units at the grid edge, every mask family with and without the sink,
q tiles of 64/128/256, kv tiles of 64/128 and head dims 64/128.  Tile maps and
permutations must match the oracle bit for bit; outputs within the tolerance.
"""
import numpy as np
import pytest

import oracle
import workloads as W
from _helpers import PathRun, torch_bf16

pytestmark = pytest.mark.gpu

S = W.mask_spec

CASES = {
    # name: (grid, unit, Bq, Bk, D, specs)
    "mixed_1x8x16": ((5, 13, 20), (1, 8, 16), 128, 128, 128,
                     [S("spatial", 1, rt=1), S("temporal", 1, rh=2, rw=3),
                      S("stripe", 1, Tw=2, To=1, Ts=3, Sw=20, So=5, Ss=47), S("full"),
                      S("sta", 0, kt=3, kh=1, kw=1), S("stripe", 0, Tw=1, To=0, Ts=2, Sw=7, So=0, Ss=9)]),
    "token_units_ragged_tail": ((3, 7, 9), (1, 1, 1), 128, 128, 64,
                                [S("temporal", 1, rh=1, rw=1),
                                 S("stripe", 1, Tw=1, To=1, Ts=2, Sw=3, So=2, Ss=5),
                                 S("spatial", 0, rt=0)]),
    "q64_k64_deep_units_tail": ((6, 9, 17), (2, 4, 8), 64, 64, 128,
                                [S("spatial", 0, rt=0),
                                 S("stripe", 1, Tw=2, To=0, Ts=3, Sw=9, So=4, Ss=20),
                                 S("sta", 1, kt=1, kh=3, kw=3), S("temporal", 0, rh=3, rw=2)]),
    "q256_k128_d64": ((4, 16, 32), (1, 8, 16), 256, 128, 64,
                      [S("temporal", 1, rh=2, rw=5), S("stripe", 1, Tw=1, To=0, Ts=4, Sw=40, So=16, Ss=100),
                       S("full")]),
    # 256-row q tiles run as two 128-row sub-tiles of one CTA
    "q256_k128_mixed": ((5, 13, 20), (1, 8, 16), 256, 128, 128,
                        [S("spatial", 1, rt=1), S("temporal", 1, rh=2, rw=3),
                         S("stripe", 1, Tw=2, To=1, Ts=3, Sw=20, So=5, Ss=47), S("full"),
                         S("sta", 0, kt=3, kh=1, kw=1), S("stripe", 0, Tw=1, To=0, Ts=2, Sw=7, So=0, Ss=9)]),
    "q256_k128_multibox": ((4, 16, 32), (1, 8, 8), 256, 128, 128,
                           [S("spatial", 1, rt=1), S("temporal", 1, rh=1, rw=2),
                            S("stripe", 1, Tw=1, To=0, Ts=4, Sw=40, So=16, Ss=100)]),
    "q256_k64_frame0_rounded": ((4, 9, 11), (1, 8, 8), 256, 64, 128,
                                [S("temporal", 1, rh=1, rw=2, layout=1), S("spatial", 0, rt=0, tile_round=1),
                                 S("full")]),
    "q256_token_units_tail": ((3, 7, 9), (1, 1, 1), 256, 128, 64,
                              [S("temporal", 1, rh=1, rw=1), S("stripe", 1, Tw=1, To=1, Ts=2, Sw=3, So=2, Ss=5),
                               S("spatial", 0, rt=0)]),
    "q128_k64_units_of_64": ((4, 16, 32), (1, 8, 8), 128, 64, 128,
                             [S("spatial", 1, rt=1), S("temporal", 1, rh=1, rw=1),
                              S("sta", 0, kt=3, kh=1, kw=3)]),
    "q64_k128_unit128": ((2, 8, 8), (2, 8, 8), 64, 128, 128,
                         [S("spatial", 0, rt=0), S("stripe", 1, Tw=1, To=1, Ts=5, Sw=3, So=0, Ss=8)]),
    "q64_k64_tiny_tail_half_empty": ((2, 3, 5), (1, 1, 1), 64, 64, 64,
                                     [S("temporal", 1, rh=1, rw=1), S("full")]),
    "no_kept_pairs": ((3, 8, 16), (1, 8, 16), 128, 128, 128,
                      [S("stripe", 0, Tw=1, To=9, Ts=1000, Sw=1, So=0, Ss=1000), S("spatial", 0, rt=0)]),
    "sta_sink_d64": ((6, 16, 16), (2, 8, 8), 128, 128, 64,
                     [S("sta", 1, kt=1, kh=1, kw=1), S("sta", 0, kt=3, kh=3, kw=3)]),
    # frame-0-first heads next to tile-major ones in one plan
    "frame0_first_mixed": ((5, 13, 20), (1, 8, 16), 128, 128, 128,
                           [S("temporal", 1, rh=2, rw=3, layout=1), S("temporal", 0, rh=1, rw=5, layout=1),
                            S("full", 0, layout=1), S("spatial", 1, rt=1)]),
    "frame0_first_q64_k64_d64": ((4, 9, 11), (1, 8, 8), 64, 64, 64,
                                 [S("temporal", 1, rh=1, rw=2, layout=1), S("temporal", 1, rh=0, rw=0, layout=1),
                                  S("temporal", 0, rh=2, rw=1)]),
    "frame0_first_ragged": ((3, 7, 9), (1, 1, 1), 128, 64, 64,
                            [S("temporal", 1, rh=1, rw=1, layout=1), S("full", 1, layout=1)]),
    "frame0_first_one_frame": ((1, 8, 16), (1, 8, 16), 128, 128, 128,
                               [S("temporal", 0, rh=1, rw=2, layout=1), S("temporal", 1, rh=1, rw=2, layout=1)]),
    # tile-aligned rounding (lossy mode), next to exact heads
    "rounded_mixed": ((5, 13, 20), (1, 8, 16), 128, 128, 128,
                      [S("temporal", 1, rh=2, rw=3, tile_round=1), S("spatial", 1, rt=1, tile_round=1),
                       S("temporal", 1, rh=1, rw=4, layout=1, tile_round=1), S("full", 0, tile_round=1),
                       S("temporal", 1, rh=2, rw=3)]),
    "rounded_q64_k64_d64": ((4, 9, 11), (1, 8, 8), 64, 64, 64,
                            [S("temporal", 0, rh=1, rw=2, tile_round=1), S("spatial", 0, rt=0, tile_round=1)]),
    "rounded_token_units": ((3, 7, 9), (1, 1, 1), 128, 64, 64,
                            [S("temporal", 1, rh=1, rw=1, tile_round=1), S("spatial", 1, rt=0, tile_round=1)]),
}


def _workload(name):
    grid, unit, Bq, Bk, D, specs = CASES[name]
    return W.Workload(name, 1, grid[0], grid[1], grid[2], len(specs), D, unit, Bq, Bk, tuple(specs),
                      seeds=(11, 12, 13))


@pytest.fixture(scope="module", params=sorted(CASES))
def run(request):
    w = _workload(request.param)
    r = PathRun(w)
    yield r
    r.close()


def test_tile_map_bit_exact(run):
    w = run.w
    gmap = run.plan.tile_map()
    for h in range(w.heads):
        fn = oracle.rounded_tile_map if w.specs[h].get("tile_round", 0) else oracle.tile_map
        ref = fn(w.specs[h], run.grid, w.unit, run.plan.n_slots, w.q_tile, w.kv_tile)
        assert (gmap[h] == ref).all(), f"head {h}: {np.argwhere(gmap[h] != ref)[:5]}"
    counts = run.plan.tile_counts()
    for h in range(w.heads):
        assert counts[h].tolist() == np.bincount(gmap[h].ravel(), minlength=3).tolist()


def test_exec_steps_follow_the_map(run):
    w = run.w
    gmap = run.plan.tile_map()
    steps = run.plan.exec_steps()
    for h in range(w.heads):
        nz = gmap[h] != 0
        if w.q_tile == 64:
            per_block = nz.reshape(-1, 2, nz.shape[1]).any(axis=1)
            want = int(per_block.sum())
        elif w.q_tile == 128:
            want = int(nz.sum())
        else:
            want = 2 * int(nz.sum())
        assert int(steps[h]) == want


def test_perm_matches_oracle(run):
    assert (run.plan.perm() == run.perm).all()
    for layout in (0, 1):
        want = oracle.tile_major_order(run.grid, run.w.unit, run.plan.n_slots, layout=layout)
        assert (run.plan.perm(layout=layout) == want).all()


def test_permute_bit_exact_and_round_trip(run):
    import torch
    import block_sparse_attention_mask_b200 as vsa
    w = run.w
    x = run.q
    xd = torch_bf16(x)
    xt = vsa.permute(run.plan, xd)
    got = xt.view(torch.int16).cpu().numpy().view(np.uint16)
    want = np.zeros((w.B, w.heads, run.plan.n_slots, w.D), dtype=np.uint16)
    for h in range(w.heads):
        real = run.perms[h] >= 0
        want[:, h, real] = x[:, h, run.perms[h][real]]
    assert (got == want).all()
    back = vsa.unpermute(run.plan, xt)
    assert torch.equal(back.view(torch.int16), xd.view(torch.int16))


def test_permute_qkv_matches_single_permutes(run):
    import torch
    import block_sparse_attention_mask_b200 as vsa
    xs = [torch_bf16(x) for x in (run.q, run.k, run.v)]
    fused = vsa.permute_qkv(run.plan, *xs)
    for x, f in zip(xs, fused):
        assert torch.equal(vsa.permute(run.plan, x).view(torch.int16), f.view(torch.int16))


def test_attention_all_rows(run):
    w = run.w
    for h in range(w.heads):
        run.check_rows(h, np.arange(w.N))


def test_attention_is_deterministic(run):
    import torch
    import block_sparse_attention_mask_b200 as vsa
    w = run.w
    q, k, v = (vsa.permute(run.plan, torch_bf16(x)) for x in (run.q, run.k, run.v))
    o1, l1 = vsa.sparse_attn_fwd(run.plan, q, k, v, w.scale)
    o2, l2 = vsa.sparse_attn_fwd(run.plan, q, k, v, w.scale)
    torch.cuda.synchronize()
    run.plan.check()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1, l2)


def test_plan_rebuild_is_identical(run):
    m1 = run.plan.tile_map()
    c1 = run.plan.tile_counts()
    run.plan.build()
    assert (run.plan.tile_map() == m1).all()
    assert (run.plan.tile_counts() == c1).all()


def test_kept_pairs_match_oracle(run):
    w = run.w
    kept = run.plan.kept_pairs()
    for h in range(w.heads):
        assert int(kept[h]) == oracle.kept_pairs(w.specs[h], run.grid, w.unit), f"head {h}"
