"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times (all heads, B = 1, the workload's tile shape).

Outputs are compared with the oracle on R = 512 stratified sampled rows per
head (frame 0, last frame, the padded edge, corners, rows of q tiles whose
executed kv tiles are all boundary or all full, uniform rows), each row exact
over all N keys, on every head of the SVG, STA and stripe workloads and on
the first and last head of each scaling grid (both of its masks).  Tile maps
are compared with the oracle's brute-force classes on sampled q-tile rows
here, and bit for bit on every head in ``test_gpu_full_maps.py``; their
per-head totals also with closed forms where one exists.
"""
import numpy as np
import pytest

import oracle
import workloads as W
from _helpers import PathRun, oracle_map_rows, parity_rows, sample_qtiles

pytestmark = pytest.mark.gpu

_INPUTS = {}


def _inputs(w):
    key = (w.T, w.H, w.W, w.heads, w.D, w.seeds)
    if key not in _INPUTS:
        _INPUTS.clear()
        _INPUTS[key] = tuple(W.full_tensor(w, x) for x in "qkv")
    return _INPUTS[key]


def _check(w, heads, rows_per_head, map_heads, qtiles_per_head=6):
    r = PathRun(w, _inputs(w))
    try:
        errs = []
        for h in heads:
            rows = np.arange(w.N) if rows_per_head >= w.N else parity_rows(w, h, rows_per_head)
            errs.append(r.check_rows(h, rows))
        gmap = r.plan.tile_map()
        for h in map_heads:
            qt = sample_qtiles(gmap.shape[1], qtiles_per_head, seed=h)
            ref = oracle_map_rows(w, h, r.plan.n_slots, qt)
            assert (gmap[h][qt] == ref).all(), f"head {h}"
        return r.plan.tile_counts(), errs
    finally:
        r.close()


def _spatial_closed_form(T, Bq, Bk):
    """Full / boundary tiles of one SVG spatial head (rt=1, sink) on T x 45 x 80.

    (4T-4) kept frame pairs; per frame the q tiles and the kv tiles split into
    those holding real rows only and those reaching the padded rows 45..47.
    """
    unit_w = 8 if min(Bq, Bk) == 64 else 16
    units = 6 * (80 // unit_w)                 # units per padded frame
    unit_tokens = 8 * unit_w
    q_per_frame = units * unit_tokens // Bq
    kv_per_frame = units * unit_tokens // Bk
    kv_padded = (80 // unit_w) * unit_tokens // Bk if Bk >= unit_tokens else (80 // unit_w)
    pairs = 4 * T - 4
    return pairs * q_per_frame * (kv_per_frame - kv_padded), pairs * q_per_frame * kv_padded


def test_tiny_all_rows():
    w = W.tiny()
    counts, _ = _check(w, range(w.heads), w.N, range(w.heads), qtiles_per_head=4)
    assert counts.tolist() == [[4, 0, 12], [0, 12, 4]]


def test_tiny_error_against_the_fp32_draw():
    """Information: the tiny configuration names fp32 inputs; the kernel sees
    their bf16 rounding.  Printed per head: the GPU output against the fp64
    dense attention of the unrounded fp32 draw, next to the share the input
    rounding alone explains (the oracle on the bf16 values against the same).
    Asserted only what the parity bound implies by the triangle inequality."""
    from _helpers import TOL_MAX, TOL_MEAN
    w = W.tiny()
    grid = (w.T, w.H, w.W)
    rows = np.arange(w.N)
    r = PathRun(w, _inputs(w))
    try:
        for h, spec in enumerate(w.specs):
            draw = [W.head_draw_f32(seed, 0, h, w.N, w.D) for seed in w.seeds]
            o_f32, _ = oracle.attention_dense_real(spec, grid, w.unit, w.scale, *draw)
            o_bf16, _ = oracle.attention_rows(spec, grid, w.unit, w.D, w.scale, r.q[0, h], r.k[0, h], r.v[0, h],
                                              rows)
            e_gpu = np.abs(r.o_rows(0, h, rows) - o_f32)
            e_in = np.abs(o_bf16 - o_f32)
            print(f"tiny head {h}: GPU vs fp32-draw attention max {e_gpu.max():.3e} mean {e_gpu.mean():.3e}; "
                  f"bf16 input rounding alone max {e_in.max():.3e} mean {e_in.mean():.3e}")
            assert e_gpu.max() <= e_in.max() + TOL_MAX
            assert e_gpu.mean() <= e_in.mean() + TOL_MEAN
    finally:
        r.close()


def test_svg_wan720p():
    w = W.svg_wan720p()
    counts, _ = _check(w, range(w.heads), 512, [0, 7])
    for h in range(5):
        assert counts[h].tolist() == [324900, 12000, 60000]
    for h in range(5, 10):
        assert counts[h].tolist() == [290640, 90510, 15750]
    import block_sparse_attention_mask_b200 as vsa
    plan = vsa.Plan(list(w.specs), (w.T, w.H, w.W), w.unit, w.q_tile, w.kv_tile)
    kept = plan.kept_pairs()
    plan.close()
    # spatial: 80 of 441 frame pairs; temporal: 21 sink frame pairs + 420 x 465 x 1288
    assert kept.tolist() == [80 * 3600 ** 2] * 5 + [21 * 3600 ** 2 + 420 * 465 * 1288] * 5


def test_svg_wan720p_temporal_frame0_first():
    # the temporal heads in the frame-0-first, position-major order: maps of
    # sampled q tiles against the oracle in that order, outputs of sampled
    # rows, and the layout-invariant kept pairs; far fewer executed tiles
    w = W.svg_wan720p(temporal_layout=1)
    counts, _ = _check(w, range(w.heads), 512, [5, 9], qtiles_per_head=8)
    for h in range(5):
        assert counts[h].tolist() == [324900, 12000, 60000]
    base = W.svg_wan720p()
    import block_sparse_attention_mask_b200 as vsa
    plan = vsa.Plan(list(w.specs), (w.T, w.H, w.W), w.unit, w.q_tile, w.kv_tile)
    plan0 = vsa.Plan(list(base.specs), (base.T, base.H, base.W), base.unit, base.q_tile, base.kv_tile)
    try:
        assert (plan.kept_pairs() == plan0.kept_pairs()).all()
        steps, steps0 = plan.exec_steps(), plan0.exec_steps()
        assert (steps[:5] == steps0[:5]).all()
        assert int(steps[5:].sum()) < int(steps0[5:].sum())
    finally:
        plan.close()
        plan0.close()


@pytest.mark.parametrize("layout", [0, 1])
def test_svg_wan720p_tile_rounded(layout):
    # the lossy tile-aligned rounding on the full SVG workload: sampled maps
    # against the oracle's rounded map, sampled rows against attention under
    # the rounded mask; boundary tiles remain only where a kv tile has padding
    w = W.svg_wan720p(temporal_layout=layout, tile_round=1)
    counts, _ = _check(w, [0, 5, 9], 512, [0, 5], qtiles_per_head=6)
    import block_sparse_attention_mask_b200 as vsa
    plan = vsa.Plan(list(w.specs), (w.T, w.H, w.W), w.unit, w.q_tile, w.kv_tile)
    try:
        gmap = plan.tile_map()
        for h in range(w.heads):
            perm = oracle.tile_major_order((w.T, w.H, w.W), w.unit, plan.n_slots, layout=int(w.specs[h]["layout"]))
            padded_kv = (perm.reshape(-1, w.kv_tile) < 0).any(axis=1)
            assert not (gmap[h][:, ~padded_kv] == 1).any()
    finally:
        plan.close()


def test_sta_hunyuan720p():
    w = W.sta_hunyuan720p()
    counts, _ = _check(w, range(w.heads), 512, [0])
    # 900 q tiles of 128 each see 45 window units x 3 tiles; no boundary tiles
    for h in range(w.heads):
        assert counts[h].tolist() == [810000 - 121500, 0, 121500]


def test_stripe_wan720p():
    w = W.stripe_wan720p()
    counts, _ = _check(w, range(w.heads), 512, range(0, 40, 3), qtiles_per_head=4)
    assert (counts.sum(axis=1) == 630 * 630).all()


@pytest.mark.parametrize("T", W.SCALING_T)
@pytest.mark.parametrize("mask", ["full", "spatial"])
def test_scaling(T, mask):
    w = W.scaling(T, mask)
    counts, _ = _check(w, [0, 39], 512, [0])
    n_tiles = (3840 * T // 128) ** 2
    if mask == "full":
        # only the kv tiles holding padded rows (5 of 30 per frame) are boundary
        assert counts[0].tolist() == [0, n_tiles // 6, n_tiles - n_tiles // 6]
    else:
        full, bnd = _spatial_closed_form(T, 128, 128)
        assert counts[0].tolist() == [n_tiles - full - bnd, bnd, full]


@pytest.mark.parametrize("mask", ["full", "spatial"])
def test_scaling_T5_all_rows(mask):
    # the smallest scaling grid (5 x 45 x 80, 18,000 tokens) on every query
    # row of head 0, each row exact over all keys
    w = W.scaling(5, mask)
    _check(w, [0], w.N, [0], qtiles_per_head=4)


@pytest.mark.parametrize("q_tile,kv_tile", [(q, k) for q in W.SWEEP_Q for k in W.SWEEP_KV
                                            if (q, k) != (128, 128)])
def test_tile_sweep(q_tile, kv_tile):
    w = W.scaling(21, "spatial", q_tile, kv_tile)
    counts, _ = _check(w, [0, 39], 512, [0])
    full, bnd = _spatial_closed_form(21, q_tile, kv_tile)
    assert counts[0][2] == full and counts[0][1] == bnd
    assert bnd * 5 == full  # boundary share of executed tiles is 1/6


def test_execution_pairs_follow_identical_lists():
    """How the kernel groups 128-row blocks (execution only; the map is
    unchanged): SVG spatial heads pair neighbouring blocks inside a frame,
    temporal heads pair a block with the same unit one frame later (their kv
    tiles do not depend on the query's frame), and every pair's two blocks
    list the same kv tiles in the oracle's map."""
    import block_sparse_attention_mask_b200 as vsa
    w = W.svg_wan720p()
    plan = vsa.Plan(list(w.specs), (w.T, w.H, w.W), w.unit, w.q_tile, w.kv_tile)
    try:
        pairs = plan.exec_pairs()
        gmap = plan.tile_map()
    finally:
        plan.close()
    nE = pairs.shape[1]
    per_frame = 30                                  # 48 x 80 padded frame / 128
    for h in range(w.heads):
        lead = np.nonzero(pairs[h] >= 0)[0]
        stride = 1 if h < 5 else per_frame
        assert (pairs[h][lead] == lead + stride).all(), h
        assert (pairs[h][lead + stride] == -2).all()
        n_pairs = nE // 2 if h < 5 else per_frame * (w.T // 2)
        assert len(lead) == n_pairs, (h, len(lead))
        for e in lead[::37]:
            assert ((gmap[h][e] != 0) == (gmap[h][e + stride] != 0)).all()
    # 256-row q tiles always pair their halves; 64-row q tiles never pair
    for q, expect in ((256, True), (64, False)):
        ws = W.scaling(5, "spatial", q, 64)
        plan = vsa.Plan(list(ws.specs), (ws.T, ws.H, ws.W), ws.unit, ws.q_tile, ws.kv_tile)
        try:
            pr = plan.exec_pairs()
        finally:
            plan.close()
        if expect:
            assert (pr[:, 0::2] == np.arange(1, pr.shape[1], 2)).all() and (pr[:, 1::2] == -2).all()
        else:
            assert (pr == -1).all()
