"""GPU parity of SVG routing (sampled-query profiling of spatial vs temporal
masks) against the oracle, and of the fixed-shape switch that applies it.

Tolerance of a deviation: the GPU outputs behind it are each within the
output tolerance of the oracle's, so with eps the rms error of a difference
of two outputs (eps = 5e-3 from the mean-abs bound 2e-3 of each, rms over
mean-abs about 1.25) the deviation err = mean(d^2) moves by at most
2 sqrt(err) eps + eps^2.  A flag must match the oracle's wherever the two
deviations differ by more than the sum of their tolerances, and must always
agree with the GPU's own deviations.
"""
import numpy as np
import pytest

import oracle
import workloads as W
from _helpers import torch_bf16

pytestmark = pytest.mark.gpu

EPS = 5e-3


def _tol(e):
    return 2.0 * np.sqrt(np.maximum(e, 0.0)) * EPS + EPS * EPS


def _route_gpu(w, q, k, v, rows, plan=None):
    import torch
    import block_sparse_attention_mask_b200 as vsa
    own = plan is None
    if own:
        plan = vsa.Plan(list(w.specs), (w.T, w.H, w.W), w.unit, w.q_tile, w.kv_tile)
    plan.set_route_candidates([a for a, _ in w.route_specs], [b for _, b in w.route_specs])
    qd, kd, vd = (torch_bf16(x) for x in (q, k, v))
    rd = torch.as_tensor(np.asarray(rows, dtype=np.int32)).cuda()
    err, flags = vsa.svg_route(plan, qd, kd, vd, rd, scale=w.scale)
    torch.cuda.synchronize()
    plan.check()
    out = err.cpu().numpy().astype(np.float64), flags.cpu().numpy()
    if own:
        plan.close()
    return out


def _oracle_route(w, q, k, v, rows):
    return oracle.svg_route([a for a, _ in w.route_specs], [b for _, b in w.route_specs],
                            (w.T, w.H, w.W), w.D, w.scale, q, k, v, rows)


def _check(err_g, flags_g, err_o, flags_o):
    tol = _tol(err_o)
    assert np.all(np.abs(err_g - err_o) <= tol), f"deviations {err_g} vs oracle {err_o}"
    assert np.array_equal(flags_g, (err_g[:, 1] < err_g[:, 0]).astype(flags_g.dtype))
    decisive = np.abs(err_o[:, 0] - err_o[:, 1]) > tol[:, 0] + tol[:, 1]
    assert np.array_equal(flags_g[decisive], flags_o[decisive]), (flags_g, flags_o)


def _workload(name, B, grid, heads, D, structure, sp, tm, amp=10.0):
    T, H, Wd = grid
    return W.Workload(name, B, T, H, Wd, heads, D, (1, 8, 16), 128, 128, tuple([sp] * heads),
                      structure=tuple(structure), structure_amp=amp,
                      route_specs=tuple([(sp, tm)] * heads))


S = W.mask_spec
CASES = {
    # B=2, d=64, one ragged kv tile pair, 13 sampled rows
    "tiny": (W.tiny_routing(), 0.05),
    # 200 rows: two row tiles, the second ragged
    "tiny_two_row_tiles": (W.tiny_routing(), 200 / 256),
    # d=128, 960 tokens = 7.5 kv tiles (last one half padding), sink off on one side
    "d128_ragged": (_workload("route_d128", 1, (5, 12, 16), 3, 128, ("frame", "position", ""),
                              S("spatial", 1, rt=1), S("temporal", 0, rh=2, rw=3)), 0.2),
    # wide spatial window, temporal window wider than the grid in w
    "d64_wide": (_workload("route_d64_wide", 2, (7, 9, 11), 2, 64, ("position", "frame"),
                           S("spatial", 0, rt=2), S("temporal", 1, rh=1, rw=20)), 0.1),
    # a single sampled row
    "one_row": (_workload("route_one_row", 1, (4, 8, 16), 2, 128, ("frame", "position"),
                          S("spatial", 1, rt=0), S("temporal", 1, rh=1, rw=1)), 1 / 512),
}


@pytest.mark.parametrize("name", list(CASES))
def test_route_small(name):
    w, frac = CASES[name]
    q, k, v = (W.full_tensor(w, x) for x in "qkv")
    rows = W.route_rows(w.N, frac)
    err_g, flags_g = _route_gpu(w, q, k, v, rows)
    err_o, flags_o = _oracle_route(w, q, k, v, rows)
    _check(err_g, flags_g, err_o, flags_o)
    # structured heads have a clear answer (frame -> spatial, position ->
    # temporal) unless the sample only holds rows both masks serve alike
    # (e.g. frame-0 rows, which both candidates' sinks cover)
    for h, kind in enumerate(w.structure):
        lo, hi = sorted(err_o[h])
        if kind and hi > 10 * lo:
            assert flags_g[h] == (1 if kind == "position" else 0), (h, kind, err_g[h])


def test_route_full_size_wan720p():
    # the Wan 720p grid with structured heads; the oracle checks 48 of the
    # sampled rows (every CTA split and both row tiles of the kernel still run
    # on the full 1% sample for the flags)
    w = W.svg_wan720p_routing()
    q, k, v = (W.full_tensor(w, x) for x in "qkv")
    rows_full = W.route_rows(w.N, 0.01)
    err_full, flags_full = _route_gpu(w, q, k, v, rows_full)
    assert list(flags_full) == [0] * 5 + [1] * 5, err_full
    rows = rows_full[:: len(rows_full) // 48][:48]
    err_g, flags_g = _route_gpu(w, q, k, v, rows)
    err_o, flags_o = _oracle_route(w, q, k, v, rows)
    _check(err_g, flags_g, err_o, flags_o)


def test_route_rows_out_of_range_flag_device_error():
    import torch
    import block_sparse_attention_mask_b200 as vsa
    w = W.tiny_routing()
    plan = vsa.Plan(list(w.specs), (w.T, w.H, w.W), w.unit, w.q_tile, w.kv_tile)
    plan.set_route_candidates([a for a, _ in w.route_specs], [b for _, b in w.route_specs])
    q, k, v = (torch_bf16(W.full_tensor(w, x)) for x in "qkv")
    rows = torch.tensor([3, w.N + 5, 7], dtype=torch.int32, device="cuda")
    vsa.svg_route(plan, q, k, v, rows, scale=w.scale)
    with pytest.raises(vsa.VsaError) as e:
        plan.check()
    assert e.value.code == -7                   # VSA_ERR_DEVICE
    plan.check()                                # cleared
    plan.close()


def test_route_needs_candidates_and_workspace():
    import torch
    import block_sparse_attention_mask_b200 as vsa
    w = W.tiny_routing()
    plan = vsa.Plan(list(w.specs), (w.T, w.H, w.W), w.unit, w.q_tile, w.kv_tile)
    q, k, v = (torch_bf16(W.full_tensor(w, x)) for x in "qkv")
    rows = torch.tensor([3], dtype=torch.int32, device="cuda")
    with pytest.raises(vsa.VsaError):
        vsa.svg_route(plan, q, k, v, rows)
    with pytest.raises(vsa.VsaError):            # a spatial slot given a temporal spec
        plan.set_route_candidates([S("temporal", 1, rh=1, rw=1)] * 4, [S("temporal", 1, rh=1, rw=1)] * 4)
    plan.set_route_candidates([a for a, _ in w.route_specs], [b for _, b in w.route_specs])
    need = vsa.vsa_svg_route_workspace_size(plan.handle, w.B, w.D, 1)
    small = torch.empty(need - 1, dtype=torch.uint8, device="cuda")
    with pytest.raises(ValueError):
        vsa.svg_route(plan, q, k, v, rows, workspace=small)
    plan.close()


def _apply_and_run(w, tm_layout, graph):
    """Route, apply, then permute + attention + unpermute with the new specs;
    optionally as one captured CUDA graph (fixed shapes)."""
    import torch
    import block_sparse_attention_mask_b200 as vsa
    tm = dict(w.route_specs[0][1], layout=tm_layout)
    cands = [(a, tm) for a, _ in w.route_specs]
    w2 = W.Workload(w.name, w.B, w.T, w.H, w.W, w.heads, w.D, w.unit, w.q_tile, w.kv_tile, w.specs,
                    structure=w.structure, structure_amp=w.structure_amp, route_specs=tuple(cands))
    plan = vsa.Plan(list(w2.specs), (w.T, w.H, w.W), w.unit, w.q_tile, w.kv_tile)
    plan.set_route_candidates([a for a, _ in cands], [b for _, b in cands])
    qn, kn, vn = (W.full_tensor(w, x) for x in "qkv")
    q, k, v = (torch_bf16(x) for x in (qn, kn, vn))
    rows = torch.as_tensor(W.route_rows(w.N, 0.05).astype(np.int32)).cuda()
    ws = torch.empty(vsa.vsa_svg_route_workspace_size(plan.handle, w.B, w.D, rows.numel()),
                     dtype=torch.uint8, device="cuda")
    err = torch.empty((w.heads, 2), dtype=torch.float32, device="cuda")
    flags = torch.empty((w.heads,), dtype=torch.int32, device="cuda")

    def step():
        vsa.svg_route(plan, q, k, v, rows, scale=w.scale, workspace=ws, err=err, flags=flags)
        plan.apply_route(flags)
        return vsa.attention(plan, q, k, v, scale=w.scale)

    if graph:
        step()                                   # warm up outside the capture
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            o, lse = step()
        g.replay()
    else:
        o, lse = step()
    torch.cuda.synchronize()
    plan.check()
    fl = flags.cpu().numpy()
    chosen = [cands[h][int(fl[h])] for h in range(w.heads)]
    # tile map of the plan = the oracle's map of the chosen specs
    tmap = plan.tile_map()
    for h, spec in enumerate(chosen):
        want = oracle.tile_map(spec, (w.T, w.H, w.W), w.unit, plan.n_slots, w.q_tile, w.kv_tile)
        assert np.array_equal(tmap[h], want), f"head {h}"
    # outputs of every head under its chosen mask
    from _helpers import TOL_MAX, TOL_MEAN
    rows_chk = W.sample_rows(w, 0, 64)
    for b in range(w.B):
        for h, spec in enumerate(chosen):
            o_ref, _ = oracle.attention_rows(spec, (w.T, w.H, w.W), w.unit, w.D, w.scale,
                                             qn[b, h], kn[b, h], vn[b, h], rows_chk)
            o_gpu = o[b, h].index_select(0, torch.as_tensor(rows_chk, device="cuda")).float().cpu().numpy()
            e = np.abs(o_gpu - o_ref)
            assert e.max() <= TOL_MAX and e.mean() <= TOL_MEAN, (b, h, e.max(), e.mean())
    plan.close()
    return fl


@pytest.mark.parametrize("tm_layout", [0, 1])
def test_apply_route_switches_specs_and_order(tm_layout):
    fl = _apply_and_run(W.tiny_routing(), tm_layout, graph=False)
    assert fl[0] == 0 and fl[1] == 1 and fl[3] == 0


def test_route_apply_attention_in_one_cuda_graph():
    fl = _apply_and_run(W.tiny_routing(), 1, graph=True)
    assert fl[0] == 0 and fl[1] == 1 and fl[3] == 0
