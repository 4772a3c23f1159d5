"""The no-allocation tile map (vsa_tile_map_noalloc) against the plan API.

vsa_tile_map_noalloc exists for callers that cannot allocate device memory
themselves (a framework-owned memory pool, or a serving loop that cannot
afford cudaMalloc's device synchronisation).  It keeps its working memory in
one static device array shared by every call, so these tests call it through
the C ABI several times in a row, with different head counts and grid sizes,
and require each map to equal, bit for bit, the map vsa_plan_create builds.
"""
import ctypes

import numpy as np
import pytest

import block_sparse_attention_mask_b200 as vsa
import workloads as W

S = W.mask_spec


def _noalloc(specs, grid, unit, q_tile, kv_tile):
    import torch
    info = vsa.vsa_layout_info(len(specs), grid, unit, q_tile, kv_tile)
    out = torch.full((info["map_bytes"],), -1, dtype=torch.int8, device="cuda")
    arr = (vsa.vsa_mask_spec * len(specs))(*[vsa.make_spec(s) for s in specs])
    T, H, Wd = grid
    bt, bh, bw = unit
    rc = vsa.lib.vsa_tile_map_noalloc(arr, len(specs), T, H, Wd, bt, bh, bw, q_tile, kv_tile,
                                      ctypes.c_void_p(out.data_ptr()), out.numel(),
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, vsa.vsa_status_string(rc)
    torch.cuda.synchronize()
    return out.cpu().numpy().reshape(len(specs), info["n_q_tiles"], info["n_kv_tiles"])


def _with_plan(specs, grid, unit, q_tile, kv_tile):
    plan = vsa.Plan(list(specs), grid, unit, q_tile, kv_tile)
    try:
        return plan.tile_map()
    finally:
        plan.close()


CALLS = [
    # 40 stripe heads with the sink on the Wan 720p latent: the largest offset tables
    (list(W.stripe_wan720p().specs), (21, 45, 80), (1, 8, 16), 128, 128),
    # fewer heads and a smaller frame: the shared array still holds the first call's tables
    ([S("stripe", 1, Tw=2, To=1, Ts=3, Sw=20, So=5, Ss=47), S("temporal", 1, rh=2, rw=3),
      S("spatial", 1, rt=1), S("sta", 0, kt=3, kh=1, kw=1)], (5, 13, 20), (1, 8, 16), 128, 128),
    # no stripe head, other tile shape
    (list(W.svg_wan720p().specs), (21, 45, 80), (1, 8, 8), 64, 64),
    # temporal heads in the frame-0-first order
    (list(W.svg_wan720p(temporal_layout=1).specs), (21, 45, 80), (1, 8, 16), 128, 128),
]


@pytest.mark.gpu
def test_noalloc_map_equals_plan_map_on_consecutive_calls():
    got = [_noalloc(*c) for c in CALLS]          # back to back, sharing the scratch
    for c, g in zip(CALLS, got):
        assert (g == _with_plan(*c)).all()
    again = _noalloc(*CALLS[1])                  # a repeat after a different call
    assert (again == got[1]).all()


def test_noalloc_rejects_requests_beyond_its_scratch():
    spec = vsa.make_spec(S("stripe", 0, Tw=1, To=0, Ts=2, Sw=1, So=0, Ss=3))
    many = (vsa.vsa_mask_spec * (vsa_max_heads() + 1))(*([spec] * (vsa_max_heads() + 1)))
    rc = vsa.lib.vsa_tile_map_noalloc(many, vsa_max_heads() + 1, 4, 8, 8, 1, 8, 8, 64, 64,
                                      ctypes.c_void_p(16), 1 << 20, None)
    assert rc == -2
    # 64 stripe heads on a 256 x 256 frame need about 2 MiB of offset tables
    big = (vsa.vsa_mask_spec * 64)(*([spec] * 64))
    rc = vsa.lib.vsa_tile_map_noalloc(big, 64, 1, 256, 256, 1, 8, 8, 64, 64,
                                      ctypes.c_void_p(16), 1 << 30, None)
    assert rc == -2


def vsa_max_heads():
    return 64
