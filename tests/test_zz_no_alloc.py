"""The no-allocation tile map (vsa_tile_map_noalloc) against the plan API.

vsa_tile_map_noalloc exists for callers that cannot allocate device memory
themselves (a framework-owned memory pool, or a serving loop that cannot
afford cudaMalloc's device synchronisation).  It keeps its working memory in
one static device array shared by every call, so these tests call it through
the C ABI several times in a row, with different head counts and grid sizes,
and require each map to equal, bit for bit, the map vsa_plan_create builds,
and the device's free memory to stay the same across the calls.

Every pointer handed to the C entry point here is a real buffer of the size
the call is told: a rejection test never relies on the order of the host-side
checks to keep a kernel from running.
"""
import ctypes

import numpy as np
import pytest

import block_sparse_attention_mask_b200 as vsa
import workloads as W

S = W.mask_spec
MAX_HEADS = 64


def _raw_call(specs, grid, unit, q_tile, kv_tile, ptr, nbytes, stream):
    arr = (vsa.vsa_mask_spec * len(specs))(*[vsa.make_spec(s) for s in specs])
    T, H, Wd = grid
    bt, bh, bw = unit
    return vsa.lib.vsa_tile_map_noalloc(arr, len(specs), T, H, Wd, bt, bh, bw, q_tile, kv_tile,
                                        ctypes.c_void_p(ptr), nbytes, ctypes.c_void_p(stream))


def _out_buffer(specs, grid, unit, q_tile, kv_tile):
    import torch
    info = vsa.vsa_layout_info(len(specs), grid, unit, q_tile, kv_tile)
    out = torch.full((info["map_bytes"],), -1, dtype=torch.int8, device="cuda")
    return out, (len(specs), info["n_q_tiles"], info["n_kv_tiles"])


def _noalloc_into(out, call):
    import torch
    rc = _raw_call(*call, out.data_ptr(), out.numel(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0, vsa.vsa_status_string(rc)


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
    import torch
    outs = [_out_buffer(*c) for c in CALLS]
    # one call of each kind first: the first launch of a kernel may load its
    # module, which is the library's one-time set-up, not the call's
    for c, (o, _) in zip(CALLS, outs):
        _noalloc_into(o, c)
    again = torch.full_like(outs[1][0], -1)
    for o, _ in outs:
        o.fill_(-1)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    for c, (o, _) in zip(CALLS, outs):         # back to back, sharing the scratch
        _noalloc_into(o, c)
    _noalloc_into(again, CALLS[1])             # a repeat after a different call
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    # neither torch's allocator nor the device saw an allocation
    assert torch.cuda.memory_allocated() == alloc0
    assert free1 == free0, f"device free memory changed by {free0 - free1} bytes"
    got = [o.cpu().numpy().reshape(shape) for o, shape in outs]
    for c, g in zip(CALLS, got):
        assert (g == _with_plan(*c)).all()
    assert (again.cpu().numpy().reshape(outs[1][1]) == got[1]).all()


@pytest.mark.gpu
def test_noalloc_rejects_requests_beyond_its_scratch():
    import torch
    spec = S("stripe", 0, Tw=1, To=0, Ts=2, Sw=1, So=0, Ss=3)
    stream = torch.cuda.current_stream().cuda_stream
    # more heads than the spec area holds
    call = ([spec] * (MAX_HEADS + 1), (4, 8, 8), (1, 8, 8), 64, 64)
    out, _ = _out_buffer(*call)
    assert _raw_call(*call, out.data_ptr(), out.numel(), stream) == -2
    # 64 stripe heads on a 256 x 256 frame need about 2 MiB of offset tables
    call = ([spec] * MAX_HEADS, (1, 256, 256), (1, 8, 8), 64, 64)
    out, _ = _out_buffer(*call)
    assert _raw_call(*call, out.data_ptr(), out.numel(), stream) == -2
    torch.cuda.synchronize()
    assert (out == -1).all()                   # nothing was written


@pytest.mark.gpu
def test_noalloc_rejects_a_map_that_is_not_device_memory():
    import torch
    call = CALLS[1]
    out, _ = _out_buffer(*call)
    host = torch.full((out.numel(),), -1, dtype=torch.int8).pin_memory()
    stream = torch.cuda.current_stream().cuda_stream
    assert _raw_call(*call, host.data_ptr(), host.numel(), stream) == -1
    # a map buffer smaller than the map
    assert _raw_call(*call, out.data_ptr(), out.numel() - 1, stream) == -1
    torch.cuda.synchronize()
    assert (host == -1).all() and (out == -1).all()
    # the Python wrapper refuses views and wrong types before the C call
    with pytest.raises(vsa.VsaError):
        vsa.vsa_tile_map_noalloc(call[0], *call[1:], out[::2])
    with pytest.raises(vsa.VsaError):
        vsa.vsa_tile_map_noalloc(call[0], *call[1:], host)
    with pytest.raises(vsa.VsaError):
        vsa.vsa_tile_map_noalloc(call[0], *call[1:], out.view(torch.uint8))
    # a view that starts inside a buffer is bounded by what remains of it
    with pytest.raises(vsa.VsaError):
        vsa.vsa_tile_map_noalloc(call[0], *call[1:], out[1:])
    vsa.vsa_tile_map_noalloc(call[0], *call[1:], out)
    torch.cuda.synchronize()
    assert (out.cpu().numpy().reshape(_out_buffer(*call)[1]) == _with_plan(*call)).all()


def test_noalloc_rejects_bad_arguments_on_the_host():
    """Null buffers and head counts out of range are refused before any
    device work; no pointer other than NULL is passed."""
    spec = S("spatial", 1, rt=1)
    assert _raw_call([spec], (4, 8, 8), (1, 8, 8), 64, 64, None, 1 << 20, None) == -1
    arr = (vsa.vsa_mask_spec * 1)(vsa.make_spec(spec))
    assert vsa.lib.vsa_tile_map_noalloc(arr, 0, 4, 8, 8, 1, 8, 8, 64, 64, None, 1 << 20, None) == -1
