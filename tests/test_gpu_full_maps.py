"""GPU tile maps at full size, bit-exact against the oracle for every head.

``tests/golden/full_maps.json`` holds, for every parity workload (the tiny
grid, the SVG Wan 720p workload in both token orders with and without
tile-aligned rounding, STA HunyuanVideo, the 40 stripe heads, the scaling grids
T = 5..33 with the dense and spatial masks, and the tile sweep), the SHA-256 of
each head's full int8 map as the CPU oracle classifies it by brute force, and
its tile counts; ``tests/golden/make_full_maps.py`` wrote it, calling only the
oracle.  Here the plan is built on the GPU in the launch configuration the
benchmark times and every head's map is hashed and compared.
"""
import hashlib
import json
import os

import numpy as np
import pytest

import workloads as W
from _helpers import heads_of

pytestmark = pytest.mark.gpu

_GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "full_maps.json")
with open(_GOLDEN) as _f:
    FULL = json.load(_f)["workloads"]

WORKLOADS = {w.name: w for w in W.all_parity_workloads()}


@pytest.mark.parametrize("name", sorted(FULL))
def test_full_map_every_head(name):
    import block_sparse_attention_mask_b200 as vsa
    w = WORKLOADS[name]
    ref = FULL[name]
    heads = heads_of(ref)
    assert [dict(s) for s in w.specs] == [hd["spec"] for hd in heads]
    plan = vsa.Plan(list(w.specs), (w.T, w.H, w.W), w.unit, w.q_tile, w.kv_tile)
    try:
        assert plan.n_slots == ref["n_slots"]
        gmap = plan.tile_map()
        counts = plan.tile_counts()
        plan.check()
    finally:
        plan.close()
    assert gmap.shape[0] == w.heads
    bad = []
    for h in range(w.heads):
        m = np.ascontiguousarray(gmap[h], dtype=np.int8)
        assert list(m.shape) == heads[h]["shape"]
        if hashlib.sha256(m.tobytes()).hexdigest() != heads[h]["sha256"]:
            bad.append(h)
        assert counts[h].tolist() == heads[h]["counts"], f"head {h} counts"
    assert not bad, f"heads whose map differs from the oracle's: {bad}"
