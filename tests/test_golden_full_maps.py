"""CPU checks of ``tests/golden/full_maps.json`` (the oracle's full-size map
digests that the GPU maps are compared with).

The file must cover every parity workload with its current specs; its tile
counts must agree with the closed forms derived from the mask definitions
(SVG heads on the Wan 720p latent, STA's Eq. 4 block count, the scaling
grids); one head's digest and the q-tile strata are recomputed with the
oracle, so the file is reproducible from the committed script.
"""
import hashlib

import numpy as np
import pytest

import oracle
import workloads as W
from _helpers import full_maps, heads_of

FULL = full_maps()
PARITY = {w.name: w for w in W.all_parity_workloads()}


def test_every_parity_workload_is_covered_with_its_specs():
    assert set(FULL) == set(PARITY)
    for name, w in PARITY.items():
        rec = FULL[name]
        heads = heads_of(rec)
        assert [h["spec"] for h in heads] == [dict(s) for s in w.specs]
        assert (rec["q_tile"], rec["kv_tile"], tuple(rec["unit"])) == (w.q_tile, w.kv_tile, w.unit)
        assert len(heads) == w.heads
        for h in heads:
            assert sum(h["counts"]) == h["shape"][0] * h["shape"][1]


def test_svg_counts_equal_the_closed_forms():
    # 80 kept frame pairs x 30 q units x (25 full + 5 boundary kv units) for a
    # spatial head; the temporal head's frame-0 column and 16 x 13 unit pairs
    # of the 420 other frame pairs ("Sparse VideoGen ... on TPU", SVG heads)
    for name in ("svg_wan720p_21x45x80",):
        heads = heads_of(FULL[name])
        for h in range(5):
            assert heads[h]["counts"] == [324900, 12000, 60000]
        for h in range(5, 10):
            assert heads[h]["counts"] == [290640, 90510, 15750]


def test_sta_counts_equal_eq4():
    # every 128-row q tile sees 45 window units of 3 kv tiles, all full
    # ("Fast Video Generation with Sliding Tile Attention", section 3, Eq. 4)
    for h in heads_of(FULL["sta_hunyuan720p_30x48x80"]):
        assert h["counts"] == [810000 - 121500, 0, 121500]


@pytest.mark.parametrize("T", W.SCALING_T)
def test_scaling_counts_equal_the_closed_forms(T):
    n = (3840 * T // 128) ** 2
    dense = heads_of(FULL[W.scaling(T, "full").name])
    # only kv tiles holding padded rows (5 of 30 per frame) are boundary
    assert all(h["counts"] == [0, n // 6, n - n // 6] for h in dense)
    # spatial |dt| <= 1 with the sink: (4T - 4) kept frame pairs of 30 x 30 tiles
    spatial = heads_of(FULL[W.scaling(T, "spatial").name])
    pairs = 4 * T - 4
    assert all(h["counts"] == [n - pairs * 900, pairs * 150, pairs * 750] for h in spatial)


def test_one_digest_and_the_strata_recompute():
    w = W.svg_wan720p()
    rec = FULL[w.name]
    spec = w.specs[0]
    m = oracle.tile_map(spec, (w.T, w.H, w.W), w.unit, rec["n_slots"], w.q_tile, w.kv_tile)
    assert hashlib.sha256(np.ascontiguousarray(m, dtype=np.int8).tobytes()).hexdigest() == \
        heads_of(rec)[0]["sha256"]
    for name in (w.name, "stripe_wan720p_21x45x80"):
        ww = PARITY[name]
        r = FULL[name]
        for h in (0, ww.heads - 1):
            head = heads_of(r)[h]
            for key, cls in (("boundary_only_qtiles", 1), ("full_only_qtiles", 2)):
                qt = head[key]
                if not qt:
                    continue
                rows = oracle.tile_map(ww.specs[h], (ww.T, ww.H, ww.W), ww.unit, r["n_slots"],
                                       ww.q_tile, ww.kv_tile, qt)
                executed = rows != 0
                assert executed.any(axis=1).all()
                assert (rows[executed] == cls).all()


def test_strata_follow_from_the_masks():
    # With the frame-0 sink in the tile-major order, the 25 padding-free
    # frame-0 kv units are full for every q tile, so no q tile is
    # boundary-only; the kept frames' padded kv units are boundary, so SVG and
    # dense q tiles are not full-only either.  Every STA q tile is full-only
    # (all its tiles are full or empty).
    for name in ("svg_wan720p_21x45x80", "stripe_wan720p_21x45x80"):
        assert all(h["n_boundary_only"] == 0 for h in heads_of(FULL[name]))
    svg = heads_of(FULL["svg_wan720p_21x45x80"])
    assert all(h["n_full_only"] == 0 for h in svg)
    for T in W.SCALING_T:
        for mask in ("full", "spatial"):
            hs = heads_of(FULL[W.scaling(T, mask).name])
            assert all(h["n_full_only"] == 0 and h["n_boundary_only"] == 0 for h in hs)
    sta = heads_of(FULL["sta_hunyuan720p_30x48x80"])
    assert all(h["n_full_only"] == 900 and h["n_boundary_only"] == 0 for h in sta)
