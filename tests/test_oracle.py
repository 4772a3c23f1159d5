"""Pins of the CPU oracle against what the pages and the mathematics fix.

No GPU.  Every check here compares the oracle with something other than itself:
values printed on the pages or derived by hand (tests/golden), closed forms,
a textbook softmax written with numpy, brute force on tiny grids, and the
degenerate stripe settings that reduce to the SVG and STA masks.
"""
import json
import os

import numpy as np
import pytest

import oracle
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _spec(d):
    d = dict(d)
    kind = d.pop("kind")
    return W.mask_spec(kind, **d)


# ---------------------------------------------------------------------------
# layout


def test_layout_fixture():
    g = _golden("layout.json")
    assert int(np.prod(g["wan720p_grid"])) == g["wan720p_tokens"]
    assert oracle.padded_tokens(g["wan720p_grid"], g["psablock"]) == g["psablock_padded_tokens"]
    assert int(np.prod(g["psablock_padded_grid"])) == g["psablock_padded_tokens"]
    so = g["small_order"]
    perm = oracle.tile_major_order(so["grid"], so["unit"])
    assert perm[:24].tolist() == so["first_24_slots"]


@pytest.mark.parametrize("grid,unit,extra", [((2, 3, 5), (1, 2, 2), 0), ((5, 7, 9), (2, 4, 4), 17),
                                              ((4, 8, 8), (1, 8, 8), 0), ((3, 5, 6), (3, 1, 6), 5)])
def test_order_is_a_bijection(grid, unit, extra):
    npad = oracle.padded_tokens(grid, unit)
    perm = oracle.tile_major_order(grid, unit, npad + extra)
    real = perm[perm >= 0]
    assert sorted(real.tolist()) == list(range(int(np.prod(grid))))
    assert (perm[npad:] == -1).all()
    # every unit occupies a contiguous run of slots and holds a 3D box
    T, H, Wd = grid
    U = unit[0] * unit[1] * unit[2]
    for u in range(npad // U):
        blk = perm[u * U:(u + 1) * U]
        r = blk[blk >= 0]
        if len(r) == 0:
            continue
        t, h, w = r // (H * Wd), (r // Wd) % H, r % Wd
        assert t.max() - t.min() < unit[0] and h.max() - h.min() < unit[1] and w.max() - w.min() < unit[2]


def test_tiny_order_is_identity():
    w = W.tiny()
    perm = oracle.tile_major_order((w.T, w.H, w.W), w.unit)
    assert (perm == np.arange(w.N)).all()


# ---------------------------------------------------------------------------
# mask predicate


@pytest.mark.parametrize("case", _golden("mask_cases.json")["cases"], ids=lambda c: c["name"])
def test_mask_cases(case):
    spec = _spec(case["spec"])
    grid = tuple(case["grid"])
    for nq, nk, want in case["points"]:
        assert oracle.keep(spec, grid, (1, 1, 1), nq, nk) == want, (nq, nk)
    assert oracle.kept_pairs(spec, grid) == case["kept_pairs"]
    assert int(oracle.keep_matrix(spec, grid, (1, 1, 1)).sum()) == case["kept_pairs"]


def _random_grid(g, tmax=5, hmax=6, wmax=7):
    return (int(g.integers(1, tmax + 1)), int(g.integers(1, hmax + 1)), int(g.integers(1, wmax + 1)))


def test_degenerate_stripe_equals_svg_spatial():
    g = np.random.default_rng(3)
    for _ in range(12):
        T, H, Wd = _random_grid(g)
        rt = int(g.integers(0, 3))
        for sink in (0, 1):
            a = oracle.keep_matrix(W.mask_spec("spatial", sink=sink, rt=rt), (T, H, Wd), (1, 1, 1))
            b = oracle.keep_matrix(W.mask_spec("stripe", sink=sink, Tw=rt + 1, To=0, Ts=T + 1,
                                               Sw=H * Wd, So=0, Ss=H * Wd), (T, H, Wd), (1, 1, 1))
            assert (a == b).all()


def test_degenerate_stripe_equals_svg_temporal():
    g = np.random.default_rng(4)
    for _ in range(12):
        T, _, Wd = _random_grid(g)
        rw = int(g.integers(0, 4))
        for sink in (0, 1):
            a = oracle.keep_matrix(W.mask_spec("temporal", sink=sink, rh=int(g.integers(0, 3)), rw=rw),
                                   (T, 1, Wd), (1, 1, 1))
            b = oracle.keep_matrix(W.mask_spec("stripe", sink=sink, Tw=T, To=0, Ts=T, Sw=rw + 1,
                                               So=0, Ss=Wd), (T, 1, Wd), (1, 1, 1))
            assert (a == b).all()
        # zero radii: same spatial position in every frame, on any grid
        T, H, Wd = _random_grid(g)
        a = oracle.keep_matrix(W.mask_spec("temporal", sink=1, rh=0, rw=0), (T, H, Wd), (1, 1, 1))
        b = oracle.keep_matrix(W.mask_spec("stripe", sink=1, Tw=T, To=0, Ts=T, Sw=1, So=0, Ss=H * Wd),
                               (T, H, Wd), (1, 1, 1))
        assert (a == b).all()


def test_degenerate_stripe_equals_sta_unclamped_rows():
    g = np.random.default_rng(5)
    for _ in range(10):
        T, Wd = int(g.integers(5, 9)), int(g.integers(5, 11))
        kt, kw = int(g.choice([1, 3, 5])), int(g.choice([1, 3]))
        sta = oracle.keep_matrix(W.mask_spec("sta", kt=kt, kh=1, kw=kw), (T, 1, Wd), (1, 1, 1))
        st = oracle.keep_matrix(W.mask_spec("stripe", Tw=kt // 2 + 1, To=0, Ts=T + 1, Sw=kw // 2 + 1,
                                            So=0, Ss=Wd + 1), (T, 1, Wd), (1, 1, 1))
        for nq in range(T * Wd):
            t, w = nq // Wd, nq % Wd
            unclamped = (kt // 2 <= t <= T - 1 - kt // 2) and (kw // 2 <= w <= Wd - 1 - kw // 2)
            if unclamped:
                assert (sta[nq] == st[nq]).all()
            # the clamped window still holds exactly kt*kw keys
            assert sta[nq].sum() == min(kt, T) * min(kw, Wd)


def test_rows_never_empty_with_sink_or_sta():
    g = np.random.default_rng(6)
    for _ in range(8):
        grid = _random_grid(g)
        T, H, Wd = grid
        specs = [W.mask_spec("spatial", sink=1, rt=0),
                 W.mask_spec("temporal", sink=1, rh=0, rw=0),
                 W.mask_spec("stripe", sink=1, Tw=1, To=int(g.integers(0, 3)), Ts=int(g.integers(1, 6)),
                             Sw=1, So=int(g.integers(0, 5)), Ss=int(g.integers(1, 9))),
                 W.mask_spec("sta", kt=1, kh=1, kw=1)]
        for s in specs:
            m = oracle.keep_matrix(s, grid, (1, 1, 1))
            assert (m.sum(axis=1) >= 1).all()


def test_sta_sparsity_matches_printed_table():
    """Table 2 / Table 4 sparsities, on the 5x6x10 tile grid of a 30x48x80 latent."""
    fx = _golden("sta_sparsity.json")
    T, H, Wd = fx["grid"]
    bt, bh, bw = fx["unit"]
    for case in fx["cases"]:
        kt, kh, kw = case["window_tiles"]
        assert [a // b for a, b in zip(case["window_tokens"], fx["unit"])] == [kt, kh, kw]
        spec = W.mask_spec("sta", kt=kt, kh=kh, kw=kw)
        # one token per tile: the same tile grid, every tile pair is one pair
        grid1 = (T // bt, H // bh, Wd // bw)
        kept = oracle.kept_pairs(spec, grid1)
        n_tiles = int(np.prod(grid1))
        assert round(100.0 * (1 - kept / n_tiles ** 2), 2) == case["sparsity_pct"]
        # 2x2x2 tokens per tile: the map at tile granularity is full/empty only
        grid2 = tuple(2 * x for x in grid1)
        cls = oracle.tile_map(spec, grid2, (2, 2, 2), 8 * n_tiles, 8, 8)
        assert (cls != 1).all()
        assert round(100.0 * (1 - (cls == 2).sum() / cls.size), 2) == case["sparsity_pct"]


def test_sta_eq4_dense_block_count():
    for case in _golden("sta_eq4.json")["cases"]:
        L, Tt, Wt = case["L"], case["T"], case["W"]
        k = Wt // Tt
        spec = W.mask_spec("sta", kt=k, kh=k, kw=k)
        B = Tt ** 3
        cls = oracle.tile_map(spec, (L, L, L), (Tt, Tt, Tt), L ** 3, B, B)
        assert int((cls == 2).sum()) == case["dense_blocks"]
        assert int((cls == 1).sum()) == case["mixed_blocks"]


def test_tiny_maps_and_counts():
    fx = _golden("tiny_maps.json")
    w = W.tiny()
    for h in range(2):
        cls = oracle.tile_map(w.specs[h], (w.T, w.H, w.W), w.unit, w.N, 64, 64)
        assert cls.tolist() == fx["maps"][h]
        assert oracle.kept_pairs(w.specs[h], (w.T, w.H, w.W)) == fx["kept_pairs"][h]


def test_single_token_tiles_are_the_predicate():
    """With 1-slot tiles every tile is full or empty, and full exactly where keep holds."""
    g = np.random.default_rng(8)
    for _ in range(6):
        grid = _random_grid(g, 3, 5, 6)
        unit = (1, int(g.integers(1, 4)), int(g.integers(1, 4)))
        spec = W.mask_spec("stripe", sink=int(g.integers(0, 2)), Tw=int(g.integers(1, 3)),
                           To=int(g.integers(0, 2)), Ts=int(g.integers(1, 4)),
                           Sw=int(g.integers(1, 5)), So=int(g.integers(0, 4)), Ss=int(g.integers(1, 9)))
        perm = oracle.tile_major_order(grid, unit)
        n = len(perm)
        cls = oracle.tile_map(spec, grid, unit, n, 1, 1)
        km = oracle.keep_matrix(spec, grid, (1, 1, 1))
        for a in range(n):
            for b in range(n):
                if perm[a] < 0 or perm[b] < 0:
                    assert cls[a, b] == 0
                else:
                    assert cls[a, b] == (2 if km[perm[a], perm[b]] else 0)


def test_tile_counts_aggregate_the_predicate():
    """Counts per tile pair equal a numpy sum of the predicate matrix over the tile's slots."""
    g = np.random.default_rng(9)
    for _ in range(6):
        grid = _random_grid(g, 4, 6, 6)
        unit = (1, 2, 2)
        npad = oracle.padded_tokens(grid, unit)
        Bq = int(g.choice([4, 8]))
        Bk = int(g.choice([4, 8]))
        n_slots = int(np.ceil(npad / 8) * 8) + 8
        spec = W.mask_spec("temporal", sink=1, rh=1, rw=int(g.integers(0, 3)))
        perm = oracle.tile_major_order(grid, unit, n_slots)
        km = oracle.keep_matrix(spec, grid, (1, 1, 1))
        full = np.zeros((n_slots, n_slots), dtype=np.int64)
        real = perm >= 0
        full[np.ix_(real, real)] = km[np.ix_(perm[real], perm[real])]
        want = full.reshape(n_slots // Bq, Bq, n_slots // Bk, Bk).sum(axis=(1, 3))
        counts, real_q = oracle.tile_counts(spec, grid, unit, n_slots, Bq, Bk)
        assert (counts == want).all()
        assert (real_q == real.reshape(-1, Bq).sum(axis=1)).all()
        cls = oracle.classes_from_counts(counts, real_q, Bk)
        # a kv tile holding padding is never full
        kv_has_pad = (~real).reshape(-1, Bk).any(axis=1)
        assert not (cls[:, kv_has_pad] == 2).any()


@pytest.mark.slow
def test_svg_wan720p_closed_forms():
    fx = _golden("svg_wan720p_counts.json")
    grid, unit = tuple(fx["grid"]), tuple(fx["unit"])
    for key in ("spatial", "temporal"):
        spec = _spec(fx[key]["spec"])
        assert oracle.kept_pairs(spec, grid) == fx[key]["kept_pairs"]
        cls = oracle.tile_map(spec, grid, unit, oracle.padded_tokens(grid, unit), 128, 128)
        tiles = fx[key]["tiles"]
        assert int((cls == 2).sum()) == tiles["full"]
        assert int((cls == 1).sum()) == tiles["boundary"]
        assert int((cls == 0).sum()) == tiles["empty"]
    assert fx["spatial"]["kept_pairs"] * fx["spatial"]["kept_fraction_den"] == \
        fx["spatial"]["kept_fraction_num"] * (75600 ** 2)


# ---------------------------------------------------------------------------
# attention


def _textbook(q, k, v, scale, keep):
    """softmax(q k^T * scale with dropped pairs at -inf) v and its log-sum-exp, numpy fp64."""
    s = (q @ k.T) * scale
    s = np.where(keep, s, -np.inf)
    mx = s.max(axis=1, keepdims=True)
    e = np.exp(s - mx)
    l = e.sum(axis=1, keepdims=True)
    return (e @ v) / l, (mx + np.log(l))[:, 0]


@pytest.mark.parametrize("kind", ["full", "spatial", "temporal", "sta", "stripe"])
def test_attention_matches_textbook(kind):
    g = np.random.default_rng(11)
    grid = (3, 5, 6)
    N = int(np.prod(grid))
    D = 16
    spec = {"full": W.mask_spec("full"),
            "spatial": W.mask_spec("spatial", sink=1, rt=0),
            "temporal": W.mask_spec("temporal", sink=1, rh=1, rw=2),
            "sta": W.mask_spec("sta", kt=1, kh=3, kw=3),
            "stripe": W.mask_spec("stripe", sink=1, Tw=1, To=1, Ts=2, Sw=3, So=2, Ss=7)}[kind]
    q16 = W.bf16_bits_from_f32(g.standard_normal((N, D)).astype(np.float32))
    k16 = W.bf16_bits_from_f32(g.standard_normal((N, D)).astype(np.float32))
    v16 = W.bf16_bits_from_f32(g.standard_normal((N, D)).astype(np.float32))
    q, k, v = (W.bf16_bits_to_f32(x).astype(np.float64) for x in (q16, k16, v16))
    scale = 1 / np.sqrt(D)
    unit = (1, 1, 1)
    keepm = oracle.keep_matrix(spec, grid, unit)
    o_ref, lse_ref = _textbook(q, k, v, scale, keepm)
    o, lse = oracle.attention_rows(spec, grid, unit, D, scale, q16, k16, v16, range(N))
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-12)
    if kind == "full":
        # the full mask is unmasked attention
        o2, _ = _textbook(q, k, v, scale, np.ones((N, N), bool))
        np.testing.assert_allclose(o, o2, rtol=0, atol=1e-12)
    # the numpy dense form for real-valued inputs agrees with the C oracle on
    # the same (bf16-valued) numbers
    o3, lse3 = oracle.attention_dense_real(spec, grid, unit, scale, q, k, v)
    np.testing.assert_allclose(o3, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse3, lse, rtol=0, atol=1e-12)


def test_attention_dense_real_on_fp32_inputs():
    """On unrounded fp32 inputs: weights sum to one (v = 1 gives o = 1), lse is
    the log-sum-exp of the kept scores, and the result moves from the bf16
    oracle by no more than the input rounding can explain (a few 1e-3)."""
    g = np.random.default_rng(21)
    grid, unit, D = (3, 4, 5), (1, 2, 5), 32
    N = int(np.prod(grid))
    spec = W.mask_spec("temporal", sink=1, rh=1, rw=1)
    q, k, v = (g.standard_normal((N, D)).astype(np.float32) for _ in range(3))
    scale = D ** -0.5
    keepm = oracle.keep_matrix(spec, grid, unit)
    o1, lse = oracle.attention_dense_real(spec, grid, unit, scale, q, k, np.ones((N, D), np.float32))
    np.testing.assert_allclose(o1, 1.0, rtol=0, atol=1e-14)
    s = scale * (q.astype(np.float64) @ k.astype(np.float64).T)
    for i in range(N):
        kept = s[i][keepm[i]]
        assert abs(lse[i] - (kept.max() + np.log(np.exp(kept - kept.max()).sum()))) < 1e-12
    o, _ = oracle.attention_dense_real(spec, grid, unit, scale, q, k, v)
    b16 = [W.bf16_bits_from_f32(x) for x in (q, k, v)]
    ob, _ = oracle.attention_rows(spec, grid, unit, D, scale, *b16, range(N))
    assert 0 < np.abs(o - ob).max() < 2e-2


def test_attention_weights_sum_to_one():
    """With v = 1 every output element is the row sum of the attention weights."""
    g = np.random.default_rng(12)
    grid = (4, 3, 5)
    N, D = 60, 8
    spec = W.mask_spec("stripe", sink=1, Tw=2, To=0, Ts=3, Sw=4, So=1, Ss=6)
    q16 = W.bf16_bits_from_f32(g.standard_normal((N, D)).astype(np.float32) * 3)
    k16 = W.bf16_bits_from_f32(g.standard_normal((N, D)).astype(np.float32) * 3)
    ones = W.bf16_bits_from_f32(np.ones((N, D), np.float32))
    o, _ = oracle.attention_rows(spec, grid, (1, 1, 1), D, 0.25, q16, k16, ones, range(N))
    np.testing.assert_allclose(o, 1.0, rtol=0, atol=1e-13)


def test_attention_on_tiny_workload_rows_subset():
    w = W.tiny()
    q = W.head_tensor(w, "q", 0, 1)
    k = W.head_tensor(w, "k", 0, 1)
    v = W.head_tensor(w, "v", 0, 1)
    rows = [0, 5, 63, 64, 200, 255]
    o_all, lse_all = oracle.attention_rows(w.specs[1], (w.T, w.H, w.W), w.unit, w.D, w.scale,
                                           q, k, v, range(w.N))
    o, lse = oracle.attention_rows(w.specs[1], (w.T, w.H, w.W), w.unit, w.D, w.scale, q, k, v, rows)
    np.testing.assert_array_equal(o, o_all[rows])
    np.testing.assert_array_equal(lse, lse_all[rows])


# ---------------------------------------------------------------------------
# inputs


def test_bf16_rounding_ties_to_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 3.0e38], dtype=np.float32)
    b = W.bf16_bits_from_f32(x)
    back = W.bf16_bits_to_f32(b)
    assert back[0] == 1.0
    assert back[1] == 1.0                       # tie rounds to the even mantissa
    assert back[2] == 1.0 + 4 * 2 ** -8         # tie rounds up to even
    assert back[3] == -2.5
    assert np.isfinite(back[4])


def test_stripe_parameter_draw_is_in_range_and_seeded():
    p1 = W.draw_stripe_params(40, 100)
    p2 = W.draw_stripe_params(40, 100)
    assert p1 == p2
    for p in p1:
        assert 1 <= p["Tw"] <= 4 and 0 <= p["To"] <= 2 and p["Ts"] in (21, 7, 5)
        assert 80 <= p["Sw"] <= 720 and p["So"] in (0, 80, 160) and p["Ss"] in (3600, 1200, 400)


# --- layout 1 (frame 0 first, then position-major) for temporal heads -------------


def test_frame0_first_order_structure():
    # "Sparse VideoGen ... on TPU", "arranging tokens for efficient temporal
    # access": tokens of one spatial position across frames become contiguous;
    # frame 0 (the sink) comes first.
    T, H, Wd = 4, 3, 5
    HW, N = H * Wd, T * H * Wd
    perm = oracle.tile_major_order((T, H, Wd), (1, 1, 1), 128, layout=1)
    assert sorted(perm[:N].tolist()) == list(range(N))          # a bijection onto the real tokens
    assert (perm[N:] == -1).all()
    t, h, w = perm[:N] // HW, (perm[:N] % HW) // Wd, perm[:N] % Wd
    assert (t[:HW] == 0).all() and (h[:HW] * Wd + w[:HW] == np.arange(HW)).all()
    runs = (h[HW:] * Wd + w[HW:]).reshape(HW, T - 1)             # one run of T-1 slots per position
    assert (runs == np.arange(HW)[:, None]).all()
    assert (t[HW:].reshape(HW, T - 1) == np.arange(1, T)[None, :]).all()


def test_layout1_counts_match_keep_matrix_and_total():
    # the brute-force tile counts under layout 1, recomputed from the dense keep
    # matrix permuted by the order, and the total against the kept-pair routine
    grid, unit = (5, 4, 6), (1, 1, 1)
    spec = dict(W.mask_spec("temporal", sink=1, rh=1, rw=2), layout=1)
    n_slots, B = 128, 32
    perm = oracle.tile_major_order(grid, unit, n_slots, layout=1)
    km = oracle.keep_matrix(spec, grid, unit).astype(np.int64)
    real = perm >= 0
    kp = np.zeros((n_slots, n_slots), dtype=np.int64)
    kp[np.ix_(real, real)] = km[np.ix_(perm[real], perm[real])]
    ref = kp.reshape(n_slots // B, B, n_slots // B, B).sum(axis=(1, 3))
    counts, real_q = oracle.tile_counts(spec, grid, unit, n_slots, B, B)
    assert (counts == ref).all()
    assert real_q.sum() == np.prod(grid)
    assert counts.sum() == oracle.kept_pairs(spec, grid, unit)
    spec0 = dict(spec, layout=0)
    c0, _ = oracle.tile_counts(spec0, grid, unit, n_slots, B, B)
    assert c0.sum() == counts.sum()                                # the order does not change the pairs


def test_layout1_temporal_keys_form_bands():
    # a temporal head's kept keys past frame 0 are one contiguous band per
    # kept latent row: at most 2 rh + 1 runs per query
    grid = (6, 7, 9)
    T, H, Wd = grid
    HW = H * Wd
    rh, rw = 1, 2
    spec = dict(W.mask_spec("temporal", sink=1, rh=rh, rw=rw), layout=1)
    perm = oracle.tile_major_order(grid, (1, 1, 1), T * HW, layout=1)
    km = oracle.keep_matrix(spec, grid, (1, 1, 1))
    for q in (0, 17, 3 * HW + 40, T * HW - 1):
        row = km[q, perm[HW:]].astype(np.int8)                    # keys of frames >= 1 in layout order
        starts = int(((row[1:] == 1) & (row[:-1] == 0)).sum() + row[0])
        hq = (q % HW) // Wd
        assert starts == min(hq + rh, H - 1) - max(hq - rh, 0) + 1
        assert km[q, perm[:HW]].all()                               # the sink keeps all of frame 0


# --- tile-aligned rounding (lossy mode) ---------------------------------------------


def _rounded_from_keep_matrix(spec, grid, unit, n_slots, B):
    # the rounding rule restated on the dense keep matrix permuted into the head's order
    perm = oracle.tile_major_order(grid, unit, n_slots, layout=int(spec.get("layout", 0)))
    km = oracle.keep_matrix(spec, grid, unit).astype(np.int64)
    real = perm >= 0
    kp = np.zeros((n_slots, n_slots), dtype=np.int64)
    kp[np.ix_(real, real)] = km[np.ix_(perm[real], perm[real])]
    cnt = kp.reshape(n_slots // B, B, n_slots // B, B).sum(axis=(1, 3))
    rq = real.reshape(-1, B).sum(axis=1)
    pairs = rq[:, None] * rq[None, :]
    keep = (cnt > 0) & (2 * cnt >= pairs)
    return np.where(keep, np.where(rq[None, :] == B, 2, 1), 0), cnt, pairs


@pytest.mark.parametrize("layout", [0, 1])
def test_rounded_map_rule_and_exact_tiles(layout):
    grid, unit, n_slots, B = (5, 4, 6), (1, 2, 3), 128, 32
    spec = dict(W.mask_spec("temporal", sink=1, rh=1, rw=1), layout=layout, tile_round=1)
    got = oracle.rounded_tile_map(spec, grid, unit, n_slots, B, B)
    want, cnt, pairs = _rounded_from_keep_matrix(spec, grid, unit, n_slots, B)
    assert (got == want).all()
    exact = oracle.tile_map(spec, grid, unit, n_slots, B, B)
    assert (got[exact == 0] == 0).all() and (got[exact == 2] == 2).all()   # only boundary tiles move
    assert ((got == 1) <= (exact == 1)).all()
    moved = exact == 1
    assert ((got[moved] != 0) == (2 * cnt[moved] >= pairs[moved])).all()


def test_rounding_a_full_mask_changes_nothing():
    grid, unit = (3, 7, 9), (1, 1, 1)
    spec = dict(W.mask_spec("full"), tile_round=1)
    assert (oracle.rounded_tile_map(spec, grid, unit, 256, 64, 64) ==
            oracle.tile_map(spec, grid, unit, 256, 64, 64)).all()


def test_rounded_attention_is_exact_for_a_tile_aligned_mask():
    # spatial |dt| <= 0 with one frame per tile: every tile pair is full or
    # empty, so rounding must not change a single output
    grid, unit, B, D = (4, 4, 8), (1, 4, 8), 32, 64
    spec = W.mask_spec("spatial", sink=0, rt=0)
    rspec = dict(spec, tile_round=1)
    w = W.Workload("t", 1, *grid, 1, D, unit, B, B, (spec,))
    q, k, v = (W.head_tensor(w, x, 0, 0) for x in "qkv")
    rows = np.arange(int(np.prod(grid)))
    o1, l1 = oracle.attention_rows(spec, grid, unit, D, w.scale, q, k, v, rows)
    o2, l2 = oracle.attention_rows_rounded(rspec, grid, unit, 128, B, B, D, w.scale, q, k, v, rows)
    assert np.allclose(o1, o2, atol=1e-12) and np.allclose(l1, l2, atol=1e-12)


def test_rounded_attention_against_dense_reference():
    # the rounded keep matrix, dense fp64 softmax by hand
    grid, unit, B, D = (5, 4, 6), (1, 2, 3), 32, 64
    spec = dict(W.mask_spec("temporal", sink=1, rh=1, rw=1), tile_round=1)
    cls, _, _ = _rounded_from_keep_matrix(spec, grid, unit, 128, B)
    perm = oracle.tile_major_order(grid, unit, 128)
    w = W.Workload("t", 1, *grid, 1, D, unit, B, B, (spec,))
    q, k, v = (W.head_tensor(w, x, 0, 0) for x in "qkv")
    f = lambda b: (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    qf, kf, vf = f(q), f(k), f(v)
    N = int(np.prod(grid))
    slot_of = np.empty(N, dtype=np.int64)
    slot_of[perm[perm >= 0]] = np.nonzero(perm >= 0)[0]
    keep = np.zeros((N, N), dtype=bool)
    for n in range(N):
        for m in range(N):
            keep[n, m] = cls[slot_of[n] // B, slot_of[m] // B] != 0
    s = qf @ kf.T * w.scale
    s[~keep] = -np.inf
    mx = s.max(axis=1, keepdims=True)
    p = np.exp(s - mx)
    o_ref = (p @ vf) / p.sum(axis=1, keepdims=True)
    o, _ = oracle.attention_rows_rounded(spec, grid, unit, 128, B, B, D, w.scale, q, k, v, np.arange(N))
    assert np.abs(o - o_ref).max() < 1e-12


# ---------------------------------------------------------------------------
# SVG routing (sampled-query profiling of spatial vs temporal masks)


def _route(sp, tm, grid, D, q, k, v, rows, scale=None):
    scale = scale if scale is not None else 1.0 / np.sqrt(D)
    return oracle.svg_route(sp, tm, grid, D, scale, q, k, v, rows)


def _rand_bits(shape, seed):
    g = np.random.Generator(np.random.PCG64(seed))
    return W.bf16_bits_from_f32(g.standard_normal(shape, dtype=np.float32))


def test_route_uniform_weights_closed_form():
    # q = 0 makes every kept key weigh the same, so each output is the mean of
    # v over the kept keys.  Grid T=3, H=2, W=3 (token n = (t*2 + h)*3 + w).
    # Row 17 = (t2, h1, w2): spatial rt=0 + sink keeps frames 0 and 2 = tokens
    # 0..5, 12..17; temporal rh=0, rw=1 keeps h=1, w in {1,2} of every frame =
    # tokens 4,5,10,11,16,17.  Row 0 = (t0, h0, w0): spatial keeps frame 0 =
    # 0..5; temporal keeps h=0, w in {0,1} = 0,1,6,7,12,13.
    grid, D = (3, 2, 3), 4
    q = np.zeros((1, 1, 18, D), dtype=np.uint16)
    k = _rand_bits((1, 1, 18, D), 1)
    v = _rand_bits((1, 1, 18, D), 2)
    vf = W.bf16_bits_to_f32(v[0, 0]).astype(np.float64)
    sp = [W.mask_spec("spatial", sink=1, rt=0)]
    tm = [W.mask_spec("temporal", sink=0, rh=0, rw=1)]
    err, flags = _route(sp, tm, grid, D, q, k, v, [0, 17])
    full = vf.mean(axis=0)
    keep = {(17, 0): list(range(6)) + list(range(12, 18)), (17, 1): [4, 5, 10, 11, 16, 17],
            (0, 0): list(range(6)), (0, 1): [0, 1, 6, 7, 12, 13]}
    for c in (0, 1):
        want = sum(((vf[keep[(r, c)]].mean(axis=0) - full) ** 2).sum() for r in (0, 17)) / (2 * D)
        assert err[0, c] == pytest.approx(want, rel=1e-12, abs=1e-300)
    assert flags[0] == int(err[0, 1] < err[0, 0])


def test_route_keep_all_candidate_has_zero_deviation():
    grid, D = (4, 3, 5), 8
    N = 60
    q, k, v = (_rand_bits((2, 2, N, D), s) for s in (3, 4, 5))
    rows = [0, 7, 33, 59]
    # head 0: the spatial candidate keeps every key; head 1: the temporal one
    sp = [W.mask_spec("spatial", sink=0, rt=3), W.mask_spec("spatial", sink=0, rt=0)]
    tm = [W.mask_spec("temporal", sink=1, rh=0, rw=0), W.mask_spec("temporal", sink=0, rh=2, rw=4)]
    err, flags = _route(sp, tm, grid, D, q, k, v, rows)
    assert err[0, 0] == 0.0 and err[0, 1] > 0.0 and flags[0] == 0
    assert err[1, 1] == 0.0 and err[1, 0] > 0.0 and flags[1] == 1


def test_route_tie_goes_spatial_and_batches_average():
    grid, D = (3, 4, 4), 8
    N = 48
    q, k, v = (_rand_bits((2, 1, N, D), s) for s in (6, 7, 8))
    rows = [1, 20, 47]
    same = W.mask_spec("spatial", sink=1, rt=0)
    err, flags = _route([same], [same], grid, D, q, k, v, rows)
    assert err[0, 0] == err[0, 1] > 0.0 and flags[0] == 0
    # the deviation is a mean over the batch: the two batches' own deviations
    tm = W.mask_spec("temporal", sink=1, rh=1, rw=1)
    e2, _ = _route([same], [tm], grid, D, q, k, v, rows)
    e0, _ = _route([same], [tm], grid, D, q[:1], k[:1], v[:1], rows)
    e1, _ = _route([same], [tm], grid, D, q[1:], k[1:], v[1:], rows)
    np.testing.assert_allclose(e2, (e0 + e1) / 2, rtol=1e-12)


def test_route_picks_the_pattern_the_heads_follow():
    # frame-structured q/k attend within their frame (the pages' spatial
    # heads), position-structured ones to their position across frames (the
    # temporal heads)
    w = W.tiny_routing()
    q, k, v = (W.full_tensor(w, x) for x in "qkv")
    rows = W.route_rows(w.N, 0.05)
    sp = [a for a, _ in w.route_specs]
    tm = [b for _, b in w.route_specs]
    err, flags = _route(sp, tm, (w.T, w.H, w.W), w.D, q, k, v, rows)
    assert flags[0] == 0 and flags[1] == 1 and flags[3] == 0
    assert err[0, 0] < 1e-3 * err[0, 1] and err[1, 1] < 1e-3 * err[1, 0]


def test_route_rows_sample():
    r = W.route_rows(75600, 0.01)
    assert len(r) == 756 and len(np.unique(r)) == 756 and r.min() >= 0 and r.max() < 75600
    assert np.all(np.diff(r) > 0)
