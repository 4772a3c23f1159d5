"""CPU: the seeded input generators hold to the recipe the design states
(per-(tensor, batch, head) N(0,1) streams rounded to bf16 ties-to-even, the
stripe parameter ranges, the routing sample, the stratified parity rows).
The module is shared by the oracle and the CUDA path, so a change here moves
both sides at once; these checks keep it fixed."""
import numpy as np
import pytest

import workloads as W


def test_bf16_rounding_matches_torch():
    torch = pytest.importorskip("torch")
    g = np.random.Generator(np.random.PCG64(3))
    normal = g.standard_normal(100_000).astype(np.float32)
    # exact ties: a bf16 value plus half of its last place
    base = g.integers(0x0080, 0x7F00, 4000).astype(np.uint32) << np.uint32(16)
    ties = (base + np.uint32(0x8000)).view(np.float32)
    special = np.array([0.0, -0.0, np.inf, -np.inf, 1e-40, -1e-40, 3.0e38, 3.4e38, 1.0, -2.5], np.float32)
    x = np.concatenate([normal, ties, -ties, special])
    ours = W.bf16_bits_from_f32(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    # a tie goes to the even neighbour: 1 + 2^-8 -> 1.0, 1 + 3 * 2^-8 -> 1 + 2^-6
    assert W.bf16_bits_from_f32(np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8], np.float32)).tolist() == [0x3F80, 0x3F82]


def test_bf16_round_trip_is_exact_on_bf16_values():
    bits = np.arange(0, 0x7F80, 7, dtype=np.uint16)
    assert np.array_equal(W.bf16_bits_from_f32(W.bf16_bits_to_f32(bits)), bits)


def test_head_tensors_follow_the_stated_streams():
    w = W.tiny()
    assert tuple(w.seeds) == (0, 1, 2)
    for which, seed in zip("qkv", w.seeds):
        for b, h in ((0, 0), (0, 1)):
            g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, b, h])))
            draw = g.standard_normal(w.N * w.D, dtype=np.float32).reshape(w.N, w.D)
            assert np.array_equal(W.head_tensor(w, which, b, h), W.bf16_bits_from_f32(draw)), (which, b, h)
    # streams differ between tensors, heads and batches
    q00, k00, q01 = W.head_tensor(w, "q", 0, 0), W.head_tensor(w, "k", 0, 0), W.head_tensor(w, "q", 0, 1)
    assert not np.array_equal(q00, k00) and not np.array_equal(q00, q01)
    assert not np.array_equal(q00, W.head_tensor(w, "q", 1, 0))


def test_full_tensor_independent_of_threads():
    w = W.tiny()
    a = W.full_tensor(w, "v", threads=1)
    b = W.full_tensor(w, "v", threads=4)
    assert np.array_equal(a, b)
    assert np.array_equal(a[0, 1], W.head_tensor(w, "v", 0, 1))


def test_structured_heads_move_q_and_k_only():
    w = W.tiny_routing()
    for h, kind in enumerate(w.structure):
        plain_v = W.bf16_bits_from_f32(W.head_draw_f32(w.seeds[2], 0, h, w.N, w.D))
        assert np.array_equal(W.head_tensor(w, "v", 0, h), plain_v)
        plain_q = W.bf16_bits_from_f32(W.head_draw_f32(w.seeds[0], 0, h, w.N, w.D))
        assert np.array_equal(W.head_tensor(w, "q", 0, h), plain_q) == (not kind)


def test_stripe_parameters_in_their_ranges():
    ps = W.draw_stripe_params(40)
    assert ps == W.draw_stripe_params(40)
    for p in ps:
        assert 1 <= p["Tw"] <= 4 and 0 <= p["To"] <= 2 and p["Ts"] in (21, 7, 5)
        assert 80 <= p["Sw"] <= 720 and p["So"] in (0, 80, 160) and p["Ss"] in (3600, 1200, 400)
    for key, values in (("Tw", {1, 2, 3, 4}), ("To", {0, 1, 2}), ("Ts", {21, 7, 5}), ("So", {0, 80, 160}),
                        ("Ss", {3600, 1200, 400})):
        assert {p[key] for p in ps} == values, key
    w = W.stripe_wan720p()
    assert w.heads == 40
    assert [dict(s) for s in w.specs] == [W.mask_spec("stripe", 1, **p) for p in ps]


def test_route_rows_sample():
    r = W.route_rows(75600, 0.01)
    assert len(r) == 756 and r.dtype == np.int64
    assert np.all(np.diff(r) > 0) and r[0] >= 0 and r[-1] < 75600
    assert np.array_equal(r, W.route_rows(75600, 0.01))
    assert not np.array_equal(r, W.route_rows(75600, 0.01, seed=12))
    assert len(W.route_rows(50, 0.001)) == 1
    assert np.array_equal(W.route_rows(10, 5.0), np.arange(10))


def test_sample_rows_cover_corners_and_edges():
    w = W.svg_wan720p()
    r = W.sample_rows(w, 0, 64)
    assert len(r) == 64 and np.all(np.diff(r) > 0) and r[0] >= 0 and r[-1] < w.N
    HW = w.H * w.W
    for t in (0, w.T - 1):
        for h in (0, w.H - 1):
            for x in (0, w.W - 1):
                assert (t * w.H + h) * w.W + x in set(r.tolist())
    assert np.any(r < HW) and np.any(r >= (w.T - 1) * HW)
    t_small = W.tiny()
    assert np.array_equal(W.sample_rows(t_small, 0, 10_000), np.arange(t_small.N))
