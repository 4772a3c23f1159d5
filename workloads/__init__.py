"""Seeded synthetic workloads for block-sparse 3D-video attention.

This module only describes inputs: grid shapes, head counts, per-head mask
parameters, tile shapes, and seeded N(0,1) draws rounded to bf16.  It holds
none of the method's arithmetic (no mask predicate, no permutation, no
attention), so both the CPU oracle and the CUDA path can consume it.

Workloads (stand-ins for the video-DiT activations the pages measure on;
weights and prompts are not available, so inputs are iid N(0,1)):

* ``tiny``            4x8x8 grid, 2 heads, d=64, SVG spatial + temporal heads,
                      64x64 tiles over (1,8,8) units.
* ``svg_wan720p``     21x45x80 grid (Wan 720p latent, 75,600 tokens), 10 heads,
                      d=128; 5 SVG spatial + 5 SVG temporal heads with the
                      frame-0 sink; 128x128 tiles over (1,8,16) units.
* ``sta_hunyuan720p`` 30x48x80 grid (115,200 tokens), 24 heads, d=128,
                      Sliding Tile Attention window (3,3,5) tiles of (6,8,8).
* ``stripe_wan720p``  21x45x80 grid, 40 heads, d=128, one stripe mask
                      M(Tw,To,Ts,Sw,So,Ss) per head drawn from a seed, + sink.
* ``scaling``         T x 45 x 80 grids, 40 heads, d=128, dense or SVG spatial
                      mask, with a q-tile / kv-tile sweep.

Random streams: tensor ``which`` in {q,k,v} of batch ``b``, head ``h`` is drawn
from ``numpy.random.Generator(PCG64(SeedSequence([seed_which, b, h])))`` as
``standard_normal(N*D, float32)`` in natural (t,h,w)-major token order, then
rounded to bf16 with round-to-nearest-even.  Both sides consume the bf16 values.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

MASK_KINDS = {"full": 0, "spatial": 1, "temporal": 2, "sta": 3, "stripe": 4}

SPEC_KEYS = ("kind", "sink", "rt", "rh", "rw", "kt", "kh", "kw",
             "Tw", "To", "Ts", "Sw", "So", "Ss", "layout", "tile_round")


def mask_spec(kind: str, sink: int = 0, **params) -> Dict[str, int]:
    """A per-head mask description as a plain dict of integers.

    kind     one of ``MASK_KINDS``
    sink     1: every query also keeps all real keys of frame 0
    rt       SVG spatial radius in frames
    rh, rw   SVG temporal radii in latent rows / columns
    kt,kh,kw STA window, counted in 3D units (clamped to the unit grid)
    Tw,To,Ts,Sw,So,Ss  stripe width / offset / stride, inter-frame (T*) and
             intra-frame (S*, over s = h*W + w)
    layout   token order of the head: 0 tile-major over 3D units, 1 frame 0
             first, then every spatial position with its other frames
             (temporal heads only)
    tile_round  1: tile-aligned rounding of the mask (lossy; SVG and full heads)
    """
    if kind not in MASK_KINDS:
        raise ValueError(f"unknown mask kind {kind!r}")
    spec = {k: 0 for k in SPEC_KEYS}
    spec["kind"] = MASK_KINDS[kind]
    spec["sink"] = int(sink)
    for k, v in params.items():
        if k not in SPEC_KEYS:
            raise ValueError(f"unknown mask parameter {k!r}")
        spec[k] = int(v)
    # strides of 0 would make the stripe undefined; default to "no period"
    if kind == "stripe":
        for k in ("Ts", "Ss"):
            if spec[k] <= 0:
                raise ValueError("stripe strides must be positive")
    return spec


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    H: int
    W: int
    heads: int
    D: int
    unit: Tuple[int, int, int]
    q_tile: int
    kv_tile: int
    specs: Tuple[Dict[str, int], ...]
    seeds: Tuple[int, int, int] = (0, 1, 2)
    note: str = ""
    # per-head structure of the q/k draws: "" iid, "frame" or "position" (see
    # ``head_tensor``); empty tuple = iid everywhere
    structure: Tuple[str, ...] = ()
    structure_amp: float = 0.0
    # candidate masks for SVG routing (one pair per head), empty if not routed
    route_specs: Tuple[Tuple[Dict[str, int], Dict[str, int]], ...] = ()
    # global index of local head 0: a shard holding heads [lo, hi) of a
    # workload draws exactly the inputs those heads have in the whole one
    head_offset: int = 0

    @property
    def N(self) -> int:
        return self.T * self.H * self.W

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.D))

    def with_tiles(self, q_tile: int, kv_tile: int,
                   unit: Optional[Tuple[int, int, int]] = None) -> "Workload":
        return replace(self, q_tile=q_tile, kv_tile=kv_tile,
                       unit=unit if unit is not None else self.unit)

    def head_shard(self, lo: int, hi: int) -> "Workload":
        """Heads [lo, hi) of this workload as a workload of their own (same
        grid, tiles and per-head masks; inputs drawn as in the whole one)."""
        if not 0 <= lo < hi <= self.heads:
            raise ValueError(f"head range [{lo}, {hi}) outside {self.heads} heads")
        return replace(self, heads=hi - lo, specs=self.specs[lo:hi],
                       structure=self.structure[lo:hi] if self.structure else (),
                       route_specs=self.route_specs[lo:hi] if self.route_specs else (),
                       head_offset=self.head_offset + lo)

    def describe(self) -> Dict[str, object]:
        return {"workload": self.name, "B": self.B, "grid": [self.T, self.H, self.W],
                "tokens": self.N, "heads": self.heads, "d": self.D,
                "unit": list(self.unit), "q_tile": self.q_tile,
                "kv_tile": self.kv_tile}


def tiny() -> Workload:
    specs = (mask_spec("spatial", sink=1, rt=1),
             mask_spec("temporal", sink=1, rh=1, rw=1))
    return Workload("tiny_4x8x8", 1, 4, 8, 8, 2, 64, (1, 8, 8), 64, 64, specs,
                    note="fp32 N(0,1) draw seen by the kernel as bf16")


def svg_wan720p(temporal_layout: int = 0, tile_round: int = 0) -> Workload:
    """SVG on the Wan 720p latent: 5 spatial + 5 temporal heads with the sink.
    temporal_layout=1 puts the temporal heads in the frame-0-first,
    position-major order (the temporal-head permutation); same keep sets.
    tile_round=1 rounds every head's mask to whole tiles (lossy)."""
    specs = tuple([mask_spec("spatial", sink=1, rt=1, tile_round=tile_round)] * 5 +
                  [mask_spec("temporal", sink=1, rh=5, rw=8, layout=temporal_layout,
                             tile_round=tile_round)] * 5)
    name = ("svg_wan720p_21x45x80" + ("_temporal_frame0_first" if temporal_layout else "") +
            ("_tile_rounded" if tile_round else ""))
    return Workload(name, 1, 21, 45, 80, 10, 128, (1, 8, 16), 128, 128, specs)


def svg_wan720p_routing(amp: float = 10.0, temporal_layout: int = 0) -> Workload:
    """SVG routing on the Wan 720p latent: every head has both candidates
    (spatial |dt| <= 1 and temporal |dh| <= 5, |dw| <= 8, both with the
    frame-0 sink).  The q/k draws of heads 0-4 carry a per-frame embedding and
    those of heads 5-9 a per-position embedding, so that the former attend
    within their frame (spatial heads) and the latter to their position across
    frames (temporal heads).  The plan starts with every head spatial.
    temporal_layout=1 gives the temporal candidate the frame-0-first order,
    which the routed heads then take."""
    sp = mask_spec("spatial", sink=1, rt=1)
    tm = mask_spec("temporal", sink=1, rh=5, rw=8, layout=temporal_layout)
    name = "svg_wan720p_routing_21x45x80" + ("_temporal_frame0_first" if temporal_layout else "")
    return Workload(name, 1, 21, 45, 80, 10, 128, (1, 8, 16), 128, 128,
                    tuple([sp] * 10), structure=tuple(["frame"] * 5 + ["position"] * 5),
                    structure_amp=amp, route_specs=tuple([(sp, tm)] * 10))


def tiny_routing(amp: float = 10.0) -> Workload:
    """4x8x8 grid, 4 heads (frame, position, iid, frame structure), d=64,
    candidates spatial |dt| <= 1 and temporal |dh|, |dw| <= 1, with the sink."""
    sp = mask_spec("spatial", sink=1, rt=1)
    tm = mask_spec("temporal", sink=1, rh=1, rw=1)
    return Workload("tiny_routing_4x8x8", 2, 4, 8, 8, 4, 64, (1, 8, 8), 64, 64, tuple([sp] * 4),
                    structure=("frame", "position", "", "frame"), structure_amp=amp,
                    route_specs=tuple([(sp, tm)] * 4))


def sta_hunyuan720p() -> Workload:
    specs = tuple([mask_spec("sta", sink=0, kt=3, kh=3, kw=5)] * 24)
    return Workload("sta_hunyuan720p_30x48x80", 1, 30, 48, 80, 24, 128, (6, 8, 8),
                    128, 128, specs)


def draw_stripe_params(heads: int, seed_p: int = 100) -> List[Dict[str, int]]:
    """Per-head stripe parameters, drawn in a fixed order from one stream.

    Tw in [1,4], To in [0,2], Ts in {21,7,5}, Sw in [80,720],
    So in {0,80,160}, Ss in {3600,1200,400}; integer ranges inclusive.
    """
    g = np.random.Generator(np.random.PCG64(seed_p))
    out = []
    for _ in range(heads):
        Tw = int(g.integers(1, 5))
        To = int(g.integers(0, 3))
        Ts = int(g.choice([21, 7, 5]))
        Sw = int(g.integers(80, 721))
        So = int(g.choice([0, 80, 160]))
        Ss = int(g.choice([3600, 1200, 400]))
        out.append(dict(Tw=Tw, To=To, Ts=Ts, Sw=Sw, So=So, Ss=Ss))
    return out


def stripe_wan720p(seed_p: int = 100) -> Workload:
    specs = tuple(mask_spec("stripe", sink=1, **p)
                  for p in draw_stripe_params(40, seed_p))
    return Workload("stripe_wan720p_21x45x80", 1, 21, 45, 80, 40, 128, (1, 8, 16),
                    128, 128, specs, note=f"stripe params seed {seed_p}")


SCALING_T = (5, 9, 13, 21, 33)
SWEEP_Q = (64, 128, 256)
SWEEP_KV = (64, 128)


def scaling(T: int, mask: str = "full", q_tile: int = 128, kv_tile: int = 128) -> Workload:
    if mask == "full":
        spec = mask_spec("full")
    elif mask == "spatial":
        spec = mask_spec("spatial", sink=1, rt=1)
    else:
        raise ValueError(mask)
    unit = (1, 8, 8) if min(q_tile, kv_tile) == 64 else (1, 8, 16)
    return Workload(f"scaling_{mask}_{T}x45x80_q{q_tile}_k{kv_tile}", 1, T, 45, 80,
                    40, 128, unit, q_tile, kv_tile, tuple([spec] * 40))


def all_parity_workloads() -> List[Workload]:
    out = [tiny(), svg_wan720p(), svg_wan720p(temporal_layout=1), svg_wan720p(tile_round=1),
           svg_wan720p(temporal_layout=1, tile_round=1), sta_hunyuan720p(), stripe_wan720p()]
    for T in SCALING_T:
        out.append(scaling(T, "full"))
        out.append(scaling(T, "spatial"))
    for q in SWEEP_Q:
        for k in SWEEP_KV:
            if (q, k) != (128, 128):
                out.append(scaling(21, "spatial", q, k))
    return out


# ---------------------------------------------------------------------------
# seeded tensors


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (round to nearest, ties to even); returns uint16 bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (b >> np.uint32(16)) & np.uint32(1)
    r = (b + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def head_draw_f32(seed: int, b: int, h: int, n: int, d: int) -> np.ndarray:
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, b, h])))
    return g.standard_normal(n * d, dtype=np.float32).reshape(n, d)


def structure_embedding(w: Workload, h: int) -> Tuple[np.ndarray, np.ndarray]:
    """(class index of every natural token [N], unit-norm embeddings [C, D])
    of head ``h``: class = frame t for "frame", (h, w) position for
    "position".  Drawn from ``PCG64(SeedSequence([seeds[0] + 1000, h]))``."""
    kind = w.structure[h]
    hg = w.head_offset + h
    n = np.arange(w.N)
    if kind == "frame":
        cls, C = n // (w.H * w.W), w.T
    elif kind == "position":
        cls, C = n % (w.H * w.W), w.H * w.W
    else:
        raise ValueError(f"no structure for head {h}")
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([w.seeds[0] + 1000, hg])))
    e = g.standard_normal((C, w.D))
    e /= np.linalg.norm(e, axis=1, keepdims=True)
    return cls, e.astype(np.float32)


def head_tensor(w: Workload, which: str, b: int, h: int) -> np.ndarray:
    """bf16 bits [N, D] of tensor ``which`` for batch ``b``, head ``h`` (natural order).

    With a structured head, q and k both get ``structure_amp`` times the
    head's embedding of each token's class added to the N(0,1) draw before
    the bf16 rounding; v stays iid."""
    seed = w.seeds["qkv".index(which)]
    x = head_draw_f32(seed, b, w.head_offset + h, w.N, w.D)
    if which in "qk" and w.structure and w.structure[h]:
        cls, e = structure_embedding(w, h)
        x += np.float32(w.structure_amp) * e[cls]
    return bf16_bits_from_f32(x)


def full_tensor(w: Workload, which: str, heads: Optional[Sequence[int]] = None,
                threads: Optional[int] = None) -> np.ndarray:
    """bf16 bits [B, Hh, N, D] (natural order); only ``heads`` filled if given.

    Heads are drawn in parallel threads; each head has its own stream, so the
    result does not depend on the thread count.
    """
    from concurrent.futures import ThreadPoolExecutor
    import os

    out = np.zeros((w.B, w.heads, w.N, w.D), dtype=np.uint16)
    hs = list(range(w.heads) if heads is None else heads)
    jobs = [(b, h) for b in range(w.B) for h in hs]

    def fill(job):
        b, h = job
        out[b, h] = head_tensor(w, which, b, h)

    n = threads or min(len(jobs), os.cpu_count() or 1, 16)
    if n <= 1:
        for j in jobs:
            fill(j)
    else:
        with ThreadPoolExecutor(n) as ex:
            list(ex.map(fill, jobs))
    return out


def route_rows(N: int, frac: float = 0.01, seed: int = 11) -> np.ndarray:
    """The query sample of SVG routing: round(frac * N) (at least 1) distinct
    natural token indices drawn uniformly from ``PCG64(seed)``, ascending."""
    R = max(1, int(round(frac * N)))
    g = np.random.Generator(np.random.PCG64(seed))
    return np.sort(g.choice(N, size=min(R, N), replace=False)).astype(np.int64)


def sample_rows(w: Workload, head: int, R: int, seed: int = 7) -> np.ndarray:
    """Stratified natural query indices for sampled parity checks.

    Includes frame 0, the last frame, the last latent row (which lands in the
    padded edge of 3D units when H is not a multiple of the unit height), the
    grid corners and uniform random rows.
    """
    T, H, W = w.T, w.H, w.W
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, head])))
    picks: Dict[int, None] = {}
    for t in (0, T - 1):
        for h in (0, H - 1):
            for x in (0, W - 1):
                picks[(t * H + h) * W + x] = None
    k = max(1, R // 8)
    for t in (0, T - 1):
        for _ in range(k):
            picks[(t * H + int(g.integers(0, H))) * W + int(g.integers(0, W))] = None
    for _ in range(k):
        t = int(g.integers(0, T))
        h = H - 1 - int(g.integers(0, min(H, 5)))
        picks[(t * H + h) * W + int(g.integers(0, W))] = None
    target = min(R, w.N)
    while len(picks) < target:
        picks[int(g.integers(0, w.N))] = None
    return np.array(sorted(list(picks)[:target]), dtype=np.int64)
