"""CPU oracle for block-sparse 3D-video attention -- test infrastructure.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  It wraps ``vsa_oracle.c`` (plain fp64 C, built
with gcc into ``liborc.so`` beside it) through ctypes and shares no code with
the CUDA library.  What each function follows is stated in ``vsa_oracle.c``.

Classification of a tile pair from brute-force counts (the three tile kinds of
"Sparse VideoGen: accelerating video diffusion attention on TPU", section
"logical sparsity is not physical sparsity"): 0 empty when no (real query,
key slot) pair is kept, 2 full when every such pair is kept (a kv tile holding
padding is therefore never full), 1 boundary otherwise.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Iterable, Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "vsa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liborc.so")
_lib = None


class _Mask(ctypes.Structure):
    _fields_ = [(k, ctypes.c_int32) for k in
                ("kind", "sink", "rt", "rh", "rw", "kt", "kh", "kw",
                 "Tw", "To", "Ts", "Sw", "So", "Ss", "layout", "tile_round")]


class _Grid(ctypes.Structure):
    _fields_ = [(k, ctypes.c_int32) for k in ("T", "H", "W", "bt", "bh", "bw")]


def build_oracle(force: bool = False) -> str:
    """Compile liborc.so with gcc (plain C, -O2, pthreads)."""
    if force or not os.path.exists(_LIB_PATH) or \
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-Wall", "-shared", "-fPIC",
                               "-o", tmp, _SRC, "-lpthread", "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build_oracle())
        P = ctypes.POINTER
        lib.orc_padded_tokens.restype = ctypes.c_int64
        lib.orc_padded_tokens.argtypes = [P(_Grid)]
        lib.orc_tile_major_order.restype = ctypes.c_int64
        lib.orc_tile_major_order.argtypes = [P(_Grid), ctypes.c_int64, ctypes.c_void_p]
        lib.orc_frame0_first_order.restype = ctypes.c_int64
        lib.orc_frame0_first_order.argtypes = [P(_Grid), ctypes.c_int64, ctypes.c_void_p]
        lib.orc_keep.restype = ctypes.c_int
        lib.orc_keep.argtypes = [P(_Mask), P(_Grid), ctypes.c_int64, ctypes.c_int64]
        lib.orc_keep_matrix.restype = ctypes.c_int
        lib.orc_keep_matrix.argtypes = [P(_Mask), P(_Grid), ctypes.c_void_p]
        lib.orc_attention_rows.restype = ctypes.c_int
        lib.orc_attention_rows.argtypes = [P(_Mask), P(_Grid), ctypes.c_int, ctypes.c_double,
                                           ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                           ctypes.c_int64, ctypes.c_void_p,
                                           ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        lib.orc_tile_counts.restype = ctypes.c_int
        lib.orc_tile_counts.argtypes = [P(_Mask), P(_Grid), ctypes.c_int64, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_int64, ctypes.c_void_p,
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        lib.orc_kept_pairs.restype = ctypes.c_int64
        lib.orc_kept_pairs.argtypes = [P(_Mask), P(_Grid), ctypes.c_int]
        _lib = lib
    return _lib


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:  # pragma: no cover
        return os.cpu_count() or 1


def _mask(spec: Dict[str, int]) -> _Mask:
    m = _Mask()
    for k, _ in _Mask._fields_:
        setattr(m, k, int(spec.get(k, 0)))
    return m


def _grid(grid: Sequence[int], unit: Sequence[int]) -> _Grid:
    g = _Grid()
    g.T, g.H, g.W = (int(x) for x in grid)
    g.bt, g.bh, g.bw = (int(x) for x in unit)
    return g


def padded_tokens(grid, unit) -> int:
    return int(_load().orc_padded_tokens(ctypes.byref(_grid(grid, unit))))


def tile_major_order(grid, unit, n_slots: Optional[int] = None, layout: int = 0) -> np.ndarray:
    """perm[slot] = natural token index or -1 (padding), for a head's layout:
    0 tile-major over 3D units, 1 frame 0 first then position-major."""
    g = _grid(grid, unit)
    if n_slots is None:
        n_slots = padded_tokens(grid, unit)
    perm = np.empty(n_slots, dtype=np.int32)
    fn = _load().orc_frame0_first_order if layout == 1 else _load().orc_tile_major_order
    r = fn(ctypes.byref(g), n_slots, perm.ctypes.data)
    if r < 0:
        raise ValueError("n_slots smaller than the grid")
    return perm


def keep(spec, grid, unit, nq: int, nk: int) -> bool:
    return bool(_load().orc_keep(ctypes.byref(_mask(spec)), ctypes.byref(_grid(grid, unit)),
                                 int(nq), int(nk)))


def keep_matrix(spec, grid, unit) -> np.ndarray:
    N = int(np.prod(grid))
    out = np.empty((N, N), dtype=np.uint8)
    r = _load().orc_keep_matrix(ctypes.byref(_mask(spec)), ctypes.byref(_grid(grid, unit)),
                                out.ctypes.data)
    if r != 0:
        raise ValueError("grid too large for a full predicate matrix")
    return out.astype(bool)


def attention_rows(spec, grid, unit, D: int, scale: float, q: np.ndarray, k: np.ndarray,
                   v: np.ndarray, rows: Iterable[int], nthreads: Optional[int] = None
                   ) -> Tuple[np.ndarray, np.ndarray]:
    """fp64 masked attention for the given natural query rows of one (batch, head).

    q, k, v: uint16 bf16 bits [N, D] in natural order.  Returns (o [R, D], lse [R]).
    """
    rows = np.ascontiguousarray(np.asarray(list(rows) if not isinstance(rows, np.ndarray)
                                           else rows, dtype=np.int64))
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    v = np.ascontiguousarray(v, dtype=np.uint16)
    N = int(np.prod(grid))
    assert q.shape == (N, D) and k.shape == (N, D) and v.shape == (N, D)
    o = np.zeros((len(rows), D), dtype=np.float64)
    lse = np.zeros(len(rows), dtype=np.float64)
    r = _load().orc_attention_rows(ctypes.byref(_mask(spec)), ctypes.byref(_grid(grid, unit)),
                                   int(D), float(scale), q.ctypes.data, k.ctypes.data,
                                   v.ctypes.data, len(rows), rows.ctypes.data,
                                   o.ctypes.data, lse.ctypes.data,
                                   int(nthreads or default_threads()))
    if r != 0:
        raise ValueError("bad arguments to orc_attention_rows")
    return o, lse


def attention_dense_real(spec, grid, unit, scale: float, q: np.ndarray, k: np.ndarray,
                         v: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """fp64 masked attention of every natural query row from real-valued
    inputs (any float dtype, e.g. the unrounded fp32 draw), small grids only.

    softmax over the kept keys of scale * q k^T, then times v, with the keep
    matrix of ``keep_matrix``; the dense formula written out in numpy, so it
    shares no arithmetic with ``vsa_oracle.c``.  Returns (o [N, D], lse [N]).
    """
    q64, k64, v64 = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    s = scale * (q64 @ k64.T)
    s[~keep_matrix(spec, grid, unit)] = -np.inf
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    l = p.sum(axis=1, keepdims=True)
    return (p @ v64) / l, (m + np.log(l))[:, 0]


def tile_counts(spec, grid, unit, n_slots: int, Bq: int, Bk: int,
                qtiles: Optional[Iterable[int]] = None, nthreads: Optional[int] = None
                ) -> Tuple[np.ndarray, np.ndarray]:
    """Brute-force kept-pair counts [len(qtiles), n_slots/Bk] and real queries per q tile."""
    if qtiles is None:
        qtiles = range(n_slots // Bq)
    qt = np.ascontiguousarray(np.asarray(list(qtiles), dtype=np.int64))
    counts = np.zeros((len(qt), n_slots // Bk), dtype=np.int64)
    real_q = np.zeros(len(qt), dtype=np.int64)
    r = _load().orc_tile_counts(ctypes.byref(_mask(spec)), ctypes.byref(_grid(grid, unit)),
                                int(n_slots), int(Bq), int(Bk), len(qt), qt.ctypes.data,
                                counts.ctypes.data, real_q.ctypes.data,
                                int(nthreads or default_threads()))
    if r != 0:
        raise ValueError("bad arguments to orc_tile_counts")
    return counts, real_q


def classes_from_counts(counts: np.ndarray, real_q: np.ndarray, Bk: int) -> np.ndarray:
    full = counts == (real_q[:, None] * Bk)
    cls = np.where(counts == 0, 0, np.where(full, 2, 1)).astype(np.int8)
    return cls


def tile_map(spec, grid, unit, n_slots: int, Bq: int, Bk: int,
             qtiles: Optional[Iterable[int]] = None, nthreads: Optional[int] = None
             ) -> np.ndarray:
    """int8 classes [len(qtiles), n_slots/Bk]: 0 empty, 1 boundary, 2 full."""
    counts, real_q = tile_counts(spec, grid, unit, n_slots, Bq, Bk, qtiles, nthreads)
    return classes_from_counts(counts, real_q, Bk)


def kept_pairs(spec, grid, unit=(1, 1, 1), nthreads: Optional[int] = None) -> int:
    return int(_load().orc_kept_pairs(ctypes.byref(_mask(spec)), ctypes.byref(_grid(grid, unit)),
                                      int(nthreads or default_threads())))


def rounded_tile_map(spec, grid, unit, n_slots: int, Bq: int, Bk: int,
                     qtiles: Optional[Iterable[int]] = None, nthreads: Optional[int] = None
                     ) -> np.ndarray:
    """Tile-aligned rounding of the mask ("Sparse VideoGen: accelerating video
    diffusion attention on TPU", "aligning the sparse mask with execution",
    B3).  Reading: a tile pair with some kept (real query, real key) pairs
    becomes kept whole when at least half of its real pairs are kept and is
    dropped otherwise, which rounds outward and inward in balance; a kept kv
    tile holding padding slots stays class 1, its padding masked.  Classes
    from the brute-force counts in the head's token order."""
    counts, real_q = tile_counts(spec, grid, unit, n_slots, Bq, Bk, qtiles, nthreads)
    perm = tile_major_order(grid, unit, n_slots, layout=int(spec.get("layout", 0)))
    real_k = (perm.reshape(-1, Bk) >= 0).sum(axis=1)
    pairs = real_q[:, None] * real_k[None, :]
    kept = (counts > 0) & (2 * counts >= pairs)
    return np.where(kept, np.where(real_k[None, :] == Bk, 2, 1), 0).astype(np.int8)


def attention_rows_rounded(spec, grid, unit, n_slots: int, Bq: int, Bk: int, D: int, scale: float,
                           q: np.ndarray, k: np.ndarray, v: np.ndarray, rows) -> Tuple[np.ndarray, np.ndarray]:
    """fp64 softmax(scale q k^T) v of natural query rows under the rounded mask:
    query n keeps every real key of every kv tile that the rounded map keeps for
    n's q tile.  q, k, v are one head's bf16 bits [N, D] in natural order."""
    perm = tile_major_order(grid, unit, n_slots, layout=int(spec.get("layout", 0)))
    n_tok = int(np.prod(grid))
    slot_of = np.full(n_tok, -1, dtype=np.int64)
    real = perm >= 0
    slot_of[perm[real]] = np.nonzero(real)[0]
    rows = np.asarray(rows, dtype=np.int64)
    qt_of = slot_of[rows] // Bq
    qts = np.unique(qt_of)
    cls = rounded_tile_map(spec, grid, unit, n_slots, Bq, Bk, qts)
    f64 = lambda b: (np.asarray(b, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)
    qf, kf, vf = f64(q), f64(k), f64(v)
    o = np.zeros((len(rows), D))
    lse = np.full(len(rows), -np.inf)
    for i, (n, qt) in enumerate(zip(rows, qt_of)):
        kv_tiles = np.nonzero(cls[np.searchsorted(qts, qt)] != 0)[0]
        if len(kv_tiles) == 0:
            continue
        slots = (kv_tiles[:, None] * Bk + np.arange(Bk)[None, :]).ravel()
        keys = perm[slots]
        keys = keys[keys >= 0]
        s = (kf[keys] @ qf[n]) * scale
        mx = s.max()
        p = np.exp(s - mx)
        o[i] = (p @ vf[keys]) / p.sum()
        lse[i] = mx + np.log(p.sum())
    return o, lse


def svg_route(spatial_specs, temporal_specs, grid, D: int, scale: float,
              q: np.ndarray, k: np.ndarray, v: np.ndarray, rows,
              nthreads: Optional[int] = None) -> Tuple[np.ndarray, np.ndarray]:
    """SVG online profiling: route every head to its spatial or temporal mask.

    "Sparse VideoGen: accelerating video diffusion attention on TPU", section
    on SVG heads: a few query rows are sampled, their outputs are computed
    under full attention and under each head's spatial and temporal masks,
    and the head takes the sparse mask whose outputs deviate least from the
    full ones (the sample is 1-2% of the tokens, "Video diffusion
    long-sequence attention and sparsity", section 7).  Readings: the
    deviation is the mean squared difference over the sampled rows, the batch
    and the head dimension; a head goes temporal only when its temporal
    deviation is strictly smaller; the candidates' exact predicates are
    compared (their token order and rounding switches only change execution).

    q, k, v: bf16 bits [B, Hh, N, D] in natural order; rows: sampled natural
    token indices, shared by all heads and batches.  Returns (err [Hh, 2]
    float64 = (spatial, temporal) deviations, flags [Hh] int32, 1 = temporal).
    """
    q = np.asarray(q, dtype=np.uint16)
    B, Hh, N, Dq = q.shape
    assert Dq == D and N == int(np.prod(grid))
    rows = np.asarray(rows, dtype=np.int64)
    full = {f: 0 for f, _ in _Mask._fields_}     # kind 0: every real key kept
    unit = (1, 1, 1)                              # SVG predicates use no 3D unit
    err = np.zeros((Hh, 2), dtype=np.float64)
    for h in range(Hh):
        for b in range(B):
            qs, ks, vs = q[b, h], k[b, h], v[b, h]
            o_full, _ = attention_rows(full, grid, unit, D, scale, qs, ks, vs, rows, nthreads)
            for c, spec in enumerate((spatial_specs[h], temporal_specs[h])):
                o_c, _ = attention_rows(spec, grid, unit, D, scale, qs, ks, vs, rows, nthreads)
                err[h, c] += float(((o_c - o_full) ** 2).sum())
    err /= float(B * len(rows) * D)
    flags = (err[:, 1] < err[:, 0]).astype(np.int32)
    return err, flags


def shard_offsets(n_tokens: int, world: int):
    """Sequence shards of the head-sharded exchange: rank r holds natural
    tokens [off[r], off[r+1]), off[r] = floor(r * N / world)."""
    return [r * n_tokens // world for r in range(world + 1)]


def ulysses_exchange(x: np.ndarray, world: int):
    """The all-to-all of head-sharded attention ("Sparse VideoGen:
    accelerating video diffusion attention on TPU", "performing layout
    transformation on local heads": [B,S/N,H,D] -> [B,S,H/N,D]), written out
    from its definition.  x: [B, Hh, N, D] (natural token order).  Returns
    (shards, head_local): shards[r] = [B, n_r, Hh, D], the tokens rank r
    holds for every head; head_local[g] = [B, Hh/world, N, D], every token of
    rank g's heads [g Hh/world, (g+1) Hh/world)."""
    B, Hh, N, D = x.shape
    assert Hh % world == 0
    off = shard_offsets(N, world)
    hpr = Hh // world
    shards = [np.ascontiguousarray(x[:, :, off[r]:off[r + 1], :].transpose(0, 2, 1, 3)) for r in range(world)]
    head_local = [np.ascontiguousarray(x[:, g * hpr:(g + 1) * hpr]) for g in range(world)]
    return shards, head_local


def layout_gather(x_head_local: np.ndarray, perms) -> np.ndarray:
    """[B, heads, N, D] natural order -> [B, heads, n_slots, D] in each head's
    slot order (perms[h][p] = natural token of slot p, -1 = padding -> 0)."""
    B, Hh, N, D = x_head_local.shape
    S = len(perms[0])
    out = np.zeros((B, Hh, S, D), dtype=x_head_local.dtype)
    for h in range(Hh):
        real = perms[h] >= 0
        out[:, h, real] = x_head_local[:, h, perms[h][real]]
    return out
