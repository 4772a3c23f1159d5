"""Shared helpers for the GPU parity tests (test infrastructure).

The CUDA path and the oracle only meet here: both consume the same seeded bf16
inputs from ``workloads``, and their outputs are compared element by element.
"""
from __future__ import annotations

import numpy as np

import oracle
import workloads as W

# Output tolerance on N(0,1) inputs (max-abs and mean-abs against the fp64
# oracle), and the lse tolerance.
TOL_MAX = 2e-2
TOL_MEAN = 2e-3
TOL_LSE = 1e-2


def torch_bf16(bits: np.ndarray):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def inverse_perm(perm: np.ndarray, n_tokens: int) -> np.ndarray:
    inv = np.full(n_tokens, -1, dtype=np.int64)
    real = perm >= 0
    inv[perm[real]] = np.nonzero(real)[0]
    assert (inv >= 0).all()
    return inv


class PathRun:
    """Run the whole path (plan, permute, forward, unpermute) on one workload."""

    def __init__(self, w: W.Workload, inputs=None):
        import torch
        import block_sparse_attention_mask_b200 as vsa
        self.w = w
        self.grid = (w.T, w.H, w.W)
        if inputs is None:
            inputs = tuple(W.full_tensor(w, x) for x in "qkv")
        self.q, self.k, self.v = inputs
        self.plan = vsa.Plan(list(w.specs), self.grid, w.unit, w.q_tile, w.kv_tile)
        qd, kd, vd = (torch_bf16(x) for x in (self.q, self.k, self.v))
        o, lse = vsa.attention(self.plan, qd, kd, vd, scale=w.scale)
        torch.cuda.synchronize()
        self.plan.check()
        del qd, kd, vd
        self.o_dev = o                                  # natural order, on the GPU
        self.lse_tm = lse.cpu().numpy().astype(np.float64)
        self.perm = oracle.tile_major_order(self.grid, w.unit, self.plan.n_slots)
        # each head's own token order (its layout field)
        self.perms = [oracle.tile_major_order(self.grid, w.unit, self.plan.n_slots,
                                              layout=int(spec.get("layout", 0))) for spec in w.specs]
        self.invs = [inverse_perm(p, w.N) for p in self.perms]

    def o_rows(self, b: int, h: int, rows) -> np.ndarray:
        import torch
        idx = torch.as_tensor(np.asarray(rows, dtype=np.int64), device=self.o_dev.device)
        return self.o_dev[b, h].index_select(0, idx).float().cpu().numpy().astype(np.float64)

    def lse_natural(self, b: int, h: int) -> np.ndarray:
        return self.lse_tm[b, h][self.invs[h]]

    def compare_rows(self, h: int, rows, b: int = 0):
        """Oracle vs GPU on natural query rows of head h; returns (max, mean, lse max)."""
        w = self.w
        rows = np.asarray(rows, dtype=np.int64)
        if w.specs[h].get("tile_round", 0):
            o_ref, lse_ref = oracle.attention_rows_rounded(w.specs[h], self.grid, w.unit, self.plan.n_slots,
                                                           w.q_tile, w.kv_tile, w.D, w.scale,
                                                           self.q[b, h], self.k[b, h], self.v[b, h], rows)
        else:
            o_ref, lse_ref = oracle.attention_rows(w.specs[h], self.grid, w.unit, w.D, w.scale,
                                                   self.q[b, h], self.k[b, h], self.v[b, h], rows)
        o_gpu = self.o_rows(b, h, rows)
        lse_gpu = self.lse_natural(b, h)[rows]
        assert np.isfinite(o_gpu).all(), "GPU output has non-finite values"
        err = np.abs(o_gpu - o_ref)
        fin = np.isfinite(lse_ref)
        assert (np.isfinite(lse_gpu) == fin).all(), "rows with no kept key disagree"
        assert (o_gpu[~fin] == 0).all()
        lerr = float(np.abs(lse_gpu[fin] - lse_ref[fin]).max()) if fin.any() else 0.0
        return float(err.max()), float(err.mean()), lerr

    def check_rows(self, h: int, rows, b: int = 0):
        mx, mean, lerr = self.compare_rows(h, rows, b)
        assert mx <= TOL_MAX, f"head {h}: max abs err {mx}"
        assert mean <= TOL_MEAN, f"head {h}: mean abs err {mean}"
        assert lerr <= TOL_LSE, f"head {h}: lse max abs err {lerr}"
        return mx, mean, lerr

    def close(self):
        self.plan.close()
        self.o_dev = None


def oracle_map_rows(w: W.Workload, h: int, n_slots: int, qtiles) -> np.ndarray:
    fn = oracle.rounded_tile_map if w.specs[h].get("tile_round", 0) else oracle.tile_map
    return fn(w.specs[h], (w.T, w.H, w.W), w.unit, n_slots, w.q_tile, w.kv_tile, qtiles)


_FULL_MAPS = None


def full_maps() -> dict:
    """The oracle's full-size map digests, tile counts and q-tile strata per
    parity workload (``tests/golden/full_maps.json``)."""
    global _FULL_MAPS
    if _FULL_MAPS is None:
        import json
        import os
        path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "full_maps.json")
        with open(path) as f:
            _FULL_MAPS = json.load(f)["workloads"]
    return _FULL_MAPS


def heads_of(rec: dict) -> list:
    """Per-head view of a workload record of ``full_maps()``: each head's mask record."""
    return [rec["maps"][i] for i in rec["head_mask"]]


def parity_rows(w: W.Workload, h: int, R: int = 512, seed: int = 7) -> np.ndarray:
    """R stratified natural query rows of head h for a sampled parity check.

    The strata of ``workloads.sample_rows`` (frame 0, the last frame, the
    padded-edge latent rows, the grid corners, uniform rows) plus rows of q
    tiles whose executed kv tiles are all boundary and of q tiles whose
    executed kv tiles are all full, as the oracle's full map of the head
    classifies them (q tiles listed in ``tests/golden/full_maps.json``).  Up
    to R/4 rows come from those q tiles, spread evenly over them."""
    rec = full_maps()[w.name]
    head = heads_of(rec)[h]
    perm = oracle.tile_major_order((w.T, w.H, w.W), w.unit, rec["n_slots"],
                                   layout=int(w.specs[h].get("layout", 0)))
    tiles = head["boundary_only_qtiles"] + head["full_only_qtiles"]
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, h, 1])))
    picks = {}
    if tiles:
        per_tile = max(1, (R // 4) // len(tiles))
        for qt in tiles:
            nat = perm[qt * w.q_tile:(qt + 1) * w.q_tile]
            nat = nat[nat >= 0]
            for n in g.choice(nat, size=min(per_tile, len(nat)), replace=False):
                picks[int(n)] = None
    target = min(R, w.N)
    for n in W.sample_rows(w, h, max(1, target - len(picks)), seed=seed):
        picks[int(n)] = None
    while len(picks) < target:                  # rows both strata picked
        picks[int(g.integers(0, w.N))] = None
    return np.array(sorted(picks), dtype=np.int64)


def sample_qtiles(n_q: int, k: int, seed: int) -> np.ndarray:
    g = np.random.default_rng(seed)
    pick = {0, n_q - 1, n_q // 2}
    while len(pick) < min(k, n_q):
        pick.add(int(g.integers(0, n_q)))
    return np.array(sorted(pick), dtype=np.int64)
