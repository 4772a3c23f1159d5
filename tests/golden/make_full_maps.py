"""Write ``full_maps.json``: SHA-256 digests of every head's full int8 tile map
at the parity workloads' full sizes, computed by the CPU oracle alone.

    python tests/golden/make_full_maps.py [--only NAME_SUBSTRING]

Every map is the oracle's brute-force classification ("Sparse VideoGen:
accelerating video diffusion attention on TPU", section "logical sparsity is
not physical sparsity": a tile pair with no kept (real query, key slot) pair is
empty, one where every such pair is kept is full, anything else is boundary),
or, for heads with tile-aligned rounding, the oracle's rounded map of the same
page's "aligning the sparse mask with execution".  Per distinct mask of a
workload the file stores the digest of the map's bytes ([n_q_tiles][n_kv_tiles],
row-major, int8), its (empty, boundary, full) tile counts and the q-tile strata
below; per head, the index of its mask.  Only ``oracle`` and ``workloads`` (seeded inputs, no arithmetic
of the method) are imported.

The number of tile-major slots follows the library's documented rule: the
padded grid rounded up to a multiple of max(128, q_tile, kv_tile).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import sys
import time

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
import workloads as W  # noqa: E402

OUT = os.path.join(HERE, "full_maps.json")


def n_slots_of(w: W.Workload) -> int:
    L = max(128, w.q_tile, w.kv_tile)
    npad = oracle.padded_tokens((w.T, w.H, w.W), w.unit)
    return -(-npad // L) * L


def head_map(w: W.Workload, spec, n_slots: int) -> np.ndarray:
    grid = (w.T, w.H, w.W)
    fn = oracle.rounded_tile_map if spec.get("tile_round", 0) else oracle.tile_map
    return fn(spec, grid, w.unit, n_slots, w.q_tile, w.kv_tile)


def strata(m: np.ndarray, seed: int, k: int = 8) -> dict:
    """Up to k q tiles (seeded pick) whose executed kv tiles are all boundary,
    and up to k whose executed kv tiles are all full: the parity tests draw
    query rows from them."""
    executed = (m != 0).sum(axis=1)
    bnd_only = np.nonzero((executed > 0) & ((m == 1).sum(axis=1) == executed))[0]
    full_only = np.nonzero((executed > 0) & ((m == 2).sum(axis=1) == executed))[0]
    g = np.random.Generator(np.random.PCG64(seed))
    pick = lambda a: sorted(int(x) for x in (g.choice(a, size=min(k, len(a)), replace=False) if len(a) else []))
    return {"boundary_only_qtiles": pick(bnd_only), "full_only_qtiles": pick(full_only),
            "n_boundary_only": int(len(bnd_only)), "n_full_only": int(len(full_only))}


def workload_record(w: W.Workload) -> dict:
    """One record per distinct mask ("maps", with its spec), and per head the
    index of its mask ("head_mask")."""
    n_slots = n_slots_of(w)
    maps, index, head_mask = [], {}, []
    for spec in w.specs:
        key = tuple(sorted(spec.items()))
        if key not in index:
            m = np.ascontiguousarray(head_map(w, spec, n_slots), dtype=np.int8)
            index[key] = len(maps)
            maps.append({"spec": dict(spec), "sha256": hashlib.sha256(m.tobytes()).hexdigest(),
                         "counts": [int((m == c).sum()) for c in range(3)],
                         "shape": list(m.shape), **strata(m, seed=len(maps))})
        head_mask.append(index[key])
    return {"grid": [w.T, w.H, w.W], "unit": list(w.unit), "q_tile": w.q_tile,
            "kv_tile": w.kv_tile, "n_slots": n_slots, "maps": maps, "head_mask": head_mask}


def heads_of(rec: dict) -> list:
    """Per-head view of a workload record: the record of each head's mask."""
    return [rec["maps"][i] for i in rec["head_mask"]]


def source_digest() -> str:
    h = hashlib.sha256()
    for f in ("vsa_oracle.c", "__init__.py"):
        with open(os.path.join(ROOT, "oracle", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--only", default="", help="recompute only workloads whose name contains this")
    args = ap.parse_args()
    data = {}
    if os.path.exists(OUT):
        with open(OUT) as f:
            data = json.load(f)
    data["source"] = ("brute-force tile classes of the CPU oracle ('Sparse VideoGen: accelerating video "
                      "diffusion attention on TPU', 'logical sparsity is not physical sparsity'; rounded "
                      "heads: 'aligning the sparse mask with execution'), per head of every parity workload")
    data["provenance"] = {"script": "tests/golden/make_full_maps.py",
                          "command": "python tests/golden/make_full_maps.py",
                          "inputs": "workload specs only (stripe parameters: PCG64 seed 100)",
                          "oracle_sources_sha256_16": source_digest()}
    wl = data.setdefault("workloads", {})
    for w in W.all_parity_workloads():
        if args.only and args.only not in w.name:
            continue
        t0 = time.time()
        wl[w.name] = workload_record(w)
        print(f"{w.name}: {time.time() - t0:.1f} s", flush=True)
        write(data)


def write(data: dict) -> None:
    """Indented by workload and mask; each mask record on one line."""
    lines = ["{"]
    top = [k for k in sorted(data) if k != "workloads"]
    for k in top:
        lines.append(f" {json.dumps(k)}: {json.dumps(data[k], sort_keys=True)},")
    lines.append(' "workloads": {')
    names = sorted(data["workloads"])
    for i, name in enumerate(names):
        rec = data["workloads"][name]
        lines.append(f"  {json.dumps(name)}: {{")
        keys = [k for k in sorted(rec) if k != "maps"]
        for k in keys:
            lines.append(f"   {json.dumps(k)}: {json.dumps(rec[k])},")
        lines.append('   "maps": [')
        for j, m in enumerate(rec["maps"]):
            lines.append("    " + json.dumps(m, sort_keys=True) + ("," if j + 1 < len(rec["maps"]) else ""))
        lines.append("   ]")
        lines.append("  }" + ("," if i + 1 < len(names) else ""))
    lines.append(" }")
    lines.append("}")
    with open(OUT, "w") as f:
        f.write("\n".join(lines) + "\n")


if __name__ == "__main__":
    main()
