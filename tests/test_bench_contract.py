"""CPU: the benchmark's command-line contract on its CPU arm (the oracle timed
on host cores): one JSON line with the keys and types the contract names,
nothing from ranks other than 0, and warm-up below three refused."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=600)


def test_reference_arm_line():
    r = _run(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "3"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key, typ in (("impl", str), ("metric", str), ("value", float), ("unit", str), ("n_gpus", int),
                     ("steps", int), ("warmup", int), ("ms_per_step", float), ("higher_is_better", bool),
                     ("scaling", str), ("dtype", str), ("data", str), ("config", dict),
                     ("cpu_baseline", dict), ("e2e", dict)):
        assert isinstance(d[key], typ), key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["vs_baseline"] is None and d["value"] > 0 and d["ms_per_step"] > 0
    assert d["config"]["workload"] == "tiny_4x8x8"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_silent():
    r = _run(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "3"],
             {"WORLD_SIZE": "2", "RANK": "1", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_warmup_below_three_refused():
    r = _run(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "2"])
    assert r.returncode != 0
    assert "warmup" in r.stderr


def test_reference_arm_flops_equal_the_oracle_goldens():
    """The CPU arm counts executed tiles with the oracle over every q tile; on
    the SVG workload that must equal the full-map counts stored in
    tests/golden/full_maps.json (so both arms divide the same FLOPs)."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    import workloads as W
    from _helpers import full_maps, heads_of
    w = W.svg_wan720p()
    flops, how = bench.oracle_exec_flops(w, 8)
    executed = sum(h["counts"][1] + h["counts"][2] for h in heads_of(full_maps()[w.name]))
    assert "every q tile" in how
    assert flops == 4.0 * w.D * w.q_tile * w.kv_tile * executed
