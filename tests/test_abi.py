"""C-ABI library checks that need no GPU: it loads, exports every entry point
the public header declares, and rejects bad arguments on the host before any
device work.  Also the host-side layout rules (slot counts, tile counts)."""
import ctypes
import os
import re

import pytest

import block_sparse_attention_mask_b200 as vsa
import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(vsa_[a-z_0-9]+)\s*\(", src))
    return names


def test_header_symbols_are_exported():
    names = _declared()
    assert {"vsa_plan_create", "vsa_permute", "vsa_unpermute", "vsa_sparse_attn_fwd",
            "vsa_check_status"} <= names
    lib = ctypes.CDLL(vsa.LIB_PATH)
    for n in sorted(names):
        assert hasattr(lib, n), n


def test_version_and_status_strings():
    assert vsa.vsa_version() == 1
    for code in range(0, -8, -1):
        assert vsa.vsa_status_string(code) not in ("", "unknown status")
    assert vsa.vsa_status_string(-99) == "unknown status"


def _create_raw(specs, grid=(4, 8, 8), unit=(1, 8, 8), q=64, k=64):
    arr = (vsa.vsa_mask_spec * max(1, len(specs)))(*[vsa.make_spec(s) for s in specs])
    out = ctypes.c_void_p(1234)
    T, H, Wd = grid
    bt, bh, bw = unit
    rc = vsa.lib.vsa_plan_create(arr if specs else None, len(specs), T, H, Wd, bt, bh, bw, q, k,
                                 None, ctypes.byref(out))
    return rc, out.value


def test_plan_create_rejects_bad_arguments_on_host():
    ok = W.mask_spec("spatial", 1, rt=1)
    cases = [
        ([], dict(), -1),                                   # no heads / null specs
        ([ok], dict(grid=(0, 8, 8)), -1),                  # empty grid
        ([ok], dict(unit=(1, 8, 0)), -1),                  # empty unit
        ([ok], dict(q=96), -2),                            # tile size not supported
        ([ok], dict(k=256), -2),
        ([ok], dict(unit=(1, 8, 12)), -2),                 # bw not a power of two
        ([ok], dict(unit=(3, 5, 4), q=128, k=128), -2),    # tile neither whole units nor a unit box
        ([dict(ok, kind=9)], dict(), -1),                  # bad mask kind
        ([dict(ok, sink=2)], dict(), -1),
        ([W.mask_spec("sta", kt=0, kh=1, kw=1)], dict(), -1),
        ([dict(W.mask_spec("stripe", Tw=1, Ts=1, Sw=1, Ss=1), Ts=0)], dict(), -1),
        ([W.mask_spec("temporal", rh=-1, rw=0)], dict(), -1),
        ([W.mask_spec("stripe", Tw=1, Ts=2, Sw=1, Ss=3)], dict(grid=(2, 300, 300), unit=(1, 8, 8)), -2),
        ([dict(ok, layout=1)], dict(), -2),                # frame-0-first order: temporal / full heads only
        ([dict(ok, layout=2)], dict(), -1),                # unknown layout
        ([dict(W.mask_spec("sta", kt=1, kh=1, kw=1), tile_round=1)], dict(), -2),  # rounding: SVG / full only
        ([dict(ok, tile_round=2)], dict(), -1),
    ]
    for specs, kw, want in cases:
        rc, handle = _create_raw(specs, **kw)
        assert rc == want, (specs, kw, rc)
        assert handle is None


def test_calls_reject_null_plan_on_host():
    L = vsa.lib
    assert L.vsa_plan_build(None, None) == -1
    assert L.vsa_plan_info(None, None) == -1
    assert L.vsa_plan_tile_map(None, None, 0, None) == -1
    assert L.vsa_plan_tile_counts(None, None, 0, None) == -1
    assert L.vsa_plan_perm(None, None, 0, None) == -1
    assert L.vsa_plan_layout_perm(None, 0, None, 0, None) == -1
    assert L.vsa_plan_exec_steps(None, None, 0, None) == -1
    assert L.vsa_plan_exec_pairs(None, None, 0, None) == -1
    assert L.vsa_plan_destroy(None) == -1
    assert L.vsa_permute(None, None, None, 1, 128, None) == -1
    assert L.vsa_unpermute(None, None, None, 1, 128, None) == -1
    assert L.vsa_sparse_attn_fwd(None, None, None, None, None, None, 1, 128, 0.1, None) == -1
    assert L.vsa_check_status(None, None) == -1
    assert L.vsa_selftest_watchdog(None, 1000, None) == -1
    assert L.vsa_plan_set_route_candidates(None, None, None, None) == -1
    n = ctypes.c_size_t(0)
    assert L.vsa_svg_route_workspace_size(None, 1, 128, 1, ctypes.byref(n)) == -1
    assert L.vsa_svg_route(None, None, None, None, 1, 128, None, 1, 0.1, None, None, None, 0, None) == -1
    assert L.vsa_plan_apply_route(None, None, None) == -1
    assert L.vsa_ulysses_permute(None, None, 1, 128, 0, 1, None, None, None) == -1
    assert L.vsa_permute_qkv(None, None, None, None, None, None, None, 1, 128, None) == -1
    assert L.vsa_pipeline_run(None, None, None, None, None, None, 0.1, None) == -1
    assert L.vsa_pipeline_check_status(None, None) == -1
    assert L.vsa_pipeline_destroy(None) == -1
    h = ctypes.c_void_p()
    assert L.vsa_pipeline_create(None, 1, 2, 2, 2, 1, 1, 1, 128, 128, 1, 128, 1, ctypes.byref(h)) == -1
    assert L.vsa_ulysses_unpermute(None, None, 1, 128, 0, 1, None, None, None) == -1
    assert L.vsa_plan_kept_pairs(None, None, 0, None) == -1
    assert L.vsa_tile_map_noalloc(None, 1, 2, 8, 8, 1, 8, 8, 64, 64, None, 0, None) == -1
    assert L.vsa_plan_create(None, 1, 2, 8, 8, 1, 8, 8, 64, 64, None, ctypes.byref(h)) == -1
    assert L.vsa_plan_create(None, 1, 2, 8, 8, 1, 8, 8, 64, 64, None, None) == -1


def test_every_declared_entry_point_is_checked_here():
    # each entry point of the header appears in this file's host-side checks
    # (null arguments above, malformed shapes and strings in the other tests)
    src = open(__file__).read()
    for name in sorted(_declared()):
        assert name in src, name


def test_layout_slot_counts():
    # 21 x 45 x 80 = 75,600 tokens; natural order with 128-token blocks gives
    # 591 blocks per side ("video diffusion long-sequence attention and
    # sparsity", section 7.3)
    info = vsa.vsa_layout_info(1, (21, 45, 80), (1, 1, 1), 128, 128)
    assert info["n_tokens"] == 75600
    assert info["n_kv_tiles"] == 591 and info["n_q_tiles"] == 591
    assert info["n_slots"] == 591 * 128
    # PSABlock 3x8x16 pads 45 -> 48 ("Parameterized Stripe Attention", complete example)
    info = vsa.vsa_layout_info(40, (21, 45, 80), (3, 8, 16), 128, 128)
    assert info["n_padded"] == 21 * 48 * 80 and info["n_slots"] == 80640
    # (1,8,16) units: 630 tiles of 128 per side; q tiles of 256 round the slots to 256
    info = vsa.vsa_layout_info(10, (21, 45, 80), (1, 8, 16), 128, 128)
    assert (info["n_q_tiles"], info["n_kv_tiles"], info["map_bytes"]) == (630, 630, 10 * 630 * 630)
    info = vsa.vsa_layout_info(1, (5, 45, 80), (1, 8, 8), 256, 64)
    assert info["n_slots"] == 19200 and info["n_q_tiles"] == 75 and info["n_kv_tiles"] == 300
    # a ragged tail: 3x7x9 tokens in 128-slot tiles
    info = vsa.vsa_layout_info(1, (3, 7, 9), (1, 1, 1), 128, 64)
    assert info["n_padded"] == 189 and info["n_slots"] == 256
    # every workload the benchmark and the parity tests use is supported
    for w in W.all_parity_workloads():
        info = vsa.vsa_layout_info(w.heads, (w.T, w.H, w.W), w.unit, w.q_tile, w.kv_tile)
        assert info["n_slots"] % max(128, w.q_tile, w.kv_tile) == 0


def test_layout_rejects_unsupported():
    with pytest.raises(vsa.VsaError):
        vsa.vsa_layout_info(1, (4, 8, 8), (1, 8, 8), 32, 64)
    with pytest.raises(vsa.VsaError):
        vsa.vsa_layout_info(1, (4, 8, 8), (1, 8, 64), 128, 128)
