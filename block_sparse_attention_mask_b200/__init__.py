"""Python binding for libvsa (block-sparse 3D-video attention on B200).

Argument marshalling only: every step runs in the CUDA kernels of libvsa.so,
built in-tree by ``block_sparse_attention_mask_b200.build``.  Importing this
package raises if the library cannot be built or loaded; there is no CPU or
library fallback.  PyTorch is used for device memory and streams.

The C entry points are exposed under their own names (``vsa_plan_create``,
``vsa_permute``, ``vsa_unpermute``, ``vsa_sparse_attn_fwd``, ...), taking
torch tensors where the C call takes device pointers.  ``Plan`` wraps a plan
handle; ``attention`` runs permute -> forward -> unpermute.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Dict, Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvsa.so")

VSA_OK = 0
STATUS_NAMES = {0: "VSA_OK", -1: "VSA_ERR_INVALID_ARG", -2: "VSA_ERR_UNSUPPORTED",
                -3: "VSA_ERR_ALIGNMENT", -4: "VSA_ERR_CUDA", -5: "VSA_ERR_OOM",
                -6: "VSA_ERR_TIMEOUT", -7: "VSA_ERR_DEVICE"}
MASK_KINDS = {"full": 0, "spatial": 1, "temporal": 2, "sta": 3, "stripe": 4}
TILE_EMPTY, TILE_BOUNDARY, TILE_FULL = 0, 1, 2


class VsaError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        name = STATUS_NAMES.get(code, str(code))
        msg = _lib.vsa_status_string(code).decode() if _lib is not None else name
        super().__init__(f"{what}: {name} ({msg})" if what else f"{name} ({msg})")


class vsa_mask_spec(ctypes.Structure):
    _fields_ = [(k, ctypes.c_int32) for k in
                ("kind", "sink", "rt", "rh", "rw", "kt", "kh", "kw",
                 "Tw", "To", "Ts", "Sw", "So", "Ss", "layout", "tile_round")]


class vsa_plan_info_t(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("W", ctypes.c_int32),
                ("bt", ctypes.c_int32), ("bh", ctypes.c_int32), ("bw", ctypes.c_int32),
                ("num_heads", ctypes.c_int32), ("q_tile", ctypes.c_int32),
                ("kv_tile", ctypes.c_int32), ("n_q_tiles", ctypes.c_int32),
                ("n_kv_tiles", ctypes.c_int32), ("n_tokens", ctypes.c_int64),
                ("n_padded", ctypes.c_int64), ("n_slots", ctypes.c_int64),
                ("map_bytes", ctypes.c_int64)]


def _load() -> ctypes.CDLL:
    from . import build as _build
    if not _build.up_to_date():
        _build.build()
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
    P = ctypes.POINTER
    sig = {
        "vsa_plan_create": ([P(vsa_mask_spec), i32, i32, i32, i32, i32, i32, i32, i32, i32, vp,
                             P(vp)], i32),
        "vsa_plan_build": ([vp, vp], i32),
        "vsa_layout_info": ([i32, i32, i32, i32, i32, i32, i32, i32, i32, P(vsa_plan_info_t)], i32),
        "vsa_plan_info": ([vp, P(vsa_plan_info_t)], i32),
        "vsa_plan_tile_map": ([vp, vp, sz, vp], i32),
        "vsa_plan_tile_counts": ([vp, vp, sz, vp], i32),
        "vsa_plan_perm": ([vp, vp, sz, vp], i32),
        "vsa_plan_layout_perm": ([vp, i32, vp, sz, vp], i32),
        "vsa_plan_exec_steps": ([vp, vp, sz, vp], i32),
        "vsa_plan_exec_pairs": ([vp, vp, sz, vp], i32),
        "vsa_plan_kept_pairs": ([vp, vp, sz, vp], i32),
        "vsa_plan_destroy": ([vp], i32),
        "vsa_permute": ([vp, vp, vp, i32, i32, vp], i32),
        "vsa_unpermute": ([vp, vp, vp, i32, i32, vp], i32),
        "vsa_permute_qkv": ([vp, vp, vp, vp, vp, vp, vp, i32, i32, vp], i32),
        "vsa_sparse_attn_fwd": ([vp, vp, vp, vp, vp, vp, i32, i32, f32, vp], i32),
        "vsa_check_status": ([vp, vp], i32),
        "vsa_selftest_watchdog": ([vp, ctypes.c_longlong, vp], i32),
        "vsa_tile_map_noalloc": ([P(vsa_mask_spec), i32, i32, i32, i32, i32, i32, i32, i32, i32, vp,
                                  sz, vp], i32),
        "vsa_plan_set_route_candidates": ([vp, P(vsa_mask_spec), P(vsa_mask_spec), vp], i32),
        "vsa_svg_route_workspace_size": ([vp, i32, i32, i32, P(sz)], i32),
        "vsa_svg_route": ([vp, vp, vp, vp, i32, i32, vp, i32, f32, vp, vp, vp, sz, vp], i32),
        "vsa_plan_apply_route": ([vp, vp, vp], i32),
        "vsa_ulysses_permute": ([vp, vp, i32, i32, i32, i32, vp, P(vp), vp], i32),
        "vsa_ulysses_unpermute": ([vp, vp, i32, i32, i32, i32, vp, P(vp), vp], i32),
        "vsa_pipeline_create": ([P(vsa_mask_spec), i32, i32, i32, i32, i32, i32, i32, i32, i32, i32, i32, i32,
                                 P(vp)], i32),
        "vsa_pipeline_run": ([vp, vp, vp, vp, vp, vp, f32, vp], i32),
        "vsa_pipeline_check_status": ([vp, vp], i32),
        "vsa_pipeline_destroy": ([vp], i32),
        "vsa_status_string": ([i32], ctypes.c_char_p),
        "vsa_version": ([], i32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


_lib: Optional[ctypes.CDLL] = None
_lib = _load()
lib = _lib


def _check(code: int, what: str) -> None:
    if code != VSA_OK:
        raise VsaError(code, what)


def _stream(stream) -> Optional[int]:
    """cudaStream_t handle: an int, a torch.cuda.Stream, or None (torch's current stream)."""
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if hasattr(t, "data_ptr"):
        return t.data_ptr()
    return int(t)


def make_spec(d: Dict[str, int]) -> vsa_mask_spec:
    s = vsa_mask_spec()
    for k, _ in vsa_mask_spec._fields_:
        setattr(s, k, int(d.get(k, 0)))
    return s


# ---------------------------------------------------------------------------
# C entry points under their own names


def vsa_plan_create(specs: Sequence[Dict[str, int]], grid: Sequence[int], unit: Sequence[int],
                    q_tile: int, kv_tile: int, stream=None) -> int:
    arr = (vsa_mask_spec * len(specs))(*[make_spec(s) for s in specs])
    out = ctypes.c_void_p()
    T, H, W = (int(x) for x in grid)
    bt, bh, bw = (int(x) for x in unit)
    _check(_lib.vsa_plan_create(arr, len(specs), T, H, W, bt, bh, bw, int(q_tile), int(kv_tile),
                                _stream(stream), ctypes.byref(out)), "vsa_plan_create")
    return out.value


def vsa_plan_build(plan: int, stream=None) -> None:
    _check(_lib.vsa_plan_build(plan, _stream(stream)), "vsa_plan_build")


def vsa_layout_info(num_heads: int, grid: Sequence[int], unit: Sequence[int], q_tile: int,
                    kv_tile: int) -> Dict[str, int]:
    info = vsa_plan_info_t()
    T, H, W = (int(x) for x in grid)
    bt, bh, bw = (int(x) for x in unit)
    _check(_lib.vsa_layout_info(int(num_heads), T, H, W, bt, bh, bw, int(q_tile), int(kv_tile),
                                ctypes.byref(info)), "vsa_layout_info")
    return {k: getattr(info, k) for k, _ in vsa_plan_info_t._fields_}


def vsa_plan_info(plan: int) -> Dict[str, int]:
    info = vsa_plan_info_t()
    _check(_lib.vsa_plan_info(plan, ctypes.byref(info)), "vsa_plan_info")
    return {k: getattr(info, k) for k, _ in vsa_plan_info_t._fields_}


def vsa_plan_tile_map(plan: int, stream=None) -> np.ndarray:
    info = vsa_plan_info(plan)
    out = np.empty((info["num_heads"], info["n_q_tiles"], info["n_kv_tiles"]), dtype=np.int8)
    _check(_lib.vsa_plan_tile_map(plan, out.ctypes.data, out.nbytes, _stream(stream)),
           "vsa_plan_tile_map")
    return out


def vsa_plan_tile_counts(plan: int, stream=None) -> np.ndarray:
    info = vsa_plan_info(plan)
    out = np.empty((info["num_heads"], 3), dtype=np.int64)
    _check(_lib.vsa_plan_tile_counts(plan, out.ctypes.data, out.size, _stream(stream)),
           "vsa_plan_tile_counts")
    return out


def vsa_plan_perm(plan: int, stream=None) -> np.ndarray:
    info = vsa_plan_info(plan)
    out = np.empty(info["n_slots"], dtype=np.int32)
    _check(_lib.vsa_plan_perm(plan, out.ctypes.data, out.size, _stream(stream)), "vsa_plan_perm")
    return out


def vsa_plan_layout_perm(plan: int, layout: int, stream=None) -> np.ndarray:
    info = vsa_plan_info(plan)
    out = np.empty(info["n_slots"], dtype=np.int32)
    _check(_lib.vsa_plan_layout_perm(plan, int(layout), out.ctypes.data, out.size, _stream(stream)),
           "vsa_plan_layout_perm")
    return out


def vsa_plan_exec_steps(plan: int, stream=None) -> np.ndarray:
    info = vsa_plan_info(plan)
    out = np.empty(info["num_heads"], dtype=np.int64)
    _check(_lib.vsa_plan_exec_steps(plan, out.ctypes.data, out.size, _stream(stream)),
           "vsa_plan_exec_steps")
    return out


def vsa_plan_exec_pairs(plan: int, stream=None) -> np.ndarray:
    """[heads, n_blocks] int32: partner of a pair's leader, -1 alone, -2 in the leader's CTA."""
    info = vsa_plan_info(plan)
    nE = info["n_slots"] // 128
    out = np.empty((info["num_heads"], nE), dtype=np.int32)
    _check(_lib.vsa_plan_exec_pairs(plan, out.ctypes.data, out.size, _stream(stream)),
           "vsa_plan_exec_pairs")
    return out


def vsa_plan_kept_pairs(plan: int, stream=None) -> np.ndarray:
    info = vsa_plan_info(plan)
    out = np.empty(info["num_heads"], dtype=np.int64)
    _check(_lib.vsa_plan_kept_pairs(plan, out.ctypes.data, out.size, _stream(stream)),
           "vsa_plan_kept_pairs")
    return out


def vsa_plan_destroy(plan: int) -> None:
    _check(_lib.vsa_plan_destroy(plan), "vsa_plan_destroy")


def vsa_permute(plan: int, x_in, x_out, B: int, D: int, stream=None) -> None:
    _check(_lib.vsa_permute(plan, _ptr(x_in), _ptr(x_out), int(B), int(D), _stream(stream)),
           "vsa_permute")


def vsa_unpermute(plan: int, x_in, x_out, B: int, D: int, stream=None) -> None:
    _check(_lib.vsa_unpermute(plan, _ptr(x_in), _ptr(x_out), int(B), int(D), _stream(stream)),
           "vsa_unpermute")


def vsa_permute_qkv(plan: int, q, k, v, q_out, k_out, v_out, B: int, D: int, stream=None) -> None:
    _check(_lib.vsa_permute_qkv(plan, _ptr(q), _ptr(k), _ptr(v), _ptr(q_out), _ptr(k_out), _ptr(v_out), B, D,
                                _stream(stream)), "vsa_permute_qkv")


def vsa_sparse_attn_fwd(q, k, v, o, lse, plan: int, B: int, D: int, scale: float,
                        stream=None) -> None:
    _check(_lib.vsa_sparse_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), plan, int(B),
                                    int(D), float(scale), _stream(stream)), "vsa_sparse_attn_fwd")


def vsa_tile_map_noalloc(specs: Sequence[Dict[str, int]], grid: Sequence[int], unit: Sequence[int],
                         q_tile: int, kv_tile: int, map_out, stream=None) -> None:
    """Tile map into a caller-owned int8 CUDA tensor; the library allocates nothing.

    ``map_out`` must be a contiguous int8 CUDA tensor on the current device;
    the bound passed to the library is the bytes its storage really holds from
    the tensor's first element on, so a view can never let the kernel write
    past its allocation."""
    import torch
    if not (isinstance(map_out, torch.Tensor) and map_out.is_cuda and map_out.dtype == torch.int8
            and map_out.is_contiguous() and map_out.device.index == torch.cuda.current_device()):
        raise VsaError(-1, "vsa_tile_map_noalloc: map_out must be a contiguous int8 CUDA tensor "
                           "on the current device")
    arr = (vsa_mask_spec * len(specs))(*[make_spec(s) for s in specs])
    T, H, W = (int(x) for x in grid)
    bt, bh, bw = (int(x) for x in unit)
    nbytes = min(map_out.numel(),
                 map_out.untyped_storage().nbytes() - map_out.storage_offset() * map_out.element_size())
    _check(_lib.vsa_tile_map_noalloc(arr, len(specs), T, H, W, bt, bh, bw, int(q_tile), int(kv_tile),
                                     _ptr(map_out), nbytes, _stream(stream)),
           "vsa_tile_map_noalloc")


def vsa_check_status(plan: int, stream=None) -> None:
    _check(_lib.vsa_check_status(plan, _stream(stream)), "vsa_check_status")


def vsa_selftest_watchdog(plan: int, cycles: int, stream=None) -> None:
    _check(_lib.vsa_selftest_watchdog(plan, int(cycles), _stream(stream)), "vsa_selftest_watchdog")


def vsa_status_string(code: int) -> str:
    return _lib.vsa_status_string(int(code)).decode()


def vsa_version() -> int:
    return int(_lib.vsa_version())


def vsa_plan_set_route_candidates(plan: int, spatial: Sequence[Dict[str, int]],
                                  temporal: Sequence[Dict[str, int]], stream=None) -> None:
    n = len(spatial)
    if len(temporal) != n:
        raise ValueError("one spatial and one temporal candidate per head")
    sa = (vsa_mask_spec * n)(*[make_spec(d) for d in spatial])
    ta = (vsa_mask_spec * n)(*[make_spec(d) for d in temporal])
    _check(_lib.vsa_plan_set_route_candidates(plan, sa, ta, _stream(stream)),
           "vsa_plan_set_route_candidates")


def vsa_svg_route_workspace_size(plan: int, B: int, D: int, n_rows: int) -> int:
    out = ctypes.c_size_t(0)
    _check(_lib.vsa_svg_route_workspace_size(plan, B, D, n_rows, ctypes.byref(out)),
           "vsa_svg_route_workspace_size")
    return int(out.value)


def vsa_svg_route(plan: int, q, k, v, B: int, D: int, rows, n_rows: int, scale: float, err, flags,
                  workspace, workspace_bytes: int, stream=None) -> None:
    _check(_lib.vsa_svg_route(plan, _ptr(q), _ptr(k), _ptr(v), B, D, _ptr(rows), n_rows, scale,
                              _ptr(err), _ptr(flags), _ptr(workspace), workspace_bytes,
                              _stream(stream)), "vsa_svg_route")


def _ptr_array(ptrs) -> "ctypes.Array":
    return (ctypes.c_void_p * len(ptrs))(*[_ptr(p) for p in ptrs])


def vsa_ulysses_permute(plan: int, x, B: int, D: int, rank: int, world: int, head_layout, dst,
                        stream=None) -> None:
    _check(_lib.vsa_ulysses_permute(plan, _ptr(x), B, D, rank, world, _ptr(head_layout), _ptr_array(dst),
                                    _stream(stream)), "vsa_ulysses_permute")


def vsa_ulysses_unpermute(plan: int, o, B: int, D: int, rank: int, world: int, head_layout, dst,
                          stream=None) -> None:
    _check(_lib.vsa_ulysses_unpermute(plan, _ptr(o), B, D, rank, world, _ptr(head_layout), _ptr_array(dst),
                                      _stream(stream)), "vsa_ulysses_unpermute")


def shard_offsets(n_tokens: int, world: int) -> list:
    """Token offsets of the sequence shards: rank r holds [off[r], off[r+1])."""
    return [r * n_tokens // world for r in range(world + 1)]


def vsa_plan_apply_route(plan: int, flags, stream=None) -> None:
    _check(_lib.vsa_plan_apply_route(plan, _ptr(flags), _stream(stream)), "vsa_plan_apply_route")


# ---------------------------------------------------------------------------
# convenience wrapper


class Plan:
    """Owns a plan handle; shapes as in ``include/vsa.h``."""

    def __init__(self, specs: Sequence[Dict[str, int]], grid: Sequence[int], unit: Sequence[int],
                 q_tile: int = 128, kv_tile: int = 128, stream=None):
        self.handle = vsa_plan_create(specs, grid, unit, q_tile, kv_tile, stream)
        self.info = vsa_plan_info(self.handle)
        self.heads = self.info["num_heads"]
        self.n_slots = self.info["n_slots"]
        self.n_tokens = self.info["n_tokens"]

    def close(self) -> None:
        if getattr(self, "handle", None):
            vsa_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):  # pragma: no cover - best effort
        try:
            self.close()
        except Exception:
            pass

    def build(self, stream=None) -> None:
        vsa_plan_build(self.handle, stream)

    def tile_map(self, stream=None) -> np.ndarray:
        return vsa_plan_tile_map(self.handle, stream)

    def tile_counts(self, stream=None) -> np.ndarray:
        return vsa_plan_tile_counts(self.handle, stream)

    def perm(self, stream=None, layout: int = 0) -> np.ndarray:
        return vsa_plan_layout_perm(self.handle, layout, stream)

    def exec_steps(self, stream=None) -> np.ndarray:
        return vsa_plan_exec_steps(self.handle, stream)

    def exec_pairs(self, stream=None) -> np.ndarray:
        return vsa_plan_exec_pairs(self.handle, stream)

    def kept_pairs(self, stream=None) -> np.ndarray:
        return vsa_plan_kept_pairs(self.handle, stream)

    def check(self, stream=None) -> None:
        vsa_check_status(self.handle, stream)

    def set_route_candidates(self, spatial: Sequence[Dict[str, int]],
                             temporal: Sequence[Dict[str, int]], stream=None) -> None:
        vsa_plan_set_route_candidates(self.handle, spatial, temporal, stream)

    def apply_route(self, flags, stream=None) -> None:
        """Switch every head to its temporal (flag 1) or spatial candidate and
        rebuild the maps on the device; ``flags`` is a device int32 [heads]."""
        vsa_plan_apply_route(self.handle, flags, stream)


def _require_bf16(t, shape: Tuple[int, ...], name: str) -> None:
    import torch
    if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")
    if tuple(t.shape) != shape:
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {shape}")


def permute(plan: Plan, x, out=None, stream=None):
    """natural [B, Hh, N, D] -> tile-major [B, Hh, n_slots, D]."""
    import torch
    B, Hh, N, D = x.shape
    _require_bf16(x, (B, plan.heads, plan.n_tokens, D), "x")
    if out is None:
        out = torch.empty((B, Hh, plan.n_slots, D), dtype=torch.bfloat16, device=x.device)
    _require_bf16(out, (B, Hh, plan.n_slots, D), "out")
    vsa_permute(plan.handle, x, out, B, D, stream)
    return out


def unpermute(plan: Plan, x, out=None, stream=None):
    """tile-major [B, Hh, n_slots, D] -> natural [B, Hh, N, D]."""
    import torch
    B, Hh, S, D = x.shape
    _require_bf16(x, (B, plan.heads, plan.n_slots, D), "x")
    if out is None:
        out = torch.empty((B, Hh, plan.n_tokens, D), dtype=torch.bfloat16, device=x.device)
    _require_bf16(out, (B, Hh, plan.n_tokens, D), "out")
    vsa_unpermute(plan.handle, x, out, B, D, stream)
    return out


def sparse_attn_fwd(plan: Plan, q, k, v, scale: Optional[float] = None, o=None, lse=None,
                    stream=None):
    """Tile-major q, k, v -> (o, lse), both tile-major."""
    import torch
    B, Hh, S, D = q.shape
    for name, t in (("q", q), ("k", k), ("v", v)):
        _require_bf16(t, (B, plan.heads, plan.n_slots, D), name)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hh, S), dtype=torch.float32, device=q.device)
    vsa_sparse_attn_fwd(q, k, v, o, lse, plan.handle, B, D, scale, stream)
    return o, lse


def permute_qkv(plan: Plan, q, k, v, stream=None):
    """natural [B, Hh, N, D] x3 -> tile-major [B, Hh, n_slots, D] x3 in one launch."""
    import torch
    B, Hh, N, D = q.shape
    for name, t in (("q", q), ("k", k), ("v", v)):
        _require_bf16(t, (B, plan.heads, plan.n_tokens, D), name)
    outs = [torch.empty((B, Hh, plan.n_slots, D), dtype=torch.bfloat16, device=q.device) for _ in range(3)]
    vsa_permute_qkv(plan.handle, q, k, v, *outs, B, D, stream)
    return tuple(outs)


def attention(plan: Plan, q, k, v, scale: Optional[float] = None, stream=None):
    """Natural-order q, k, v [B, Hh, N, D] -> (o natural [B, Hh, N, D], lse tile-major)."""
    qp, kp, vp = permute_qkv(plan, q, k, v, stream=stream)
    op, lse = sparse_attn_fwd(plan, qp, kp, vp, scale, stream=stream)
    return unpermute(plan, op, stream=stream), lse


def svg_route(plan: Plan, q, k, v, rows, scale: Optional[float] = None, workspace=None,
              err=None, flags=None, stream=None):
    """Sampled-query routing of every head (natural-order q, k, v [B, Hh, N, D]
    bf16; rows: device int32 [R] natural token indices).  Returns (err fp32
    [Hh, 2] spatial / temporal deviations, flags int32 [Hh], 1 = temporal),
    both on the device; nothing synchronises."""
    import torch
    B, Hh, N, D = q.shape
    for name, t in (("q", q), ("k", k), ("v", v)):
        _require_bf16(t, (B, plan.heads, plan.n_tokens, D), name)
    if rows.dtype != torch.int32 or not rows.is_cuda or not rows.is_contiguous() or rows.dim() != 1:
        raise ValueError("rows must be a contiguous int32 CUDA vector")
    R = int(rows.shape[0])
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    need = vsa_svg_route_workspace_size(plan.handle, B, D, R)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if workspace.numel() * workspace.element_size() < need:
        raise ValueError(f"workspace needs {need} bytes")
    if err is None:
        err = torch.empty((Hh, 2), dtype=torch.float32, device=q.device)
    if flags is None:
        flags = torch.empty((Hh,), dtype=torch.int32, device=q.device)
    vsa_svg_route(plan.handle, q, k, v, B, D, rows, R, scale, err, flags, workspace,
                  workspace.numel() * workspace.element_size(), stream)
    return err, flags


class Pipeline:
    """Attention from host buffers with the PCIe copies overlapped with the
    compute, chunk by chunk of heads (see ``vsa_pipeline_run`` in
    ``include/vsa.h``)."""

    def __init__(self, specs: Sequence[Dict[str, int]], grid: Sequence[int], unit: Sequence[int],
                 q_tile: int = 128, kv_tile: int = 128, B: int = 1, D: int = 128, chunk_heads: int = 1):
        arr = (vsa_mask_spec * len(specs))(*[make_spec(d) for d in specs])
        h = ctypes.c_void_p()
        _check(_lib.vsa_pipeline_create(arr, len(specs), int(grid[0]), int(grid[1]), int(grid[2]),
                                        int(unit[0]), int(unit[1]), int(unit[2]), q_tile, kv_tile, B, D,
                                        chunk_heads, ctypes.byref(h)), "vsa_pipeline_create")
        self.handle = h.value
        self.B, self.D, self.heads = B, D, len(specs)

    def run(self, q_host, k_host, v_host, o_host, lse_host, scale: float, stream=None) -> None:
        """Host tensors (pinned): q, k, v, o bf16 [B, Hh, N, D]; lse fp32 [B, Hh, n_slots]."""
        _check(_lib.vsa_pipeline_run(self.handle, _ptr(q_host), _ptr(k_host), _ptr(v_host), _ptr(o_host),
                                     _ptr(lse_host), scale, _stream(stream)), "vsa_pipeline_run")

    def check(self, stream=None) -> None:
        _check(_lib.vsa_pipeline_check_status(self.handle, _stream(stream)), "vsa_pipeline_check_status")

    def close(self) -> None:
        if getattr(self, "handle", None):
            _check(_lib.vsa_pipeline_destroy(self.handle), "vsa_pipeline_destroy")
            self.handle = None

    def __del__(self):  # pragma: no cover - best effort
        try:
            self.close()
        except Exception:
            pass

