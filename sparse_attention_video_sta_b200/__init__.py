"""Sliding Tile Attention (STA) forward and backward for NVIDIA B200 (sm_100a).

Thin ctypes binding of the C-ABI library ``libsta.so`` (declared in
``include/sta.h``).  This module only marshals arguments -- tensor pointers,
sizes and the current CUDA stream -- and checks that tensor shapes match the
plan; every step of the computation runs in the library's CUDA kernels.  There
is no CPU fallback: importing this package fails if ``libsta.so`` is missing.

The functions carry the C names:

    sta_plan / sta_plan_host -> Plan  (per-head key-tile lists + work list)
    sta_tile_reorder / sta_tile_unreorder  (raster <-> tile-major tokens)
    sta_forward                             (STA attention on tile-major tensors)
    sta_forward_raster                      (same, raster tensors, permutation fused)
    sta_backward                            (dQ, dK, dV on tile-major tensors)
    sta_last_device_status, sta_status_string, sta_debug_inject_timeout

``sta_attention`` / ``sta_attention_backward`` chain them for raster-order
tensors, and ``StaAttention`` wraps both as a ``torch.autograd.Function``.
``sta_window_stats`` / ``sta_window_search`` profile candidate windows per head
(attention recall and output error against full attention).
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

__all__ = [
    "StaError", "Plan", "sta_plan", "sta_plan_host", "sta_tile_reorder", "sta_tile_unreorder",
    "sta_forward", "sta_forward_raster", "sta_forward_noalloc", "sta_last_device_status",
    "sta_status_string", "sta_debug_inject_timeout", "sta_attention", "raster_supported", "library_path", "EXPORTED_SYMBOLS",
    "sta_backward", "sta_attention_backward", "StaAttention", "sta_window_stats", "sta_window_search",
    "Pipe", "sta_pipe_create", "sta_backward_raster", "sta_window_pick",
]

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
# STA_LIBRARY=debug loads libsta_debug.so, the build whose kernels check every
# plan index before use (status STA_ERR_BOUNDS instead of a fault).
_LIB_NAME = "libsta_debug.so" if os.environ.get("STA_LIBRARY", "") == "debug" else "libsta.so"
_LIB_PATH = os.path.join(_PKG_DIR, _LIB_NAME)

STA_OK = 0
STA_ERR_INVALID_ARG = 1
STA_ERR_UNSUPPORTED = 2
STA_ERR_CUDA = 3
STA_ERR_TIMEOUT = 4
STA_ERR_OOM = 5
STA_ERR_BOUNDS = 6

EXPORTED_SYMBOLS = (
    "sta_plan", "sta_plan_host", "sta_plan_destroy", "sta_plan_query", "sta_plan_stats",
    "sta_plan_work_items", "sta_tile_reorder", "sta_tile_unreorder", "sta_forward",
    "sta_forward_raster", "sta_forward_noalloc", "sta_last_device_status", "sta_status_string", "sta_debug_inject_timeout",
    "sta_last_error_detail", "sta_plan_key_query", "sta_backward", "sta_window_stats",
    "sta_pipe_create", "sta_pipe_submit", "sta_pipe_wait", "sta_pipe_destroy", "sta_backward_raster",
    "sta_plan_backward_items", "sta_plan_validate", "sta_debug_plan_poke", "sta_window_pick",
)


class _Geom(ctypes.Structure):
    _fields_ = [("lat_t", ctypes.c_int32), ("lat_h", ctypes.c_int32), ("lat_w", ctypes.c_int32),
                ("tile_t", ctypes.c_int32), ("tile_h", ctypes.c_int32), ("tile_w", ctypes.c_int32)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"{_LIB_NAME} not found at {_LIB_PATH}; build it with "
            "`python sparse_attention_video_sta_b200/_build.py --debug` (nvcc, sm_100a)")
    L = ctypes.CDLL(_LIB_PATH)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    G = ctypes.POINTER(_Geom)
    i32p, i64p = ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int64)
    sig = {
        "sta_plan": [G, i32, i32, i32p, vp, ctypes.POINTER(vp)],
        "sta_plan_host": [G, i32, i32, i32p, ctypes.POINTER(vp)],
        "sta_plan_destroy": [vp],
        "sta_plan_query": [vp, i32, i32, i32p, i32, i32p],
        "sta_plan_key_query": [vp, i32, i32, i32p, i32, i32p],
        "sta_plan_stats": [vp, i64p, i64p],
        "sta_plan_work_items": [vp, i32p, i64, i64p],
        "sta_plan_backward_items": [vp, i32, i32p, i64, i64p],
        "sta_tile_reorder": [vp, vp, i64, i32, G, vp],
        "sta_tile_unreorder": [vp, vp, i64, i32, G, vp],
        "sta_forward": [vp, vp, vp, vp, vp, vp, i32, ctypes.c_float, vp],
        "sta_forward_raster": [vp, vp, vp, vp, vp, vp, i32, ctypes.c_float, vp],
        "sta_forward_noalloc": [G, i32, i32, i32p, vp, vp, vp, vp, vp, i32, ctypes.c_float, vp],
        "sta_backward": [vp] * 11 + [i32, ctypes.c_float, vp],
        "sta_backward_raster": [vp] * 11 + [i32, ctypes.c_float, vp],
        "sta_window_stats": [vp, vp, vp, vp, i64, i64, i32, vp, vp, vp],
        "sta_pipe_create": [vp, i32, ctypes.c_float, i32, ctypes.POINTER(vp)],
        "sta_pipe_submit": [vp, vp, vp, vp, vp, vp],
        "sta_pipe_wait": [vp],
        "sta_pipe_destroy": [vp],
        "sta_last_device_status": [vp, vp],
        "sta_debug_inject_timeout": [i32, i32],
        "sta_plan_validate": [vp],
        "sta_debug_plan_poke": [vp, i32, i64, i32],
        "sta_window_pick": [G, i32, i32, i32p, vp, vp, ctypes.c_double, ctypes.c_double, i32p],
    }
    for name, args in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    L.sta_status_string.argtypes = [ctypes.c_int]
    L.sta_status_string.restype = ctypes.c_char_p
    L.sta_last_error_detail.argtypes = []
    L.sta_last_error_detail.restype = ctypes.c_char_p
    return L


_lib = _load()


def library_path() -> str:
    return _LIB_PATH


def sta_status_string(status: int) -> str:
    return _lib.sta_status_string(int(status)).decode()


def sta_last_error_detail() -> str:
    return _lib.sta_last_error_detail().decode()


class StaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = int(status)
        msg = f"{what}: {sta_status_string(status)}"
        if self.status in (STA_ERR_CUDA, STA_ERR_OOM):
            msg += f" ({sta_last_error_detail()})"
        super().__init__(msg)


def _check(status: int, what: str) -> None:
    if status != STA_OK:
        raise StaError(status, what)


def _geom(latent, tile) -> _Geom:
    return _Geom(int(latent[0]), int(latent[1]), int(latent[2]),
                 int(tile[0]), int(tile[1]), int(tile[2]))


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _device(tensors, plan=None) -> torch.device:
    """The one CUDA device of ``tensors`` (and of ``plan``, when it has one).
    Calls into the library run with it current, so the library's device
    checks and the default stream refer to the tensors' device."""
    idx = {t.device.index for t in tensors if t is not None and t.is_cuda}
    if plan is not None and plan.device is not None:
        idx.add(plan.device)
    if len(idx) != 1:
        raise ValueError(f"tensors and plan must be on one CUDA device (got devices {sorted(idx)})")
    return torch.device("cuda", idx.pop())


def _windows(heads: int, windows) -> ctypes.Array:
    w = torch.as_tensor(windows, dtype=torch.int32).reshape(-1, 3)
    if w.shape[0] == 1 and heads > 1:
        w = w.expand(heads, 3)
    if w.shape[0] != heads:
        raise ValueError(f"expected {heads} windows, got {w.shape[0]}")
    flat = w.contiguous().flatten().tolist()
    return (ctypes.c_int32 * len(flat))(*flat)


class Plan:
    """Owner of a ``sta_plan_t`` handle (freed on ``destroy`` / garbage collection)."""

    def __init__(self, handle: int, latent, tile, batch: int, heads: int, windows, device: int | None = None):
        self._h = ctypes.c_void_p(handle)
        self.device = device  # CUDA device index of a device plan; None for a host-only plan
        self.latent = tuple(int(x) for x in latent)
        self.tile = tuple(int(x) for x in tile)
        self.batch = int(batch)
        self.heads = int(heads)
        self.windows = torch.as_tensor(windows, dtype=torch.int32).reshape(-1, 3)

    @property
    def handle(self) -> ctypes.c_void_p:
        if not self._h:
            raise ValueError("plan already destroyed")
        return self._h

    @property
    def tokens(self) -> int:
        """Raster tokens per head (the latent)."""
        return self.latent[0] * self.latent[1] * self.latent[2]

    @property
    def tiles_per_head(self) -> int:
        """Tiles per head; an axis that is not a multiple of the tile is padded to whole tiles."""
        return math.prod(-(-self.latent[i] // self.tile[i]) for i in range(3))

    @property
    def padded_tokens(self) -> int:
        """Rows per head of the tile-major layout (whole tiles; equals ``tokens``
        when every axis is a multiple of the tile)."""
        return self.tiles_per_head * self.tile[0] * self.tile[1] * self.tile[2]

    def query(self, head: int, q_tile: int) -> list:
        """Ascending key-tile ids attended by query tile ``q_tile`` of ``head``."""
        count = ctypes.c_int32(0)
        _check(_lib.sta_plan_query(self.handle, head, q_tile, None, 0, ctypes.byref(count)),
               "sta_plan_query")
        buf = (ctypes.c_int32 * max(count.value, 1))()
        _check(_lib.sta_plan_query(self.handle, head, q_tile, buf, count.value, ctypes.byref(count)),
               "sta_plan_query")
        return list(buf[:count.value])

    def key_query(self, head: int, k_tile: int) -> list:
        """Ascending query-tile ids whose window holds key tile ``k_tile`` of ``head``."""
        count = ctypes.c_int32(0)
        _check(_lib.sta_plan_key_query(self.handle, head, k_tile, None, 0, ctypes.byref(count)),
               "sta_plan_key_query")
        buf = (ctypes.c_int32 * max(count.value, 1))()
        _check(_lib.sta_plan_key_query(self.handle, head, k_tile, buf, count.value, ctypes.byref(count)),
               "sta_plan_key_query")
        return list(buf[:count.value])

    def stats(self) -> tuple:
        """(computed query-tile/key-tile pairs over all b, h; work items)."""
        pairs, items = ctypes.c_int64(0), ctypes.c_int64(0)
        _check(_lib.sta_plan_stats(self.handle, ctypes.byref(pairs), ctypes.byref(items)),
               "sta_plan_stats")
        return pairs.value, items.value

    def work_items(self):
        """The forward's work list as (bh, query row block, -1, window id)
        tuples, in the order the kernel hands them out."""
        count = ctypes.c_int64(0)
        _check(_lib.sta_plan_work_items(self.handle, None, 0, ctypes.byref(count)), "sta_plan_work_items")
        buf = (ctypes.c_int32 * max(4 * count.value, 4))()
        _check(_lib.sta_plan_work_items(self.handle, buf, count.value, ctypes.byref(count)),
               "sta_plan_work_items")
        flat = list(buf[:4 * count.value])
        return [tuple(flat[4 * i:4 * i + 4]) for i in range(count.value)]

    def backward_items(self, which: int):
        """Backward work list (0: dQ query blocks, 1: dK / dV key blocks) as
        (bh, block, -1, window id) tuples, in the order the CTAs take them."""
        count = ctypes.c_int64(0)
        _check(_lib.sta_plan_backward_items(self.handle, int(which), None, 0, ctypes.byref(count)),
               "sta_plan_backward_items")
        buf = (ctypes.c_int32 * max(4 * count.value, 4))()
        _check(_lib.sta_plan_backward_items(self.handle, int(which), buf, count.value, ctypes.byref(count)),
               "sta_plan_backward_items")
        flat = list(buf[:4 * count.value])
        return [tuple(flat[4 * i:4 * i + 4]) for i in range(count.value)]

    def flops(self, head_dim: int) -> float:
        """Attention FLOPs over computed tiles: pairs * 4 * |tile|^2 * d."""
        vol = self.tile[0] * self.tile[1] * self.tile[2]
        return float(self.stats()[0]) * 4.0 * vol * vol * head_dim

    def validate(self) -> None:
        """Check every index of the plan's host copy (sta_plan_validate)."""
        _check(_lib.sta_plan_validate(self.handle), "sta_plan_validate")

    def destroy(self) -> None:
        if self._h:
            _check(_lib.sta_plan_destroy(self._h), "sta_plan_destroy")
            self._h = ctypes.c_void_p(0)

    def __del__(self):
        try:
            if self._h:
                _lib.sta_plan_destroy(self._h)
                self._h = ctypes.c_void_p(0)
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.destroy()


def sta_plan(latent, tile, batch: int, heads: int, windows, stream=None) -> Plan:
    """Build a plan on the current CUDA device (windows: ``[heads, 3]`` tokens)."""
    h = ctypes.c_void_p(0)
    g = _geom(latent, tile)
    dev = torch.cuda.current_device()
    _check(_lib.sta_plan(ctypes.byref(g), int(batch), int(heads), _windows(heads, windows),
                         _stream(stream), ctypes.byref(h)), "sta_plan")
    return Plan(h.value, latent, tile, batch, heads, windows, device=dev)


def sta_plan_host(latent, tile, batch: int, heads: int, windows) -> Plan:
    """Host-only plan (no device memory): for ``query`` / ``stats`` without a GPU."""
    h = ctypes.c_void_p(0)
    g = _geom(latent, tile)
    _check(_lib.sta_plan_host(ctypes.byref(g), int(batch), int(heads), _windows(heads, windows),
                              ctypes.byref(h)), "sta_plan_host")
    return Plan(h.value, latent, tile, batch, heads, windows)


def _padded_tokens(latent, tile) -> int:
    return math.prod(-(-int(latent[i]) // int(tile[i])) * int(tile[i]) for i in range(3))


def _tile_major_like(x: torch.Tensor, plan: Plan, token_dim: int = 2) -> torch.Tensor:
    """Empty tensor shaped like raster ``x`` with the token dimension padded to whole tiles."""
    shape = list(x.shape)
    shape[token_dim] = plan.padded_tokens
    return torch.empty(shape, dtype=x.dtype, device=x.device)


def _perm_args(src: torch.Tensor, dst: torch.Tensor, tokens: int, token_dim: int,
               src_tokens: int | None = None, dst_tokens: int | None = None):
    if not (src.is_cuda and dst.is_cuda):
        raise ValueError("sta_tile_reorder/unreorder need CUDA tensors")
    if src.dtype != dst.dtype or src.dim() != dst.dim():
        raise ValueError("src and dst must have the same dtype and rank")
    if not (src.is_contiguous() and dst.is_contiguous()):
        raise ValueError("src and dst must be contiguous")
    td = token_dim % src.dim()
    for name, t, n in (("src", src, src_tokens), ("dst", dst, dst_tokens)):
        if t.shape[td] != n:
            raise ValueError(f"{name} dimension {td} has {t.shape[td]} tokens, expected {n}")
    if src.shape[:td] != dst.shape[:td] or src.shape[td + 1:] != dst.shape[td + 1:]:
        raise ValueError("src and dst may differ only in the token dimension")
    outer = math.prod(src.shape[:td]) if td > 0 else 1
    row_bytes = math.prod(src.shape[td + 1:]) * src.element_size()
    return outer, row_bytes


def sta_tile_reorder(src: torch.Tensor, dst: torch.Tensor, latent, tile, token_dim: int = 2,
                     stream=None) -> torch.Tensor:
    """dst = src with the token dimension permuted raster -> tile-major (dst's
    token dimension padded to whole tiles, padding rows zeroed)."""
    N = latent[0] * latent[1] * latent[2]
    outer, row_bytes = _perm_args(src, dst, N, token_dim, N, _padded_tokens(latent, tile))
    g = _geom(latent, tile)
    with torch.cuda.device(_device((src, dst))):
        _check(_lib.sta_tile_reorder(ctypes.c_void_p(src.data_ptr()), ctypes.c_void_p(dst.data_ptr()),
                                     outer, row_bytes, ctypes.byref(g), _stream(stream)),
               "sta_tile_reorder")
    return dst


def sta_tile_unreorder(src: torch.Tensor, dst: torch.Tensor, latent, tile, token_dim: int = 2,
                       stream=None) -> torch.Tensor:
    """dst = src with the token dimension permuted tile-major -> raster (src's
    padding rows are dropped)."""
    N = latent[0] * latent[1] * latent[2]
    outer, row_bytes = _perm_args(src, dst, N, token_dim, _padded_tokens(latent, tile), N)
    g = _geom(latent, tile)
    with torch.cuda.device(_device((src, dst))):
        _check(_lib.sta_tile_unreorder(ctypes.c_void_p(src.data_ptr()), ctypes.c_void_p(dst.data_ptr()),
                                       outer, row_bytes, ctypes.byref(g), _stream(stream)),
               "sta_tile_unreorder")
    return dst


def _forward_args(plan: Plan, q, k, v, o, lse, raster: bool = False):
    B, H = plan.batch, plan.heads
    N = plan.tokens if raster else plan.padded_tokens
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor")
        if t.dim() != 4 or tuple(t.shape[:3]) != (B, H, N):
            raise ValueError(f"{name} has shape {tuple(t.shape)}, plan expects [{B}, {H}, {N}, d]")
    d = q.shape[3]
    if k.shape[3] != d or v.shape[3] != d or o.shape[3] != d:
        raise ValueError("q, k, v, o must share the head dimension")
    if not lse.is_cuda or lse.dtype != torch.float32 or not lse.is_contiguous() \
            or tuple(lse.shape) != (B, H, N):
        raise ValueError(f"lse must be a contiguous CUDA fp32 tensor of shape [{B}, {H}, {N}]")
    return (ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
            ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lse.data_ptr()), int(d))


def sta_forward(plan: Plan, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                o: torch.Tensor, lse: torch.Tensor, softmax_scale: float, stream=None):
    """STA forward on tile-major ``[B, H, N, d]`` bf16 tensors; writes ``o`` and ``lse``."""
    args = _forward_args(plan, q, k, v, o, lse)
    with torch.cuda.device(_device((q, k, v, o, lse), plan)):
        _check(_lib.sta_forward(plan.handle, *args, float(softmax_scale), _stream(stream)), "sta_forward")
    return o, lse


def sta_forward_raster(plan: Plan, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                       o: torch.Tensor, lse: torch.Tensor, softmax_scale: float, stream=None):
    """STA forward on raster-order ``[B, H, N, d]`` bf16 tensors (permutation fused)."""
    args = _forward_args(plan, q, k, v, o, lse, raster=True)
    with torch.cuda.device(_device((q, k, v, o, lse), plan)):
        _check(_lib.sta_forward_raster(plan.handle, *args, float(softmax_scale), _stream(stream)),
               "sta_forward_raster")
    return o, lse


def _backward_call(fn, what: str, plan: Plan, q, k, v, o, lse, dout, softmax_scale, dq, dk, dv, workspace,
                   stream, raster: bool):
    args = _forward_args(plan, q, k, v, o, lse, raster=raster)
    B, H = plan.batch, plan.heads
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for name, t in (("dout", dout), ("dq", dq), ("dk", dk), ("dv", dv)):
        if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() or t.shape != q.shape:
            raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor of shape {tuple(q.shape)}")
    n_ws = 2 * B * H * plan.padded_tokens
    if workspace is None:
        workspace = torch.empty(n_ws, dtype=torch.float32, device=q.device)
    if not workspace.is_cuda or workspace.dtype != torch.float32 or not workspace.is_contiguous() \
            or workspace.numel() < n_ws:
        raise ValueError(f"workspace must be a contiguous CUDA fp32 tensor of {n_ws} floats")
    qp, kp, vp_, op, lp, hd = args
    with torch.cuda.device(_device((q, k, v, o, lse, dout, dq, dk, dv, workspace), plan)):
        _check(fn(plan.handle, qp, kp, vp_, op, ctypes.c_void_p(dout.data_ptr()), lp,
                  ctypes.c_void_p(dq.data_ptr()), ctypes.c_void_p(dk.data_ptr()), ctypes.c_void_p(dv.data_ptr()),
                  ctypes.c_void_p(workspace.data_ptr()), hd, float(softmax_scale), _stream(stream)), what)
    return dq, dk, dv


def sta_backward(plan: Plan, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
                 lse: torch.Tensor, dout: torch.Tensor, softmax_scale: float, dq=None, dk=None, dv=None,
                 workspace=None, stream=None):
    """STA backward on tile-major ``[B, H, N_tiles, d]`` bf16 tensors (``o`` and
    ``lse`` from ``sta_forward``).  Returns ``(dq, dk, dv)``; outputs and the fp32
    workspace (``2 * B * H * N_tiles`` floats) are allocated when not given."""
    return _backward_call(_lib.sta_backward, "sta_backward", plan, q, k, v, o, lse, dout, softmax_scale,
                          dq, dk, dv, workspace, stream, raster=False)


def sta_backward_raster(plan: Plan, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
                        lse: torch.Tensor, dout: torch.Tensor, softmax_scale: float, dq=None, dk=None, dv=None,
                        workspace=None, stream=None):
    """STA backward on raster-order ``[B, H, N, d]`` bf16 tensors (``o`` and
    ``lse`` from ``sta_forward_raster``), the permutation fused into the kernels."""
    return _backward_call(_lib.sta_backward_raster, "sta_backward_raster", plan, q, k, v, o, lse, dout,
                          softmax_scale, dq, dk, dv, workspace, stream, raster=True)


def raster_supported(tile, latent=None) -> bool:
    """Whether the fused raster path handles this tile shape (see sta.h); with
    ``latent``, also that one block's box is no larger than the latent."""
    T = [int(x) for x in tile]
    L = [int(x) for x in latent] if latent is not None else [1 << 30] * 3
    hw = T[1] * T[2]
    if T[2] > 256 or T[2] > L[2]:
        return False
    if 128 % hw == 0:
        box_t = 128 // hw
        return T[0] % box_t == 0 and T[1] <= 256 and box_t <= L[0] and T[1] <= L[1]
    return hw % 128 == 0 and 128 % T[2] == 0 and 128 // T[2] <= L[1]


def sta_forward_noalloc(latent, tile, batch: int, heads: int, windows, q: torch.Tensor,
                        k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, lse: torch.Tensor,
                        softmax_scale: float, stream=None):
    """STA forward without any device allocation by the library: the plan is
    kept in the library's fixed scratch array (see ``include/sta.h``).  Same
    tile-major tensors as ``sta_forward``; calls must not overlap on the GPU."""
    B, H = int(batch), int(heads)
    N = int(latent[0]) * int(latent[1]) * int(latent[2])
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor")
        if t.dim() != 4 or tuple(t.shape[:3]) != (B, H, N) or t.shape[3] != q.shape[3]:
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected [{B}, {H}, {N}, d]")
    if not lse.is_cuda or lse.dtype != torch.float32 or not lse.is_contiguous() \
            or tuple(lse.shape) != (B, H, N):
        raise ValueError(f"lse must be a contiguous CUDA fp32 tensor of shape [{B}, {H}, {N}]")
    g = _geom(latent, tile)
    with torch.cuda.device(_device((q, k, v, o, lse))):
        _check(_lib.sta_forward_noalloc(ctypes.byref(g), B, H, _windows(H, windows),
                                        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                        ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(o.data_ptr()),
                                        ctypes.c_void_p(lse.data_ptr()), int(q.shape[3]),
                                        float(softmax_scale), _stream(stream)), "sta_forward_noalloc")
    return o, lse


def sta_last_device_status(plan: Plan, stream=None) -> int:
    """Synchronise and return (clearing it) the plan's device status code."""
    if plan.device is None:
        return int(_lib.sta_last_device_status(plan.handle, None))  # host-only plan: INVALID_ARG
    with torch.cuda.device(plan.device):
        return int(_lib.sta_last_device_status(plan.handle, _stream(stream)))


def sta_debug_inject_timeout(mode, limit_ms: int = 50) -> None:
    """Debug: make a device-side wait of the next forward calls run out
    (``mode`` 0 off, 1 or True: before any copy, 2: at a CTA's second work
    item with copies issued); see sta.h."""
    _check(_lib.sta_debug_inject_timeout(int(mode), int(limit_ms)), "sta_debug_inject_timeout")


def sta_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, plan: Plan,
                  softmax_scale: float | None = None, stream=None, fused: bool = True):
    """STA attention on raster-order ``[B, H, N, d]`` bf16 tensors.

    With ``fused`` (and a tile shape the fused kernel handles) one kernel reads
    and writes raster order directly; otherwise Q, K, V are permuted to
    tile-major order, the forward kernel runs, and O and LSE are permuted back.
    Both give the same bits.  Returns ``(O bf16 [B, H, N, d], LSE fp32 [B, H, N])``.
    """
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(q.shape[-1])
    lat, tile = plan.latent, plan.tile
    if fused and raster_supported(tile, lat):
        o = torch.empty_like(q)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
        return sta_forward_raster(plan, q, k, v, o, lse, softmax_scale, stream=stream)
    qt, kt, vt = (_tile_major_like(x, plan) for x in (q, k, v))
    sta_tile_reorder(q, qt, lat, tile, stream=stream)
    sta_tile_reorder(k, kt, lat, tile, stream=stream)
    sta_tile_reorder(v, vt, lat, tile, stream=stream)
    ot = torch.empty_like(qt)
    lset = torch.empty(qt.shape[:3], dtype=torch.float32, device=q.device)
    sta_forward(plan, qt, kt, vt, ot, lset, softmax_scale, stream=stream)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    sta_tile_unreorder(ot, o, lat, tile, stream=stream)
    sta_tile_unreorder(lset, lse, lat, tile, stream=stream)
    return o, lse


def sta_attention_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
                           lse: torch.Tensor, dout: torch.Tensor, plan: Plan,
                           softmax_scale: float | None = None, stream=None, fused: bool = True):
    """Gradients ``(dq, dk, dv)`` of ``sta_attention`` on raster-order tensors.

    With ``fused`` (and a tile shape the fused kernels handle) the kernels read
    and write raster order directly; otherwise the inputs are permuted to
    tile-major order, ``sta_backward`` runs, and the gradients are permuted
    back.  Both give the same bits."""
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(q.shape[-1])
    lat, tile = plan.latent, plan.tile
    if fused and raster_supported(tile, lat):
        return sta_backward_raster(plan, q, k, v, o, lse, dout, softmax_scale, stream=stream)

    def to_tiles(x):
        y = _tile_major_like(x, plan)
        sta_tile_reorder(x, y, lat, tile, stream=stream)
        return y

    qt, kt, vt, ot, dot, lset = (to_tiles(x) for x in (q, k, v, o, dout, lse))
    dqt, dkt, dvt = sta_backward(plan, qt, kt, vt, ot, lset, dot, softmax_scale, stream=stream)
    out = []
    for x, like in ((dqt, q), (dkt, k), (dvt, v)):
        y = torch.empty_like(like)
        sta_tile_unreorder(x, y, lat, tile, stream=stream)
        out.append(y)
    return tuple(out)


class StaAttention(torch.autograd.Function):
    """``O = StaAttention.apply(q, k, v, plan, softmax_scale)`` on raster-order
    bf16 tensors, with gradients for q, k and v through ``sta_backward``."""

    @staticmethod
    def forward(ctx, q, k, v, plan, softmax_scale=None):
        scale = 1.0 / math.sqrt(q.shape[-1]) if softmax_scale is None else float(softmax_scale)
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        o, lse = sta_attention(q, k, v, plan, scale)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.plan, ctx.scale = plan, scale
        return o

    @staticmethod
    def backward(ctx, dout):
        q, k, v, o, lse = ctx.saved_tensors
        dq, dk, dv = sta_attention_backward(q, k, v, o, lse, dout.contiguous(), ctx.plan, ctx.scale)
        return dq, dk, dv, None, None


def sta_window_stats(lse_w: torch.Tensor, lse_full: torch.Tensor, o_w: torch.Tensor, o_full: torch.Tensor,
                     stream=None):
    """Per-(b, h) attention recall (mean of exp(lse_w - lse_full)) and output
    mean squared error of a candidate window against the full window.
    Returns ``(recall, mse)``, fp64 CUDA tensors of shape ``[B, H]``."""
    if o_w.shape != o_full.shape or lse_w.shape != lse_full.shape or tuple(lse_w.shape) != tuple(o_w.shape[:3]):
        raise ValueError("o_w / o_full must be [B, H, N, d] and lse_w / lse_full [B, H, N], matching")
    for name, t, dt in (("lse_w", lse_w, torch.float32), ("lse_full", lse_full, torch.float32),
                        ("o_w", o_w, torch.bfloat16), ("o_full", o_full, torch.bfloat16)):
        if not t.is_cuda or t.dtype != dt or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA {dt} tensor")
    B, H, N, d = o_w.shape
    dev = _device((lse_w, lse_full, o_w, o_full))
    recall = torch.empty((B, H), dtype=torch.float64, device=dev)
    mse = torch.empty_like(recall)
    with torch.cuda.device(dev):
        _check(_lib.sta_window_stats(ctypes.c_void_p(lse_w.data_ptr()), ctypes.c_void_p(lse_full.data_ptr()),
                                     ctypes.c_void_p(o_w.data_ptr()), ctypes.c_void_p(o_full.data_ptr()),
                                     B * H, N, d, ctypes.c_void_p(recall.data_ptr()),
                                     ctypes.c_void_p(mse.data_ptr()), _stream(stream)), "sta_window_stats")
    return recall, mse


def sta_window_search(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, latent, tile, candidates,
                      softmax_scale: float | None = None, max_mse: float | None = None,
                      min_recall: float | None = None, stream=None) -> dict:
    """Profile candidate windows per head on raster-order inputs and pick one.

    For every candidate (a window in tokens, used for all heads) the STA
    forward runs once, and once with a window covering the volume;
    ``sta_window_stats`` gives each (b, h) its recall and output error, which
    are averaged over the batch (the inputs the search averages over).  Each
    head gets the candidate with the fewest attended tiles that meets every
    given bound (``max_mse``, ``min_recall``); the full window when none does.
    Returns ``{"windows": [H][3], "recall": [C, H], "mse": [C, H],
    "candidates": [C][3], "tiles": [C]}`` (host values, fp64)."""
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(q.shape[-1])
    B, H = int(q.shape[0]), int(q.shape[1])
    lat = tuple(int(x) for x in latent)
    cands = [tuple(int(x) for x in c) for c in candidates]
    dev = _device((q, k, v))
    with torch.cuda.device(dev):  # plans live on the inputs' device
        full = sta_plan(lat, tile, B, H, [lat] * H, stream=stream)
    o_full, lse_full = sta_attention(q, k, v, full, softmax_scale, stream=stream)
    n = [-(-lat[i] // int(tile[i])) for i in range(3)]  # tiles per axis (padded latents: whole tiles)
    tiles, rec, err = [], [], []
    for c in cands:
        with torch.cuda.device(dev):
            plan = sta_plan(lat, tile, B, H, [c] * H, stream=stream)
        o_c, lse_c = sta_attention(q, k, v, plan, softmax_scale, stream=stream)
        r, m = sta_window_stats(lse_c, lse_full, o_c, o_full, stream=stream)
        rec.append(r.mean(dim=0))
        err.append(m.mean(dim=0))
        tiles.append(math.prod(min(c[i] // int(tile[i]), n[i]) for i in range(3)))
        plan.destroy()
    full.destroy()
    recall = torch.stack(rec).cpu().double().contiguous() if rec else None
    mse = torch.stack(err).cpu().double().contiguous() if err else None
    chosen = sta_window_pick(lat, tile, H, cands, recall, mse, max_mse, min_recall)
    return {"windows": chosen, "recall": recall.numpy() if rec else None, "mse": mse.numpy() if err else None,
            "candidates": [list(c) for c in cands], "tiles": tiles}


def sta_window_pick(latent, tile, heads: int, candidates, recall, mse, max_mse: float | None = None,
                    min_recall: float | None = None) -> list:
    """Per head, the candidate window with the fewest attended tiles meeting
    the bounds (the C call ``sta_window_pick``); recall and mse are
    ``[len(candidates), heads]`` host arrays.  Returns ``[heads][3]``."""
    cands = [tuple(int(x) for x in c) for c in candidates]
    C, H = len(cands), int(heads)
    flat = (ctypes.c_int32 * max(3 * C, 3))(*[x for c in cands for x in c])
    r = torch.as_tensor(recall if C else [0.0], dtype=torch.float64).contiguous()
    m = torch.as_tensor(mse if C else [0.0], dtype=torch.float64).contiguous()
    if C and (tuple(r.shape) != (C, H) or tuple(m.shape) != (C, H)):
        raise ValueError(f"recall and mse must be [{C}, {H}]")
    out = (ctypes.c_int32 * (3 * H))()
    geom = _geom(latent, tile)
    _check(_lib.sta_window_pick(ctypes.byref(geom), H, C, flat, ctypes.c_void_p(r.data_ptr()),
                                ctypes.c_void_p(m.data_ptr()), -1.0 if max_mse is None else float(max_mse),
                                -1.0 if min_recall is None else float(min_recall), out), "sta_window_pick")
    return [list(out[3 * h:3 * h + 3]) for h in range(H)]


class Pipe:
    """STA forward from host memory with copy-in, forward and copy-out of
    consecutive calls overlapped (``sta_pipe_*`` in ``include/sta.h``)."""

    def __init__(self, handle: int, plan: Plan, head_dim: int):
        self._h = ctypes.c_void_p(handle)
        self.plan = plan  # kept alive: the pipeline uses it
        self.head_dim = int(head_dim)

    def submit(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
               lse: torch.Tensor) -> None:
        """Enqueue one call on pinned host tensors (raster order): reads q, k, v,
        writes o and lse once ``wait`` returns."""
        B, H, N, d = self.plan.batch, self.plan.heads, self.plan.tokens, self.head_dim
        for name, t, shape, dt in (("q", q, (B, H, N, d), torch.bfloat16), ("k", k, (B, H, N, d), torch.bfloat16),
                                   ("v", v, (B, H, N, d), torch.bfloat16), ("o", o, (B, H, N, d), torch.bfloat16),
                                   ("lse", lse, (B, H, N), torch.float32)):
            if t.is_cuda or t.dtype != dt or not t.is_contiguous() or tuple(t.shape) != shape:
                raise ValueError(f"{name} must be a contiguous host {dt} tensor of shape {shape}")
            if not t.is_pinned():
                raise ValueError(f"{name} must be in pinned host memory (tensor.pin_memory())")
        with torch.cuda.device(self.plan.device):
            _check(_lib.sta_pipe_submit(self._h, ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                        ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(o.data_ptr()),
                                        ctypes.c_void_p(lse.data_ptr())), "sta_pipe_submit")

    def wait(self) -> None:
        with torch.cuda.device(self.plan.device):
            _check(_lib.sta_pipe_wait(self._h), "sta_pipe_wait")

    def destroy(self) -> None:
        if self._h:
            _check(_lib.sta_pipe_destroy(self._h), "sta_pipe_destroy")
            self._h = ctypes.c_void_p(0)

    def __del__(self):
        try:
            if self._h:
                _lib.sta_pipe_destroy(self._h)
                self._h = ctypes.c_void_p(0)
        except Exception:
            pass


def sta_pipe_create(plan: Plan, head_dim: int, softmax_scale: float | None = None, depth: int = 2) -> Pipe:
    """Pipeline of ``depth`` device buffer sets for ``plan``, on the plan's device."""
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(head_dim)
    if plan.device is None:
        raise ValueError("sta_pipe_create needs a device plan (sta_plan), not a host-only one")
    h = ctypes.c_void_p(0)
    with torch.cuda.device(plan.device):
        _check(_lib.sta_pipe_create(plan.handle, int(head_dim), float(softmax_scale), int(depth), ctypes.byref(h)),
               "sta_pipe_create")
    return Pipe(h.value, plan, head_dim)
