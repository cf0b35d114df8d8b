"""CPU oracle for Sliding Tile Attention (STA) -- test infrastructure only.

This package is the checker, not the product.  Only ``tests/``, the smoke
check in ``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may
import it.  It shares no code with the CUDA library: the arithmetic lives in
``sta_oracle.c`` (plain C, fp64), compiled here with gcc and called through
ctypes.  The method it follows is the one described in "Fast Video Generation
with Sliding Tile Attention" (tile-by-tile sliding window, per-head window,
exact softmax over the attended tiles); the readings of points the pages leave
open are listed at the top of ``sta_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sta_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle_sta.so")

_lock = threading.Lock()
_lib = None


class _Geom(ctypes.Structure):
    _fields_ = [("lat", ctypes.c_int32 * 3), ("tile", ctypes.c_int32 * 3)]


def build(force: bool = False) -> str:
    """Compile ``sta_oracle.c`` into ``_build/liboracle_sta.so``; return its path."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-fPIC", "-shared", "-pthread",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            path = build()
            L = ctypes.CDLL(path)
            G = ctypes.POINTER(_Geom)
            i32p = ctypes.POINTER(ctypes.c_int32)
            L.ora_num_tokens.argtypes = [G]
            L.ora_num_tokens.restype = ctypes.c_int64
            L.ora_key_allowed.argtypes = [G, i32p, ctypes.c_int64, ctypes.c_int64]
            L.ora_key_allowed.restype = ctypes.c_int
            L.ora_mask_row.argtypes = [G, i32p, ctypes.c_int64, ctypes.c_void_p]
            L.ora_mask_row.restype = ctypes.c_int
            L.ora_tile_major_index.argtypes = [G, ctypes.c_int64]
            L.ora_tile_major_index.restype = ctypes.c_int64
            L.ora_sta_attention.argtypes = [
                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, G,
                ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, i32p, ctypes.c_float,
                ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                ctypes.c_int32]
            L.ora_sta_attention.restype = ctypes.c_int
            bw = [ctypes.c_void_p] * 4 + [G, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, i32p,
                                          ctypes.c_float, ctypes.c_void_p, ctypes.c_int64]
            L.ora_sta_backward_dq.argtypes = bw + [ctypes.c_void_p, ctypes.c_int32]
            L.ora_sta_backward_dq.restype = ctypes.c_int
            L.ora_sta_backward_dkdv.argtypes = bw + [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32]
            L.ora_sta_backward_dkdv.restype = ctypes.c_int
            L.ora_window_recall.argtypes = [ctypes.c_void_p, ctypes.c_void_p, G, ctypes.c_int64, ctypes.c_int64,
                                            ctypes.c_int32, i32p, ctypes.c_float, ctypes.c_void_p,
                                            ctypes.c_int64, ctypes.c_void_p, ctypes.c_int32]
            L.ora_window_recall.restype = ctypes.c_int
            _lib = L
    return _lib


def _geom(latent, tile) -> _Geom:
    g = _Geom()
    for i in range(3):
        g.lat[i] = int(latent[i])
        g.tile[i] = int(tile[i])
    return g


def _win(window) -> ctypes.Array:
    w = (ctypes.c_int32 * 3)()
    for i in range(3):
        w[i] = int(window[i])
    return w


def num_tokens(latent) -> int:
    return int(latent[0]) * int(latent[1]) * int(latent[2])


def key_allowed(latent, tile, window, qi: int, kj: int) -> int:
    """1 if raster query token ``qi`` may attend raster key token ``kj``."""
    r = lib().ora_key_allowed(ctypes.byref(_geom(latent, tile)), _win(window), int(qi), int(kj))
    if r < 0:
        raise ValueError("oracle: bad arguments to key_allowed")
    return r


def mask_row(latent, tile, window, qi: int) -> np.ndarray:
    """Token-level STA mask row of raster query token ``qi`` (bool, length N)."""
    out = np.zeros(num_tokens(latent), dtype=np.uint8)
    r = lib().ora_mask_row(ctypes.byref(_geom(latent, tile)), _win(window), int(qi),
                           out.ctypes.data)
    if r != 0:
        raise ValueError("oracle: bad arguments to mask_row")
    return out.astype(bool)


def tile_major_index(latent, tile, tokens) -> np.ndarray:
    """Tile-major position of each raster token in ``tokens``."""
    g = _geom(latent, tile)
    L = lib()
    toks = np.asarray(tokens, dtype=np.int64).ravel()
    out = np.empty_like(toks)
    for i, t in enumerate(toks):
        out[i] = L.ora_tile_major_index(ctypes.byref(g), int(t))
        if out[i] < 0:
            raise ValueError("oracle: bad arguments to tile_major_index")
    return out


def tile_tokens(latent, tile, tile_id: int) -> np.ndarray:
    """Raster indices of the real tokens of tile ``tile_id`` (tiles numbered in
    raster order over the tile grid of ceil(L / T) tiles per axis), in raster
    order; a tile at a padded edge holds fewer than a full tile."""
    n = [-(-latent[i] // tile[i]) for i in range(3)]
    it, rem = divmod(int(tile_id), n[1] * n[2])
    ih, iw = divmod(rem, n[2])
    t = np.arange(tile[0]) + it * tile[0]
    h = np.arange(tile[1]) + ih * tile[1]
    w = np.arange(tile[2]) + iw * tile[2]
    t, h, w = t[t < latent[0]], h[h < latent[1]], w[w < latent[2]]
    tt, hh, ww = np.meshgrid(t, h, w, indexing="ij")
    return ((tt * latent[1] + hh) * latent[2] + ww).ravel().astype(np.int64)


def _as_u16(x) -> np.ndarray:
    """bf16 tensor (torch) or uint16 array -> contiguous uint16 numpy array."""
    if hasattr(x, "view") and hasattr(x, "dtype") and "bfloat16" in str(x.dtype):
        import torch
        return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    a = np.ascontiguousarray(x)
    if a.dtype != np.uint16:
        raise TypeError("oracle: expected bf16 tensor or uint16 bit array")
    return a


def sta_attention(q, k, v, latent, tile, windows, softmax_scale: float,
                  rows=None, nthreads: int | None = None):
    """fp64 STA attention.

    q, k, v : bf16 ``[B, H, N, d]`` in raster token order (torch bf16 or uint16 bits)
    windows : ``[H, 3]`` window per head in tokens
    rows    : optional ``[R, 2]`` int64 pairs ``(b * H + h, raster token)``;
              default is every row of every head
    Returns ``(O [R, d] float64, LSE [R] float64)``; with ``rows=None`` the
    results are reshaped to ``[B, H, N, d]`` and ``[B, H, N]``.
    """
    qa, ka, va = _as_u16(q), _as_u16(k), _as_u16(v)
    if qa.ndim != 4 or qa.shape != ka.shape or qa.shape != va.shape:
        raise ValueError("oracle: q, k, v must share a [B, H, N, d] shape")
    B, H, N, d = qa.shape
    if N != num_tokens(latent):
        raise ValueError("oracle: N does not match the latent")
    win = np.ascontiguousarray(np.asarray(windows, dtype=np.int32).reshape(H, 3))
    full = rows is None
    if full:
        bh = np.repeat(np.arange(B * H, dtype=np.int64), N)
        tok = np.tile(np.arange(N, dtype=np.int64), B * H)
        rows_a = np.stack([bh, tok], axis=1)
    else:
        rows_a = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 2))
    R = rows_a.shape[0]
    out_o = np.empty((R, d), dtype=np.float64)
    out_lse = np.empty((R,), dtype=np.float64)
    if nthreads is None:
        nthreads = max(1, os.cpu_count() or 1)
    r = lib().ora_sta_attention(
        qa.ctypes.data, ka.ctypes.data, va.ctypes.data, ctypes.byref(_geom(latent, tile)),
        B, H, d, win.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), float(softmax_scale),
        rows_a.ctypes.data, R, out_o.ctypes.data, out_lse.ctypes.data, int(nthreads))
    if r != 0:
        raise ValueError(f"oracle: ora_sta_attention failed with status {r}")
    if full:
        return out_o.reshape(B, H, N, d), out_lse.reshape(B, H, N)
    return out_o, out_lse


def _rows_or_all(rows, B, H, N):
    if rows is None:
        bh = np.repeat(np.arange(B * H, dtype=np.int64), N)
        tok = np.tile(np.arange(N, dtype=np.int64), B * H)
        return np.stack([bh, tok], axis=1), True
    return np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 2)), False


def _bw_args(q, k, v, dout, latent, windows):
    qa, ka, va, da = _as_u16(q), _as_u16(k), _as_u16(v), _as_u16(dout)
    if qa.ndim != 4 or any(x.shape != qa.shape for x in (ka, va, da)):
        raise ValueError("oracle: q, k, v, dout must share a [B, H, N, d] shape")
    B, H, N, d = qa.shape
    if N != num_tokens(latent):
        raise ValueError("oracle: N does not match the latent")
    win = np.ascontiguousarray(np.asarray(windows, dtype=np.int32).reshape(H, 3))
    return qa, ka, va, da, win, (B, H, N, d)


def sta_backward_dq(q, k, v, dout, latent, tile, windows, softmax_scale: float,
                    rows=None, nthreads: int | None = None):
    """fp64 gradient of STA attention with respect to Q, for upstream gradient
    ``dout`` (same shape as O).

    rows : optional ``[R, 2]`` pairs ``(b * H + h, raster query token)``;
           default every row, returned as ``[B, H, N, d]``, else ``[R, d]``.
    """
    qa, ka, va, da, win, (B, H, N, d) = _bw_args(q, k, v, dout, latent, windows)
    rows_a, full = _rows_or_all(rows, B, H, N)
    out = np.empty((rows_a.shape[0], d), dtype=np.float64)
    r = lib().ora_sta_backward_dq(
        qa.ctypes.data, ka.ctypes.data, va.ctypes.data, da.ctypes.data,
        ctypes.byref(_geom(latent, tile)), B, H, d,
        win.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), float(softmax_scale),
        rows_a.ctypes.data, rows_a.shape[0], out.ctypes.data,
        int(nthreads or max(1, os.cpu_count() or 1)))
    if r != 0:
        raise ValueError(f"oracle: ora_sta_backward_dq failed with status {r}")
    return out.reshape(B, H, N, d) if full else out


def sta_backward_dkdv(q, k, v, dout, latent, tile, windows, softmax_scale: float,
                      keys=None, nthreads: int | None = None):
    """fp64 gradients of STA attention with respect to K and V.

    keys : optional ``[R, 2]`` pairs ``(b * H + h, raster key token)``;
           default every key.  Returns ``(dK, dV)``, ``[B, H, N, d]`` each for
           all keys, else ``[R, d]`` each.
    """
    qa, ka, va, da, win, (B, H, N, d) = _bw_args(q, k, v, dout, latent, windows)
    keys_a, full = _rows_or_all(keys, B, H, N)
    R = keys_a.shape[0]
    dk = np.empty((R, d), dtype=np.float64)
    dv = np.empty((R, d), dtype=np.float64)
    r = lib().ora_sta_backward_dkdv(
        qa.ctypes.data, ka.ctypes.data, va.ctypes.data, da.ctypes.data,
        ctypes.byref(_geom(latent, tile)), B, H, d,
        win.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), float(softmax_scale),
        keys_a.ctypes.data, R, dk.ctypes.data, dv.ctypes.data,
        int(nthreads or max(1, os.cpu_count() or 1)))
    if r != 0:
        raise ValueError(f"oracle: ora_sta_backward_dkdv failed with status {r}")
    if full:
        return dk.reshape(B, H, N, d), dv.reshape(B, H, N, d)
    return dk, dv


def sta_backward(q, k, v, dout, latent, tile, windows, softmax_scale: float,
                 nthreads: int | None = None):
    """All three fp64 gradients ``(dQ, dK, dV)``, each ``[B, H, N, d]``."""
    dq = sta_backward_dq(q, k, v, dout, latent, tile, windows, softmax_scale, nthreads=nthreads)
    dk, dv = sta_backward_dkdv(q, k, v, dout, latent, tile, windows, softmax_scale, nthreads=nthreads)
    return dq, dk, dv


def window_recall(q, k, latent, tile, windows, softmax_scale: float, rows=None,
                  nthreads: int | None = None) -> np.ndarray:
    """Attention recall of query rows: the share of each row's full-attention
    softmax mass on the keys its STA window attends.  ``rows`` as in
    ``sta_attention``; default every row, returned as ``[B, H, N]``."""
    qa, ka = _as_u16(q), _as_u16(k)
    if qa.ndim != 4 or qa.shape != ka.shape:
        raise ValueError("oracle: q, k must share a [B, H, N, d] shape")
    B, H, N, d = qa.shape
    if N != num_tokens(latent):
        raise ValueError("oracle: N does not match the latent")
    win = np.ascontiguousarray(np.asarray(windows, dtype=np.int32).reshape(H, 3))
    rows_a, full = _rows_or_all(rows, B, H, N)
    out = np.empty((rows_a.shape[0],), dtype=np.float64)
    r = lib().ora_window_recall(qa.ctypes.data, ka.ctypes.data, ctypes.byref(_geom(latent, tile)), B, H, d,
                                win.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), float(softmax_scale),
                                rows_a.ctypes.data, rows_a.shape[0], out.ctypes.data,
                                int(nthreads or max(1, os.cpu_count() or 1)))
    if r != 0:
        raise ValueError(f"oracle: ora_window_recall failed with status {r}")
    return out.reshape(B, H, N) if full else out
