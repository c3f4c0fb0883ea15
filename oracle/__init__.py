"""CPU oracle for the vision PatchEmbed -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it and the
two share no code; the only thing both sides consume is the seeded input
generator in ``workloads``.

The arithmetic lives in ``pe_oracle.c`` (plain C, fp64 accumulation, OpenMP over
output rows).  This module compiles it with gcc on first use and marshals numpy
arrays through ctypes; it adds no arithmetic of its own except concatenating
the rows of a grouped call in list order (Optimize VLM PatchEmbed, the vision
model's forward: ``hidden_states`` of shape (seq_len, ...) with ``grid_thw`` of
shape (num_images_or_videos, 3)).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libpe_oracle.so")
_lib = None
# A test may point this at a deliberately broken build of pe_oracle.c to check
# that the pins catch it; normal use leaves it unset.
_LIB_OVERRIDE = os.environ.get("PE_ORACLE_LIB")

_CFLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-std=c11",
           "-shared", "-fPIC"]


def compile_source(src: str, out: str) -> str:
    """Compile a C source of the oracle into a shared library at ``out``."""
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", *_CFLAGS, src, "-o", tmp, "-lm"])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile pe_oracle.c into libpe_oracle.so next to it (gcc)."""
    if force or not os.path.exists(_LIB_PATH) or \
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        compile_source(_SRC, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(_LIB_OVERRIDE or build())
        f32p = ctypes.POINTER(ctypes.c_float)
        f64p = ctypes.POINTER(ctypes.c_double)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        lib.oracle_bf16_round.argtypes = [ctypes.c_float]
        lib.oracle_bf16_round.restype = ctypes.c_float
        lib.oracle_bf16_round_array.argtypes = [f32p, f32p, ctypes.c_int64]
        lib.oracle_normalize_pixel.argtypes = [ctypes.c_float] * 3
        lib.oracle_normalize_pixel.restype = ctypes.c_float
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_row_index.argtypes = [ctypes.c_int64] * 5 + [ctypes.c_int]
        lib.oracle_row_index.restype = ctypes.c_int64
        lib.oracle_conv3d_patches.argtypes = [
            f32p, ctypes.c_int64, f32p, f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, u8p, f64p, f64p]
        lib.oracle_conv3d_patches_fp32.argtypes = lib.oracle_conv3d_patches.argtypes
        lib.oracle_patch_merger.argtypes = [
            f32p, ctypes.c_int64, ctypes.c_int, ctypes.c_int, f32p, f32p, ctypes.c_double, f32p, f32p, f32p, f32p,
            ctypes.c_int, u8p, f64p, f64p]
        lib.oracle_conv3d_frames.argtypes = [
            f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, f32p, f32p, f32p, f32p, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, u8p, f64p, f64p]
        lib.oracle_conv3d_frames.restype = ctypes.c_int
        lib.oracle_patchify.argtypes = [
            f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, f32p, f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            f32p]
        lib.oracle_patchify.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f32(a) -> np.ndarray:
    """Host fp32 C-contiguous copy of a numpy array or CPU torch tensor (bf16 widens exactly)."""
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").float().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _p(a: Optional[np.ndarray], ct):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ct))


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def bf16_round(a) -> np.ndarray:
    a = _f32(a)
    out = np.empty_like(a)
    _load().oracle_bf16_round_array(_p(a, ctypes.c_float), _p(out, ctypes.c_float), a.size)
    return out


def normalize_pixel(x: float, mean: float, std: float) -> float:
    return float(_load().oracle_normalize_pixel(x, mean, std))


def row_index(g_t: int, g_h: int, g_w: int, h: int, w: int, merge: int) -> int:
    return int(_load().oracle_row_index(g_t, g_h, g_w, h, w, merge))


def _mask(row_mask, n):
    if row_mask is None:
        return None
    m = np.ascontiguousarray(np.asarray(row_mask, dtype=np.uint8))
    assert m.shape == (n,)
    return m


def conv3d_patches(x, w, bias, C: int, tp: int, p: int, row_mask=None
                   ) -> Tuple[np.ndarray, np.ndarray]:
    """Patches form. Returns (out[N,E] fp64, absdot[N,E] fp64); masked-out rows are NaN."""
    x = _f32(x)
    w = _f32(w)
    E = int(w.shape[0])
    K = C * tp * p * p
    assert w.size == E * K and x.ndim == 2 and x.shape[1] == K
    N = int(x.shape[0])
    b = None if bias is None else _f32(bias)
    out = np.full((N, E), np.nan)
    mag = np.full((N, E), np.nan)
    m = _mask(row_mask, N)
    _load().oracle_conv3d_patches(_p(x, ctypes.c_float), N, _p(w, ctypes.c_float),
                                  _p(b, ctypes.c_float), E, C, tp, p,
                                  _p(m, ctypes.c_uint8), _p(out, ctypes.c_double),
                                  _p(mag, ctypes.c_double))
    return out, mag


def conv3d_patches_fp32(x, w, bias, C: int, tp: int, p: int, row_mask=None
                        ) -> Tuple[np.ndarray, np.ndarray]:
    """Patches form on the fp32 values as given (no bf16 rounding): the Conv3d
    definition in fp64.  Returns (out[N,E], absdot[N,E]); masked-out rows NaN."""
    x = _f32(x)
    w = _f32(w)
    E = int(w.shape[0])
    K = C * tp * p * p
    assert w.size == E * K and x.ndim == 2 and x.shape[1] == K
    N = int(x.shape[0])
    b = None if bias is None else _f32(bias)
    out = np.full((N, E), np.nan)
    mag = np.full((N, E), np.nan)
    m = _mask(row_mask, N)
    _load().oracle_conv3d_patches_fp32(_p(x, ctypes.c_float), N, _p(w, ctypes.c_float),
                                       _p(b, ctypes.c_float), E, C, tp, p,
                                       _p(m, ctypes.c_uint8), _p(out, ctypes.c_double),
                                       _p(mag, ctypes.c_double))
    return out, mag


def patch_merger(x, m2: int, gamma, beta, eps: float, w1, b1, w2, b2, v_mask=None
                 ) -> Tuple[np.ndarray, np.ndarray]:
    """PatchMerger on rows in merge order: x [V*m2, E] -> (out [V, H], absdot [V, H])
    fp64 (LayerNorm, concat of m2 rows, fc1 + exact GELU, fc2; the LayerNorm and
    GELU outputs and the weights rounded to bf16).  Masked-out rows are NaN."""
    x = _f32(x)
    E = int(x.shape[1])
    assert x.shape[0] % m2 == 0
    V = x.shape[0] // m2
    D = E * m2
    w1 = _f32(w1)
    w2 = _f32(w2)
    H = int(w2.shape[0])
    assert w1.shape == (D, D) and w2.shape == (H, D)
    gm, bt = _f32(gamma), _f32(beta)                 # held for the duration of the call
    b1a = None if b1 is None else _f32(b1)
    b2a = None if b2 is None else _f32(b2)
    out = np.full((V, H), np.nan)
    mag = np.full((V, H), np.nan)
    m = _mask(v_mask, V)
    _load().oracle_patch_merger(_p(x, ctypes.c_float), V, E, m2, _p(gm, ctypes.c_float), _p(bt, ctypes.c_float),
                                float(eps), _p(w1, ctypes.c_float), _p(b1a, ctypes.c_float), _p(w2, ctypes.c_float),
                                _p(b2a, ctypes.c_float), H, _p(m, ctypes.c_uint8), _p(out, ctypes.c_double),
                                _p(mag, ctypes.c_double))
    return out, mag


def conv3d_frames(frames, grid: Sequence[int], merge: int, mean, std, w, bias,
                  C: int, tp: int, p: int, row_mask=None) -> Tuple[np.ndarray, np.ndarray]:
    """Frames form for one item (frames [T,C,H,W]). Returns (out, absdot) [N,E] fp64."""
    return _frames(frames, grid, merge, mean, std, w, bias, C, tp, p, row_mask, True)


def _frames(frames, grid, merge, mean, std, w, bias, C, tp, p, row_mask, fill):
    """conv3d_frames; with fill=False the rows a row_mask leaves out are left
    unwritten (np.empty: pages that nothing touches cost nothing)."""
    f = _f32(frames)
    T, Cf, H, W = f.shape
    assert Cf == C
    w = _f32(w)
    E = int(w.shape[0])
    gt, gh, gw = (int(v) for v in grid)
    N = gt * gh * gw
    mu = _f32(np.asarray(mean, dtype=np.float32).reshape(C))
    sd = _f32(np.asarray(std, dtype=np.float32).reshape(C))
    b = None if bias is None else _f32(bias)
    make = (lambda shape: np.full(shape, np.nan)) if fill or row_mask is None else np.empty
    out = make((N, E))
    mag = make((N, E))
    m = _mask(row_mask, N)
    rc = _load().oracle_conv3d_frames(
        _p(f, ctypes.c_float), T, H, W, gt, gh, gw, merge, _p(mu, ctypes.c_float),
        _p(sd, ctypes.c_float), _p(w, ctypes.c_float), _p(b, ctypes.c_float), E, C, tp, p,
        _p(m, ctypes.c_uint8), _p(out, ctypes.c_double), _p(mag, ctypes.c_double))
    if rc != 0:
        raise ValueError("oracle_conv3d_frames: inconsistent sizes")
    return out, mag


def conv3d_grouped(items, merge: int, mean, std, w, bias, C: int, tp: int, p: int,
                   row_mask=None, compact: bool = False) -> Tuple[np.ndarray, np.ndarray]:
    """Grouped frames form: items' rows concatenated in list order.
    ``items`` is a sequence of (frames, grid).  With ``compact`` (and a
    row_mask) only the selected rows are returned, in row order, and items
    without a selected row are not computed at all; the arithmetic of every
    computed row is the same."""
    w = _f32(w)                                    # converted once for all items
    bias = None if bias is None else _f32(bias)
    mask = None if row_mask is None else np.asarray(row_mask, dtype=np.uint8)
    compact = compact and mask is not None
    outs, mags = [], []
    off = 0
    for frames, grid in items:
        n = int(grid[0]) * int(grid[1]) * int(grid[2])
        sub = None if mask is None else mask[off:off + n]
        off += n
        if compact and not sub.any():
            continue
        o, m = _frames(frames, grid, merge, mean, std, w, bias, C, tp, p, sub, not compact)
        if compact:
            sel = np.flatnonzero(sub)
            o, m = o[sel], m[sel]
        outs.append(o)
        mags.append(m)
    if not outs:
        E = int(w.shape[0])
        return np.empty((0, E)), np.empty((0, E))
    return np.concatenate(outs, 0), np.concatenate(mags, 0)


def patchify(frames, grid: Sequence[int], merge: int, mean, std, C: int, tp: int, p: int
             ) -> np.ndarray:
    """Normalised patch rows [N, K] fp32 (bf16-valued) in output-row order."""
    f = _f32(frames)
    T, Cf, H, W = f.shape
    assert Cf == C
    gt, gh, gw = (int(v) for v in grid)
    K = C * tp * p * p
    mu = _f32(np.asarray(mean, dtype=np.float32).reshape(C))
    sd = _f32(np.asarray(std, dtype=np.float32).reshape(C))
    rows = np.empty((gt * gh * gw, K), dtype=np.float32)
    rc = _load().oracle_patchify(_p(f, ctypes.c_float), T, H, W, gt, gh, gw, merge,
                                 _p(mu, ctypes.c_float), _p(sd, ctypes.c_float), C, tp, p,
                                 _p(rows, ctypes.c_float))
    if rc != 0:
        raise ValueError("oracle_patchify: inconsistent sizes")
    return rows
