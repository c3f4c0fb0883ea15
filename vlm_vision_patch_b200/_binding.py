"""ctypes binding of libpe.so: argument marshalling only.

Every function here has the name and argument order of the C entry point it
wraps (include/pe.h).  Tensors are passed as raw device pointers; streams as
the raw CUDA stream handle.  There is no fallback: if libpe.so is missing or a
call fails, an exception is raised.
"""
from __future__ import annotations

import array
import ctypes
import operator
import os
from typing import Optional, Sequence

HERE = os.path.dirname(os.path.abspath(__file__))
# PE_LIB selects another build of the same library (the bounds-checking
# libpe_debug.so); by default the in-tree libpe.so
LIB_PATH = os.environ.get("PE_LIB") or os.path.join(HERE, "libpe.so")

PE_F32, PE_BF16 = 0, 1
STATUS = {
    0: "PE_OK", 1: "PE_ERR_INVALID_ARG", 2: "PE_ERR_SHAPE", 3: "PE_ERR_DTYPE",
    4: "PE_ERR_ALIGN", 5: "PE_ERR_NO_WEIGHT", 6: "PE_ERR_CUDA", 7: "PE_ERR_UNSUPPORTED",
    8: "PE_ERR_DEVICE_TIMEOUT", 9: "PE_ERR_HOST_MEMORY", 10: "PE_ERR_DEVICE_BOUNDS",
}
PE_INLINE_ITEMS = 16
PE_MAX_PATCH = 32
PE_NOALLOC_MAX_ITEMS = 1024

# Every symbol include/pe.h declares.
EXPORTS = (
    "pe_create", "pe_set_weight", "pe_set_norm", "pe_forward_patches", "pe_forward_frames",
    "pe_forward_frames_grouped", "pe_forward_frames_grouped_noalloc", "pe_patchify", "pe_num_patches", "pe_last_error",
    "pe_status_string", "pe_destroy", "pe_device", "pe_profile_begin", "pe_profile_end",
    "pe_set_temporal_fold", "pe_forward_patches_pos", "pe_forward_frames_grouped_pos", "pe_set_tf32",
    "pe_merger_create", "pe_merger_set_weights", "pe_merger_forward", "pe_merger_last_error", "pe_merger_destroy",
    "pe_merger_profile_begin", "pe_merger_profile_end", "pe_forward_frames_grouped_host", "pe_forward_patches_host",
    "pe_selftest_wait_timeout", "pe_profile_target",
)


class PEError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        self.status = STATUS.get(code, str(code))
        super().__init__(f"{fn} failed: {self.status} ({status_string(code)})")


_lib = None


def load(path: Optional[str] = None) -> ctypes.CDLL:
    """Load libpe.so (build it first with vlm_vision_patch_b200.build)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"libpe.so not found at {p}: build it with "
                           "`python -m vlm_vision_patch_b200.build` (no CPU fallback exists)")
    lib = ctypes.CDLL(p)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    i32p = ctypes.POINTER(ctypes.c_int32)
    f32p = ctypes.POINTER(ctypes.c_float)
    sig = {
        "pe_create": ([i32, i32, i32, i32, i32, ctypes.POINTER(vp)], i32),
        "pe_set_weight": ([vp, vp, i32, vp, i32, vp], i32),
        "pe_set_norm": ([vp, f32p, f32p], i32),
        "pe_set_temporal_fold": ([vp, i32], i32),
        "pe_set_tf32": ([vp, i32], i32),
        "pe_merger_create": ([i32, i32, i32, ctypes.c_float, ctypes.POINTER(vp)], i32),
        "pe_merger_set_weights": ([vp, vp, vp, vp, vp, vp, vp, i32, vp], i32),
        "pe_merger_forward": ([vp, vp, i64, vp, i32, vp], i32),
        "pe_merger_last_error": ([vp], i32),
        "pe_merger_destroy": ([vp], None),
        "pe_merger_profile_begin": ([vp, i32], i32),
        "pe_merger_profile_end": ([vp, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(i32),
                                   ctypes.POINTER(ctypes.c_int64)], i32),
        "pe_forward_patches": ([vp, vp, i32, i64, vp, i32, vp], i32),
        "pe_forward_patches_pos": ([vp, vp, i32, i64, vp, i32, vp, i32, vp], i32),
        "pe_forward_frames_grouped_pos": ([vp, i32, ctypes.POINTER(vp), i32, i32p, i32p, i32, vp, i32, vp, i32, vp],
                                          i32),
        "pe_forward_frames": ([vp, vp, i32, i32, i32, i32, i32p, i32, vp, i32, vp], i32),
        "pe_forward_frames_grouped": ([vp, i32, ctypes.POINTER(vp), i32, i32p, i32p, i32, vp, i32, vp], i32),
        "pe_forward_frames_grouped_noalloc": ([vp, i32, ctypes.POINTER(vp), i32, i32p, i32p, i32, vp, i32, vp], i32),
        "pe_patchify": ([vp, i32, ctypes.POINTER(vp), i32, i32p, i32p, i32, vp, i32, vp], i32),
        "pe_forward_frames_grouped_host": ([vp, i32, ctypes.POINTER(vp), i32, i32p, i32p, i32, vp, i32, vp], i32),
        "pe_forward_patches_host": ([vp, vp, i32, i64, vp, i32, vp], i32),
        "pe_num_patches": ([i32p, i32], i64),
        "pe_last_error": ([vp], i32),
        "pe_selftest_wait_timeout": ([vp, vp], i32),
        "pe_status_string": ([i32], ctypes.c_char_p),
        "pe_destroy": ([vp], None),
        "pe_device": ([vp], i32),
        "pe_profile_begin": ([vp, i32], i32),
        "pe_profile_target": ([vp, i32], i32),
        "pe_profile_end": ([vp, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(i32),
                            ctypes.POINTER(ctypes.c_int64)], i32),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    if path is None:
        _lib = lib
    return lib


def _check(fn: str, code: int) -> None:
    if code != 0:
        raise PEError(fn, code)


assert array.array("i").itemsize == 4 and array.array("Q").itemsize == 8


def _i32arr(vals: Sequence[int]):
    # array.array fills the buffer in C: several times faster than building
    # the ctypes array element by element; the ctypes view keeps it alive
    a = array.array("i", vals)
    return (ctypes.c_int32 * len(a)).from_buffer(a)


def _i32rows(rows) -> "ctypes.Array":
    """int32 array of [n, 3] values given as n triples or already flat."""
    if len(rows):
        try:
            operator.index(rows[0])          # an integer: already flat
        except TypeError:
            rows = [v for r in rows for v in r]
    return _i32arr(rows)


def _f32arr(vals: Sequence[float]):
    return (ctypes.c_float * len(vals))(*[float(v) for v in vals])


def _ptrs(ptrs: Sequence[int]):
    a = array.array("Q", ptrs)
    return (ctypes.c_void_p * len(a)).from_buffer(a)


# ----------------------------------------------------------- raw entry points

def status_string(code: int) -> str:
    return load().pe_status_string(int(code)).decode()


def pe_create(E: int, C: int, tp: int, p: int, has_bias: bool) -> int:
    h = ctypes.c_void_p()
    _check("pe_create", load().pe_create(E, C, tp, p, int(bool(has_bias)), ctypes.byref(h)))
    return h.value


def pe_destroy(h: int) -> None:
    load().pe_destroy(h)


def pe_device(h: int) -> int:
    return int(load().pe_device(h))


def pe_set_weight(h: int, w_ptr: int, w_dt: int, bias_ptr: Optional[int], b_dt: int, stream: int) -> None:
    _check("pe_set_weight", load().pe_set_weight(h, w_ptr, w_dt, bias_ptr, b_dt, stream))


def pe_set_norm(h: int, mean: Sequence[float], std: Sequence[float]) -> None:
    _check("pe_set_norm", load().pe_set_norm(h, _f32arr(mean), _f32arr(std)))


def pe_set_temporal_fold(h: int, enable: bool) -> None:
    _check("pe_set_temporal_fold", load().pe_set_temporal_fold(h, int(bool(enable))))


def pe_set_tf32(h: int, enable: bool) -> None:
    _check("pe_set_tf32", load().pe_set_tf32(h, int(bool(enable))))


def pe_forward_patches(h: int, x_ptr: int, x_dt: int, N: int, out_ptr: int, out_dt: int, stream: int) -> None:
    _check("pe_forward_patches", load().pe_forward_patches(h, x_ptr, x_dt, N, out_ptr, out_dt, stream))


def pe_forward_patches_pos(h: int, x_ptr: int, x_dt: int, N: int, pos_ptr: int, pos_dt: int, out_ptr: int,
                           out_dt: int, stream: int) -> None:
    _check("pe_forward_patches_pos",
           load().pe_forward_patches_pos(h, x_ptr, x_dt, N, pos_ptr, pos_dt, out_ptr, out_dt, stream))


def pe_forward_frames_grouped_pos(h: int, f_ptrs: Sequence[int], f_dt: int, THW: Sequence[Sequence[int]],
                                  grid_thw: Sequence[Sequence[int]], merge: int, pos_ptr: int, pos_dt: int,
                                  out_ptr: int, out_dt: int, stream: int) -> None:
    n = len(f_ptrs)
    _check("pe_forward_frames_grouped_pos", load().pe_forward_frames_grouped_pos(
        h, n, _ptrs(f_ptrs), f_dt, _i32rows(THW),
        _i32rows(grid_thw), merge, pos_ptr, pos_dt, out_ptr, out_dt, stream))


def pe_forward_frames(h: int, f_ptr: int, f_dt: int, T: int, H: int, W: int, grid_thw: Sequence[int],
                      merge: int, out_ptr: int, out_dt: int, stream: int) -> None:
    _check("pe_forward_frames", load().pe_forward_frames(h, f_ptr, f_dt, T, H, W, _i32arr(grid_thw), merge,
                                                          out_ptr, out_dt, stream))


def pe_forward_frames_grouped(h: int, f_ptrs: Sequence[int], f_dt: int, THW: Sequence[Sequence[int]],
                              grid_thw: Sequence[Sequence[int]], merge: int, out_ptr: int, out_dt: int,
                              stream: int) -> None:
    n = len(f_ptrs)
    _check("pe_forward_frames_grouped", load().pe_forward_frames_grouped(
        h, n, _ptrs(f_ptrs), f_dt, _i32rows(THW),
        _i32rows(grid_thw), merge, out_ptr, out_dt, stream))


def pe_forward_frames_grouped_noalloc(h: int, f_ptrs: Sequence[int], f_dt: int, THW: Sequence[Sequence[int]],
                                      grid_thw: Sequence[Sequence[int]], merge: int, out_ptr: int, out_dt: int,
                                      stream: int) -> None:
    n = len(f_ptrs)
    _check("pe_forward_frames_grouped_noalloc", load().pe_forward_frames_grouped_noalloc(
        h, n, _ptrs(f_ptrs), f_dt, _i32rows(THW),
        _i32rows(grid_thw), merge, out_ptr, out_dt, stream))


def pe_forward_frames_grouped_host(h: int, f_ptrs: Sequence[int], f_dt: int, THW: Sequence[Sequence[int]],
                                   grid_thw: Sequence[Sequence[int]], merge: int, out_ptr: int, out_dt: int,
                                   stream: int) -> None:
    """Host pointers in and out (see include/pe.h)."""
    n = len(f_ptrs)
    _check("pe_forward_frames_grouped_host", load().pe_forward_frames_grouped_host(
        h, n, _ptrs(f_ptrs), f_dt, _i32rows(THW),
        _i32rows(grid_thw), merge, out_ptr, out_dt, stream))


def pe_forward_patches_host(h: int, x_ptr: int, x_dt: int, N: int, out_ptr: int, out_dt: int, stream: int) -> None:
    _check("pe_forward_patches_host", load().pe_forward_patches_host(h, x_ptr, x_dt, N, out_ptr, out_dt, stream))


def pe_patchify(h: int, f_ptrs: Sequence[int], f_dt: int, THW: Sequence[Sequence[int]],
                grid_thw: Sequence[Sequence[int]], merge: int, rows_ptr: int, rows_dt: int,
                stream: int) -> None:
    n = len(f_ptrs)
    _check("pe_patchify", load().pe_patchify(
        h, n, _ptrs(f_ptrs), f_dt, _i32rows(THW),
        _i32rows(grid_thw), merge, rows_ptr, rows_dt, stream))


def pe_num_patches(grid_thw: Sequence[Sequence[int]]) -> int:
    flat = [v for g in grid_thw for v in g]
    return int(load().pe_num_patches(_i32arr(flat) if flat else None, len(grid_thw)))


def pe_profile_begin(h: int, max_calls: int) -> None:
    _check("pe_profile_begin", load().pe_profile_begin(h, max_calls))


def pe_profile_target(h: int, target: int) -> None:
    """0: profile the contraction kernel (default); 1: the kernel before it."""
    _check("pe_profile_target", load().pe_profile_target(h, target))


def pe_profile_end(h: int, max_calls: int):
    """Returns (per-call contraction-kernel ms, kernels launched in the window)."""
    ms = (ctypes.c_float * max(1, max_calls))()
    n = ctypes.c_int(max_calls)
    launches = ctypes.c_int64(0)
    _check("pe_profile_end", load().pe_profile_end(h, ms, ctypes.byref(n), ctypes.byref(launches)))
    return [float(ms[i]) for i in range(n.value)], int(launches.value)


def pe_merger_create(E: int, m: int, H: int, eps: float) -> int:
    h = ctypes.c_void_p()
    _check("pe_merger_create", load().pe_merger_create(E, m, H, eps, ctypes.byref(h)))
    return h.value


def pe_merger_set_weights(pm: int, gamma: int, beta: int, w1: int, b1: Optional[int], w2: int, b2: Optional[int],
                          dt: int, stream: int) -> None:
    _check("pe_merger_set_weights", load().pe_merger_set_weights(pm, gamma, beta, w1, b1, w2, b2, dt, stream))


def pe_merger_forward(pm: int, x_ptr: int, N: int, out_ptr: int, out_dt: int, stream: int) -> None:
    _check("pe_merger_forward", load().pe_merger_forward(pm, x_ptr, N, out_ptr, out_dt, stream))


def pe_merger_profile_begin(pm: int, max_calls: int) -> None:
    _check("pe_merger_profile_begin", load().pe_merger_profile_begin(pm, max_calls))


def pe_merger_profile_end(pm: int, max_calls: int):
    """Returns (per-linear-layer ms, alternating fc1/fc2; kernels launched)."""
    ms = (ctypes.c_float * max(1, max_calls))()
    n = ctypes.c_int(max_calls)
    launches = ctypes.c_int64(0)
    _check("pe_merger_profile_end", load().pe_merger_profile_end(pm, ms, ctypes.byref(n), ctypes.byref(launches)))
    return [float(ms[i]) for i in range(n.value)], int(launches.value)


def pe_merger_last_error(pm: int) -> int:
    return int(load().pe_merger_last_error(pm))


def pe_merger_destroy(pm: int) -> None:
    load().pe_merger_destroy(pm)


def pe_selftest_wait_timeout(h: int, stream: int) -> None:
    _check("pe_selftest_wait_timeout", load().pe_selftest_wait_timeout(h, stream))


def pe_last_error(h: int) -> int:
    return int(load().pe_last_error(h))
