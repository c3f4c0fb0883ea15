"""B200-native vision PatchEmbed (Qwen2-VL / Qwen2.5-VL) over the libpe.so C ABI.

``PatchEmbed`` is a convenience wrapper holding one ``pe_handle``; every method
forwards to the same-named C entry point (``_binding``) with torch tensors
turned into raw device pointers and the current CUDA stream.  PyTorch only
provides device memory and streams here; all arithmetic runs in libpe.so.
"""
from __future__ import annotations

from typing import Optional, Sequence

import torch

from . import _binding as B
from ._binding import PE_BF16, PE_F32, PEError, load  # noqa: F401

__all__ = ["PatchEmbed", "PatchMerger", "PEError", "PE_F32", "PE_BF16", "load", "num_patches"]


def _dt(t: torch.dtype) -> int:
    if t == torch.float32:
        return PE_F32
    if t == torch.bfloat16:
        return PE_BF16
    raise TypeError(f"unsupported dtype {t}; use torch.float32 or torch.bfloat16")


def _dev(t: torch.Tensor, name: str, device: Optional[int] = None) -> int:
    d = t.get_device()            # -1 for a host tensor
    if d < 0:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and d != device:
        raise ValueError(f"{name} is on cuda:{d}, the handle on cuda:{device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _host(t: torch.Tensor, name: str) -> int:
    if t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _host_out(shape, out, out_dtype) -> torch.Tensor:
    if out is None:
        out = torch.empty(shape, dtype=out_dtype, pin_memory=torch.cuda.is_available())
    _need(out, shape, "out")
    return out


def _need(t: torch.Tensor, shape: Sequence[int], name: str) -> None:
    """The C ABI takes raw pointers and trusts the documented layout, so a tensor
    of the wrong shape would be read or written past its end: refuse it here."""
    if tuple(t.shape) != tuple(int(v) for v in shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}; expected {tuple(int(v) for v in shape)}")


def _need_frames(frames: Sequence[torch.Tensor], C: int) -> None:
    for f in frames:
        if f.dim() != 4 or f.shape[1] != C:
            raise ValueError(f"frames must be [T, {C}, H, W]; got {tuple(f.shape)}")


# the current stream's raw handle without building a Stream object (a few
# microseconds per call otherwise); the public route where torch lacks it
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream) -> int:
    if stream is None:
        if _raw_stream is not None:
            return int(_raw_stream(torch.cuda.current_device()))
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _sync(stream) -> None:
    """Wait for `stream` (None: the current stream; a raw handle: the device)."""
    if stream is None:
        torch.cuda.current_stream().synchronize()
    elif isinstance(stream, torch.cuda.Stream):
        stream.synchronize()
    else:
        torch.cuda.synchronize()


def num_patches(grid_thw: Sequence[Sequence[int]]) -> int:
    return B.pe_num_patches(grid_thw)


class PatchEmbed:
    """Conv3d(C, E, kernel=stride=(tp, p, p)) on sm_100a kernels (C ABI in include/pe.h)."""

    def __init__(self, E: int, C: int = 3, tp: int = 2, p: int = 14, bias: bool = False):
        self.E, self.C, self.tp, self.p, self.has_bias = E, C, tp, p, bias
        self.K = C * tp * p * p
        self.h = B.pe_create(E, C, tp, p, bias)
        self.dev = B.pe_device(self.h)

    # ------------------------------------------------------------ lifetime
    def close(self) -> None:
        if getattr(self, "h", None):
            B.pe_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ------------------------------------------------------------ state
    def set_weight(self, w: torch.Tensor, bias: Optional[torch.Tensor] = None, stream=None) -> None:
        """w: [E, C, tp, p, p] (or [E, K] flattened in that order); bias: [E]."""
        if w.shape[:1] != (self.E,) or w.numel() != self.E * self.K:
            raise ValueError(f"weight has shape {tuple(w.shape)}; expected "
                             f"{(self.E, self.C, self.tp, self.p, self.p)}")
        if bias is not None and bias.numel() != self.E:
            raise ValueError(f"bias has shape {tuple(bias.shape)}; expected {(self.E,)}")
        B.pe_set_weight(self.h, _dev(w, "weight", self.dev), _dt(w.dtype),
                        None if bias is None else _dev(bias, "bias", self.dev),
                        _dt(bias.dtype) if bias is not None else PE_F32, _stream(stream))

    def set_norm(self, mean: Sequence[float], std: Sequence[float]) -> None:
        B.pe_set_norm(self.h, mean, std)

    def set_tf32(self, enable: bool) -> None:
        """Opt-in: fp32 patch rows are contracted in tf32 (rows and weight rounded
        to tf32, fp32 accumulation) instead of bf16."""
        B.pe_set_tf32(self.h, enable)

    def set_temporal_fold(self, enable: bool) -> None:
        """Opt-in: single-frame items use the summed temporal slices of the weight
        (half the contraction; one more bf16 rounding per weight term)."""
        B.pe_set_temporal_fold(self.h, enable)

    def last_error(self) -> int:
        return B.pe_last_error(self.h)

    # ------------------------------------------------------------ forward
    def _out(self, n: int, out, out_dtype, device):
        if out is None:
            out = torch.empty((n, self.E), dtype=out_dtype, device=device)
        _need(out, (n, self.E), "out")
        return out

    def forward_patches(self, x: torch.Tensor, out: Optional[torch.Tensor] = None,
                        out_dtype: torch.dtype = torch.bfloat16, stream=None,
                        pos: Optional[torch.Tensor] = None) -> torch.Tensor:
        """out = x @ W^T (+ bias) (+ pos, a [N, E] table added in the same epilogue)."""
        if x.dim() != 2 or x.shape[1] != self.K:
            raise ValueError(f"x must be [N, {self.K}]; got {tuple(x.shape)}")
        out = self._out(x.shape[0], out, out_dtype, x.device)
        if pos is not None:
            _need(pos, (x.shape[0], self.E), "pos")
        d = self.dev
        if pos is None:
            B.pe_forward_patches(self.h, _dev(x, "x", d), _dt(x.dtype), x.shape[0], _dev(out, "out", d),
                                 _dt(out.dtype), _stream(stream))
        else:
            B.pe_forward_patches_pos(self.h, _dev(x, "x", d), _dt(x.dtype), x.shape[0], _dev(pos, "pos", d),
                                     _dt(pos.dtype), _dev(out, "out", d), _dt(out.dtype), _stream(stream))
        return out

    def forward_frames(self, frames: torch.Tensor, grid_thw: Sequence[int], merge: int = 2,
                       out: Optional[torch.Tensor] = None, out_dtype: torch.dtype = torch.bfloat16,
                       stream=None) -> torch.Tensor:
        _need_frames([frames], self.C)
        if len(grid_thw) != 3:
            raise ValueError("grid_thw must be (t, h, w)")
        T, C, H, W = frames.shape
        n = int(grid_thw[0]) * int(grid_thw[1]) * int(grid_thw[2])
        out = self._out(n, out, out_dtype, frames.device)
        B.pe_forward_frames(self.h, _dev(frames, "frames", self.dev), _dt(frames.dtype), T, H, W, grid_thw, merge,
                            _dev(out, "out", self.dev), _dt(out.dtype), _stream(stream))
        return out

    def _items(self, frames, grid_thw):
        """One pass over the items: the grids, layouts and dtypes checked, and the
        frame sizes (T, H, W) and grids flattened for the C call.  Returns
        (patch count, flat THW, flat grids, frames dtype)."""
        if len(frames) == 0 or len(frames) != len(grid_thw):
            raise ValueError(f"{len(frames)} frame tensors for {len(grid_thw)} grids; need one per item, at least one")
        C = self.C
        thw, grids, n, dt = [], [], 0, None
        for f, g in zip(frames, grid_thw):
            if len(g) != 3:
                raise ValueError("every grid_thw entry must be (t, h, w)")
            s = f.shape
            if len(s) != 4 or s[1] != C:
                raise ValueError(f"frames must be [T, {C}, H, W]; got {tuple(s)}")
            if dt is None:
                dt = f.dtype
            elif f.dtype != dt:
                raise TypeError("all items must share one dtype")
            t, h, w = int(g[0]), int(g[1]), int(g[2])
            grids += (t, h, w)
            thw += (s[0], s[2], s[3])
            n += t * h * w
        return n, thw, grids, dt

    def forward_frames_grouped(self, frames: Sequence[torch.Tensor], grid_thw: Sequence[Sequence[int]],
                               merge: int = 2, out: Optional[torch.Tensor] = None,
                               out_dtype: torch.dtype = torch.bfloat16, stream=None,
                               pos: Optional[torch.Tensor] = None) -> torch.Tensor:
        """All items in one launch; `pos`, if given, is a [N, E] table in output row
        order added in the same epilogue."""
        n, thw, grids, fdt = self._items(frames, grid_thw)
        out = self._out(n, out, out_dtype, frames[0].device)
        if pos is not None:
            _need(pos, (n, self.E), "pos")
        d = self.dev
        ptrs = [_dev(f, "frames", d) for f in frames]
        if pos is None:
            B.pe_forward_frames_grouped(self.h, ptrs, _dt(fdt), thw, grids, merge,
                                        _dev(out, "out", d), _dt(out.dtype), _stream(stream))
        else:
            B.pe_forward_frames_grouped_pos(self.h, ptrs, _dt(fdt), thw, grids, merge,
                                            _dev(pos, "pos", d), _dt(pos.dtype), _dev(out, "out", d),
                                            _dt(out.dtype), _stream(stream))
        return out

    def forward_frames_grouped_host(self, frames: Sequence[torch.Tensor], grid_thw: Sequence[Sequence[int]],
                                    merge: int = 2, out: Optional[torch.Tensor] = None,
                                    out_dtype: torch.dtype = torch.bfloat16, stream=None,
                                    blocking: bool = True) -> torch.Tensor:
        """forward_frames_grouped with host (CPU) frames and a host output: the
        library copies the frames in and the rows out in pipelined chunks.  Pinned
        tensors (``pin_memory()``) overlap the copies; the default output is
        pinned.  With ``blocking=False`` the output is complete only once the
        stream has drained."""
        n, thw, grids, fdt = self._items(frames, grid_thw)
        out = _host_out((n, self.E), out, out_dtype)
        ptrs = [_host(f, "frames") for f in frames]
        st = _stream(stream)
        B.pe_forward_frames_grouped_host(self.h, ptrs, _dt(fdt), thw, grids, merge,
                                         _host(out, "out"), _dt(out.dtype), st)
        if blocking:
            _sync(stream)
        return out

    def forward_patches_host(self, x: torch.Tensor, out: Optional[torch.Tensor] = None,
                             out_dtype: torch.dtype = torch.bfloat16, stream=None,
                             blocking: bool = True) -> torch.Tensor:
        """forward_patches with host (CPU) rows in and out, pipelined in chunks
        (see forward_frames_grouped_host)."""
        if x.dim() != 2 or x.shape[1] != self.K:
            raise ValueError(f"x must be [N, {self.K}]; got {tuple(x.shape)}")
        out = _host_out((x.shape[0], self.E), out, out_dtype)
        st = _stream(stream)
        B.pe_forward_patches_host(self.h, _host(x, "x"), _dt(x.dtype), x.shape[0], _host(out, "out"),
                                  _dt(out.dtype), st)
        if blocking:
            _sync(stream)
        return out

    def patchify(self, frames: Sequence[torch.Tensor], grid_thw: Sequence[Sequence[int]], merge: int = 2,
                 rows_dtype: torch.dtype = torch.bfloat16, stream=None) -> torch.Tensor:
        n, thw, grids, fdt = self._items(frames, grid_thw)
        rows = torch.empty((n, self.K), dtype=rows_dtype, device=frames[0].device)
        B.pe_patchify(self.h, [_dev(f, "frames", self.dev) for f in frames], _dt(fdt), thw, grids, merge,
                      _dev(rows, "rows"), _dt(rows.dtype), _stream(stream))
        return rows


class PatchMerger:
    """LayerNorm -> concat of the m*m rows of each merge window -> GELU MLP
    D -> D -> H on rows in merge order (the PatchEmbed output).  Thin wrapper
    over the pe_merger_* C calls."""

    def __init__(self, E: int, m: int, H: int, eps: float = 1e-6):
        self.E, self.m2, self.H = E, m * m, H
        self.D = E * m * m
        self.h = B.pe_merger_create(E, m, H, eps)
        self.dev = torch.cuda.current_device()   # the device pe_merger_create bound the handle to

    def set_weights(self, gamma: torch.Tensor, beta: torch.Tensor, w1: torch.Tensor, b1: Optional[torch.Tensor],
                    w2: torch.Tensor, b2: Optional[torch.Tensor], stream=None) -> None:
        """gamma, beta: [E]; w1: [D, D], b1: [D]; w2: [H, D], b2: [H] (D = m*m*E)."""
        E, D, H = self.E, self.D, self.H
        for t, shape, name in ((gamma, (E,), "gamma"), (beta, (E,), "beta"), (w1, (D, D), "w1"),
                               (b1, (D,), "b1"), (w2, (H, D), "w2"), (b2, (H,), "b2")):
            if t is not None:
                _need(t, shape, name)
        ts = [gamma, beta, w1, w2] + [t for t in (b1, b2) if t is not None]
        if len({t.dtype for t in ts}) != 1:
            raise TypeError("all merger weights must share one dtype")
        self._keep = ts
        d = self.dev
        B.pe_merger_set_weights(self.h, _dev(gamma, "gamma", d), _dev(beta, "beta", d), _dev(w1, "w1", d),
                                None if b1 is None else _dev(b1, "b1", d), _dev(w2, "w2", d),
                                None if b2 is None else _dev(b2, "b2", d), _dt(w1.dtype), _stream(stream))

    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None, out_dtype: torch.dtype = torch.bfloat16,
                stream=None) -> torch.Tensor:
        if x.dim() != 2 or x.shape[1] != self.E:
            raise ValueError(f"x must be [N, {self.E}]; got {tuple(x.shape)}")
        V = x.shape[0] // self.m2
        if out is None:
            out = torch.empty((V, self.H), dtype=out_dtype, device=x.device)
        _need(out, (V, self.H), "out")
        B.pe_merger_forward(self.h, _dev(x, "x", self.dev), x.shape[0], _dev(out, "out", self.dev), _dt(out.dtype),
                            _stream(stream))
        return out

    def last_error(self) -> int:
        return B.pe_merger_last_error(self.h)

    def close(self) -> None:
        if getattr(self, "h", None):
            B.pe_merger_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

