"""The allocation-free grouped call, against the CPU oracle.

pe_forward_frames_grouped_noalloc exists for callers that cannot allocate
device memory while serving: their memory is all handed to their own pool up
front, and cudaMalloc would also synchronise the device.  It keeps its item
table in a fixed array of the library's static device memory instead of the
handle's workspace, and fills it with small kernels whose launch parameters
carry the descriptors.  Checked here, through the C ABI:
  - the output against the oracle at the parity tolerance of the other GPU
    tests, twice in a row with different item lists (the shared table is
    overwritten in between), and against the plain grouped call;
  - a first call on a fresh handle leaves the device's free memory unchanged;
  - a group small enough to pass its items inside the launch (no table);
  - more items than the table holds is refused before anything runs.
The file sits last in collection order and passes both on its own in a fresh
process and after the rest.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from vlm_vision_patch_b200 import PatchEmbed, _binding as B
from tests.gpu_util import assert_within_tolerance

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
C, TP, P, E = 3, 2, 14, 256


def _items(seed, n):
    rng = np.random.default_rng(seed)
    grids = [(1, int(2 * rng.integers(1, 4)), int(2 * rng.integers(1, 5))) for _ in range(n)]
    frames = [workloads.uniform01((1, C, g[1] * P, g[2] * P), seed * 1000 + i) for i, g in enumerate(grids)]
    return frames, grids


def _weight(seed=5):
    return workloads.normal((E, C, TP, P, P), seed, std=0.02, dtype=torch.bfloat16)


def _handle(w):
    pe = PatchEmbed(E, C, TP, P, False)
    pe.set_weight(w.to(DEV))
    pe.set_norm(workloads.CLIP_MEAN, workloads.CLIP_STD)
    return pe


def _call(fn, pe, frames_dev, grids, out):
    getattr(B, fn)(pe.h, [f.data_ptr() for f in frames_dev], B.PE_BF16,
                   [(f.shape[0], f.shape[2], f.shape[3]) for f in frames_dev], grids, 2, out.data_ptr(), B.PE_BF16,
                   torch.cuda.current_stream().cuda_stream)


def _oracle(frames, grids, w):
    return oracle.conv3d_grouped(list(zip(frames, grids)), 2, workloads.CLIP_MEAN, workloads.CLIP_STD, w, None,
                                 C, TP, P)


def test_noalloc_matches_oracle_twice_in_a_row():
    w = _weight()
    pe = _handle(w)
    for seed, n in ((1, 40), (2, 23)):          # both above the inline-item limit: the static table
        frames, grids = _items(seed, n)
        fd = [f.to(DEV) for f in frames]
        N = sum(g[0] * g[1] * g[2] for g in grids)
        plain = torch.empty(N, E, dtype=torch.bfloat16, device=DEV)
        new_out = torch.full((N, E), float("nan"), dtype=torch.bfloat16, device=DEV)
        _call("pe_forward_frames_grouped", pe, fd, grids, plain)
        _call("pe_forward_frames_grouped_noalloc", pe, fd, grids, new_out)
        torch.cuda.synchronize()
        assert pe.last_error() == 0
        ref, mag = _oracle(frames, grids, w)
        assert_within_tolerance(new_out, ref, mag, what=f"noalloc n={n} vs oracle")
        assert_within_tolerance(new_out, plain.double().cpu().numpy(), mag, what=f"noalloc n={n} vs grouped")


def test_noalloc_first_call_on_a_fresh_handle_allocates_nothing():
    w = _weight(7)
    frames, grids = _items(3, 40)
    fd = [f.to(DEV) for f in frames]
    N = sum(g[0] * g[1] * g[2] for g in grids)
    out = torch.full((N, E), float("nan"), dtype=torch.bfloat16, device=DEV)
    # load the kernels the call launches (a first launch may map code) on another handle
    warm = _handle(w)
    _call("pe_forward_frames_grouped_noalloc", warm, fd, grids, out)
    torch.cuda.synchronize()
    pe = _handle(w)                              # a fresh handle: its own buffers are allocated here
    out.fill_(float("nan"))
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    _call("pe_forward_frames_grouped_noalloc", pe, fd, grids, out)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, f"device free memory changed by {free0 - free1} bytes"
    assert pe.last_error() == 0
    ref, mag = _oracle(frames, grids, w)
    assert_within_tolerance(out, ref, mag, what="noalloc first call on a fresh handle")


def test_noalloc_inline_items():
    w = _weight(9)
    pe = _handle(w)
    frames, grids = _items(4, 11)               # at most PE_INLINE_ITEMS: no table at all
    fd = [f.to(DEV) for f in frames]
    N = sum(g[0] * g[1] * g[2] for g in grids)
    out = torch.full((N, E), float("nan"), dtype=torch.bfloat16, device=DEV)
    _call("pe_forward_frames_grouped_noalloc", pe, fd, grids, out)
    torch.cuda.synchronize()
    assert pe.last_error() == 0
    ref, mag = _oracle(frames, grids, w)
    assert_within_tolerance(out, ref, mag, what="noalloc inline items")


def test_noalloc_rejects_too_many_items():
    pe = _handle(_weight(6))
    f = torch.zeros(1, C, 2 * P, 2 * P, dtype=torch.bfloat16, device=DEV)
    n = B.PE_NOALLOC_MAX_ITEMS + 1
    out = torch.empty(4 * n, E, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(B.PEError) as e:
        _call("pe_forward_frames_grouped_noalloc", pe, [f] * n, [(1, 2, 2)] * n, out)
    assert e.value.status == "PE_ERR_UNSUPPORTED"
