"""Shapes at the edges the C ABI accepts, against the CPU oracle.

pe_create takes E up to 65535 (E % 8 == 0), C up to 4 and p up to
PE_MAX_PATCH = 32, so K = C*tp*p*p reaches 8192.  These cases run the
largest of each through the paths that take them:
  - patch rows with K = 8192 (C = 4, tp = 2, p = 32): 64 weight stages per tile;
  - E = 65528, the largest accepted hidden size: 256 weight tiles per M-block;
  - frames with p = 32 (the fused frames kernel: 64 KB A stages), video and a
    single image, merge 2 and raster order.
Same tolerance as the other parity tests.
"""
import pytest
import torch

import oracle
import workloads
from vlm_vision_patch_b200 import PatchEmbed
from tests.gpu_util import assert_within_tolerance

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _pe(E, C, tp, p, w, b):
    pe = PatchEmbed(E, C, tp, p, b is not None)
    pe.set_weight(w.to(DEV), None if b is None else b.to(DEV))
    return pe


@pytest.mark.parametrize("C,tp,p,E,N,x_dtype,out_dtype", [
    (4, 2, 32, 256, 300, torch.bfloat16, torch.float32),     # K = 8192
    (4, 2, 32, 128, 70, torch.float32, torch.bfloat16),      # K = 8192, fp32 rows (cast, then TMA)
    (3, 2, 2, 65528, 300, torch.bfloat16, torch.bfloat16),   # E = 65528
])
def test_patches_at_abi_limits(C, tp, p, E, N, x_dtype, out_dtype):
    K = C * tp * p * p
    x = workloads.normal((N, K), 900 + p, dtype=x_dtype)
    w = workloads.normal((E, C, tp, p, p), 901 + p, std=0.02, dtype=torch.bfloat16)
    b = workloads.normal((E,), 902, std=0.02, dtype=torch.bfloat16)
    pe = _pe(E, C, tp, p, w, b)
    out = pe.forward_patches(x.to(DEV), out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert pe.last_error() == 0
    ref, mag = oracle.conv3d_patches(x, w, b, C, tp, p)
    assert_within_tolerance(out, ref, mag, what=f"patches K={K} E={E}")


@pytest.mark.parametrize("T,gh,gw,merge,E", [
    (3, 2, 4, 2, 128),     # video, odd T (last frame repeated)
    (1, 4, 2, 2, 96),      # one image
    (2, 3, 5, 1, 64),      # raster order, odd grid
])
def test_frames_p32(T, gh, gw, merge, E):
    C, tp, p = 3, 2, 32
    frames = workloads.uniform01((T, C, gh * p, gw * p), 910 + T)
    w = workloads.normal((E, C, tp, p, p), 911, std=0.02, dtype=torch.bfloat16)
    b = workloads.normal((E,), 912, std=0.02, dtype=torch.bfloat16)
    pe = _pe(E, C, tp, p, w, b)
    pe.set_norm(workloads.CLIP_MEAN, workloads.CLIP_STD)
    grid = (-(-T // tp), gh, gw)
    out = pe.forward_frames(frames.to(DEV), grid, merge, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert pe.last_error() == 0
    ref, mag = oracle.conv3d_frames(frames, grid, merge, workloads.CLIP_MEAN, workloads.CLIP_STD, w, b, C, tp, p)
    assert_within_tolerance(out, ref, mag, what=f"frames p=32 T={T} grid={grid} merge={merge}")


@pytest.mark.parametrize("C", [1, 2, 4])
@pytest.mark.parametrize("path", ["staged", "fused", "astat"])
def test_frames_other_channel_counts(C, path, monkeypatch):
    """Grayscale (C = 1), two-channel and four-channel frames (pe_create takes
    C up to 4) through every frames path: a group of images and, for the
    staged and fused paths, a video item; against the oracle."""
    tp, p, E = 2, 14, 256
    monkeypatch.setenv("PE_FRAMES_PATH", path)
    items = [(1, 6, 8), (1, 4, 10)] if path == "astat" else [(1, 6, 8), (3, 4, 6), (1, 2, 2)]
    frames = [workloads.uniform01((T, C, gh * p, gw * p), 920 + 7 * C + i) for i, (T, gh, gw) in enumerate(items)]
    grids = [(-(-T // tp), gh, gw) for T, gh, gw in items]
    w = workloads.normal((E, C, tp, p, p), 921 + C, std=0.02, dtype=torch.bfloat16)
    b = workloads.normal((E,), 922, std=0.02, dtype=torch.bfloat16)
    mean, std = (0.5, 0.45, 0.4, 0.35)[:C], (0.25, 0.26, 0.27, 0.28)[:C]
    pe = _pe(E, C, tp, p, w, b)
    pe.set_norm(mean, std)
    out = pe.forward_frames_grouped([f.to(DEV) for f in frames], grids, 2, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert pe.last_error() == 0
    ref, mag = oracle.conv3d_grouped(list(zip(frames, grids)), 2, mean, std, w, b, C, tp, p)
    assert_within_tolerance(out, ref, mag, what=f"C={C} {path}")


@pytest.mark.parametrize("T,tp,p,merge", [(5, 3, 14, 2), (1, 3, 8, 2), (6, 4, 6, 1), (3, 4, 14, 2)])
def test_frames_temporal_patch_3_and_4(T, tp, p, merge):
    """Temporal patch sizes above 2 (pe_create takes tp up to 4) run the fused
    frames kernel: the last frame repeated up to a multiple of tp (T = 1 with
    tp = 3 is one image three times), against the oracle."""
    C, E, gh, gw = 3, 192, 4, 6
    frames = workloads.uniform01((T, C, gh * p, gw * p), 930 + T + tp)
    w = workloads.normal((E, C, tp, p, p), 931 + tp, std=0.02, dtype=torch.bfloat16)
    b = workloads.normal((E,), 932, std=0.02, dtype=torch.bfloat16)
    pe = _pe(E, C, tp, p, w, b)
    pe.set_norm(workloads.CLIP_MEAN, workloads.CLIP_STD)
    grid = (-(-T // tp), gh, gw)
    out = pe.forward_frames(frames.to(DEV), grid, merge, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert pe.last_error() == 0
    ref, mag = oracle.conv3d_frames(frames, grid, merge, workloads.CLIP_MEAN, workloads.CLIP_STD, w, b, C, tp, p)
    assert_within_tolerance(out, ref, mag, what=f"tp={tp} T={T} p={p}")


@pytest.mark.parametrize("items,p,merge", [([(1, 6, 8), (1, 4, 10), (1, 2, 2)], 14, 2),      # single frames
                                           ([(4, 6, 8), (3, 4, 6), (1, 2, 4)], 14, 2),      # video rows
                                           ([(1, 4, 6), (2, 2, 4)], 16, 1)])
def test_fp32_frames_staged_and_fused(items, p, merge, monkeypatch):
    """fp32 frames take the staged pair (the prepare kernel's fp32 form, two
    launches) by default and the fused kernel when asked for; both within
    tolerance of the oracle."""
    from vlm_vision_patch_b200 import _binding as B
    C, tp, E = 3, 2, 256
    frames = [workloads.uniform01((T, C, gh * p, gw * p), 940 + i, dtype=torch.float32)
              for i, (T, gh, gw) in enumerate(items)]
    grids = [(-(-T // tp), gh, gw) for T, gh, gw in items]
    w = workloads.normal((E, C, tp, p, p), 941, std=0.02, dtype=torch.bfloat16)
    b = workloads.normal((E,), 942, std=0.02, dtype=torch.bfloat16)
    pe = _pe(E, C, tp, p, w, b)
    pe.set_norm(workloads.CLIP_MEAN, workloads.CLIP_STD)
    ref, mag = oracle.conv3d_grouped(list(zip(frames, grids)), merge, workloads.CLIP_MEAN, workloads.CLIP_STD,
                                     w, b, C, tp, p)
    dev_frames = [f.to(DEV) for f in frames]
    for path, launches in (("staged", 2), ("fused", 1)):
        monkeypatch.setenv("PE_FRAMES_PATH", path)
        B.pe_profile_begin(pe.h, 0)
        out = pe.forward_frames_grouped(dev_frames, grids, merge, out_dtype=torch.float32)
        _, n = B.pe_profile_end(pe.h, 0)
        torch.cuda.synchronize()
        assert pe.last_error() == 0
        assert n == launches, (path, n)
        assert_within_tolerance(out, ref, mag, what=f"fp32 frames {path} p={p}")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("p,merge", [(14, 2), (16, 1)])
def test_temporal_patch_1_staged_and_fused(p, merge, dtype, monkeypatch):
    """tp = 1 (one frame per temporal patch, a plain 2-D patch embedding per
    frame) runs the staged pair (one-slice rows against the frames-order
    weight) by default and the fused kernel when asked for: a group of a
    3-frame item and two images, against the oracle."""
    from vlm_vision_patch_b200 import _binding as B
    C, tp, E = 3, 1, 192
    items = [(3, 4, 6), (1, 6, 8), (1, 2, 2)]
    frames = [workloads.uniform01((T, C, gh * p, gw * p), 950 + i, dtype=dtype) for i, (T, gh, gw) in enumerate(items)]
    grids = [(T, gh, gw) for T, gh, gw in items]
    w = workloads.normal((E, C, tp, p, p), 951, std=0.02, dtype=torch.bfloat16)
    b = workloads.normal((E,), 952, std=0.02, dtype=torch.bfloat16)
    pe = _pe(E, C, tp, p, w, b)
    pe.set_norm(workloads.CLIP_MEAN, workloads.CLIP_STD)
    ref, mag = oracle.conv3d_grouped(list(zip(frames, grids)), merge, workloads.CLIP_MEAN, workloads.CLIP_STD,
                                     w, b, C, tp, p)
    dev_frames = [f.to(DEV) for f in frames]
    for path, launches in (("staged", 2), ("fused", 1)):
        monkeypatch.setenv("PE_FRAMES_PATH", path)
        B.pe_profile_begin(pe.h, 0)
        out = pe.forward_frames_grouped(dev_frames, grids, merge, out_dtype=torch.float32)
        _, n = B.pe_profile_end(pe.h, 0)
        torch.cuda.synchronize()
        assert pe.last_error() == 0
        assert n == launches, (path, n)
        assert_within_tolerance(out, ref, mag, what=f"tp=1 {path} p={p} {dtype}")
