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
