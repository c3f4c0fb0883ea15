"""Profiling hooks of the C ABI on a B200: pe_profile_target selects which
kernel of a forward call the event pairs time (the contraction, or the kernel
before it), and a window that only counts launches records no times."""
import pytest
import torch

import workloads
from vlm_vision_patch_b200 import PatchEmbed, PEError, _binding as B

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _pe(E=256, p=14):
    pe = PatchEmbed(E, 3, 2, p, False)
    pe.set_weight(workloads.normal((E, 3, 2, p, p), 960, std=0.02, dtype=torch.bfloat16).to(DEV))
    pe.set_norm(workloads.CLIP_MEAN, workloads.CLIP_STD)
    return pe


def _window(pe, target, calls, fn):
    B.pe_profile_target(pe.h, target)
    B.pe_profile_begin(pe.h, calls)
    for _ in range(calls):
        fn()
    ms, launches = B.pe_profile_end(pe.h, calls)
    torch.cuda.synchronize()
    B.pe_profile_target(pe.h, 0)
    return ms, launches


def test_profile_target_selects_the_kernel():
    pe = _pe()
    frames = [workloads.uniform01((1, 3, 14 * 8, 14 * 12), 961).to(DEV)]
    grids = [(1, 8, 12)]
    x = workloads.normal((500, pe.K), 962, dtype=torch.bfloat16).to(DEV)
    xf = workloads.normal((500, pe.K), 963).to(DEV)
    staged = lambda: pe.forward_frames_grouped(frames, grids, 2)
    ms_c, n_c = _window(pe, 0, 3, staged)          # contraction of a staged call
    ms_p, n_p = _window(pe, 1, 3, staged)          # its prepare kernel
    assert len(ms_c) == 3 and len(ms_p) == 3 and n_c == n_p == 6
    assert all(t > 0 for t in ms_c + ms_p)
    ms_b, n_b = _window(pe, 1, 2, lambda: pe.forward_patches(x))   # bf16 rows: no kernel before the GEMM
    assert ms_b == [] and n_b == 2
    ms_f, n_f = _window(pe, 1, 2, lambda: pe.forward_patches(xf))  # fp32 rows: the cast kernel
    assert len(ms_f) == 2 and n_f == 4 and all(t > 0 for t in ms_f)
    B.pe_profile_begin(pe.h, 0)                    # counting only: no events, launches still counted
    staged()
    staged()
    ms0, n0 = B.pe_profile_end(pe.h, 0)
    torch.cuda.synchronize()
    assert ms0 == [] and n0 == 4
    assert pe.last_error() == 0


def test_profile_target_rejects_unknown_targets():
    pe = _pe()
    with pytest.raises(PEError):
        B.pe_profile_target(pe.h, 2)
    with pytest.raises(PEError):
        B.pe_profile_target(pe.h, -1)
