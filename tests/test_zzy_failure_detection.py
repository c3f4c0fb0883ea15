"""Failure detection on the GPU without a fault: a wait that can never be
satisfied gives up after its limit, the kernel reports PE_ERR_DEVICE_TIMEOUT
through the handle's error word, pe_last_error reads and clears it, and the
context and the handle keep working (a forward afterwards matches the oracle)."""
from __future__ import annotations

import time

import pytest
import torch

import oracle
import workloads
from vlm_vision_patch_b200 import PatchEmbed
from vlm_vision_patch_b200 import _binding as B
from tests.gpu_util import assert_within_tolerance

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
PE_ERR_DEVICE_TIMEOUT = 8


def test_stalled_wait_is_reported_and_the_handle_stays_usable():
    C, tp, p, E = 3, 2, 14, 128
    w = workloads.normal((E, C, tp, p, p), 930, std=0.02, dtype=torch.bfloat16)
    pe = PatchEmbed(E, C, tp, p, False)
    pe.set_weight(w.to(DEV))
    torch.cuda.synchronize()
    assert pe.last_error() == 0
    t0 = time.perf_counter()
    B.pe_selftest_wait_timeout(pe.h, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert pe.last_error() == PE_ERR_DEVICE_TIMEOUT
    assert pe.last_error() == 0                       # read and cleared
    assert 1.0 < waited < 60.0, waited                # the 2 s limit, not a hang
    x = workloads.normal((300, C * tp * p * p), 931, dtype=torch.bfloat16)
    out = pe.forward_patches(x.to(DEV), out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert pe.last_error() == 0
    ref, mag = oracle.conv3d_patches(x, w, None, C, tp, p)
    assert_within_tolerance(out, ref, mag, what="forward after a reported timeout")
