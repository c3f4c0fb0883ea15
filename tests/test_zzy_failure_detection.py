"""Failure detection on the GPU without a fault: a wait that can never be
satisfied gives up after its limit, the kernel reports PE_ERR_DEVICE_TIMEOUT
through the handle's error word, pe_last_error reads and clears it, and the
context and the handle keep working (a forward afterwards matches the oracle).
Two forms: a probe kernel whose wait nothing satisfies, and the resident-A
pipeline itself with its wait limit forced down to a few microseconds."""
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


@pytest.mark.parametrize("cap_ns", [1, 2000, 20000])
def test_forced_wait_cap_unwinds_the_resident_a_pipeline(cap_ns, monkeypatch):
    """The forced cap on a real pipeline: PE_TEST_WAIT_NS gives the resident-A
    kernel's bounded waits a limit of `cap_ns`, so they give up at the first
    wait (1 ns) or part-way through (2 us, 20 us) instead of after 2 s.  The
    kernel then unwinds: every role stops, the MMAs already issued drain, the
    weight loads already issued land (bounded waits on their barriers), the
    TMEM is freed and PE_ERR_DEVICE_TIMEOUT is recorded.  The call returns
    without a fault or a hang, and the next forward on the same handle, with
    the default limit, matches the oracle."""
    C, tp, p, E = 3, 2, 14, 1280
    grids = [(1, 16, 64), (1, 20, 24), (1, 8, 6)]
    frames = [workloads.uniform01((1, C, g[1] * p, g[2] * p), 940 + i) for i, g in enumerate(grids)]
    w = workloads.normal((E, C, tp, p, p), 943, std=0.02, dtype=torch.bfloat16)
    pe = PatchEmbed(E, C, tp, p, False)
    pe.set_weight(w.to(DEV))
    pe.set_norm(workloads.CLIP_MEAN, workloads.CLIP_STD)
    fd = [f.to(DEV) for f in frames]
    torch.cuda.synchronize()
    assert pe.last_error() == 0
    monkeypatch.setenv("PE_FRAMES_PATH", "astat")
    monkeypatch.setenv("PE_TEST_WAIT_NS", str(cap_ns))
    B.pe_profile_begin(pe.h, 0)
    t0 = time.perf_counter()
    pe.forward_frames_grouped(fd, grids, 2)
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    _, launches = B.pe_profile_end(pe.h, 0)
    assert launches == 1, "the resident-A kernel ran"
    status = pe.last_error()
    assert waited < 30.0, waited
    if cap_ns == 1:
        assert status == PE_ERR_DEVICE_TIMEOUT
    else:
        assert status in (0, PE_ERR_DEVICE_TIMEOUT)
    assert pe.last_error() == 0
    monkeypatch.delenv("PE_TEST_WAIT_NS")
    out = pe.forward_frames_grouped(fd, grids, 2, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert pe.last_error() == 0
    ref, mag = oracle.conv3d_grouped(list(zip(frames, grids)), 2, workloads.CLIP_MEAN, workloads.CLIP_STD, w, None,
                                     C, tp, p)
    assert_within_tolerance(out, ref, mag, what=f"forward after a forced {cap_ns} ns cap")
