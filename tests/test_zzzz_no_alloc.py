"""The allocation-free grouped call against the ordinary grouped call.

pe_forward_frames_grouped_noalloc exists for callers that cannot allocate
device memory while serving (their memory is all handed to their own pool up
front, and cudaMalloc would also synchronise the device): it keeps its item
table in a fixed array of the library's static device memory instead of the
handle's workspace.  This test drives both entry points through the C ABI on
the same inputs, twice in a row with different item lists (so the shared table
is overwritten in between), and requires the outputs to agree within the
parity tolerance of the other GPU tests.  It sits in its own file, collected
last, and passes both on its own in a fresh process and after the rest.
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


def _call(fn, pe, frames_dev, grids, out):
    B_fn = getattr(B, fn)
    B_fn(pe.h, [f.data_ptr() for f in frames_dev], B.PE_BF16,
         [(f.shape[0], f.shape[2], f.shape[3]) for f in frames_dev], grids, 2, out.data_ptr(), B.PE_BF16,
         torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_grouped_twice_in_a_row():
    w = workloads.normal((E, C, TP, P, P), 5, std=0.02, dtype=torch.bfloat16)
    pe = PatchEmbed(E, C, TP, P, False)
    pe.set_weight(w.to(DEV))
    pe.set_norm(workloads.CLIP_MEAN, workloads.CLIP_STD)
    for seed, n in ((1, 40), (2, 23)):          # both above the inline-item limit
        frames, grids = _items(seed, n)
        fd = [f.to(DEV) for f in frames]
        N = sum(g[0] * g[1] * g[2] for g in grids)
        ref_out = torch.empty(N, E, dtype=torch.bfloat16, device=DEV)
        new_out = torch.full((N, E), float("nan"), dtype=torch.bfloat16, device=DEV)
        _call("pe_forward_frames_grouped", pe, fd, grids, ref_out)
        _call("pe_forward_frames_grouped_noalloc", pe, fd, grids, new_out)
        torch.cuda.synchronize()
        assert pe.last_error() == 0
        _, mag = oracle.conv3d_grouped(list(zip(frames, grids)), 2, workloads.CLIP_MEAN, workloads.CLIP_STD,
                                       w, None, C, TP, P)
        assert_within_tolerance(new_out, ref_out.double().cpu().numpy(), mag, what=f"noalloc n={n}")


def test_noalloc_rejects_too_many_items():
    pe = PatchEmbed(E, C, TP, P, False)
    pe.set_weight(workloads.normal((E, C, TP, P, P), 6, std=0.02, dtype=torch.bfloat16).to(DEV))
    f = torch.zeros(1, C, 2 * P, 2 * P, dtype=torch.bfloat16, device=DEV)
    n = B.PE_NOALLOC_MAX_ITEMS + 1
    out = torch.empty(4 * n, E, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(B.PEError) as e:
        _call("pe_forward_frames_grouped_noalloc", pe, [f] * n, [(1, 2, 2)] * n, out)
    assert e.value.status == "PE_ERR_UNSUPPORTED"
