"""The synthetic input recipe (workloads/): the documented shapes and sizes,
determinism under the seeds, the value distributions, and the 16-image grid
rule (t = 1, h and w even in [8, 96]), so that the figures quoted for each
workload cannot drift silently.  CPU only; the two multi-hundred-MB workloads
are built with stand-in generators that record the requested shapes."""
from __future__ import annotations

import math

import pytest
import torch

import workloads

SMALL = {
    # name: (N, K, E, items, p, bias, out dtype)
    "patches_fp32_1024": (1024, 1176, 1280, 0, 14, False, torch.float32),
    "image_224x896": (1024, 1176, 1280, 1, 14, False, torch.bfloat16),
    "video_8x224_p16": (784, 1536, 1152, 1, 16, True, torch.bfloat16),
    "image_448_e1152": (1024, 1176, 1152, 1, 14, False, torch.bfloat16),
    "grouped_16_images": (59204, 1176, 1280, 16, 14, False, torch.bfloat16),
}


@pytest.mark.parametrize("name", sorted(SMALL))
def test_sizes_and_determinism(name):
    N, K, E, n_items, p, bias, odt = SMALL[name]
    a, b = workloads.ALL[name](), workloads.ALL[name]()
    assert (a.N, a.K, a.E, len(a.items), a.p, a.bias is not None, a.out_dtype) == (N, K, E, n_items, p, bias, odt)
    assert a.weight.shape == (E, a.C, a.tp, p, p)
    assert torch.equal(a.weight, b.weight)
    if a.patches is not None:
        assert a.patches.shape == (N, K) and torch.equal(a.patches, b.patches)
    for x, y in zip(a.items, b.items):
        t, h, w = x.grid
        assert x.frames.shape[1:] == (a.C, h * p, w * p) and -(-x.frames.shape[0] // a.tp) == t
        assert x.grid == y.grid and torch.equal(x.frames, y.frames)


def test_value_distributions():
    x = workloads.patches_fp32_1024()
    assert abs(float(x.patches.mean())) < 0.01 and abs(float(x.patches.std()) - 1.0) < 0.01
    bound = 1.0 / math.sqrt(1176)           # kaiming_uniform(a = sqrt(5)) on fan_in 1176
    assert float(x.weight.abs().max()) <= bound and float(x.weight.abs().max()) > 0.99 * bound
    img = workloads.image_224x896()
    f = img.items[0].frames.float()
    assert img.items[0].frames.dtype == torch.bfloat16
    assert float(f.min()) >= 0.0 and float(f.max()) <= 1.0 and abs(float(f.mean()) - 0.5) < 0.01
    assert abs(float(img.weight.float().std()) - 0.02) < 0.001
    assert img.mean == workloads.CLIP_MEAN and img.std == workloads.CLIP_STD


def test_grouped_grid_rule():
    wl = workloads.grouped_16_images()
    for it in wl.items:
        t, h, w = it.grid
        assert t == 1 and it.frames.shape[0] == 1
        assert h % 2 == 0 and w % 2 == 0 and 8 <= h <= 96 and 8 <= w <= 96
    assert wl.N == sum(h * w for _, h, w in (it.grid for it in wl.items))


def test_large_workload_recipes(monkeypatch):
    """The two multi-hundred-MB workloads, built with the generators replaced
    by stand-ins that record what they are asked for: the frame and row
    shapes, seeds and grids of the recipe, without the memory."""
    asked = []

    def fake(kind):
        def gen(shape, seed, *a, **k):
            asked.append((kind, tuple(shape), seed))
            return torch.zeros(0)
        return gen
    monkeypatch.setattr(workloads, "uniform01", fake("uniform01"))
    monkeypatch.setattr(workloads, "normal", fake("normal"))
    lv = workloads.long_video_64x896()
    assert lv.items[0].grid == (32, 64, 64) and (lv.E, lv.p, lv.tp, lv.merge) == (1280, 14, 2, 2)
    assert ("uniform01", (64, 3, 896, 896), 12) in asked
    assert ("normal", (1280, 3, 2, 14, 14), 4) in asked
    asked.clear()
    pb = workloads.patches_bf16_131072()
    assert (pb.E, pb.p, pb.tp, pb.bias) == (1280, 14, 2, None)
    assert any(kind == "normal" and shape == (131072, 1176) for kind, shape, _ in asked)
