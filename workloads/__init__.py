"""Seeded synthetic inputs for the vision PatchEmbed workloads.

This module only draws random numbers and arranges them into the shapes the
workloads use. It holds none of the PatchEmbed arithmetic (no patchify, no
normalisation, no contraction), so both the CPU oracle (``oracle/``) and the
CUDA path (``vlm_vision_patch_b200``) can be fed from it without sharing any of
the method's code.

Every tensor is generated on the CPU with ``torch.Generator().manual_seed(s)``
so the oracle and the GPU see byte-identical inputs.

Workload shapes follow the pages:
  * Qwen2.5VL-Vision Encode-PatchEmbed (python验证): 1024 patch vectors of
    3x2x14x14 = 1176 values against a [1280, 3, 2, 14, 14] Conv3d weight.
  * Qwen2.5VL语言模型 (MRoPE, 示例数据): an image with grid_thw [1, 16, 64].
  * patch详解 §4.4-§4.5: an 8-frame 224x224 video with patch 16 (784 patches,
    patch_dim 1536) and a 448x448 image with patch 14 (1024 patches), hidden 1152.
  * mytransformer README §3.2/§6: embed 1280, patch 14, temporal_patch 2,
    spatial_merge 2.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Tuple

import torch

# OpenAI CLIP per-channel pixel statistics (R, G, B), the constants the Qwen2-VL
# image processor normalises with.  The pages name "CLIP" normalisation but do
# not print the numbers; these are the published values.
CLIP_MEAN = (0.48145466, 0.4578275, 0.40821073)
CLIP_STD = (0.26862954, 0.26130258, 0.27577711)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed(int(seed))
    return g


def uniform01(shape, seed: int, dtype=torch.bfloat16) -> torch.Tensor:
    """U[0,1) pixels drawn in fp32 and stored as ``dtype`` (bf16 rounds RNE)."""
    return torch.rand(shape, generator=_gen(seed), dtype=torch.float32).to(dtype)


def normal(shape, seed: int, std: float = 1.0, dtype=torch.float32) -> torch.Tensor:
    return (torch.randn(shape, generator=_gen(seed), dtype=torch.float32) * std).to(dtype)


def kaiming_uniform_conv(shape, seed: int) -> torch.Tensor:
    """PyTorch's default Conv weight init (kaiming_uniform, a=sqrt(5)): U(-b, b)
    with b = 1/sqrt(fan_in), fan_in = prod(shape[1:])."""
    fan_in = 1
    for s in shape[1:]:
        fan_in *= int(s)
    bound = 1.0 / math.sqrt(fan_in)
    u = torch.rand(shape, generator=_gen(seed), dtype=torch.float32)
    return u * (2.0 * bound) - bound


def small_ints(shape, seed: int, lo: int, hi: int) -> torch.Tensor:
    """Integers in [lo, hi] as fp32 (exactly representable in bf16 for |v| <= 256)."""
    return torch.randint(lo, hi + 1, shape, generator=_gen(seed)).to(torch.float32)


def index_frames(T: int, C: int, H: int, W: int) -> torch.Tensor:
    """Frames whose value is their own flat index (fp32, exact below 2**24)."""
    n = T * C * H * W
    assert n < (1 << 24)
    return torch.arange(n, dtype=torch.float32).reshape(T, C, H, W)


def grid_draw(n: int, seed: int, lo: int = 8, hi: int = 96) -> List[Tuple[int, int, int]]:
    """n image grids (t=1, h, w) with h, w uniform over the even values in [lo, hi]."""
    v = torch.randint(lo // 2, hi // 2 + 1, (n, 2), generator=_gen(seed)) * 2
    return [(1, int(a), int(b)) for a, b in v.tolist()]


@dataclasses.dataclass
class Item:
    frames: torch.Tensor            # [T, C, H, W] on CPU
    grid: Tuple[int, int, int]      # (t, h, w) in patch units


@dataclasses.dataclass
class Workload:
    name: str
    E: int
    C: int
    tp: int
    p: int
    weight: torch.Tensor            # [E, C, tp, p, p] (fp32 or bf16) on CPU
    bias: Optional[torch.Tensor]    # [E] or None
    out_dtype: torch.dtype
    merge: int = 2
    patches: Optional[torch.Tensor] = None      # [N, K] for the patches form
    items: List[Item] = dataclasses.field(default_factory=list)
    mean: Tuple[float, ...] = (0.0, 0.0, 0.0)
    std: Tuple[float, ...] = (1.0, 1.0, 1.0)

    @property
    def K(self) -> int:
        return self.C * self.tp * self.p * self.p

    @property
    def N(self) -> int:
        if self.patches is not None:
            return int(self.patches.shape[0])
        return sum(t * h * w for (t, h, w) in (it.grid for it in self.items))

    @property
    def flop(self) -> int:
        return 2 * self.N * self.K * self.E


def _w_bf16(E, C, tp, p, seed):
    return normal((E, C, tp, p, p), seed, std=0.02, dtype=torch.bfloat16)


def patches_fp32_1024() -> Workload:
    """pixel_values [1024,1176] fp32 ~N(0,1) (grid [1,32,32]); Kaiming-uniform
    fp32 weight [1280,3,2,14,14]; no bias; fp32 out (patches form)."""
    x = normal((1024, 1176), 1)
    w = kaiming_uniform_conv((1280, 3, 2, 14, 14), 2)
    return Workload("patches_fp32_1024", 1280, 3, 2, 14, w, None, torch.float32,
                    merge=1, patches=x)


def image_224x896() -> Workload:
    """One RGB frame [1,3,224,896] bf16 U[0,1), CLIP-normalised, duplicated to
    tp=2; grid [1,16,64] -> 1024 patches in 2x2 merge order; bf16 N(0,0.02)
    weight; bf16 out."""
    f = uniform01((1, 3, 224, 896), 3)
    return Workload("image_224x896", 1280, 3, 2, 14, _w_bf16(1280, 3, 2, 14, 4), None,
                    torch.bfloat16, merge=2, items=[Item(f, (1, 16, 64))],
                    mean=CLIP_MEAN, std=CLIP_STD)


def video_8x224_p16() -> Workload:
    """8 frames [8,3,224,224] bf16, tp=2, patch 16 -> grid [4,14,14] = 784
    patches, K=1536, E=1152 with a bf16 bias."""
    f = uniform01((8, 3, 224, 224), 5)
    return Workload("video_8x224_p16", 1152, 3, 2, 16, _w_bf16(1152, 3, 2, 16, 6),
                    normal((1152,), 7, std=0.02, dtype=torch.bfloat16), torch.bfloat16,
                    merge=2, items=[Item(f, (4, 14, 14))], mean=CLIP_MEAN, std=CLIP_STD)


def image_448_e1152() -> Workload:
    """One 448x448 image, patch 14, E=1152 -> 1024 patches; no bias."""
    f = uniform01((1, 3, 448, 448), 8)
    return Workload("image_448_e1152", 1152, 3, 2, 14, _w_bf16(1152, 3, 2, 14, 9), None,
                    torch.bfloat16, merge=2, items=[Item(f, (1, 32, 32))],
                    mean=CLIP_MEAN, std=CLIP_STD)


def grouped_16_images(n: int = 16) -> Workload:
    """n images, grid (1, h, w) with even h, w drawn in [8, 96] (seed 10); frames
    [1,3,14h,14w] bf16 U[0,1) (seed 11+i); one grouped launch; bf16 out."""
    grids = grid_draw(n, 10)
    items = [Item(uniform01((1, 3, 14 * h, 14 * w), 11 + i), (t, h, w))
             for i, (t, h, w) in enumerate(grids)]
    return Workload("grouped_16_images", 1280, 3, 2, 14, _w_bf16(1280, 3, 2, 14, 4), None,
                    torch.bfloat16, merge=2, items=items, mean=CLIP_MEAN, std=CLIP_STD)


def long_video_64x896() -> Workload:
    """[64,3,896,896] bf16 U[0,1), grid [32,64,64] -> 131072 patches; bf16 out."""
    f = uniform01((64, 3, 896, 896), 12)
    return Workload("long_video_64x896", 1280, 3, 2, 14, _w_bf16(1280, 3, 2, 14, 4), None,
                    torch.bfloat16, merge=2, items=[Item(f, (32, 64, 64))],
                    mean=CLIP_MEAN, std=CLIP_STD)


def patches_bf16_131072() -> Workload:
    """pixel_values [131072, 1176] bf16 ~N(0,1) (the long-video row count) against
    the bf16 N(0,0.02) weight: the TMA-fed patches form at full size."""
    x = normal((131072, 1176), 13, dtype=torch.bfloat16)
    return Workload("patches_bf16_131072", 1280, 3, 2, 14, _w_bf16(1280, 3, 2, 14, 4), None,
                    torch.bfloat16, merge=1, patches=x)


ALL = {
    "patches_fp32_1024": patches_fp32_1024,
    "image_224x896": image_224x896,
    "video_8x224_p16": video_8x224_p16,
    "image_448_e1152": image_448_e1152,
    "grouped_16_images": grouped_16_images,
    "long_video_64x896": long_video_64x896,
    "patches_bf16_131072": patches_bf16_131072,
}
