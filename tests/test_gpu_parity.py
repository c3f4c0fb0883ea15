"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Tolerance (per output element): |gpu - oracle| <= 1e-3 * sum_k |x_k * w_k| for
fp32 output, plus one bf16 ulp of the oracle value for bf16 output.  Integer,
one-hot and patchify cases are bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from vlm_vision_patch_b200 import PatchEmbed, PatchMerger, PEError  # noqa: F401
from tests.gpu_util import assert_within_tolerance, mask_of, sample_rows

pytestmark = pytest.mark.gpu

DEV = "cuda:0"




def _pe(wl_or_args, weight, bias, mean=None, std=None):
    E, C, tp, p = wl_or_args
    pe = PatchEmbed(E, C, tp, p, bias is not None)
    pe.set_weight(weight.to(DEV).contiguous(), None if bias is None else bias.to(DEV).contiguous())
    if mean is not None:
        pe.set_norm(mean, std)
    return pe


def _bits32(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").float().numpy().view(np.uint32)


def assert_bits_equal(got: np.ndarray, ref: np.ndarray, what: str = ""):
    assert got.shape == ref.shape, (got.shape, ref.shape)
    bad = got != ref
    if bad.any():
        idx = np.argwhere(bad)[:6]
        det = [(tuple(int(x) for x in i), hex(int(got[tuple(i)])), hex(int(ref[tuple(i)]))) for i in idx]
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} differ; first (index, got, ref): {det}")


# --------------------------------------------------------------- patches form

@pytest.mark.parametrize("x_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("N", [1, 128, 300])
def test_patches_integer_inputs_bit_exact(x_dtype, N):
    """Small integers keep every product and partial sum exact in fp32, so the
    fp32 output must equal the oracle bit for bit, and bf16 output must be its
    bf16 rounding (Optimize VLM PatchEmbed's randint check, R1 == R2)."""
    C, tp, p, E = 3, 2, 14, 1280
    K = C * tp * p * p
    x = workloads.small_ints((N, K), 31, 0, 2)
    w = workloads.small_ints((E, C, tp, p, p), 32, -4, 4)
    b = workloads.small_ints((E,), 33, -100, 100)
    ref, _ = oracle.conv3d_patches(x, w, b, C, tp, p)
    pe = _pe((E, C, tp, p), w, b)
    xd = x.to(x_dtype).to(DEV)
    out32 = pe.forward_patches(xd, out_dtype=torch.float32)
    out16 = pe.forward_patches(xd, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert pe.last_error() == 0
    assert np.array_equal(out32.cpu().double().numpy(), ref)
    ref16 = torch.from_numpy(ref.astype(np.float32)).to(torch.bfloat16)
    assert torch.equal(out16.cpu(), ref16)


def test_patches_one_hot_recovers_weight():
    C, tp, p, E = 3, 2, 14, 1280
    K = C * tp * p * p
    w = workloads.normal((E, C, tp, p, p), 34, std=0.02)
    b = workloads.normal((E,), 35, std=0.02)
    pe = _pe((E, C, tp, p), w, b)
    x = torch.eye(K, dtype=torch.bfloat16, device=DEV)
    out = pe.forward_patches(x, out_dtype=torch.float32)
    ref, _ = oracle.conv3d_patches(torch.eye(K), w, b, C, tp, p)
    torch.cuda.synchronize()
    # one product, then the fp32 bias add: the exact sum rounded once to fp32
    assert_bits_equal(out.cpu().numpy().view(np.uint32), ref.astype(np.float32).view(np.uint32), "one-hot")
    zero = pe.forward_patches(torch.zeros(5, K, dtype=torch.bfloat16, device=DEV), out_dtype=torch.float32)
    assert torch.equal(zero.cpu(), b.float().expand(5, E))


def test_patches_fp32_1024_workload():
    """pixel_values [1024, 1176] fp32 N(0,1), Kaiming-uniform fp32 weight, fp32 out."""
    wl = workloads.patches_fp32_1024()
    pe = _pe((wl.E, wl.C, wl.tp, wl.p), wl.weight, wl.bias)
    out = pe.forward_patches(wl.patches.to(DEV), out_dtype=torch.float32)
    ref, mag = oracle.conv3d_patches(wl.patches, wl.weight, wl.bias, wl.C, wl.tp, wl.p)
    torch.cuda.synchronize()
    assert pe.last_error() == 0
    assert_within_tolerance(out, ref, mag, what=wl.name)


@pytest.mark.parametrize("C,tp,p,E,N,bias,x_dtype,out_dtype", [
    (3, 2, 14, 1280, 129, False, torch.bfloat16, torch.bfloat16),
    (3, 2, 16, 1152, 1000, True, torch.bfloat16, torch.float32),
    (3, 1, 3, 72, 257, True, torch.float32, torch.float32),      # K=27: no TMA, ragged K
    (1, 2, 4, 16, 5, False, torch.bfloat16, torch.bfloat16),     # K=32
    (3, 2, 2, 40, 130, True, torch.bfloat16, torch.float32),     # K=24, E tail chunk
    (2, 2, 14, 200, 384, False, torch.float32, torch.bfloat16),  # K=784, E=200 (partial tile)
])
def test_patches_shapes(C, tp, p, E, N, bias, x_dtype, out_dtype):
    K = C * tp * p * p
    x = workloads.normal((N, K), 40 + N)
    w = workloads.normal((E, C, tp, p, p), 41 + E, std=0.05)
    b = workloads.normal((E,), 42, std=0.05) if bias else None
    pe = _pe((E, C, tp, p), w, b)
    out = pe.forward_patches(x.to(x_dtype).to(DEV), out_dtype=out_dtype)
    ref, mag = oracle.conv3d_patches(x.to(x_dtype), w, b, C, tp, p)
    torch.cuda.synchronize()
    assert pe.last_error() == 0
    assert_within_tolerance(out, ref, mag, what=f"patches {C},{tp},{p},{E},{N}")


def test_patches_empty_and_bn_override(monkeypatch):
    C, tp, p, E = 3, 2, 14, 256
    w = workloads.normal((E, C, tp, p, p), 43, std=0.02)
    pe = _pe((E, C, tp, p), w, None)
    out = pe.forward_patches(torch.empty(0, C * tp * p * p, dtype=torch.bfloat16, device=DEV))
    assert out.shape == (0, E)
    x = workloads.normal((517, C * tp * p * p), 44)
    ref, mag = oracle.conv3d_patches(x, w, None, C, tp, p)
    for bn in ("64", "128", "256"):
        monkeypatch.setenv("PE_BN", bn)
        o = pe.forward_patches(x.to(torch.bfloat16).to(DEV), out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert_within_tolerance(o, ref, mag, what=f"BN={bn}")


# ---------------------------------------------------------------- frames form

def _run_frames(wl, out_dtype=None, rows=None):
    pe = _pe((wl.E, wl.C, wl.tp, wl.p), wl.weight, wl.bias, wl.mean, wl.std)
    od = out_dtype or wl.out_dtype
    frames = [it.frames.to(DEV) for it in wl.items]
    grids = [it.grid for it in wl.items]
    if len(frames) == 1:
        out = pe.forward_frames(frames[0], grids[0], wl.merge, out_dtype=od)
    else:
        out = pe.forward_frames_grouped(frames, grids, wl.merge, out_dtype=od)
    mask = None if rows is None else mask_of(rows, wl.N)
    ref, mag = oracle.conv3d_grouped([(it.frames, it.grid) for it in wl.items], wl.merge, wl.mean, wl.std,
                                     wl.weight, wl.bias, wl.C, wl.tp, wl.p, row_mask=mask)
    torch.cuda.synchronize()
    assert pe.last_error() == 0
    return pe, out, ref, mag


@pytest.mark.parametrize("name", ["image_224x896", "video_8x224_p16", "image_448_e1152"])
def test_frames_workloads_all_rows(name):
    wl = workloads.ALL[name]()
    _, out, ref, mag = _run_frames(wl)
    assert_within_tolerance(out, ref, mag, what=name)


def test_frames_fp32_out_and_fp32_frames():
    wl = workloads.image_224x896()
    for it in wl.items:
        it.frames = it.frames.float()
    _, out, ref, mag = _run_frames(wl, out_dtype=torch.float32)
    assert out.dtype == torch.float32
    assert_within_tolerance(out, ref, mag, what="fp32 frames / fp32 out")


@pytest.mark.parametrize("T,gh,gw,merge,p,tp,E,bias", [
    (3, 4, 6, 2, 14, 2, 1280, True),     # odd T: last frame repeated
    (1, 6, 2, 1, 14, 2, 256, False),     # raster order
    (5, 2, 4, 2, 16, 2, 128, True),
    (2, 8, 10, 2, 4, 2, 64, False),      # small even p (generic kernel)
    (1, 2, 2, 2, 14, 2, 1280, False),    # 4 rows only
    (4, 10, 14, 2, 6, 1, 96, True),      # tp = 1
])
def test_frames_small_shapes(T, gh, gw, merge, p, tp, E, bias):
    C = 3
    gt = -(-T // tp)
    wl = workloads.Workload(f"frames_{T}_{gh}_{gw}_{p}", E, C, tp, p,
                            workloads.normal((E, C, tp, p, p), 50 + p, std=0.02, dtype=torch.bfloat16),
                            workloads.normal((E,), 51, std=0.02) if bias else None, torch.bfloat16, merge=merge,
                            items=[workloads.Item(workloads.uniform01((T, C, gh * p, gw * p), 52 + T), (gt, gh, gw))],
                            mean=workloads.CLIP_MEAN, std=workloads.CLIP_STD)
    _, out, ref, mag = _run_frames(wl)
    assert_within_tolerance(out, ref, mag, what=wl.name)


def test_grouped_16_images_all_rows():
    """The 16-image grouped workload at full size (59204 rows, the benchmark's
    launch), every element against the oracle."""
    wl = workloads.grouped_16_images()
    _, out, ref, mag = _run_frames(wl)
    r = assert_within_tolerance(out, ref, mag, what=wl.name)
    print(f"grouped_16_images: worst |err| / tolerance = {r:.3f}")


def test_grouped_small_items_all_rows():
    C, tp, p, E = 3, 2, 14, 1280
    grids = [(1, 2, 2), (2, 4, 6), (1, 8, 2), (1, 2, 16), (3, 6, 6)]
    items = [workloads.Item(workloads.uniform01((2 * g[0] - (i % 2 if g[0] > 1 else 0), C, g[1] * p, g[2] * p),
                                                70 + i), g) for i, g in enumerate(grids)]
    wl = workloads.Workload("grouped_small", E, C, tp, p,
                            workloads.normal((E, C, tp, p, p), 71, std=0.02, dtype=torch.bfloat16), None,
                            torch.bfloat16, merge=2, items=items, mean=workloads.CLIP_MEAN,
                            std=workloads.CLIP_STD)
    _, out, ref, mag = _run_frames(wl)
    assert_within_tolerance(out, ref, mag, what=wl.name)


def test_grouped_many_items_device_table():
    """More items than fit in the launch parameters: the item table goes through
    the handle's device workspace."""
    C, tp, p, E = 3, 2, 14, 256
    rng = np.random.default_rng(80)
    grids = [(1, int(2 * rng.integers(1, 4)), int(2 * rng.integers(1, 4))) for _ in range(40)]
    items = [workloads.Item(workloads.uniform01((1, C, g[1] * p, g[2] * p), 81 + i), g) for i, g in enumerate(grids)]
    wl = workloads.Workload("grouped_40", E, C, tp, p,
                            workloads.normal((E, C, tp, p, p), 82, std=0.02, dtype=torch.bfloat16), None,
                            torch.bfloat16, merge=2, items=items, mean=workloads.CLIP_MEAN,
                            std=workloads.CLIP_STD)
    _, out, ref, mag = _run_frames(wl)
    assert_within_tolerance(out, ref, mag, what=wl.name)


def test_long_video_sampled_rows():
    """[64, 3, 896, 896] frames, grid [32, 64, 64] -> 131072 rows, sampled."""
    wl = workloads.long_video_64x896()
    rows = sample_rows(wl.N, 768, 90)
    _, out, ref, mag = _run_frames(wl, rows=rows)
    assert_within_tolerance(out, ref, mag, rows=rows, what=wl.name)


def test_frames_deterministic():
    wl = workloads.image_448_e1152()
    pe = _pe((wl.E, wl.C, wl.tp, wl.p), wl.weight, wl.bias, wl.mean, wl.std)
    f = wl.items[0].frames.to(DEV)
    a = pe.forward_frames(f, wl.items[0].grid, 2)
    b = pe.forward_frames(f, wl.items[0].grid, 2)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


# ------------------------------------------------------------------ patchify

@pytest.mark.parametrize("T,gh,gw,merge,p,tp,fdt", [
    (1, 16, 64, 2, 14, 2, torch.bfloat16),
    (3, 4, 6, 2, 14, 2, torch.bfloat16),
    (8, 14, 14, 2, 16, 2, torch.bfloat16),
    (2, 6, 4, 1, 14, 2, torch.float32),
    (5, 4, 8, 2, 4, 2, torch.float32),
    (2, 6, 6, 2, 6, 1, torch.bfloat16),
])
def test_patchify_bit_exact(T, gh, gw, merge, p, tp, fdt):
    C = 3
    gt = -(-T // tp)
    frames = workloads.uniform01((T, C, gh * p, gw * p), 100 + p + T).to(fdt)
    pe = PatchEmbed(64, C, tp, p, False)
    pe.set_norm(workloads.CLIP_MEAN, workloads.CLIP_STD)
    rows = pe.patchify([frames.to(DEV)], [(gt, gh, gw)], merge, rows_dtype=torch.float32)
    ref = oracle.patchify(frames, (gt, gh, gw), merge, workloads.CLIP_MEAN, workloads.CLIP_STD, C, tp, p)
    torch.cuda.synchronize()
    assert_bits_equal(_bits32(rows), ref.view(np.uint32), "patchify fp32 rows")
    rows16 = pe.patchify([frames.to(DEV)], [(gt, gh, gw)], merge, rows_dtype=torch.bfloat16)
    assert_bits_equal(_bits32(rows16), ref.view(np.uint32), "patchify bf16 rows")


@pytest.mark.parametrize("mean,std", [(workloads.CLIP_MEAN, workloads.CLIP_STD),
                                      ((0.5, -0.25, 3.0), (0.5, 0.1, 7.0)),
                                      ((0.0, 0.0, 0.0), (1.0, 1.0, 1.0)),
                                      ((0.0, -0.0, 1e-30), (0.3, 1.0, 5e-40)),
                                      ((123.675, 116.28, 103.53), (58.395, 57.12, 57.375))])
def test_normalization_exhaustive_bf16(mean, std):
    """Every finite bf16 value in every channel: the kernel's fp32 (x-mean)/std
    then bf16 rounding equals the oracle's IEEE divide bit for bit."""
    vals = (np.arange(65536, dtype=np.uint32) << 16).view(np.float32)
    vals = vals[np.isfinite(vals)]
    n = vals.size                                   # 65024 values
    W = 128                                         # p = 2 -> gw = 64
    H = -(-n // W)
    H = -(-H // 4) * 4
    buf = np.zeros(H * W, dtype=np.float32)
    buf[:n] = vals
    frames = torch.from_numpy(np.stack([np.roll(buf, 977 * c) for c in range(3)]).reshape(1, 3, H, W))
    frames = frames.to(torch.bfloat16)
    pe = PatchEmbed(64, 3, 1, 2, False)
    pe.set_norm(mean, std)
    rows = pe.patchify([frames.to(DEV)], [(1, H // 2, W // 2)], 2, rows_dtype=torch.float32)
    ref = oracle.patchify(frames, (1, H // 2, W // 2), 2, mean, std, 3, 1, 2)
    torch.cuda.synchronize()
    assert_bits_equal(_bits32(rows), ref.view(np.uint32), f"normalisation mean={mean} std={std}")


# --------------------------------------------------------------- error paths

def test_error_paths():
    pe = PatchEmbed(256, 3, 2, 14, False)
    K = 3 * 2 * 14 * 14
    x = torch.zeros(4, K, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(PEError) as e:
        pe.forward_patches(x)
    assert e.value.status == "PE_ERR_NO_WEIGHT"
    w = workloads.normal((256, 3, 2, 14, 14), 1, std=0.02).to(DEV)
    with pytest.raises(PEError) as e:
        pe.set_weight(w, torch.zeros(256, device=DEV))          # handle has no bias
    assert e.value.status == "PE_ERR_INVALID_ARG"
    pe.set_weight(w)
    f = torch.zeros(1, 3, 224, 224, dtype=torch.bfloat16, device=DEV)
    for grid, merge, code in [((1, 16, 15), 2, "PE_ERR_SHAPE"), ((1, 15, 16), 2, "PE_ERR_SHAPE"),
                              ((2, 16, 16), 2, "PE_ERR_SHAPE"), ((1, 16, 16), 3, "PE_ERR_INVALID_ARG")]:
        with pytest.raises(PEError) as e:
            pe.forward_frames(f, grid, merge)
        assert e.value.status == code
    with pytest.raises(PEError) as e:
        pe.forward_patches(x.view(-1)[1:1 + 3 * K].view(3, K))   # misaligned pointer
    assert e.value.status == "PE_ERR_ALIGN"
    with pytest.raises(PEError) as e:
        pe.set_norm((0.5, 0.5, 0.5), (1.0, 0.0, 1.0))
    assert e.value.status == "PE_ERR_INVALID_ARG"
    with pytest.raises(PEError) as e:
        PatchEmbed(1004, 3, 2, 14)                                  # E % 8 != 0
    assert e.value.status == "PE_ERR_INVALID_ARG"
    odd = PatchEmbed(64, 3, 2, 3, False)
    odd.set_weight(workloads.normal((64, 3, 2, 3, 3), 2).to(DEV))
    with pytest.raises(PEError) as e:
        odd.forward_frames(torch.zeros(2, 3, 6, 6, device=DEV), (1, 2, 2), 2)
    assert e.value.status == "PE_ERR_UNSUPPORTED"
    torch.cuda.synchronize()
    assert pe.last_error() == 0


# ------------------------------------------------------ staged vs fused path

@pytest.mark.parametrize("case", ["images", "video_odd_T", "mixed", "images_p16_raster"])
def test_staged_and_fused_paths_agree(case, monkeypatch):
    """All three frames paths (fused kernel, staged pair, streamed kernel) must
    be within tolerance of the oracle.  Where some item has more than one
    frame, the fused and staged paths run the contraction in the same k order
    and tile shape, so their outputs must also be bit-identical.  When every
    item is a single frame, the staged and streamed paths both store one
    temporal slice per row and meet it with both slices of the weight in the
    same order, so those two must be bit-identical."""
    C, tp, p, E, merge = 3, 2, 14, 1280, 2
    if case == "images":
        grids = [(1, 12, 18), (1, 20, 10), (1, 8, 8)]
        Ts = [1, 1, 1]
    elif case == "video_odd_T":
        grids = [(3, 10, 12)]
        Ts = [5]
    elif case == "mixed":
        grids = [(1, 10, 14), (2, 8, 8), (1, 6, 10)]
        Ts = [1, 4, 1]
    else:   # p = 16: slice length 768 needs no padding; raster order; ragged row count
        p, E, merge = 16, 1152, 1
        grids = [(1, 7, 9), (1, 5, 11), (1, 13, 3)]
        Ts = [1, 1, 1]
    items = [workloads.Item(workloads.uniform01((T, C, g[1] * p, g[2] * p), 120 + i), g)
             for i, (T, g) in enumerate(zip(Ts, grids))]
    wl = workloads.Workload("staged_" + case, E, C, tp, p,
                            workloads.normal((E, C, tp, p, p), 121, std=0.02, dtype=torch.bfloat16),
                            workloads.normal((E,), 122, std=0.02, dtype=torch.bfloat16), torch.bfloat16,
                            merge=merge, items=items, mean=workloads.CLIP_MEAN, std=workloads.CLIP_STD)
    outs = {}
    for path in ("fused", "staged", "streamed"):
        monkeypatch.setenv("PE_FRAMES_PATH", path)
        _, out, ref, mag = _run_frames(wl)
        outs[path] = out
        assert_within_tolerance(out, ref, mag, what=f"{case} {path}")
    if any(T > 1 for T in Ts):
        assert torch.equal(outs["fused"], outs["staged"])
    else:   # staged and streamed: the same rows, tile shape and summation order
        assert torch.equal(outs["staged"], outs["streamed"])
    if case == "images":   # fp32 output from the staged path
        _, out, ref, mag = _run_frames(wl, out_dtype=torch.float32)
        assert out.dtype == torch.float32
        assert_within_tolerance(out, ref, mag, what=f"{case} staged fp32 out")


# ------------------------------------------------------------ temporal folding

def _folded_weight(w: torch.Tensor) -> torch.Tensor:
    """The weight the folded path multiplies single frames by, as a Conv3d
    weight of the original shape: bf16_rne(fp32(Ŵ0 + Ŵ1)) in slice 0, zeros in
    slice 1 (a single frame is duplicated to both slices, patch详解 §4.5)."""
    wb = w.to(torch.bfloat16).float()
    f = (wb[:, :, 0] + wb[:, :, 1]).to(torch.bfloat16).float()
    out = torch.zeros_like(wb)
    out[:, :, 0] = f
    return out


@pytest.mark.parametrize("case", ["image_224x896", "grouped_small", "p16_raster_bias", "grouped_16_images",
                                  "E200_bias_f32", "E200_bf16"])
def test_temporal_fold(case):
    """Opt-in folding: (1) within the parity tolerance of the oracle run with the
    folded weight (the same products, any summation order); (2) within the
    parity tolerance 1e-3 * sum|x̂ ŵ| (+ one bf16 ulp) of the exact, unfolded
    Conv3d on every row, the 59204-row group included.  The folded weight
    carries one more bf16 rounding per term (at most 2^-9 of |Ŵ0 + Ŵ1|); its
    errors have random signs over the C*p*p terms of a row, so on these inputs
    they stay well inside the bound (the worst ratio is printed)."""
    rows = None
    od = torch.bfloat16
    if case == "image_224x896":
        wl = workloads.image_224x896()
    elif case == "grouped_16_images":
        wl = workloads.grouped_16_images()
    else:
        C, tp = 3, 2
        if case == "grouped_small":
            p, E, merge, bias = 14, 1280, 2, None
            grids = [(1, 12, 18), (1, 20, 10), (1, 8, 8)]
        elif case.startswith("E200"):
            # rows of 400 or 800 bytes and a last 8-column chunk: the epilogue's
            # 16-byte register stores and its partial chunk
            p, E, merge = 14, 200, 2
            grids = [(1, 6, 10), (1, 4, 8)]
            bias = workloads.normal((E,), 133, std=0.5) if case == "E200_bias_f32" else None
            od = torch.float32 if case == "E200_bias_f32" else torch.bfloat16
        else:
            p, E, merge = 16, 1152, 1
            grids = [(1, 7, 9), (1, 5, 11)]
            bias = workloads.normal((E,), 132, std=0.02, dtype=torch.bfloat16)
        items = [workloads.Item(workloads.uniform01((1, C, g[1] * p, g[2] * p), 130 + i), g)
                 for i, g in enumerate(grids)]
        wl = workloads.Workload("fold_" + case, E, C, tp, p,
                                workloads.normal((E, C, tp, p, p), 131, std=0.02, dtype=torch.bfloat16),
                                bias, torch.bfloat16, merge=merge, items=items,
                                mean=workloads.CLIP_MEAN, std=workloads.CLIP_STD)
    pe = _pe((wl.E, wl.C, wl.tp, wl.p), wl.weight, wl.bias, wl.mean, wl.std)
    pe.set_temporal_fold(True)
    frames = [it.frames.to(DEV) for it in wl.items]
    out = pe.forward_frames_grouped(frames, [it.grid for it in wl.items], wl.merge, out_dtype=od)
    torch.cuda.synchronize()
    assert pe.last_error() == 0
    mask = None if rows is None else mask_of(rows, wl.N)
    its = [(it.frames, it.grid) for it in wl.items]
    ref_f, mag_f = oracle.conv3d_grouped(its, wl.merge, wl.mean, wl.std, _folded_weight(wl.weight), wl.bias,
                                         wl.C, wl.tp, wl.p, row_mask=mask)
    assert_within_tolerance(out, ref_f, mag_f, rows=rows, what=f"{case} folded-weight oracle")
    ref, mag = oracle.conv3d_grouped(its, wl.merge, wl.mean, wl.std, wl.weight, wl.bias,
                                     wl.C, wl.tp, wl.p, row_mask=mask)
    r = assert_within_tolerance(out, ref, mag, rows=rows, what=f"{case} exact oracle, parity tolerance")
    print(f"fold {case}: worst |err| / tolerance against the exact Conv3d = {r:.3f}")


def test_temporal_fold_leaves_video_and_off_state_alone():
    """Folding applies to single-frame items only; a video item, or the flag off,
    gives the unfolded result bit for bit."""
    C, tp, p, E = 3, 2, 14, 256
    w = workloads.normal((E, C, tp, p, p), 140, std=0.02, dtype=torch.bfloat16)
    vid = workloads.uniform01((4, C, 8 * p, 6 * p), 141).to(DEV)
    img = workloads.uniform01((1, C, 8 * p, 6 * p), 142).to(DEV)
    pe = _pe((E, C, tp, p), w, None, workloads.CLIP_MEAN, workloads.CLIP_STD)
    base_v = pe.forward_frames(vid, (2, 8, 6), 2)
    base_i = pe.forward_frames(img, (1, 8, 6), 2)
    pe.set_temporal_fold(True)
    fold_v = pe.forward_frames(vid, (2, 8, 6), 2)
    fold_i = pe.forward_frames(img, (1, 8, 6), 2)
    pe.set_temporal_fold(False)
    again_i = pe.forward_frames(img, (1, 8, 6), 2)
    torch.cuda.synchronize()
    assert torch.equal(base_v, fold_v)
    assert torch.equal(base_i, again_i)
    assert not torch.equal(base_i, fold_i)   # the folded path really ran


# ------------------------------------------------- position-embedding epilogue

@pytest.mark.parametrize("form,path,pos_dtype,out_dtype", [
    ("frames", "fused", torch.bfloat16, torch.bfloat16),
    ("frames", "staged", torch.float32, torch.bfloat16),
    ("frames", "fused", torch.float32, torch.float32),
    ("frames", "staged", torch.bfloat16, torch.float32),
    ("patches", "-", torch.bfloat16, torch.bfloat16),
    ("patches_f32", "-", torch.float32, torch.float32),
])
def test_position_embedding_add(form, path, pos_dtype, out_dtype, monkeypatch):
    """out = conv + bias + pos with pos a [N, E] table in output row order,
    added in fp32 before the cast (the vision model's hidden_states +
    pos_embeds right after the PatchEmbed).  Reference: the oracle's conv plus
    the table, tolerance over sum|x̂ ŵ| + |pos|."""
    C, tp, p, E = 3, 2, 14, 256
    w = workloads.normal((E, C, tp, p, p), 150, std=0.02, dtype=torch.bfloat16)
    b = workloads.normal((E,), 151, std=0.02, dtype=torch.bfloat16)
    pe = _pe((E, C, tp, p), w, b, workloads.CLIP_MEAN, workloads.CLIP_STD)
    if form == "frames":
        monkeypatch.setenv("PE_FRAMES_PATH", path)
        grids = [(1, 6, 10), (2, 4, 6), (1, 10, 4)]
        Ts = [1, 3, 1]
        items = [(workloads.uniform01((T, C, g[1] * p, g[2] * p), 152 + i), g) for i, (T, g) in enumerate(zip(Ts, grids))]
        N = sum(g[0] * g[1] * g[2] for g in grids)
        pos = workloads.normal((N, E), 160, std=1.0, dtype=pos_dtype)
        out = pe.forward_frames_grouped([f.to(DEV) for f, _ in items], grids, 2, out_dtype=out_dtype, pos=pos.to(DEV))
        ref, mag = oracle.conv3d_grouped(items, 2, workloads.CLIP_MEAN, workloads.CLIP_STD, w, b, C, tp, p)
    else:
        N = 300
        xdt = torch.float32 if form == "patches_f32" else torch.bfloat16
        x = workloads.normal((N, C * tp * p * p), 161, dtype=xdt)
        pos = workloads.normal((N, E), 162, std=1.0, dtype=pos_dtype)
        out = pe.forward_patches(x.to(DEV), out_dtype=out_dtype, pos=pos.to(DEV))
        ref, mag = oracle.conv3d_patches(x, w, b, C, tp, p)
    torch.cuda.synchronize()
    assert pe.last_error() == 0
    pv = pos.double().numpy()
    assert_within_tolerance(out, ref + pv, mag + np.abs(pv), what=f"pos {form} {path}")


@pytest.mark.parametrize("form,pos_dtype", [("patches", torch.bfloat16), ("patches", torch.float32),
                                            ("frames", torch.bfloat16), ("frames", torch.float32)])
def test_position_embedding_ragged_width(form, pos_dtype):
    """E = 200 (six whole 32-column chunks and one of 8 columns) with a bias:
    the last chunk takes the epilogue's guarded table and bias loads, the
    others the unguarded ones.  Against the oracle's conv plus the table."""
    C, tp, p, E = 3, 2, 14, 200
    w = workloads.normal((E, C, tp, p, p), 180, std=0.02, dtype=torch.bfloat16)
    b = workloads.normal((E,), 181, std=0.5)
    pe = _pe((E, C, tp, p), w, b, workloads.CLIP_MEAN, workloads.CLIP_STD)
    if form == "frames":
        grids = [(1, 6, 10), (2, 4, 6)]
        items = [(workloads.uniform01((T, C, g[1] * p, g[2] * p), 182 + i), g)
                 for i, (T, g) in enumerate(zip([1, 3], grids))]
        N = sum(g[0] * g[1] * g[2] for g in grids)
        pos = workloads.normal((N, E), 184, std=1.0, dtype=pos_dtype)
        out = pe.forward_frames_grouped([f.to(DEV) for f, _ in items], grids, 2, out_dtype=torch.float32,
                                        pos=pos.to(DEV))
        ref, mag = oracle.conv3d_grouped(items, 2, workloads.CLIP_MEAN, workloads.CLIP_STD, w, b, C, tp, p)
    else:
        N = 333
        x = workloads.normal((N, C * tp * p * p), 185, dtype=torch.bfloat16)
        pos = workloads.normal((N, E), 186, std=1.0, dtype=pos_dtype)
        out = pe.forward_patches(x.to(DEV), out_dtype=torch.float32, pos=pos.to(DEV))
        ref, mag = oracle.conv3d_patches(x, w, b, C, tp, p)
    torch.cuda.synchronize()
    assert pe.last_error() == 0
    pv = pos.double().numpy()
    assert_within_tolerance(out, ref + pv, mag + np.abs(pv), what=f"pos E=200 {form} {pos_dtype}")


def test_position_embedding_argument_errors():
    C, tp, p, E = 3, 2, 14, 64
    pe = _pe((E, C, tp, p), workloads.normal((E, C, tp, p, p), 170, std=0.02), None)
    x = torch.zeros(8, C * tp * p * p, dtype=torch.bfloat16, device=DEV)
    out = torch.empty(8, E, dtype=torch.bfloat16, device=DEV)
    pos = torch.zeros(8 * E + 8, dtype=torch.bfloat16, device=DEV)
    from vlm_vision_patch_b200 import _binding as B
    s = torch.cuda.current_stream().cuda_stream
    with pytest.raises(PEError) as e:
        B.pe_forward_patches_pos(pe.h, x.data_ptr(), B.PE_BF16, 8, 0, B.PE_BF16, out.data_ptr(), B.PE_BF16, s)
    assert e.value.status == "PE_ERR_INVALID_ARG"
    with pytest.raises(PEError) as e:
        B.pe_forward_patches_pos(pe.h, x.data_ptr(), B.PE_BF16, 8, pos.data_ptr() + 2, B.PE_BF16, out.data_ptr(),
                                 B.PE_BF16, s)
    assert e.value.status == "PE_ERR_ALIGN"
    with pytest.raises(PEError) as e:
        B.pe_forward_patches_pos(pe.h, x.data_ptr(), B.PE_BF16, 8, pos.data_ptr(), 7, out.data_ptr(), B.PE_BF16, s)
    assert e.value.status == "PE_ERR_DTYPE"


@pytest.mark.parametrize("path", ["cast", "threads"])
def test_fp32_patches_both_paths(path, monkeypatch):
    """fp32 rows: cast to bf16 by a separate kernel, then the TMA-fed contraction
    (default), or converted by producer warps inside the contraction kernel.
    Both must be within tolerance of the oracle."""
    C, tp, p, E = 3, 2, 14, 1280
    x = workloads.normal((700, C * tp * p * p), 180)
    w = workloads.kaiming_uniform_conv((E, C, tp, p, p), 181)
    pe = _pe((E, C, tp, p), w, None)
    ref, mag = oracle.conv3d_patches(x, w, None, C, tp, p)
    monkeypatch.setenv("PE_PATCHES_PATH", path)
    out = pe.forward_patches(x.to(DEV), out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert_within_tolerance(out, ref, mag, what=f"fp32 patches {path}")


# ------------------------------------------------------------ tf32 contraction

def _tf32_round(t: torch.Tensor) -> torch.Tensor:
    """fp32 -> nearest tf32 value (10 fraction bits, ties away from zero)."""
    u = t.float().contiguous().view(torch.int32).numpy().astype(np.int64)
    u = ((u + 0x1000) & 0xFFFFE000).astype(np.uint32).view(np.int32)
    return torch.from_numpy(u.copy()).view(torch.float32)


@pytest.mark.parametrize("N,E,bias,out_dtype", [
    (1024, 1280, False, torch.float32),    # the fp32 [1024, 1176] workload shape
    (300, 200, True, torch.float32),       # partial tiles in N and E
    (129, 1280, False, torch.bfloat16),
])
def test_tf32_patches(N, E, bias, out_dtype):
    """Opt-in tf32 contraction of fp32 rows: (1) within the tf32 bound
    (2^-10 + 2^-13) * sum|x w| of the exact fp32-input Conv3d; (2) within fp32
    accumulation (1e-4 * sum) of the oracle on the tf32-rounded values; (3)
    several times closer to the exact result than the default bf16 path."""
    C, tp, p = 3, 2, 14
    K = C * tp * p * p
    x = workloads.normal((N, K), 190 + N)
    w = workloads.kaiming_uniform_conv((E, C, tp, p, p), 191)
    b = workloads.normal((E,), 192, std=0.02) if bias else None
    pe = _pe((E, C, tp, p), w, b)
    xd = x.to(DEV)
    base = pe.forward_patches(xd, out_dtype=torch.float32)        # bf16 compute
    pe.set_tf32(True)
    out = pe.forward_patches(xd, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert pe.last_error() == 0
    ref, mag = oracle.conv3d_patches_fp32(x, w, b, C, tp, p)
    r_tf32 = assert_within_tolerance(out, ref, mag, what="tf32 vs exact", rel=2.0 ** -10 + 2.0 ** -13)
    ref_r, mag_r = oracle.conv3d_patches_fp32(_tf32_round(x), _tf32_round(w), b, C, tp, p)
    assert_within_tolerance(out, ref_r, mag_r, what="tf32 vs tf32-rounded oracle", rel=1e-4)
    if out_dtype == torch.float32:
        err_t = np.abs(out.cpu().double().numpy() - ref) / mag
        err_b = np.abs(base.cpu().double().numpy() - ref) / mag
        assert err_t.mean() * 4 < err_b.mean(), (err_t.mean(), err_b.mean())
    assert r_tf32 <= 1.0


def test_tf32_switch_is_per_handle_and_reversible():
    C, tp, p, E = 3, 2, 14, 256
    x = workloads.normal((64, C * tp * p * p), 195).to(DEV)
    pe = _pe((E, C, tp, p), workloads.normal((E, C, tp, p, p), 196, std=0.05), None)
    a = pe.forward_patches(x, out_dtype=torch.float32)
    pe.set_tf32(True)
    t = pe.forward_patches(x, out_dtype=torch.float32)
    pe.set_tf32(False)
    a2 = pe.forward_patches(x, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(a, a2) and not torch.equal(a, t)
    xb = x.to(torch.bfloat16)           # bf16 rows are unaffected by the switch
    pe.set_tf32(True)
    u = pe.forward_patches(xb, out_dtype=torch.float32)
    pe.set_tf32(False)
    v = pe.forward_patches(xb, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(u, v)


# ------------------------------------------------------------- PatchMerger



def _merger_case(E, m, H, V, bias, wdt, seed):
    m2 = m * m
    D = E * m2
    x = (workloads.normal((V * m2, E), seed) * 0.7 + 0.05).to(torch.bfloat16)
    gamma = (1.0 + workloads.normal((E,), seed + 1, std=0.1)).to(wdt)
    beta = workloads.normal((E,), seed + 2, std=0.05).to(wdt)
    w1 = workloads.normal((D, D), seed + 3, std=D ** -0.5).to(wdt)
    w2 = workloads.normal((H, D), seed + 4, std=D ** -0.5).to(wdt)
    b1 = workloads.normal((D,), seed + 5, std=0.02).to(wdt) if bias else None
    b2 = workloads.normal((H,), seed + 6, std=0.02).to(wdt) if bias else None
    return x, gamma, beta, w1, b1, w2, b2


@pytest.mark.parametrize("E,m,H,V,bias,wdt,out_dtype", [
    (1280, 2, 1536, 64, True, torch.bfloat16, torch.bfloat16),    # Qwen2-VL: 5120 -> 5120 -> 1536
    (1152, 2, 1024, 37, False, torch.float32, torch.float32),     # ragged V, fp32 weights
    (64, 1, 128, 300, True, torch.bfloat16, torch.float32),       # m = 1
])
def test_patch_merger(E, m, H, V, bias, wdt, out_dtype):
    """GPU PatchMerger vs the oracle at the parity tolerance 1e-3 * sum|g w2|
    (+ 1 bf16 ulp for bf16 output), g the bf16 GELU output.  The GPU rounds the
    LayerNorm and GELU outputs to bf16 like the oracle, but from fp32 rather
    than fp64 values: an element lands one bf16 ulp away only when its fp32 and
    fp64 values straddle a rounding boundary (a few per row), and one such term
    moves an output by about 2^-8 of one of the D terms of sum|g w2|.  The
    worst ratio is printed."""
    x, gamma, beta, w1, b1, w2, b2 = _merger_case(E, m, H, V, bias, wdt, 500 + E + V)
    pm = PatchMerger(E, m, H, 1e-6)
    dev = lambda t: None if t is None else t.to(DEV).contiguous()
    pm.set_weights(dev(gamma), dev(beta), dev(w1), dev(b1), dev(w2), dev(b2))
    out = pm.forward(x.to(DEV), out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert pm.last_error() == 0
    ref, mag = oracle.patch_merger(x, m * m, gamma, beta, 1e-6, w1, b1, w2, b2)
    r = assert_within_tolerance(out, ref, mag, what=f"merger {E},{m},{H},{V}")
    print(f"merger {E},{m},{H},{V}: worst |err| / tolerance = {r:.3f}")
    pm.close()


def test_patch_merger_full_size_sampled():
    """The merger on config-4-sized input (59204 patch rows -> 14801 merged rows,
    5120 -> 5120 -> 1536), sampled merged rows incl. the first and last."""
    E, m, H = 1280, 2, 1536
    V = 14801
    x, gamma, beta, w1, b1, w2, b2 = _merger_case(E, m, H, V, True, torch.bfloat16, 600)
    pm = PatchMerger(E, m, H, 1e-6)
    pm.set_weights(*(None if t is None else t.to(DEV) for t in (gamma, beta, w1, b1, w2, b2)))
    out = pm.forward(x.to(DEV))
    torch.cuda.synchronize()
    assert pm.last_error() == 0
    rows = sample_rows(V, 24, 601)
    ref, mag = oracle.patch_merger(x, 4, gamma, beta, 1e-6, w1, b1, w2, b2, v_mask=mask_of(rows, V))
    r = assert_within_tolerance(out, ref, mag, rows=rows, what="merger full size")
    print(f"merger full size: worst |err| / tolerance = {r:.3f}")
    pm.close()


def test_patch_merger_errors():
    pm = PatchMerger(64, 2, 128)
    x = torch.zeros(8, 64, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(PEError) as e:
        pm.forward(x)
    assert e.value.status == "PE_ERR_NO_WEIGHT"
    z = lambda *s: torch.zeros(*s, dtype=torch.bfloat16, device=DEV)
    pm.set_weights(z(64), z(64), z(256, 256), None, z(128, 256), None)
    with pytest.raises(PEError) as e:
        pm.forward(torch.zeros(6, 64, dtype=torch.bfloat16, device=DEV))   # 6 rows: not whole 2x2 windows
    assert e.value.status == "PE_ERR_SHAPE"
    pm.close()


# ------------------------------------------------------ more path/shape cases

@pytest.mark.parametrize("case", ["staged_E200_bias_f32", "staged_merge1_odd_gw_p16", "fold_with_pos",
                                  "fold_with_f32_pos_f32_out", "tf32_with_pos"])
def test_more_path_combinations(case, monkeypatch):
    """Combinations of options and ragged shapes on the default paths, each
    against the oracle at the parity tolerance (the tf32 case against the
    unrounded oracle at the tf32 bound)."""
    C, tp = 3, 2
    if case.startswith("tf32"):
        p, E, N = 14, 256, 200
        K = C * tp * p * p
        x = workloads.normal((N, K), 700)
        w = workloads.normal((E, C, tp, p, p), 701, std=0.03)
        pos = workloads.normal((N, E), 702, std=0.5)
        pe = _pe((E, C, tp, p), w, None)
        pe.set_tf32(True)
        out = pe.forward_patches(x.to(DEV), out_dtype=torch.float32, pos=pos.to(DEV))
        torch.cuda.synchronize()
        ref, mag = oracle.conv3d_patches_fp32(x, w, None, C, tp, p)
        pv = pos.double().numpy()
        assert_within_tolerance(out, ref + pv, mag + np.abs(pv), what=case, rel=2.0 ** -10 + 2.0 ** -13)
        return
    if case == "staged_E200_bias_f32":
        p, E, merge, grids, Ts, od = 14, 200, 2, [(2, 6, 8), (1, 4, 10)], [3, 1], torch.float32
    elif case == "staged_merge1_odd_gw_p16":
        p, E, merge, grids, Ts, od = 16, 384, 1, [(1, 5, 7), (2, 3, 9)], [1, 4], torch.bfloat16
    elif case == "fold_with_pos":
        p, E, merge, grids, Ts, od = 14, 512, 2, [(1, 8, 12), (1, 6, 6)], [1, 1], torch.bfloat16
    else:   # an fp32 table and fp32 rows through the folded path's register stores
        p, E, merge, grids, Ts, od = 14, 200, 2, [(1, 8, 12), (1, 6, 6)], [1, 1], torch.float32
    items = [(workloads.uniform01((T, C, g[1] * p, g[2] * p), 710 + i), g) for i, (T, g) in enumerate(zip(Ts, grids))]
    w = workloads.normal((E, C, tp, p, p), 720, std=0.02, dtype=torch.bfloat16)
    b = workloads.normal((E,), 721, std=0.02, dtype=torch.bfloat16)
    pe = _pe((E, C, tp, p), w, b, workloads.CLIP_MEAN, workloads.CLIP_STD)
    N = sum(g[0] * g[1] * g[2] for g in grids)
    pos = None
    if case.startswith("fold_with"):
        pe.set_temporal_fold(True)
        pos = workloads.normal((N, E), 722, std=0.5, dtype=torch.bfloat16 if case == "fold_with_pos" else torch.float32)
    out = pe.forward_frames_grouped([f.to(DEV) for f, _ in items], grids, merge, out_dtype=od,
                                    pos=None if pos is None else pos.to(DEV))
    torch.cuda.synchronize()
    assert pe.last_error() == 0
    ref, mag = oracle.conv3d_grouped(items, merge, workloads.CLIP_MEAN, workloads.CLIP_STD, w, b, C, tp, p)
    if pos is not None:
        pv = pos.double().numpy()
        ref, mag = ref + pv, mag + np.abs(pv)
    assert_within_tolerance(out, ref, mag, what=case)


# ----------------------------------------------- Qwen3-VL PatchEmbed shape

QWEN3 = dict(C=3, tp=2, p=16, E=1024)   # Optimize VLM PatchEmbed: Qwen3VLVisionPatchEmbed, bias=True, 2B hidden size


def test_qwen3_vl_shape_frames():
    """Qwen3VLVisionPatchEmbed's shape (patch 16, temporal 2, hidden 1024, with
    bias) on frames: an image and a video with an odd frame count in one
    grouped call, merge order, every row against the oracle."""
    C, tp, p, E = QWEN3["C"], QWEN3["tp"], QWEN3["p"], QWEN3["E"]
    grids, Ts = [(1, 12, 16), (2, 8, 10)], [1, 3]
    items = [(workloads.uniform01((T, C, g[1] * p, g[2] * p), 800 + i), g) for i, (T, g) in enumerate(zip(Ts, grids))]
    w = workloads.normal((E, C, tp, p, p), 801, std=0.02, dtype=torch.bfloat16)
    b = workloads.normal((E,), 802, std=0.02, dtype=torch.bfloat16)
    pe = _pe((E, C, tp, p), w, b, workloads.CLIP_MEAN, workloads.CLIP_STD)
    for od in (torch.bfloat16, torch.float32):
        out = pe.forward_frames_grouped([f.to(DEV) for f, _ in items], grids, 2, out_dtype=od)
        torch.cuda.synchronize()
        assert pe.last_error() == 0
        ref, mag = oracle.conv3d_grouped(items, 2, workloads.CLIP_MEAN, workloads.CLIP_STD, w, b, C, tp, p)
        assert_within_tolerance(out, ref, mag, what=f"Qwen3-VL frames {od}")


@pytest.mark.parametrize("x_dtype", [torch.bfloat16, torch.float32])
def test_qwen3_vl_shape_patches(x_dtype):
    """The same shape on patch rows [N, 1536] (the processor's pixel_values),
    N ragged against the 256-row tiles."""
    C, tp, p, E = QWEN3["C"], QWEN3["tp"], QWEN3["p"], QWEN3["E"]
    K = C * tp * p * p
    x = workloads.normal((777, K), 810)
    w = workloads.normal((E, C, tp, p, p), 811, std=0.02)
    b = workloads.normal((E,), 812, std=0.02)
    pe = _pe((E, C, tp, p), w, b)
    out = pe.forward_patches(x.to(x_dtype).to(DEV), out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert pe.last_error() == 0
    ref, mag = oracle.conv3d_patches(x.to(x_dtype), w, b, C, tp, p)
    assert_within_tolerance(out, ref, mag, what=f"Qwen3-VL patches {x_dtype}")
