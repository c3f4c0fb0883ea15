"""Host-buffer calls (pe_forward_frames_grouped_host, pe_forward_patches_host)
against the oracle: host frames or rows in, host embeddings out, the work cut
into chunks whose copies and contractions are pipelined over two device slots
per direction.  PE_HOST_CHUNK_ROWS forces small chunks so that many chunks,
slot reuse and the temporal split of a video are all exercised; with a single
chunk the call must equal the device-pointer call bit for bit."""
from __future__ import annotations

import pytest
import torch

import oracle
import workloads
from vlm_vision_patch_b200 import PatchEmbed, PEError
from tests.gpu_util import assert_within_tolerance, mask_of, sample_rows

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
C, TP, P, E = 3, 2, 14, 256
K = C * TP * P * P
GRIDS = [(1, 8, 10), (5, 6, 4), (1, 12, 12), (2, 4, 4), (1, 2, 2)]
TS = [1, 9, 1, 3, 1]          # 9 frames: five temporal patches, the last one a single frame


def _handle(seed: int, bias: bool = True):
    w = workloads.normal((E, C, TP, P, P), seed, std=0.02, dtype=torch.bfloat16)
    b = workloads.normal((E,), seed + 1, std=0.02, dtype=torch.bfloat16) if bias else None
    pe = PatchEmbed(E, C, TP, P, bias)
    pe.set_weight(w.to(DEV), None if b is None else b.to(DEV))
    pe.set_norm(workloads.CLIP_MEAN, workloads.CLIP_STD)
    return pe, w, b


def _items(seed: int, fdt=torch.bfloat16):
    return [(workloads.uniform01((T, C, g[1] * P, g[2] * P), seed + i, dtype=fdt), g)
            for i, (T, g) in enumerate(zip(TS, GRIDS))]


def _chunks(monkeypatch, rows):
    if rows is None:
        monkeypatch.delenv("PE_HOST_CHUNK_ROWS", raising=False)
    else:
        monkeypatch.setenv("PE_HOST_CHUNK_ROWS", str(rows))


@pytest.mark.parametrize("chunk", [None, 1, 50, 100, 1000])
@pytest.mark.parametrize("pinned", [True, False])
def test_grouped_host_all_rows(chunk, pinned, monkeypatch):
    _chunks(monkeypatch, chunk)
    pe, w, b = _handle(800)
    items = _items(810)
    frames = [f.pin_memory() if pinned else f for f, _ in items]
    out = pe.forward_frames_grouped_host(frames, [g for _, g in items], 2)
    assert out.device.type == "cpu"
    assert pe.last_error() == 0
    ref, mag = oracle.conv3d_grouped(items, 2, workloads.CLIP_MEAN, workloads.CLIP_STD, w, b, C, TP, P)
    assert_within_tolerance(out, ref, mag, what=f"host grouped, chunk {chunk}, pinned {pinned}")


@pytest.mark.parametrize("merge", [1, 2])
def test_grouped_host_fp32_frames_and_output(merge, monkeypatch):
    _chunks(monkeypatch, 64)
    pe, w, b = _handle(820)
    items = _items(830, fdt=torch.float32)
    out = pe.forward_frames_grouped_host([f.pin_memory() for f, _ in items], [g for _, g in items], merge,
                                         out_dtype=torch.float32)
    assert pe.last_error() == 0 and out.dtype == torch.float32
    ref, mag = oracle.conv3d_grouped(items, merge, workloads.CLIP_MEAN, workloads.CLIP_STD, w, b, C, TP, P)
    assert_within_tolerance(out, ref, mag, what=f"host grouped fp32, merge {merge}")


def test_grouped_host_one_chunk_equals_device_call(monkeypatch):
    """380 rows: a single chunk holding the whole call, so the host call runs
    exactly the device-pointer call on copies of the frames."""
    _chunks(monkeypatch, None)
    pe, _, _ = _handle(840)
    items = _items(850)
    grids = [g for _, g in items]
    dev = pe.forward_frames_grouped([f.to(DEV) for f, _ in items], grids, 2).cpu()
    host = pe.forward_frames_grouped_host([f.pin_memory() for f, _ in items], grids, 2)
    assert torch.equal(dev.view(torch.int16), host.view(torch.int16))


def test_grouped_host_repeat_and_side_stream(monkeypatch):
    """Slots reused across calls, and a caller stream other than the current one."""
    _chunks(monkeypatch, 50)
    pe, _, _ = _handle(860)
    items = _items(870)
    frames = [f.pin_memory() for f, _ in items]
    grids = [g for _, g in items]
    a = pe.forward_frames_grouped_host(frames, grids, 2)
    b = pe.forward_frames_grouped_host(frames, grids, 2)
    s = torch.cuda.Stream()
    c = pe.forward_frames_grouped_host(frames, grids, 2, stream=s)
    assert pe.last_error() == 0
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(a.view(torch.int16), c.view(torch.int16))


@pytest.mark.parametrize("xdt", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("chunk", [None, 300, 256])
def test_patches_host(xdt, chunk, monkeypatch):
    _chunks(monkeypatch, chunk)
    pe, w, b = _handle(880)
    N = 1000
    x = workloads.normal((N, K), 890, dtype=xdt)
    out = pe.forward_patches_host(x.pin_memory())
    assert pe.last_error() == 0
    ref, mag = oracle.conv3d_patches(x, w, b, C, TP, P)
    assert_within_tolerance(out, ref, mag, what=f"host patches {xdt}, chunk {chunk}")
    if chunk is None:   # one chunk: the device-pointer call exactly
        dev = pe.forward_patches(x.to(DEV)).cpu()
        assert torch.equal(dev.view(torch.int16), out.view(torch.int16))


def test_patches_host_empty():
    pe, _, _ = _handle(895)
    out = pe.forward_patches_host(torch.zeros(0, K, dtype=torch.bfloat16))
    assert out.shape == (0, E)


def test_grouped_host_16_images_default_chunks(monkeypatch):
    """The 16-image grouped workload (59204 rows) at the default chunking
    (about eight chunks of whole images), sampled rows incl. item boundaries."""
    _chunks(monkeypatch, None)
    wl = workloads.grouped_16_images()
    pe = PatchEmbed(wl.E, wl.C, wl.tp, wl.p, False)
    pe.set_weight(wl.weight.to(DEV))
    pe.set_norm(wl.mean, wl.std)
    grids = [it.grid for it in wl.items]
    out = pe.forward_frames_grouped_host([it.frames.pin_memory() for it in wl.items], grids, wl.merge)
    assert pe.last_error() == 0
    bounds, off = [], 0
    for g in grids:
        n = g[0] * g[1] * g[2]
        bounds += [off, off + n - 1]
        off += n
    rows = sample_rows(off, 1500, 900, bounds)
    ref, mag = oracle.conv3d_grouped([(it.frames, it.grid) for it in wl.items], wl.merge, wl.mean, wl.std,
                                     wl.weight, None, wl.C, wl.tp, wl.p, row_mask=mask_of(rows, off))
    assert_within_tolerance(out, ref, mag, rows=rows, what="host grouped 16 images")


def test_long_video_host_temporal_chunks(monkeypatch):
    """[64, 3, 896, 896], grid (32, 64, 64): the default chunking cuts the one
    video into runs of whole temporal patches; sampled rows incl. every chunk
    boundary region."""
    _chunks(monkeypatch, None)
    wl = workloads.long_video_64x896()
    pe = PatchEmbed(wl.E, wl.C, wl.tp, wl.p, False)
    pe.set_weight(wl.weight.to(DEV))
    pe.set_norm(wl.mean, wl.std)
    it = wl.items[0]
    N = it.grid[0] * it.grid[1] * it.grid[2]
    out = pe.forward_frames_grouped_host([it.frames.pin_memory()], [it.grid], wl.merge)
    assert pe.last_error() == 0
    slab = it.grid[1] * it.grid[2]
    edges = [t * slab + d for t in range(it.grid[0]) for d in (-1, 0)]
    rows = sample_rows(N, 400, 910, edges)
    ref, mag = oracle.conv3d_grouped([(it.frames, it.grid)], wl.merge, wl.mean, wl.std, wl.weight, None,
                                     wl.C, wl.tp, wl.p, row_mask=mask_of(rows, N))
    assert_within_tolerance(out, ref, mag, rows=rows, what="host long video")


def test_host_call_errors(monkeypatch):
    _chunks(monkeypatch, None)
    pe, _, _ = _handle(920)
    f = workloads.uniform01((1, C, 28, 28), 921)
    for grid, merge, code in [((1, 2, 3), 2, "PE_ERR_SHAPE"), ((2, 2, 2), 2, "PE_ERR_SHAPE"),
                              ((1, 2, 2), 3, "PE_ERR_INVALID_ARG")]:
        with pytest.raises(PEError) as e:
            pe.forward_frames_grouped_host([f], [grid], merge)
        assert e.value.status == code
    fresh = PatchEmbed(E, C, TP, P, False)
    with pytest.raises(PEError) as e:
        fresh.forward_patches_host(torch.zeros(4, K, dtype=torch.bfloat16))
    assert e.value.status == "PE_ERR_NO_WEIGHT"
    torch.cuda.synchronize()
    assert pe.last_error() == 0
