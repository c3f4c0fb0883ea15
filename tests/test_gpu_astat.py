"""The resident-A frames kernel (single images, one launch) vs the CPU oracle.

Groups whose items are all single frames (T = 1, duplicated to tp = 2) run
through pe_astat_kernel with PE_FRAMES_PATH=astat and in the allocation-free
call: each 256-row block's normalised A is built
once in shared memory from the raw frames and every weight tile streams past
it, so the [N, K] patch matrix never exists in global memory (patch详解 §4.3,
the Conv3d cuts and projects in one step).  Checked here:
  - parity with the oracle at the tolerance of the other GPU tests
    (1e-3 * sum|x̂ ŵ| per element, + one bf16 ulp for bf16 output);
  - bit-equality with the staged path, which issues the same MMAs in the same
    order on the same bf16 operands (a row's k-step meets slice 0 then
    slice 1 of the weight), so any difference is an indexing error;
  - one kernel launch per call;
  - every weight-ring depth and staging-buffer count the planner can pick,
    every tile width, M-block switches inside a pair's range, ragged N,
    both merge orders, bias / no bias, fp32 / bf16 output, the fused
    position-table add, per-channel normalisation modes, generic patch sizes,
    more items than fit inline (device item table).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from vlm_vision_patch_b200 import PatchEmbed, _binding as B
from tests.gpu_util import assert_within_tolerance, mask_of, sample_rows

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
C, TP = 3, 2


def _wl(grids, E=1280, p=14, merge=2, bias=True, seed=200, mean=workloads.CLIP_MEAN, std=workloads.CLIP_STD):
    items = [workloads.Item(workloads.uniform01((1, C, g[1] * p, g[2] * p), seed + i), g) for i, g in enumerate(grids)]
    return workloads.Workload(f"astat_{len(grids)}", E, C, TP, p,
                              workloads.normal((E, C, TP, p, p), seed + 99, std=0.02, dtype=torch.bfloat16),
                              workloads.normal((E,), seed + 98, std=0.02, dtype=torch.bfloat16) if bias else None,
                              torch.bfloat16, merge=merge, items=items, mean=mean, std=std)


def _pe(wl):
    pe = PatchEmbed(wl.E, C, TP, wl.p, wl.bias is not None)
    pe.set_weight(wl.weight.to(DEV), None if wl.bias is None else wl.bias.to(DEV))
    pe.set_norm(wl.mean, wl.std)
    return pe


def _forward(pe, wl, frames, out_dtype, path, monkeypatch, pos=None):
    monkeypatch.setenv("PE_FRAMES_PATH", path)
    B.pe_profile_begin(pe.h, 0)
    out = pe.forward_frames_grouped(frames, [it.grid for it in wl.items], wl.merge, out_dtype=out_dtype, pos=pos)
    _, launches = B.pe_profile_end(pe.h, 0)
    torch.cuda.synchronize()
    assert pe.last_error() == 0
    return out, launches


def _oracle(wl, rows=None):
    mask = None if rows is None else mask_of(rows, wl.N)
    return oracle.conv3d_grouped([(it.frames, it.grid) for it in wl.items], wl.merge, wl.mean, wl.std, wl.weight,
                                 wl.bias, C, TP, wl.p, row_mask=mask)


CASES = {
    # name: (grids, E, merge, bias, out dtype)
    "image_224x896": ([(1, 16, 64)], 1280, 2, False, torch.bfloat16),
    "three_ragged": ([(1, 12, 18), (1, 20, 10), (1, 8, 8)], 1280, 2, True, torch.bfloat16),
    "raster_e1152_f32": ([(1, 7, 9), (1, 5, 11), (1, 13, 3)], 1152, 1, True, torch.float32),
    "image_448_e1152": ([(1, 32, 32)], 1152, 2, False, torch.bfloat16),
    "tiny_4_rows": ([(1, 2, 2)], 1280, 2, True, torch.float32),
    "e16": ([(1, 6, 8), (1, 4, 4)], 16, 2, True, torch.bfloat16),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_astat_matches_oracle_and_staged_bitwise(name, monkeypatch):
    grids, E, merge, bias, od = CASES[name]
    wl = _wl(grids, E=E, merge=merge, bias=bias)
    pe = _pe(wl)
    frames = [it.frames.to(DEV) for it in wl.items]
    out_a, launches = _forward(pe, wl, frames, od, "astat", monkeypatch)
    assert launches == 1, "one launch from frames to embeddings"
    out_s, launches_s = _forward(pe, wl, frames, od, "staged", monkeypatch)
    assert launches_s == 2
    ref, mag = _oracle(wl)
    assert_within_tolerance(out_a, ref, mag, what=f"resident A {name}")
    assert torch.equal(out_a, out_s), "resident-A and staged outputs differ"


@pytest.mark.parametrize("bn", ["64", "128", "256"])
def test_astat_every_tile_width(bn, monkeypatch):
    monkeypatch.setenv("PE_BN", bn)
    wl = _wl([(1, 12, 18), (1, 20, 10), (1, 8, 8)], E=1280)
    pe = _pe(wl)
    frames = [it.frames.to(DEV) for it in wl.items]
    out_a, _ = _forward(pe, wl, frames, torch.bfloat16, "astat", monkeypatch)
    out_s, _ = _forward(pe, wl, frames, torch.bfloat16, "staged", monkeypatch)
    ref, mag = _oracle(wl)
    assert_within_tolerance(out_a, ref, mag, what=f"resident A BN={bn}")
    assert torch.equal(out_a, out_s)


@pytest.mark.parametrize("bn,nb,bufs", [("256", 2, 0), ("128", 2, 2), ("128", 3, 1), ("128", 4, 0),
                                         ("64", 2, 2), ("64", 6, 2), ("64", 5, 0)])
def test_astat_ring_depths_and_staging(bn, nb, bufs, monkeypatch):
    """Weight-ring depths and epilogue forms the planner can choose (staging
    boxes for TMA stores, or stores straight from registers when no boxes fit)
    give the same bits (the pipeline shape changes no arithmetic)."""
    wl = _wl([(1, 20, 24), (1, 16, 10), (1, 6, 14)], E=1280, seed=230)
    pe = _pe(wl)
    frames = [it.frames.to(DEV) for it in wl.items]
    monkeypatch.setenv("PE_BN", bn)
    base, _ = _forward(pe, wl, frames, torch.bfloat16, "staged", monkeypatch)
    monkeypatch.setenv("PE_ASTAT_NB", str(nb))
    monkeypatch.setenv("PE_ASTAT_EPIBUFS", str(bufs))
    out, launches = _forward(pe, wl, frames, torch.bfloat16, "astat", monkeypatch)
    assert launches == 1
    assert torch.equal(out, base)


def test_astat_block_switches_within_a_pair(monkeypatch):
    """Enough rows that every CTA pair's range crosses several M-blocks
    (each block's A rebuilt while the previous block's last pass drains):
    bit-equal to the staged path on every row, and the oracle on sampled rows
    including every item boundary."""
    grids = [(1, 32, 32)] * 40 + [(1, 10, 6)] * 3     # 41140 rows: 161 blocks of 256 rows
    wl = _wl(grids, E=1280, seed=240)
    pe = _pe(wl)
    frames = [it.frames.to(DEV) for it in wl.items]
    out_a, _ = _forward(pe, wl, frames, torch.bfloat16, "astat", monkeypatch)
    out_s, _ = _forward(pe, wl, frames, torch.bfloat16, "staged", monkeypatch)
    assert torch.equal(out_a, out_s)
    bounds, off = [], 0
    for g in grids:
        n = g[0] * g[1] * g[2]
        bounds += [off, off + n - 1]
        off += n
    rows = sample_rows(wl.N, 1500, 241, bounds)
    ref, mag = _oracle(wl, rows)
    assert_within_tolerance(out_a, ref, mag, rows=rows, what="block switches")


@pytest.mark.parametrize("pos_dtype,out_dtype", [(torch.bfloat16, torch.bfloat16), (torch.float32, torch.float32)])
def test_astat_position_table(pos_dtype, out_dtype, monkeypatch):
    wl = _wl([(1, 6, 10), (1, 10, 4), (1, 8, 8)], E=256, seed=250)
    pe = _pe(wl)
    frames = [it.frames.to(DEV) for it in wl.items]
    pos = workloads.normal((wl.N, wl.E), 251, std=1.0, dtype=pos_dtype)
    out, launches = _forward(pe, wl, frames, out_dtype, "astat", monkeypatch, pos=pos.to(DEV))
    assert launches == 1
    ref, mag = _oracle(wl)
    pv = pos.double().numpy()
    assert_within_tolerance(out, ref + pv, mag + np.abs(pv), what="resident A + position table")


@pytest.mark.parametrize("mean,std", [((0.0, 0.0, 0.0), (1.0, 1.0, 1.0)),          # identity: raw words
                                      ((0.0, 0.5, 0.25), (1.0, 0.25, 3.0)),        # identity in one channel
                                      ((1e-30, -0.3, 0.7), (0.2, 1e12, 1.0))])      # IEEE divide in two channels
def test_astat_normalisation_modes(mean, std, monkeypatch):
    wl = _wl([(1, 8, 12), (1, 4, 6)], E=512, seed=260, mean=mean, std=std)
    pe = _pe(wl)
    frames = [it.frames.to(DEV) for it in wl.items]
    out_a, _ = _forward(pe, wl, frames, torch.float32, "astat", monkeypatch)
    out_s, _ = _forward(pe, wl, frames, torch.float32, "staged", monkeypatch)
    ref, mag = _oracle(wl)
    assert_within_tolerance(out_a, ref, mag, what=f"resident A norm {mean} {std}")
    assert torch.equal(out_a, out_s)


@pytest.mark.parametrize("p,E", [(8, 256), (6, 96), (2, 64), (12, 1280)])
def test_astat_other_patch_sizes(p, E, monkeypatch):
    """Patch sizes other than 14 run the same kernel with run-time index
    arithmetic (p = 12: K = 864, a 432-column resident A)."""
    wl = _wl([(1, 6, 8), (1, 10, 4)], E=E, p=p, seed=270 + p)
    pe = _pe(wl)
    frames = [it.frames.to(DEV) for it in wl.items]
    out, launches = _forward(pe, wl, frames, torch.float32, "astat", monkeypatch)
    assert launches == 1
    ref, mag = _oracle(wl)
    assert_within_tolerance(out, ref, mag, what=f"resident A p={p}")


def test_astat_many_items_device_table(monkeypatch):
    rng = np.random.default_rng(280)
    grids = [(1, int(2 * rng.integers(1, 5)), int(2 * rng.integers(1, 5))) for _ in range(40)]
    wl = _wl(grids, E=256, seed=281)
    pe = _pe(wl)
    frames = [it.frames.to(DEV) for it in wl.items]
    out, launches = _forward(pe, wl, frames, torch.bfloat16, "astat", monkeypatch)
    assert launches == 1
    ref, mag = _oracle(wl)
    assert_within_tolerance(out, ref, mag, what="resident A, 40 items")


@pytest.mark.parametrize("bn,launches", [("64", 1), ("256", 2)])
def test_p16_images_resident_when_the_ring_fits(bn, launches, monkeypatch):
    """p = 16 makes a 768-column A (192 KB): beside 64-wide weight tiles (4 KB
    stages) it still fits and the call is one resident-A launch; with 256-wide
    tiles (16 KB stages) it does not, and the call runs the staged pair.  Both
    within tolerance of the oracle."""
    monkeypatch.setenv("PE_BN", bn)
    wl = _wl([(1, 6, 8), (1, 4, 10)], E=1024, p=16, seed=290)
    pe = _pe(wl)
    frames = [it.frames.to(DEV) for it in wl.items]
    out, n = _forward(pe, wl, frames, torch.bfloat16, "astat", monkeypatch)
    assert n == launches
    ref, mag = _oracle(wl)
    assert_within_tolerance(out, ref, mag, what=f"p=16 images, BN={bn}")
