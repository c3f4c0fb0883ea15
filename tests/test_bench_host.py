"""Host logic of bench.py's multi-rank run, on CPU: world_size-2 gloo ranks
(127.0.0.1 rendezvous) agree on the slowest rank's time, and the whole-job
value counts every rank's units over that time (weak scaling).  Also the
reference arm's rank rule: only rank 0 works and prints."""
import io
import contextlib
import json
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    local_ms = [12.5, 40.0][rank]
    m = bench.max_over_ranks(local_ms, dist, "cpu")
    v = bench.weak_scaling_value(1000, 4, world, m)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, m, v))


def test_two_gloo_ranks_agree_on_slowest_time_and_weak_scaling_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, m, v in got:
        assert m == 40.0
        assert v == pytest.approx(1000 * 4 * 2 / 0.040)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.weak_scaling_value(10, 2, 1, 20.0) == pytest.approx(1000.0)


def test_reference_arm_other_ranks_exit_without_output():
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        ns = type("A", (), dict(workload="image_224x896", ref_rows=8, steps=1, warmup=3))()
        assert bench.run_reference(ns, 1, 2) == 0
    assert buf.getvalue() == ""


def test_reference_arm_prints_one_line_on_rank0():
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        assert bench.main(["--impl", "reference", "--workload", "image_224x896", "--ref-rows", "8",
                           "--steps", "1", "--warmup", "3"]) == 0
    line = json.loads(buf.getvalue().strip())
    assert line["impl"] == "reference" and line["unit"] == "patches/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0


class _FakeNVML:
    """Three GPUs of a machine, as NVML numbers them (PCI order)."""

    class _Pci:
        def __init__(self, domain, bus, device):
            self.domain, self.bus, self.device = domain, bus, device

    def __init__(self):
        self.gpus = [(0, 0x1B, 0, b"GPU-aaaa"), (0, 0x43, 0, b"GPU-bbbb"), (0, 0x52, 0, b"GPU-cccc")]

    def nvmlDeviceGetCount(self):
        return len(self.gpus)

    def nvmlDeviceGetHandleByIndex(self, i):
        return i

    def nvmlDeviceGetPciInfo(self, h):
        return self._Pci(*self.gpus[h][:3])

    def nvmlDeviceGetUUID(self, h):
        return self.gpus[h][3]


def _props(domain, bus, device, uuid=""):
    return type("P", (), dict(pci_domain_id=domain, pci_bus_id=bus, pci_device_id=device, uuid=uuid))()


def test_clock_sampler_finds_the_cuda_device_among_all_gpus():
    """With CUDA_VISIBLE_DEVICES picking one GPU of several, CUDA device 0 is
    not NVML's GPU 0: the sampler must read the GPU at the same PCI location."""
    nv = _FakeNVML()
    assert bench.nvml_handle_for(nv, _props(0, 0x43, 0)) == (1, "pci")
    assert bench.nvml_handle_for(nv, _props(0, 0x52, 0)) == (2, "pci")
    assert bench.nvml_handle_for(nv, _props(0, 0x99, 0, "cccc")) == (2, "uuid")
    assert bench.nvml_handle_for(nv, _props(0, 0x99, 0)) == (None, None)


def test_reference_arm_for_the_merger():
    """--impl reference --merger times the CPU PatchMerger oracle with the merger
    arm's metric and unit."""
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        assert bench.main(["--impl", "reference", "--merger", "--workload", "image_224x896", "--ref-rows", "8",
                           "--steps", "1", "--warmup", "3"]) == 0
    line = json.loads(buf.getvalue().strip())
    assert line["impl"] == "reference" and line["metric"] == bench.MERGER_METRIC and line["unit"] == "patches/s"
    assert line["value"] > 0 and line["config"]["merged_rows"] == 256


def test_merger_weights_are_seeded():
    a, b = bench.merger_weights(64, 32), bench.merger_weights(64, 32)
    assert [t.shape for t in a] == [(64,), (64,), (256, 256), (256,), (32, 256), (32,)]
    assert all(torch.equal(x, y) for x, y in zip(a, b))


def test_reference_arm_for_tf32_times_the_fp32_form():
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        assert bench.main(["--impl", "reference", "--tf32", "--workload", "patches_fp32_1024", "--ref-rows", "8",
                           "--steps", "1", "--warmup", "3"]) == 0
    line = json.loads(buf.getvalue().strip())
    assert line["value"] > 0 and "unrounded fp32" in line["cpu_baseline"]["sample"]


@pytest.mark.parametrize("T,gh,gw,merge,tp,p", [(1, 4, 6, 2, 2, 14), (3, 2, 4, 2, 2, 4), (5, 6, 2, 2, 2, 3),
                                                 (2, 3, 5, 1, 2, 2), (4, 2, 2, 2, 1, 6)])
def test_eager_torch_rows_match_the_oracle_patchify(T, gh, gw, merge, tp, p):
    """The eager-torch context form of the path builds the oracle's rows bit
    for bit (normalisation, temporal padding, merge order)."""
    import numpy as np
    import oracle
    import workloads
    C = 3
    frames = workloads.uniform01((T, C, gh * p, gw * p), 77 + T)
    grid = (-(-T // tp), gh, gw)
    got = bench.torch_patch_rows(frames, grid, merge, workloads.CLIP_MEAN, workloads.CLIP_STD, tp, p)
    ref = oracle.patchify(frames, grid, merge, workloads.CLIP_MEAN, workloads.CLIP_STD, C, tp, p)
    assert got.dtype == torch.bfloat16
    assert np.array_equal(got.float().numpy().view(np.uint32), ref.view(np.uint32))


def test_measured_traffic_belongs_to_one_kernel_form_and_source(monkeypatch):
    """The per-launch DRAM figure is reported only for the kernel form it was
    captured on (a folded, position-table or tf32 launch has its own key) and
    only while the kernel sources still hash to the digest of the capture."""
    key = ("grouped_16_images", "staged")
    rec = bench.TRAFFIC[key]
    sha = bench.kernel_sha()
    if rec["kernel_sha"] == sha:
        assert bench.measured_traffic(*key) == rec["bytes"]
    assert bench.measured_traffic("grouped_16_images", "staged_pos") is None
    assert bench.measured_traffic("grouped_16_images", "no_such_path") is None
    monkeypatch.setattr(bench, "kernel_sha", lambda: "0" * 16)
    assert bench.measured_traffic(*key) is None
    # comments do not change the digest; code does
    base = bench.code_digest(["int a; // x\n", "/* y */ int b;"])
    assert bench.code_digest(["int a;  // other\n", "int b; /* z */"]) == base
    assert bench.code_digest(["int a = 1;", "int b;"]) != base
