"""Benchmark of the vision PatchEmbed on B200: raw frames (or patch rows) in,
embeddings out.

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step is one pass of the whole hot path over one batch of synthetic input:
host plan, then the kernels of the path the library takes for the workload,
over every item.  For groups of single images (the default workload, 16
images in one grouped call) that is one launch of the resident-A kernel: each
256-row block's patches are gathered from the frames, normalised and placed in
merge order once in shared memory, and every weight tile streams past them
(tcgen05 pair MMAs, bias/cast epilogue, TMA stores).  Video items take the
staged pair (a prepare kernel that writes the normalised rows once, then the
TMA-fed contraction); patch rows take the TMA-fed contraction.

The roofline object describes the dominant kernel alone: in a second timed
pass of the same K steps the library records a CUDA event pair around it on
the launching stream in every step (pe_profile_begin / pe_profile_end), and
bench divides 2*N*K*E by the mean of those durations.  The headline value
comes from the first pass, which has no events between the kernels of a step
(an event there serialises the staged path's two kernels).

For N > 1 (torchrun, one process per GPU, --gpus N must equal the number of
ranks) the global batch is N copies of the workload, cut into contiguous
output-row ranges at whole items or temporal patches (one range per rank,
weight replicated, no collective on the data path): weak scaling.  The value is
all ranks' patches over the slowest rank's device time.

Rank 0 prints one JSON line.  Timing: W untimed warm-up steps; K timed steps,
each bracketed by CUDA events on the launching stream, with an L2 flush (a
write larger than L2) before every step outside the events; barrier +
synchronize around the timed region; max over ranks.  The e2e value goes
through the library's host-buffer call (pinned host frames in, host
embeddings out, copies inside the timed region).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "PatchEmbed patches/s and TFLOP/s (% of B200 dense bf16 peak), 1 GPU"
UNIT = "patches/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one contraction
# launch, from an ncu capture, keyed by workload and path, together with the
# SHA-256 of the kernel sources it was taken on.  A changed kernel invalidates
# the figure (reported as null) until it is captured again.
TRAFFIC = {
    ("grouped_16_images", "staged"): {"bytes": 110391552 + 97005056, "kernel_sha": "1b8bf5a9bafc0d45"},
    ("grouped_16_images", "staged_fold"): {"bytes": 87545856 + 97287680, "kernel_sha": "1b8bf5a9bafc0d45"},
    ("grouped_16_images", "astat"): {"bytes": 111755008 + 99322624, "kernel_sha": "1b8bf5a9bafc0d45"},
    ("long_video_64x896", "staged"): {"bytes": 527892480 + 281080832, "kernel_sha": "1b8bf5a9bafc0d45"},
    # the PatchMerger's fc1 + GELU
    ("patch_merger_grouped_16_images", "fc1"): {"bytes": 768710912 + 135956224, "kernel_sha": "1b8bf5a9bafc0d45"},
}
KERNEL_SOURCES = ("vlm_vision_patch_b200/csrc/pe_kernels.cuh", "vlm_vision_patch_b200/csrc/pe_device.cuh",
                  "vlm_vision_patch_b200/csrc/pe_astat.cuh")


def code_digest(texts):
    """SHA-256 (16 hex) of C/CUDA sources with comments and blank space removed,
    so that a changed comment does not invalidate a measurement of the code."""
    import hashlib
    import re
    h = hashlib.sha256()
    for t in texts:
        t = re.sub(r"/\*.*?\*/", "", t, flags=re.S)
        t = re.sub(r"//[^\n]*", "", t)
        h.update(re.sub(r"\s+", " ", t).strip().encode())
    return h.hexdigest()[:16]


def kernel_sha():
    texts = []
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            texts.append(f.read())
    return code_digest(texts)


def measured_traffic(workload, path):
    rec = TRAFFIC.get((workload, path))
    if not rec or rec["kernel_sha"] != kernel_sha():
        return None
    return rec["bytes"]


def max_over_ranks(x: float, pg=None, device="cpu") -> float:
    """The largest x over all ranks (x itself without a process group)."""
    if pg is None:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank_step: int, steps: int, world: int, max_ms: float) -> float:
    """Whole-job throughput: every rank's units over the slowest rank's time."""
    return units_per_rank_step * steps * world / (max_ms / 1e3)


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


# ------------------------------------------------------------------ clocks

def nvml_handle_for(nv, props):
    """NVML handle of the CUDA device with properties `props`.  NVML numbers
    every GPU of the machine and ignores CUDA_VISIBLE_DEVICES, so the device is
    found by its PCI location (then by UUID).  Returns (handle, how) or
    (None, None)."""
    want = (int(props.pci_domain_id), int(props.pci_bus_id), int(props.pci_device_id))
    handles = [nv.nvmlDeviceGetHandleByIndex(i) for i in range(nv.nvmlDeviceGetCount())]
    for h in handles:
        pci = nv.nvmlDeviceGetPciInfo(h)
        if (int(pci.domain), int(pci.bus), int(pci.device)) == want:
            return h, "pci"
    uid = str(getattr(props, "uuid", "") or "")
    if uid:
        for h in handles:
            u = nv.nvmlDeviceGetUUID(h)
            u = u.decode() if isinstance(u, bytes) else str(u)
            if uid in u:
                return h, "uuid"
    return None, None


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running,
    on the GPU that CUDA device `index` is."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index: int, period_s: float = 0.01):
        self.index, self.period = index, period_s
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False
        self.match = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            try:
                self._h, self.match = nvml_handle_for(pynvml, torch.cuda.get_device_properties(self.index))
            except Exception:
                self._h, self.match = None, None
            if self._h is None:   # no PCI or UUID match: NVML's own numbering, flagged as such
                self._h, self.match = pynvml.nvmlDeviceGetHandleByIndex(self.index), "index (unverified)"
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            return self
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                try:
                    reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                except Exception:
                    reasons = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
                util = nv.nvmlDeviceGetUtilizationRates(self._h).gpu
                self.samples.append((mhz, int(reasons), util))
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0, "gpu_match": self.match}
        mhz = [s[0] for s in self.samples]
        bits = 0
        for s in self.samples:
            bits |= s[1]
        names = [n for b, n in self.REASONS.items() if bits & b and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(mhz)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples), "gpu_match": self.match}


# ------------------------------------------------------------------ oracle arm

def oracle_inputs(wl):
    """The workload's tensors as fp32 numpy arrays for the oracle (bf16 widens
    exactly), converted once per workload, outside every timed region: input
    marshalling, not the oracle's work."""
    if getattr(wl, "_oracle_in", None) is None:
        f32 = lambda t: None if t is None else np.ascontiguousarray(t.float().numpy())  # noqa: E731
        wl._oracle_in = {"patches": f32(wl.patches), "weight": f32(wl.weight), "bias": f32(wl.bias),
                         "items": [(f32(it.frames), it.grid) for it in wl.items]}
    return wl._oracle_in


def oracle_sample_rate(wl, n_rows: int, seed: int, fp32_form: bool = False):
    """Time the CPU oracle on n_rows sampled output rows of the workload
    (fp32_form: the unrounded fp32 Conv3d that the tf32 path is checked
    against, for fp32 patch rows).  Only the sampled rows are computed and
    returned (patch rows: the selected rows; frames: the oracle's compact
    row-mask form).  Returns (rows/s, seconds, threads)."""
    import oracle
    inp = oracle_inputs(wl)
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(wl.N, size=min(n_rows, wl.N), replace=False))
    t0 = time.perf_counter()
    if wl.patches is not None:
        form = oracle.conv3d_patches_fp32 if fp32_form else oracle.conv3d_patches
        form(inp["patches"][rows], inp["weight"], inp["bias"], wl.C, wl.tp, wl.p)
    else:
        mask = np.zeros(wl.N, np.uint8)
        mask[rows] = 1
        oracle.conv3d_grouped(inp["items"], wl.merge, wl.mean, wl.std, inp["weight"], inp["bias"],
                              wl.C, wl.tp, wl.p, row_mask=mask, compact=True)
    dt = time.perf_counter() - t0
    return len(rows) / dt, dt, oracle.num_threads()


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    wl = workloads.ALL[args.workload]()
    rows_per_step = args.ref_rows
    fp32_form = bool(args.tf32 and wl.patches is not None and wl.patches.dtype == torch.float32)
    for _ in range(args.warmup):
        oracle_sample_rate(wl, max(16, rows_per_step // 8), 1000, fp32_form)
    times, nrows = [], 0
    threads = 1
    for s in range(args.steps):
        r, dt, threads = oracle_sample_rate(wl, rows_per_step, 2000 + s, fp32_form)
        times.append(dt)
        nrows += int(round(r * dt))
    total = sum(times)
    value = nrows / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(wl, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{min(rows_per_step, wl.N)} seeded random output rows of {wl.name} per step "
                                   f"(of {wl.N}); direct fp64 Conv3d"
                                   + (" on the unrounded fp32 inputs (the tf32 path's reference)" if fp32_form else "")
                                   + ", OpenMP over rows"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm

def patchify_line(wl, pre_times):
    """The kernel before the contraction, timed with its own CUDA events: the
    staged prepare kernel (frames) or the cast of fp32 patch rows.  read_gbs is
    the unique input bytes (every pixel read once) over its time, the patchify
    read's achieved memory throughput; traffic_gbs adds the rows it writes."""
    if not pre_times:
        return None
    ms = statistics.mean(pre_times)
    if wl.patches is not None:
        kernel = "pe_cast_rows_kernel"
        rd = wl.patches.numel() * wl.patches.element_size()
        wr = wl.N * wl.K * 2
    else:
        kernel = "pe_prep_rows_kernel"
        rd = sum(it.frames.numel() * it.frames.element_size() for it in wl.items)
        one_slice = wl.tp == 1 or (wl.tp == 2 and all(it.frames.shape[0] == 1 for it in wl.items))
        row_elems = (wl.C * wl.p * wl.p + 15) // 16 * 16 if one_slice else wl.K
        wr = wl.N * row_elems * 2
    return {"kernel": kernel, "ms_mean": ms, "ms_min": min(pre_times), "read_bytes": rd, "write_bytes": wr,
            "read_gbs": rd / (ms / 1e3) / 1e9, "traffic_gbs": (rd + wr) / (ms / 1e3) / 1e9}


def torch_patch_rows(frames, grid, merge, mean, std, tp, p):
    """Normalised patch rows [N, C*tp*p*p] (bf16) of one [T, C, H, W] item in
    output-row order, written with torch tensor ops: the frames padded to
    tp*g_t by repeating the last one, bf16(fp32(fp32(x - mean) / std)) per
    channel, then a view/permute to (g_t, window row, window column, dh, dw)
    rows of (c, t, i, j) columns (raster rows for merge 1).  The eager-torch
    form of the path, timed as context only."""
    T, C, H, W = frames.shape
    gt, gh, gw = (int(v) for v in grid)
    idx = torch.clamp(torch.arange(gt * tp, device=frames.device), max=T - 1)
    f = frames[idx].float()
    mu = torch.tensor(mean, dtype=torch.float32, device=frames.device).view(1, C, 1, 1)
    sd = torch.tensor(std, dtype=torch.float32, device=frames.device).view(1, C, 1, 1)
    f = ((f - mu) / sd).to(torch.bfloat16)
    m = merge
    f = f.view(gt, tp, C, gh // m, m, p, gw // m, m, p)
    # -> (gt, gh/m, gw/m, dh, dw, C, tp, i, j)
    f = f.permute(0, 3, 6, 4, 7, 2, 1, 5, 8)
    return f.reshape(gt * gh * gw, C * tp * p * p)


def _event_ms(fn, flush_buf, dev, reps):
    for _ in range(3):
        fn()
    ts = []
    for _ in range(reps):
        flush_buf.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize(dev)
        ts.append(a.elapsed_time(b))
    return statistics.median(ts)


def library_context(wl, dev, flush_buf, reps=20):
    """Library and eager-torch forms of the same work, timed like the steps
    (L2 flushed, CUDA events): context for the path's numbers, not part of it.
      cublas_linear_bf16   torch.nn.functional.linear on [N, K] x [E, K]^T
      cudnn_conv3d_bf16    torch.nn.functional.conv3d on the rows viewed as
                           [N, C, tp, p, p] against the [E, C, tp, p, p] weight
      torch_frames_bf16    frames workloads: torch_patch_rows per item, cat,
                           then linear (+ bias): raw frames to embeddings"""
    flop = 2.0 * wl.N * wl.K * wl.E
    x = torch.randn(wl.N, wl.K, device=dev).to(torch.bfloat16)
    w = torch.randn(wl.E, wl.K, device=dev).to(torch.bfloat16) * 0.02
    ctx = {}
    ms = _event_ms(lambda: torch.nn.functional.linear(x, w), flush_buf, dev, reps)
    ctx["cublas_linear_bf16"] = {"ms": ms, "tflops": flop / (ms / 1e3) / 1e12, "shape": [wl.N, wl.K, wl.E]}
    x5 = x.view(wl.N, wl.C, wl.tp, wl.p, wl.p)
    w5 = w.view(wl.E, wl.C, wl.tp, wl.p, wl.p)
    ms = _event_ms(lambda: torch.nn.functional.conv3d(x5, w5, stride=(wl.tp, wl.p, wl.p)), flush_buf, dev, reps)
    ctx["cudnn_conv3d_bf16"] = {"ms": ms, "tflops": flop / (ms / 1e3) / 1e12}
    if wl.patches is None:
        frames = [it.frames.to(dev) for it in wl.items]
        wt = wl.weight.to(dev).to(torch.bfloat16).reshape(wl.E, wl.K)
        bias = None if wl.bias is None else wl.bias.to(dev).to(torch.bfloat16)

        def eager():
            rows = torch.cat([torch_patch_rows(f, it.grid, wl.merge, wl.mean, wl.std, wl.tp, wl.p)
                              for f, it in zip(frames, wl.items)])
            return torch.nn.functional.linear(rows, wt, bias)
        ms = _event_ms(eager, flush_buf, dev, reps)
        ctx["torch_frames_bf16"] = {"ms": ms, "patches_per_s": wl.N / (ms / 1e3), "tflops": flop / (ms / 1e3) / 1e12}
        del frames
    return ctx


E2E_PATHS = {"host": "pe_forward_frames_grouped_host / pe_forward_patches_host (C ABI, host buffers): chunked "
                     "copies in both directions pipelined with the contraction",
             "serial": "pinned copy_ in, the device-pointer call, copy_ out, one stream"}


def local_shard(wl, world, rank):
    """This rank's part of a global batch made of `world` copies of the
    workload, cut into contiguous output-row ranges at whole items or whole
    temporal patches (vlm_vision_patch_b200.shard): about one copy's rows per
    rank (weak scaling), no exchange on the data path.  The workload itself at
    world 1; patch rows shard to exactly one copy per rank."""
    if world == 1 or wl.patches is not None:
        return wl
    import dataclasses
    from vlm_vision_patch_b200.shard import shard_rows
    n = len(wl.items)
    pieces = shard_rows([it.frames.shape[0] for it in wl.items] * world, [it.grid for it in wl.items] * world,
                        wl.tp, world)[rank]
    items = [workloads.Item(wl.items[pc.item % n].frames[pc.f0:pc.f1], pc.grid) for pc in pieces]
    return dataclasses.replace(wl, items=items)


def config_of(wl, world):
    cfg = {"workload": wl.name, "N_patches": wl.N, "K": wl.K, "E": wl.E, "patch": wl.p,
           "temporal_patch": wl.tp, "merge": wl.merge, "items": max(1, len(wl.items)),
           "out_dtype": "bf16" if wl.out_dtype == torch.bfloat16 else "f32",
           "parallelism": (f"row shards x{world}: {world} copies of the workload split into contiguous output-row "
                           "ranges at whole items / temporal patches, weight replicated, no data-path collective")
                          if world > 1 else "1 gpu",
           "l2": "flushed before every timed step (write of 2x L2 outside the events)"}
    return cfg


def run_ours(args, rank, world, local):
    import vlm_vision_patch_b200 as vp
    from vlm_vision_patch_b200 import _binding as B
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist
    wl_global = workloads.ALL[args.workload]()
    wl = local_shard(wl_global, world, rank)
    total_rows = world * wl_global.N            # every rank's rows of the global batch
    pe = vp.PatchEmbed(wl.E, wl.C, wl.tp, wl.p, wl.bias is not None)
    pe.set_weight(wl.weight.to(dev), None if wl.bias is None else wl.bias.to(dev))
    pe.set_norm(wl.mean, wl.std)
    if args.fold:
        pe.set_temporal_fold(True)
    if args.tf32:
        pe.set_tf32(True)
    out = torch.empty((wl.N, wl.E), dtype=wl.out_dtype, device=dev)
    stream = torch.cuda.current_stream(dev)

    # --pos: a [N, E] bf16 position table added in the contraction's epilogue
    # (device-resident, like a model parameter)
    pos = workloads.normal((wl.N, wl.E), 97, dtype=torch.bfloat16).to(dev) if args.pos else None
    if wl.patches is not None:
        x_dev = wl.patches.to(dev)

        def step():
            pe.forward_patches(x_dev, out=out, pos=pos)
        in_bytes = wl.patches.numel() * wl.patches.element_size()
    else:
        frames_dev = [it.frames.to(dev) for it in wl.items]
        grids = [it.grid for it in wl.items]

        def step():
            pe.forward_frames_grouped(frames_dev, grids, wl.merge, out=out, pos=pos)
        in_bytes = sum(it.frames.numel() * it.frames.element_size() for it in wl.items)
    out_bytes = out.numel() * out.element_size()

    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_buf = torch.empty(2 * l2 // 4 + 1024, dtype=torch.float32, device=dev)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if pe.last_error() != 0:
        raise RuntimeError("device pipeline timeout during warm-up")

    def timed_pass(kernel_events: bool, flush: bool = True):
        """K steps, each bracketed by CUDA events on the launching stream, L2
        flushed before each step outside the events (unless `flush` is off: the
        hot figures); barrier + synchronize around the pass.  With
        kernel_events the library also records an event pair around each step's
        contraction kernel (same stream); it always counts the kernels it
        launches."""
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        B.pe_profile_begin(pe.h, args.steps if kernel_events else 0)
        if pg:
            pg.barrier()
        torch.cuda.synchronize(dev)
        for i in range(args.steps):
            if flush:
                flush_buf.zero_()
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
        torch.cuda.synchronize(dev)
        if pg:
            pg.barrier()
        kms, nl = B.pe_profile_end(pe.h, args.steps)
        return [a.elapsed_time(b) for a, b in evs], kms, nl

    with ClockSampler(local) as clk:
        # pass 1: the headline; pass 2: the same steps with the contraction
        # kernel's own events (they serialise the two kernels of a staged step,
        # so they are kept out of pass 1)
        times, _, launches = timed_pass(False)
        times_k, gemm_times, _ = timed_pass(True)
        # pass 2b: the same events around the kernel before the contraction
        # (the prepare kernel of staged frames, the cast of fp32 patch rows)
        B.pe_profile_target(pe.h, 1)
        _, pre_times, _ = timed_pass(True)
        B.pe_profile_target(pe.h, 0)
        # pass 3: L2 left warm between steps (inputs from the previous step may
        # still be cached): context beside the cold headline
        times_hot, _, _ = timed_pass(False, flush=False)
    if len(gemm_times) != args.steps:
        raise RuntimeError(f"expected {args.steps} contraction timings, got {len(gemm_times)}")
    if pe.last_error() != 0:
        raise RuntimeError("device pipeline timeout during the timed steps")
    total_max_ms = max_over_ranks(sum(times), pg, dev)
    value = total_rows * args.steps / (total_max_ms / 1e3)

    # end to end through the public API with host buffers (pinned), per step:
    # H2D of the step's frames, the forward, D2H of the embeddings.  "host"
    # (the headline): the C-ABI host-buffer call, which pipelines the copies in
    # both directions with the contraction in chunks; "serial" (context):
    # copy_ in, the device-pointer call, copy_ out, one stream.
    e2e_steps = max(3, min(args.steps, args.e2e_steps))
    if wl.patches is not None:
        host_in = [wl.patches.pin_memory()]
        dev_in = [x_dev]
    else:
        host_in = [it.frames.pin_memory() for it in wl.items]
        dev_in = frames_dev
    host_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)

    def e2e_step(mode):
        if mode == "host":
            if wl.patches is not None:
                pe.forward_patches_host(host_in[0], out=host_out, stream=stream, blocking=False)
            else:
                pe.forward_frames_grouped_host(host_in, grids, wl.merge, out=host_out, stream=stream,
                                               blocking=False)
            return
        for h_, d_ in zip(host_in, dev_in):
            d_.copy_(h_, non_blocking=True)
        step()
        host_out.copy_(out, non_blocking=True)

    def e2e_rate(mode):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for _ in range(2):
            e2e_step(mode)
        torch.cuda.synchronize(dev)
        if pg:
            pg.barrier()
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step(mode)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return total_rows * e2e_steps / (max_over_ranks(e0.elapsed_time(e1), pg, dev) / 1e3)
    # the host-buffer calls take no position table: with --pos both figures
    # come from the serial form
    e2e_mode = "serial" if args.pos else args.e2e
    other = "serial" if e2e_mode == "host" else "host"
    e2e_value = e2e_rate(e2e_mode)
    e2e_other = None if args.pos else e2e_rate(other)
    if pe.last_error() != 0:
        raise RuntimeError("device pipeline timeout during the end-to-end steps")

    result = None
    if rank == 0:
        peaks, src = load_peaks()
        folded = bool(args.fold and wl.items and wl.tp == 2 and all(it.frames.shape[0] == 1 for it in wl.items))
        k_eff = wl.C * wl.p * wl.p if folded else wl.K   # the contraction actually performed
        flop = 2.0 * wl.N * k_eff * wl.E
        mean_ms = statistics.mean(times)
        step_tflops = flop / (mean_ms / 1e3) / 1e12
        gemm_ms = statistics.mean(gemm_times)
        achieved = flop / (gemm_ms / 1e3) / 1e12
        tf32 = bool(args.tf32 and wl.patches is not None and wl.patches.dtype == torch.float32)
        # a contraction's own dtype: tf32 = the measured bf16 peak x the nominal
        # dense tf32 / bf16 ratio (1.1 / 2.25 PFLOP/s)
        peak = float(peaks["bf16_tflops"]) * (1.1 / 2.25 if tf32 else 1.0)
        staged = launches == 2 * args.steps
        kernel = "pe_fwd_kernel (contraction)"
        frames_path = os.environ.get("PE_FRAMES_PATH", "")
        if wl.patches is not None:
            if tf32:
                path = "patches: fp32 rows rounded to tf32 by a kernel, then the TMA-fed kind::tf32 pair GEMM"
            elif wl.patches.dtype == torch.float32:
                path = "patches: fp32 rows cast to bf16 by a kernel, then the TMA-fed pair GEMM"
            else:
                path = "patches: bf16 rows, TMA-fed pair GEMM"
        elif staged:
            path = "staged: prepare kernel writes the normalised rows, then the TMA-fed pair GEMM"
        elif frames_path == "astat" and wl.tp == 2 and all(it.frames.shape[0] == 1 for it in wl.items):
            path = ("fused, resident A: one kernel from frames to embeddings (each 256-row block gathered once "
                    "into shared memory, the weight streamed past it)")
            kernel = "pe_astat_kernel (fused frames -> embeddings)"
        elif frames_path == "streamed":
            path = "streamed: one cooperative kernel whose producer warps write the rows its pair GEMM reads back"
        else:
            path = "fused: one kernel from frames to embeddings (A gathered again for every weight tile)"
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            r, dt, th = oracle_sample_rate(wl, args.cpu_rows, 7)
            cpu = {"value": r, "unit": UNIT, "cores": th, "kind": "oracle",
                   "sample": f"{min(args.cpu_rows, wl.N)} seeded random output rows of {wl.name} (of {wl.N}), "
                             f"{dt:.1f} s; direct fp64 Conv3d, OpenMP over rows"}
        # the counters belong to one kernel form: the folded weight, the
        # position table and tf32 each launch another
        variant = ("staged" if staged else ("astat" if "resident A" in path else "single")) + \
            ("_fold" if folded else "") + ("_pos" if args.pos else "") + ("_tf32" if tf32 else "")
        traffic = measured_traffic(wl.name, variant)
        context = None if (args.no_context or world > 1) else library_context(wl, dev, flush_buf)
        result = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_max_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "tf32" if (args.tf32 and wl.patches is not None and wl.patches.dtype == torch.float32) else "bf16",
            "data": "synthetic (seeded U[0,1) frames, N(0,0.02) weights)",
            "config": dict(config_of(wl, world), **({"temporal_fold": True, "K_contracted": k_eff} if folded else {}),
                           **({"position_table": "bf16 [N, E], added in the epilogue"} if args.pos else {})),
            "tflops": step_tflops,
            "pct_of_peak": {f"bf16_burst_{src}": step_tflops / float(peaks["bf16_tflops"]),
                            f"bf16_sustained_{src}": step_tflops / float(peaks.get("bf16_tflops_sustained",
                                                                                   peaks["bf16_tflops"]))},
            "step_ms": {"mean": mean_ms, "median": statistics.median(times), "min": min(times)},
            "step_ms_hot": {"mean": statistics.mean(times_hot), "median": statistics.median(times_hot),
                            "note": "L2 not flushed between steps; the headline value uses the flushed steps"},
            "path": path,
            "kernel_ms": {"contraction_mean": gemm_ms, "contraction_min": min(gemm_times),
                          "step_mean_with_kernel_events": statistics.mean(times_k),
                          "rest_of_step_mean": statistics.mean(times_k) - gemm_ms},
            "patchify": patchify_line(wl, pre_times),
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": traffic,
                         # context: the same against the sustained (power-capped) figure
                         "frac_sustained": achieved / (float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
                                                       * (1.1 / 2.25 if tf32 else 1.0)),
                         "kernel": kernel + ", 2*N*K*E flop per launch over its own CUDA-event duration",
                         "peak_source": (f"{src} bf16 dense (burst), MEASURED_PEAKS.json" if src == "measured"
                                         else "fallback 1590 TFLOP/s bf16")
                                        + (" x 1.1/2.25 (nominal tf32/bf16)" if tf32 else "")},
            "cpu_baseline": cpu,
            "e2e": dict({"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": in_bytes,
                         "d2h_bytes_per_step": out_bytes, "path": E2E_PATHS[e2e_mode]},
                        **({} if args.pos else {other: {"value": e2e_other, "unit": UNIT,
                                                        "path": E2E_PATHS[other]}})),
            "gpu_launches": launches,
            "context": context,
            "clocks": clk.summary(),
        }
        print(json.dumps(result), flush=True)
    if pg:
        pg.destroy_process_group()
    pe.close()
    return 0


def merger_weights(E: int, H: int, seed: int = 77):
    """Synthetic PatchMerger weights on the CPU (bf16), for m = 2, D = 4E:
    gamma ~ 1 + N(0, 0.1), beta ~ N(0, 0.05), w1 [D, D] and w2 [H, D] ~ N(0, 1/D),
    b1, b2 ~ N(0, 0.02).  Returns (gamma, beta, w1, b1, w2, b2)."""
    D = 4 * E
    gen = torch.Generator().manual_seed(seed)
    mk = lambda *shape, std: (torch.randn(*shape, generator=gen) * std).to(torch.bfloat16)  # noqa: E731
    gamma = (1.0 + torch.randn(E, generator=gen) * 0.1).to(torch.bfloat16)
    beta, b1, b2 = mk(E, std=0.05), mk(D, std=0.02), mk(H, std=0.02)
    w1, w2 = mk(D, D, std=D ** -0.5), mk(H, D, std=D ** -0.5)
    return gamma, beta, w1, b1, w2, b2


MERGER_METRIC = "PatchMerger patches/s and TFLOP/s (% of B200 dense bf16 peak), 1 GPU"


def run_reference_merger(args, rank, world):
    """--impl reference --merger: the CPU PatchMerger oracle on sampled merged
    rows of an input shaped like the workload's PatchEmbed output (seeded
    N(0, 0.5) rows; the values do not change the work), the merger arm's
    weights, metric and unit."""
    import oracle
    if rank != 0:
        return 0
    wl = workloads.ALL[args.workload]()
    E, H = wl.E, 1536
    V = wl.N // 4
    x = (torch.randn(V * 4, E, generator=torch.Generator().manual_seed(78)) * 0.5).to(torch.bfloat16)
    gamma, beta, w1, b1, w2, b2 = merger_weights(E, H)
    per_step = max(1, min(args.ref_rows // 32, V))   # 256 merged rows (about 17 GFLOP fp64) at the default

    def sample(n, seed):
        rng = np.random.default_rng(seed)
        mask = np.zeros(V, np.uint8)
        mask[rng.choice(V, size=min(n, V), replace=False)] = 1
        t0 = time.perf_counter()
        oracle.patch_merger(x, 4, gamma, beta, 1e-6, w1, b1, w2, b2, v_mask=mask)
        return time.perf_counter() - t0
    for _ in range(args.warmup):
        sample(max(1, per_step // 8), 3000)
    times = [sample(per_step, 4000 + s) for s in range(args.steps)]
    total = sum(times)
    value = 4 * per_step * args.steps / total
    threads = oracle.num_threads()
    line = {
        "impl": "reference", "metric": MERGER_METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": dict(config_of(wl, world), merger="LayerNorm, 2x2 concat, GELU MLP "
                                            f"{4 * E} -> {4 * E} -> {H}", merged_rows=V),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{per_step} seeded random merged rows ({4 * per_step} patch rows) of {V} per "
                                   "step; fp64 LayerNorm and MLP with bf16 roundings, OpenMP over rows"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_merger(args, rank, world, local):
    """--merger: the PatchMerger (LayerNorm, 2x2 concat, GELU MLP 5120 -> 5120 ->
    1536, synthetic N(0, 1/sqrt(D)) weights) on the workload's PatchEmbed output
    (computed once, untimed).  A step is one merger forward; the roofline
    object describes its dominant kernel, fc1."""
    import vlm_vision_patch_b200 as vp
    from vlm_vision_patch_b200 import _binding as B
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist
    wl = workloads.ALL[args.workload]()
    pe = vp.PatchEmbed(wl.E, wl.C, wl.tp, wl.p, wl.bias is not None)
    pe.set_weight(wl.weight.to(dev), None if wl.bias is None else wl.bias.to(dev))
    pe.set_norm(wl.mean, wl.std)
    if wl.patches is not None:
        x = pe.forward_patches(wl.patches.to(dev))
    else:
        x = pe.forward_frames_grouped([it.frames.to(dev) for it in wl.items], [it.grid for it in wl.items], wl.merge)
    m, H = 2, 1536
    E, D = wl.E, wl.E * 4
    V = x.shape[0] // 4
    x = x[: V * 4]
    gamma, beta, w1, b1, w2, b2 = (t.to(dev) for t in merger_weights(E, H))
    pm = vp.PatchMerger(E, m, H, 1e-6)
    pm.set_weights(gamma, beta, w1, b1, w2, b2)
    out = torch.empty((V, H), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_buf = torch.empty(2 * l2 // 4 + 1024, dtype=torch.float32, device=dev)
    for _ in range(args.warmup):
        pm.forward(x, out=out)
    torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    B.pe_merger_profile_begin(pm.h, 2 * args.steps)
    with ClockSampler(local) as clk:
        if pg:
            pg.barrier()
        torch.cuda.synchronize(dev)
        for a, b in evs:
            flush_buf.zero_()
            a.record(stream)
            pm.forward(x, out=out)
            b.record(stream)
        torch.cuda.synchronize(dev)
        if pg:
            pg.barrier()
    times = [a.elapsed_time(b) for a, b in evs]
    lin, launches = B.pe_merger_profile_end(pm.h, 2 * args.steps)
    if pm.last_error() != 0:
        raise RuntimeError("device pipeline timeout in the merger")
    total_max_ms = max_over_ranks(sum(times), pg, dev)
    value = weak_scaling_value(x.shape[0], args.steps, world, total_max_ms)
    if rank == 0:
        peaks, src = load_peaks()
        peak = float(peaks["bf16_tflops"])
        flop = 2.0 * V * (D * D + D * H)
        mean_ms = statistics.mean(times)
        fc1 = [lin[i] for i in range(0, len(lin), 2)]
        fc1_ms = statistics.mean(fc1)
        achieved = 2.0 * V * D * D / (fc1_ms / 1e3) / 1e12
        print(json.dumps({
            "metric": MERGER_METRIC, "value": value,
            "unit": "patches/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total_max_ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (PatchEmbed output of the workload, "
            "seeded N(0, 1/sqrt(D)) merger weights)",
            "config": {"workload": "patch_merger_" + wl.name, "rows_in": int(x.shape[0]), "rows_out": V, "E": E,
                       "D": D, "H": H, "l2": "flushed before every timed step"},
            "tflops": flop / (mean_ms / 1e3) / 1e12,
            "kernel_ms": {"fc1_mean": fc1_ms, "fc2_mean": statistics.mean(lin[1::2]) if len(lin) > 1 else None},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": measured_traffic("patch_merger_" + wl.name, "fc1"),
                         "kernel": "pe_fwd_kernel (merger fc1 + GELU)",
                         "peak_source": f"{src} bf16 dense (burst)"},
            "cpu_baseline": None,
            "e2e": None, "gpu_launches": launches, "clocks": clk.summary()}), flush=True)
    if pg:
        pg.destroy_process_group()
    pm.close()
    pe.close()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="grouped_16_images", choices=sorted(workloads.ALL))
    ap.add_argument("--cpu-rows", type=int, default=65536,
                    help="output rows in the CPU oracle's timed sample (capped at the workload's N): about "
                         "10-30 s on the host cores")
    ap.add_argument("--ref-rows", type=int, default=8192,
                    help="output rows the reference arm's oracle computes per step (capped at the workload's N)")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--e2e", default="host", choices=["serial", "host"],
                    help="which end-to-end form is the headline e2e value (the other is reported beside it): "
                         "the library's pipelined host-buffer call, or serial copies around the device-pointer call")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-context", action="store_true", help="skip the cuBLAS context timing")
    ap.add_argument("--merger", action="store_true",
                    help="time the PatchMerger on the workload's PatchEmbed output instead of the PatchEmbed")
    ap.add_argument("--tf32", action="store_true",
                    help="opt-in tf32 contraction of fp32 patch rows (the fp32 workloads); dtype reads tf32")
    ap.add_argument("--pos", action="store_true",
                    help="add a [N, E] bf16 position-embedding table in the contraction's epilogue "
                         "(pe_forward_*_pos); e2e then times the serial form")
    ap.add_argument("--fold", action="store_true",
                    help="opt-in temporal folding of single-frame items (half the contraction; TFLOP/s then "
                         "counts the folded K)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank, world, local = dist_env()
    if args.gpus != world:
        ap.error(f"--gpus {args.gpus} but {world} process(es) were launched: run N > 1 ranks with "
                 f"python -m torch.distributed.run --nproc-per-node {args.gpus} bench.py --gpus {args.gpus} ...")
    if args.impl == "reference":
        return run_reference_merger(args, rank, world) if args.merger else run_reference(args, rank, world)
    if args.merger:
        return run_merger(args, rank, world, local)
    return run_ours(args, rank, world, local)


if __name__ == "__main__":
    sys.exit(main())
