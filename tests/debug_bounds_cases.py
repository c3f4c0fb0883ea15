"""Child process of test_gpu_debug_bounds: runs every kernel path on small
ragged shapes with whichever library PE_LIB selects and saves the outputs and
error words to the file named on the command line.

Not a test module (pytest collects test_*.py only); run as
`python tests/debug_bounds_cases.py OUT.pt`.
"""
from __future__ import annotations

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads  # noqa: E402
from vlm_vision_patch_b200 import PatchEmbed, PatchMerger, _binding as B  # noqa: E402

DEV = "cuda:0"
C, TP = 3, 2


def _pe(E, p, bias, seed, tp=TP):
    pe = PatchEmbed(E, C, tp, p, bias)
    w = workloads.normal((E, C, tp, p, p), seed, std=0.02, dtype=torch.bfloat16).to(DEV)
    b = workloads.normal((E,), seed + 1, std=0.02, dtype=torch.bfloat16).to(DEV) if bias else None
    pe.set_weight(w, b)
    pe.set_norm(workloads.CLIP_MEAN, workloads.CLIP_STD)
    return pe


def _frames(items, p, seed, dtype=torch.bfloat16):
    """items: (T, gh, gw) per item; frames [T, C, gh*p, gw*p]."""
    return [workloads.uniform01((T, C, gh * p, gw * p), seed + i, dtype=dtype).to(DEV)
            for i, (T, gh, gw) in enumerate(items)]


def _grids(items, tp=TP):
    return [((T + tp - 1) // tp, gh, gw) for T, gh, gw in items]


# name: (frames path, items (T, gh, gw), p, E, bias, frame dtype, out dtype, with pos, extra env)
FRAME_CASES = {
    "staged_video": ("staged", [(4, 6, 10), (3, 4, 8), (1, 10, 6)], 14, 1280, True, torch.bfloat16,
                     torch.bfloat16, True, {}),
    "staged_images": ("staged", [(1, 12, 18), (1, 2, 2), (1, 8, 6)], 14, 1280, False, torch.bfloat16,
                      torch.float32, False, {}),
    "astat_staging": ("astat", [(1, 12, 18), (1, 20, 10), (1, 8, 8)], 14, 1280, True, torch.bfloat16,
                      torch.bfloat16, True, {}),
    "astat_direct_store": ("astat", [(1, 12, 18), (1, 6, 10)], 14, 1280, True, torch.bfloat16,
                           torch.float32, True, {"PE_BN": "64", "PE_ASTAT_NB": "5", "PE_ASTAT_EPIBUFS": "0"}),
    "fused_video": ("fused", [(4, 6, 10), (3, 4, 8), (1, 10, 6)], 14, 1280, True, torch.bfloat16,
                    torch.bfloat16, True, {}),
    "fused_f32_frames": ("fused", [(2, 6, 4), (1, 4, 6)], 14, 256, True, torch.float32, torch.float32, False, {}),
    "staged_f32_images": ("staged", [(1, 6, 8), (1, 4, 10)], 14, 256, True, torch.float32, torch.float32, True, {}),
    "staged_f32_video": ("staged", [(4, 6, 8), (3, 4, 6)], 14, 256, True, torch.float32, torch.bfloat16, False, {}),
    "staged_tp1": ("staged", [(3, 4, 6), (1, 6, 8)], 14, 192, True, torch.bfloat16, torch.bfloat16, True, {}),
    "fused_p8": ("fused", [(2, 6, 8), (1, 4, 4)], 8, 256, False, torch.bfloat16, torch.bfloat16, False, {}),
    "streamed_video": ("streamed", [(4, 6, 10), (3, 4, 8), (1, 10, 6)], 14, 1280, True, torch.bfloat16,
                       torch.bfloat16, False, {}),
    "fused_p32": ("fused", [(3, 2, 4), (1, 4, 2)], 32, 128, True, torch.bfloat16, torch.float32, True, {}),
    "many_items": ("staged", [(1 + (i % 3), 2 + 2 * (i % 4), 2 + 2 * (i % 5)) for i in range(40)], 14, 256,
                   True, torch.bfloat16, torch.bfloat16, True, {}),
    # temporal folding: the contraction's register-store epilogue (16-byte stores
    # on 400-byte rows with a partial last chunk; 32-byte stores on fp32 rows)
    "staged_E200_fold": ("staged", [(1, 6, 10), (1, 4, 8)], 14, 200, True, torch.bfloat16, torch.bfloat16, True,
                         {}),
    "staged_f32out_fold": ("staged", [(1, 12, 18), (1, 2, 2)], 14, 1280, True, torch.bfloat16, torch.float32,
                           False, {}),
}


def run_frames(name):
    path, items, p, E, bias, fdt, odt, with_pos, env = FRAME_CASES[name]
    tp = 1 if name.endswith("_tp1") else TP
    saved = {k: os.environ.get(k) for k in list(env) + ["PE_FRAMES_PATH"]}
    os.environ.update(env)
    os.environ["PE_FRAMES_PATH"] = path
    try:
        pe = _pe(E, p, bias, 400 + len(name), tp)
        if name.endswith("_fold"):
            pe.set_temporal_fold(True)
        frames = _frames(items, p, 500 + len(name), fdt)
        grids = _grids(items, tp)
        n = B.pe_num_patches(grids)
        pos = workloads.normal((n, E), 600, dtype=odt).to(DEV) if with_pos else None
        out = pe.forward_frames_grouped(frames, grids, 2, out_dtype=odt, pos=pos)
        rows = pe.patchify(frames, grids, 2)
        torch.cuda.synchronize()
        return {"out": out.cpu(), "rows": rows.cpu()}, pe.last_error()
    finally:
        for k, v in saved.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v


def run_patches():
    pe = _pe(1280, 14, True, 700)
    x = workloads.normal((3000, pe.K), 701, dtype=torch.bfloat16).to(DEV)
    pos = workloads.normal((3000, 1280), 702, dtype=torch.float32).to(DEV)
    out = pe.forward_patches(x, out_dtype=torch.float32, pos=pos)
    torch.cuda.synchronize()
    return {"out": out.cpu()}, pe.last_error()


def run_patches_edges():
    """The largest K (C = 4, p = 32: 8192) and the largest E (65528) the ABI takes."""
    res = {}
    err = 0
    for C, tp, p, E, N in ((4, 2, 32, 256, 300), (3, 2, 2, 65528, 130)):
        K = C * tp * p * p
        pe = PatchEmbed(E, C, tp, p, True)
        pe.set_weight(workloads.normal((E, C, tp, p, p), 710 + p, std=0.02, dtype=torch.bfloat16).to(DEV),
                      workloads.normal((E,), 711, std=0.02, dtype=torch.bfloat16).to(DEV))
        x = workloads.normal((N, K), 712 + p, dtype=torch.bfloat16).to(DEV)
        out = pe.forward_patches(x, out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        res[f"K{K}_E{E}"] = out.cpu()
        err = err or pe.last_error()
    return res, err


def run_merger():
    E, m, H = 256, 2, 512
    mg = PatchMerger(E, m, H)
    D = E * m * m
    mg.set_weights(workloads.normal((E,), 800, dtype=torch.bfloat16).to(DEV),
                   workloads.normal((E,), 801, dtype=torch.bfloat16).to(DEV),
                   workloads.normal((D, D), 802, std=0.02, dtype=torch.bfloat16).to(DEV),
                   workloads.normal((D,), 803, std=0.02, dtype=torch.bfloat16).to(DEV),
                   workloads.normal((H, D), 804, std=0.02, dtype=torch.bfloat16).to(DEV),
                   workloads.normal((H,), 805, std=0.02, dtype=torch.bfloat16).to(DEV))
    x = workloads.normal((4 * 333, E), 806, dtype=torch.bfloat16).to(DEV)
    out = mg.forward(x)
    torch.cuda.synchronize()
    return {"out": out.cpu()}, mg.last_error()


def main(dst):
    res, errs = {}, {}
    for name in FRAME_CASES:
        res[name], errs[name] = run_frames(name)
    res["patches"], errs["patches"] = run_patches()
    res["patches_edges"], errs["patches_edges"] = run_patches_edges()
    res["merger"], errs["merger"] = run_merger()
    torch.save({"lib": B.LIB_PATH, "out": res, "err": errs}, dst)


if __name__ == "__main__":
    main(sys.argv[1])
