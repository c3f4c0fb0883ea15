"""The bounds-checking build (libpe_debug.so, -DPE_DEBUG_BOUNDS) on every
kernel path.

In that build each data-dependent global access of the kernels (pixel
gathers through the item table, streamed row stores, position-table loads,
register-to-global output stores) checks its address range against the
buffer it indexes; an access outside would set PE_ERR_DEVICE_BOUNDS in the
handle's error word and be skipped.  A child process runs the staged,
resident-A (staging boxes and direct stores), fused (bf16 and fp32 frames,
p = 8, p = 32), streamed, device item-table, folded (the contraction's
register stores), patch-row (including K = 8192 and E = 65528) and merger
paths on small ragged shapes, once with each library; the debug run must
report no error and give the same bits as the product library.
"""
import os
import subprocess
import sys

import pytest
import torch

from vlm_vision_patch_b200 import build

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
CHILD = os.path.join(HERE, "debug_bounds_cases.py")


def _run(lib, dst):
    env = dict(os.environ)
    env.pop("PE_FRAMES_PATH", None)
    if lib is None:
        env.pop("PE_LIB", None)
    else:
        env["PE_LIB"] = lib
    r = subprocess.run([sys.executable, CHILD, dst], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    return torch.load(dst)


def test_debug_bounds_build_is_silent_and_bit_identical(tmp_path):
    dbg_lib = build.build(debug_bounds=True)
    ref = _run(None, str(tmp_path / "product.pt"))
    dbg = _run(dbg_lib, str(tmp_path / "debug.pt"))
    assert os.path.basename(dbg["lib"]) == "libpe_debug.so"
    assert os.path.basename(ref["lib"]) == "libpe.so"
    assert set(dbg["err"]) == set(ref["err"])
    for name, code in dbg["err"].items():
        assert code == 0, f"{name}: error word {code} in the bounds-checking build"
        assert ref["err"][name] == 0, name
    for name, outs in ref["out"].items():
        for key, t in outs.items():
            assert torch.equal(t, dbg["out"][name][key]), f"{name}/{key} differs between the builds"
