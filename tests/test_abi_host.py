"""Host-side checks of the C ABI that need no GPU: the library builds for
sm_100a, loads, exports every entry point the header declares, and its pure
host functions behave."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pe.h")


@pytest.fixture(scope="module")
def lib():
    from vlm_vision_patch_b200 import build, _binding
    build.build()
    return _binding.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pe_[a-z0-9_]+)\s*\(", src)))


def test_header_matches_binding_exports():
    from vlm_vision_patch_b200 import _binding
    assert declared_functions() == sorted(_binding.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    from vlm_vision_patch_b200 import _binding
    out = subprocess.run(["nm", "-D", "--defined-only", _binding.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (pe_[a-z0-9_]+)\b", out))
    missing = [f for f in declared_functions() if f not in exported]
    assert not missing, missing
    for f in declared_functions():
        assert hasattr(lib, f)


def test_library_is_built_for_sm100a_only():
    """One -gencode, compute_100a -> sm_100a: machine code for sm_100a and no
    PTX that a JIT could take to another GPU."""
    from vlm_vision_patch_b200 import build
    flags = build.NVCC_FLAGS
    assert flags.count("-gencode") == 1
    assert flags[flags.index("-gencode") + 1] == "arch=compute_100a,code=sm_100a"


def test_build_tracks_every_source():
    """A change to any file the build reads makes the library stale."""
    from vlm_vision_patch_b200 import build
    csrc = [os.path.join(build.CSRC, f) for f in os.listdir(build.CSRC) if f.endswith((".cu", ".cuh", ".h"))]
    assert set(csrc) | {os.path.join(ROOT, "include", "pe.h")} <= set(build.DEPS)


def test_status_strings(lib):
    from vlm_vision_patch_b200 import _binding
    seen = set()
    for code in range(11):
        s = _binding.status_string(code)
        assert s and s != "unknown status"
        seen.add(s)
    assert len(seen) == 11
    assert set(_binding.STATUS) == set(range(11))
    assert _binding.status_string(99) == "unknown status"


def test_num_patches(lib):
    from vlm_vision_patch_b200 import _binding
    assert _binding.pe_num_patches([(1, 36, 54)]) == 1944
    assert _binding.pe_num_patches([(1, 16, 64), (4, 14, 14)]) == 1024 + 784
    assert _binding.pe_num_patches([]) == 0
    assert _binding.pe_num_patches([(1, 0, 4)]) == -1
    assert lib.pe_num_patches(None, 1) == -1
    big = 2**31 - 1
    assert _binding.pe_num_patches([(big, big, 2)]) == big * big * 2      # < 2^63: exact
    assert _binding.pe_num_patches([(big, big, 3)]) == -1                 # product beyond int64
    assert _binding.pe_num_patches([(big, big, 2), (big, big, 2)]) == -1  # sum beyond int64
    assert _binding.pe_num_patches([(big, big, 2), (1, 1, 1)]) == big * big * 2 + 1


def test_null_handle_calls_are_rejected(lib):
    assert lib.pe_last_error(None) == 1
    assert lib.pe_set_norm(None, None, None) == 1
    assert lib.pe_forward_patches(None, None, 1, 0, None, 1, None) == 1
    assert lib.pe_device(None) == -1
    lib.pe_destroy(None)
    h = ctypes.c_void_p()
    assert lib.pe_create(1280, 3, 2, 14, 0, None) == 1
    assert lib.pe_create(1004, 3, 2, 14, 0, ctypes.byref(h)) == 1     # E % 8 != 0
    assert lib.pe_create(1280, 5, 2, 14, 0, ctypes.byref(h)) == 1     # C > 4
    assert h.value is None


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_create_without_gpu_fails_cleanly(lib):
    h = ctypes.c_void_p()
    rc = lib.pe_create(1280, 3, 2, 14, 0, ctypes.byref(h))
    assert rc != 0 and h.value is None


def test_marshalling_helpers():
    """The binding's array builders: nested or flat grids, numpy and torch
    integers, pointers as 64-bit values; out-of-range values are refused rather
    than wrapped."""
    import numpy as np
    from vlm_vision_patch_b200 import _binding as B
    nested = [(1, 16, 64), (2, 4, 6)]
    flat = [1, 16, 64, 2, 4, 6]
    assert list(B._i32rows(nested)) == flat
    assert list(B._i32rows(flat)) == flat
    assert list(B._i32rows(np.array(nested))) == flat
    assert list(B._i32rows([torch.tensor(v) for v in flat])) == flat
    assert list(B._i32rows([])) == []
    big = 2**47 + 4096
    p = B._ptrs([big, 0, 16])
    assert [p[0], p[1], p[2]] == [big, None, 16]
    with pytest.raises(OverflowError):
        B._i32arr([2**31])
