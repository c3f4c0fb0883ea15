"""The boundary from C: include/pe.h compiles as strict C99, every call it
declares links against libpe.so, and the host-only calls answer from a plain C
program (no GPU, no Python in the call path)."""
from __future__ import annotations

import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pe.h")
LIBDIR = os.path.join(ROOT, "vlm_vision_patch_b200")

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "pe.h"

typedef void (*any_fn)(void);

/* Every declared call, so that the link fails if one is missing. */
static const any_fn table[] = {
%(table)s
};

static int fails = 0;
#define CHECK(cond) do { if (!(cond)) { printf("FAIL %%s\n", #cond); ++fails; } } while (0)

int main(void)
{
    const int32_t grids[6] = {1, 36, 54, 4, 14, 14};
    const int32_t bad[3] = {1, 0, 4};
    pe_handle *h = (pe_handle *)&fails;      /* overwritten with NULL by a refused create */
    pe_merger *pm = (pe_merger *)&fails;
    int n = 0;

    CHECK(sizeof(table) / sizeof(table[0]) == %(count)d);
    CHECK(pe_num_patches(grids, 1) == 1944);
    CHECK(pe_num_patches(grids, 2) == 1944 + 784);
    CHECK(pe_num_patches(grids, 0) == 0);
    CHECK(pe_num_patches(bad, 1) == -1);
    CHECK(pe_num_patches(NULL, 1) == -1);
    CHECK(strcmp(pe_status_string(PE_OK), "ok") == 0);
    CHECK(strcmp(pe_status_string(PE_ERR_DEVICE_TIMEOUT), "device pipeline wait timed out") == 0);
    CHECK(pe_device(NULL) == -1);
    /* argument errors are found before any CUDA call */
    CHECK(pe_create(1004, 3, 2, 14, 0, &h) == PE_ERR_INVALID_ARG && h == NULL);
    CHECK(pe_create(1280, 3, 2, 14, 0, NULL) == PE_ERR_INVALID_ARG);
    CHECK(pe_merger_create(1280, 2, 1536, 0.0f, &pm) == PE_ERR_INVALID_ARG && pm == NULL);
    CHECK(pe_forward_patches(NULL, NULL, PE_BF16, 1, NULL, PE_BF16, NULL) == PE_ERR_INVALID_ARG);
    CHECK(pe_forward_frames_grouped(NULL, 1, NULL, PE_BF16, NULL, NULL, 2, NULL, PE_BF16, NULL) ==
          PE_ERR_INVALID_ARG);
    CHECK(pe_set_norm(NULL, NULL, NULL) == PE_ERR_INVALID_ARG);
    CHECK(pe_last_error(NULL) == PE_ERR_INVALID_ARG);
    CHECK(pe_profile_end(NULL, NULL, &n, NULL) == PE_ERR_INVALID_ARG);
    CHECK(pe_merger_forward(NULL, NULL, 4, NULL, PE_BF16, NULL) == PE_ERR_INVALID_ARG);
    CHECK(pe_forward_frames_grouped_host(NULL, 1, NULL, PE_BF16, NULL, NULL, 2, NULL, PE_BF16, NULL) ==
          PE_ERR_INVALID_ARG);
    CHECK(pe_forward_patches_host(NULL, NULL, PE_BF16, 4, NULL, PE_BF16, NULL) == PE_ERR_INVALID_ARG);
    CHECK(pe_selftest_wait_timeout(NULL, NULL) == PE_ERR_INVALID_ARG);
    CHECK(pe_profile_target(NULL, 0) == PE_ERR_INVALID_ARG);
    pe_destroy(NULL);
    pe_merger_destroy(NULL);
    printf("%%d failed\n", fails);
    return fails != 0;
}
"""


def declared_calls():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^[A-Za-z_][\w \*]*?\b(pe_\w+)\s*\(", text, flags=re.M)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_header_is_c99_and_every_call_links(tmp_path):
    lib = os.path.join(LIBDIR, "libpe.so")
    if not os.path.exists(lib):
        pytest.skip("libpe.so not built")
    names = declared_calls()
    assert len(names) == len(set(names)) >= 26, names
    src = tmp_path / "abi.c"
    src.write_text(PROGRAM % {"table": ",\n".join(f"    (any_fn){n}" for n in names), "count": len(names)})
    exe = tmp_path / "abi"
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Wpedantic", "-Werror",
                         "-I", os.path.join(ROOT, "include"), str(src), "-L", LIBDIR, "-lpe",
                         f"-Wl,-rpath,{LIBDIR}", "-o", str(exe)], capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stdout + run.stderr
    assert run.stdout.strip().endswith("0 failed")
