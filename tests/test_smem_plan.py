"""The launch planners of libpe.so on every shape the ABI accepts, on the CPU:
a host-only program that includes the library's source (compiled by nvcc, run
without a GPU) calls plan_pipeline and plan_tiles directly.

Checked for every A mode and every (C, tp, p) with K = C*tp*p*p <= 8192 that
the mode accepts, and for a range of N:
  - the shared memory a launch asks for fits the B200's 227 KB per block, so
    no accepted shape fails at launch configuration;
  - both rings hold at least two stages, and the issuer warps do not outnumber
    either ring's depth;
  - the epilogue staging area sits past the rings and inside the allocation;
  - the grid is whole CTA pairs, at most one CTA per SM and no more pairs than
    tiles; the tile width is 64, 128 or 256 and covers E."""
from __future__ import annotations

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
API = os.path.join(ROOT, "vlm_vision_patch_b200", "csrc", "pe_api.cu")

PROGRAM = r"""
#include "%(api)s"
#include <cstdio>

int main() {
    pe_handle h;
    h.num_sms = 148;
    h.smem_optin = 232448;                         /* 227 KB: B200 opt-in shared memory per block */
    long cases = 0, bad = 0;
    auto fail = [&](const char *what, int mode, int C, int tp, int p, long long N) {
        if (bad++ < 20) std::printf("%%s: mode %%d C %%d tp %%d p %%d N %%lld\n", what, mode, C, tp, p, N);
    };
    for (int C = 1; C <= 4; ++C)
        for (int tp = 1; tp <= 4; ++tp)
            for (int p = 1; p <= 32; ++p) {
                const int K = C * tp * p * p;
                if (K > 8192) continue;
                h.E = 1280; h.C = C; h.tp = tp; h.p = p; h.K = K;
                h.Kpad = (K + 63) / 64 * 64;
                h.Kh = (C * p * p + 15) / 16 * 16;
                for (int mode : {(int)kAModeTma, (int)kAModePatchThreads, (int)kAModeFrames, (int)kAModeTmaShared,
                                 (int)kAModeTmaTf32}) {
                    if (mode == kAModeFrames && ((p & 1) || p > PE_MAX_PATCH)) continue;
                    if (mode == kAModeTmaShared && tp != 2) continue;
                    if (mode == kAModeTmaTf32 && (K %% 4)) continue;
                    if (mode == kAModeTma && (K %% 8)) continue;
                    FwdParams P;
                    fill_common(&h, P);
                    const size_t total = plan_pipeline(&h, P, mode, mode == kAModeTmaShared ? h.Kh : -1);
                    ++cases;
                    if (total > (size_t)h.smem_optin) fail("shared memory", mode, C, tp, p, 0);
                    if (P.nb < 2 || P.na < 2) fail("ring depth", mode, C, tp, p, 0);
                    if (P.n_iss < 1 || P.n_iss > P.nb || P.n_iss > P.na) fail("issuers", mode, C, tp, p, 0);
                    if ((size_t)P.epi_offset + 4 * 8192 + 1024 > total) fail("epilogue area", mode, C, tp, p, 0);
                }
            }
    for (int E : {16, 40, 200, 1152, 1280, 5120})
        for (long long N : {1LL, 129LL, 1024LL, 18944LL, 59204LL, 131072LL, 3000000LL}) {
            h.E = E;
            FwdParams P;
            fill_common(&h, P);
            int grid = 0;
            bool ok = false;
            plan_tiles(&h, P, N, grid, ok);
            ++cases;
            const long long mt = (N + 255) / 256;
            if (!ok || (P.bn != 64 && P.bn != 128 && P.bn != 256)) fail("tile width", -1, 0, 0, E, N);
            if ((long long)P.n_tiles_n * P.bn < E || (long long)(P.n_tiles_n - 1) * P.bn >= E) fail("E cover", -1, 0, 0, E, N);
            if (P.num_tiles != mt * P.n_tiles_n) fail("tile count", -1, 0, 0, E, N);
            if (grid %% 2 || grid > h.num_sms || grid / 2 > P.num_tiles || grid < 2) fail("grid", -1, 0, 0, E, N);
        }
    std::printf("%%s %%ld\n", bad ? "FAIL" : "ok", cases);
    return bad != 0;
}
"""


def _nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    return None


@pytest.mark.skipif(_nvcc() is None, reason="nvcc not available")
def test_launch_plans_fit_every_accepted_shape(tmp_path):
    src = tmp_path / "plan.cu"
    src.write_text(PROGRAM % {"api": API})
    exe = tmp_path / "plan"
    # PTX only (no SASS): the program runs no kernel, so the device code need not be assembled
    cc = subprocess.run([_nvcc(), "-gencode", "arch=compute_100a,code=compute_100a", "-O1", "-std=c++17", str(src),
                         "-o", str(exe)], capture_output=True, text=True, timeout=900)
    assert cc.returncode == 0, cc.stderr[-3000:]
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0 and run.stdout.strip().startswith("ok"), run.stdout + run.stderr
