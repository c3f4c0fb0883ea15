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
    tiles; the tile width is 64, 128 or 256 and covers E;
  - the resident-A kernel's plan, for every (C, p) with tp = 2: it declines
    when A does not fit and must fit for C = 3, p = 14; otherwise the weight
    ring, the resident A, the staging boxes and the barriers lie in order
    inside the allocation, and the chunk and weight-stage counts cover K."""
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
    /* resident-A kernel: every (C, p) with tp = 2 and even p; the plan either
       declines (A too large) or fits with its regions in order and in bounds */
    for (int C = 1; C <= 4; ++C)
        for (int p = 2; p <= 32; p += 2) {
            const int K = C * 2 * p * p;
            if (K > 8192) continue;
            h.E = 1280; h.C = C; h.tp = 2; h.p = p; h.K = K;
            h.Kpad = (K + 63) / 64 * 64;
            h.Kh = (C * p * p + 15) / 16 * 16;
            h.Kw = 64 * ((h.Kh + 31) / 32);
            for (int bn : {64, 128, 256})
                for (int of : {0, 1}) {
                    FwdParams P;
                    fill_common(&h, P);
                    P.bn = bn;
                    P.out_f32 = of;
                    const size_t total = plan_astat(&h, P);
                    ++cases;
                    if (total == 0) {
                        if (C == 3 && p == 14) fail("resident A must fit C=3 p=14", 100, C, 2, p, bn);
                        continue;
                    }
                    const size_t box = of ? 4096 : 2048;
                    const size_t bars = (size_t)(2 * P.nb + 2 * P.n_achunks + 5) * 8 + (size_t)(2 * P.nb + 2) * 4;
                    if (total > (size_t)h.smem_optin) fail("astat shared memory", 100, C, 2, p, bn);
                    if (P.nb < 2 || P.n_iss < 1 || P.n_iss > P.nb || P.n_iss > 3) fail("astat ring", 100, C, 2, p, bn);
                    if (P.epi_bufs < 0 || P.epi_bufs > 2) fail("astat staging", 100, C, 2, p, bn);
                    if (P.b_slot_bytes != kAsWTiles * (bn / 2) * 128) fail("astat slot", 100, C, 2, p, bn);
                    if ((size_t)P.a_offset < (size_t)P.nb * P.b_slot_bytes || P.a_offset %% 1024) fail("astat A offset", 100, C, 2, p, bn);
                    if ((size_t)P.epi_offset < (size_t)P.a_offset + (size_t)((h.Kh + 63) / 64) * kAsTileBytes ||
                        P.epi_offset %% 1024)
                        fail("astat staging offset", 100, C, 2, p, bn);
                    if ((size_t)P.bar_offset < (size_t)P.epi_offset + 4 * P.epi_bufs * box || P.bar_offset %% 8)
                        fail("astat barrier offset", 100, C, 2, p, bn);
                    if ((size_t)P.bar_offset + bars + 1024 > total) fail("astat barriers in bounds", 100, C, 2, p, bn);
                    {   /* chunks of 8 segments = p/2 k-steps: the MMA's and the producers' counts agree */
                        const int cks = kAsChunkSegs * p / 16;
                        if (P.num_ksteps * 16 != h.Kh || cks < 1 || P.n_achunks > kAsMaxChunks ||
                            P.n_achunks != (C * p + kAsChunkSegs - 1) / kAsChunkSegs ||
                            P.n_achunks != (P.num_ksteps + cks - 1) / cks)
                            fail("astat chunks", 100, C, 2, p, bn);
                    }
                    /* stage j loads weight tiles 2j, 2j + 1 (k-steps 4j .. 4j + 3); the last
                       tile any stage loads lies inside the packed weight's Kw columns */
                    if (P.n_b_stages != (h.Kh + 63) / 64 || 4 * P.n_b_stages < P.num_ksteps || P.cpp != C * p * p ||
                        64 * (2 * (P.n_b_stages - 1) + ((P.num_ksteps - 4 * (P.n_b_stages - 1)) >= 3 ? 2 : 1)) > h.Kw)
                        fail("astat weight stages", 100, C, 2, p, bn);
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
