"""Chunk planner of the host-buffer calls (csrc/pe_host_plan.h), compiled with
g++ and checked against its invariants on random groups (no GPU): every
temporal patch of every item lands in exactly one sub-item, in order; output
rows are contiguous; each sub-item's frames are the ones its temporal patches
read (ceil(T/tp) == gt, the last frame repeated only at the item's end);
input offsets inside a slot are aligned and disjoint; chunks reach the target
size except the last."""
from __future__ import annotations

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "vlm_vision_patch_b200", "csrc")

PROGRAM = r"""
#include <cstdio>
#include <cstdlib>
#include <vector>
#include "pe_host_plan.h"

static unsigned long long state = 88172645463325252ull;
static int rnd(int lo, int hi) {            /* xorshift64, inclusive range */
    state ^= state << 13; state ^= state >> 7; state ^= state << 17;
    return lo + (int)(state % (unsigned long long)(hi - lo + 1));
}

#define REQUIRE(c) do { if (!(c)) { std::printf("case %d: %s\n", cs, #c); return 1; } } while (0)

int main() {
    for (int cs = 0; cs < 4000; ++cs) {
        const int n = rnd(1, 24), tp = rnd(1, 3), C = 3, es = rnd(0, 1) ? 2 : 4;
        std::vector<int32_t> THW(3 * n), grid(3 * n);
        std::vector<int64_t> fb(n);
        int64_t N = 0;
        for (int i = 0; i < n; ++i) {
            const int T = rnd(0, 3) == 0 ? rnd(1, 40) : 1, gh = rnd(1, 12), gw = rnd(1, 12), p = 14;
            THW[3 * i] = T; THW[3 * i + 1] = gh * p; THW[3 * i + 2] = gw * p;
            grid[3 * i] = (T + tp - 1) / tp; grid[3 * i + 1] = gh; grid[3 * i + 2] = gw;
            fb[i] = (int64_t)C * gh * p * gw * p * es;
            N += (int64_t)grid[3 * i] * gh * gw;
        }
        const int64_t target = rnd(0, 1) ? pe_plan::chunk_rows(N, 1) : rnd(1, 300);
        const pe_plan::Plan pl = pe_plan::plan_frames(n, THW.data(), grid.data(), tp, fb.data(), target);

        /* sub-items: each item's temporal patches in order, rows contiguous */
        int64_t row = 0;
        int item = 0, next_t = 0;
        for (const pe_plan::SubItem &s : pl.subs) {
            if (next_t == grid[3 * item]) { ++item; next_t = 0; }
            REQUIRE(s.item == item && s.t0 == next_t && s.gt >= 1);
            const int T = THW[3 * item], gt = grid[3 * item];
            const int64_t slab = (int64_t)grid[3 * item + 1] * grid[3 * item + 2];
            REQUIRE(s.t0 + s.gt <= gt);
            REQUIRE(s.f0 == s.t0 * tp && s.T >= 1 && s.f0 + s.T <= T);
            REQUIRE((s.T + tp - 1) / tp == s.gt);
            if (s.t0 + s.gt < gt) REQUIRE(s.T == s.gt * tp);
            else REQUIRE(s.f0 + s.T == T);
            REQUIRE(s.row0 == row && s.rows == (int64_t)s.gt * slab);
            REQUIRE(s.in_bytes == (int64_t)s.T * fb[item]);
            row += s.rows;
            next_t += s.gt;
        }
        REQUIRE(item == n - 1 && next_t == grid[3 * (n - 1)] && row == N);

        /* chunks: consecutive sub-items, aligned disjoint slot offsets, sizes */
        int first = 0;
        int64_t max_in = 0, max_rows = 0, max_slab = 0;
        for (int i = 0; i < n; ++i)
            if ((int64_t)grid[3 * i + 1] * grid[3 * i + 2] > max_slab) max_slab = (int64_t)grid[3 * i + 1] * grid[3 * i + 2];
        for (size_t c = 0; c < pl.chunks.size(); ++c) {
            const pe_plan::Chunk &ch = pl.chunks[c];
            REQUIRE(ch.first == first && ch.count >= 1 && first + ch.count <= (int)pl.subs.size());
            REQUIRE(ch.row0 == pl.subs[first].row0);
            int64_t rows = 0, end = 0;
            for (int j = first; j < first + ch.count; ++j) {
                const pe_plan::SubItem &s = pl.subs[j];
                REQUIRE(s.in_off % pe_plan::kSlotAlign == 0 && s.in_off >= end);
                end = s.in_off + s.in_bytes;
                rows += s.rows;
            }
            REQUIRE(ch.rows == rows && ch.in_bytes >= end && ch.in_bytes % pe_plan::kSlotAlign == 0);
            if (c + 1 < pl.chunks.size()) REQUIRE(ch.rows >= target);
            REQUIRE(ch.rows < target + max_slab);
            if (ch.in_bytes > max_in) max_in = ch.in_bytes;
            if (ch.rows > max_rows) max_rows = ch.rows;
            first += ch.count;
        }
        REQUIRE(first == (int)pl.subs.size() && pl.max_in == max_in && pl.max_rows == max_rows);
    }
    for (long long N : {1LL, 255LL, 59204LL, 131072LL, 10000000LL}) {
        const int64_t r = pe_plan::chunk_rows(N);
        if (r % 256 != 0 || r < 8192 || (N > 8 * 8192 && r < (N + 7) / 8)) { std::printf("chunk_rows %lld\n", N); return 1; }
    }
    std::printf("ok\n");
    return 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None, reason="g++ not available")
def test_chunk_plan_invariants(tmp_path):
    src = tmp_path / "plan.cpp"
    src.write_text(PROGRAM)
    exe = tmp_path / "plan"
    cc = subprocess.run(["g++", "-std=c++17", "-O1", "-Wall", "-Wextra", "-Werror", "-I", CSRC, str(src),
                         "-o", str(exe)], capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0 and run.stdout.strip() == "ok", run.stdout + run.stderr
