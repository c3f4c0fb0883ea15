"""Race check of the host-buffer calls' event protocol (pe_plan::run_pipeline in
csrc/pe_host_plan.h, the same template the CUDA library instantiates), on CPU.

A model stands in for CUDA: each stream is an in-order queue, an event records
the last operation queued on its stream, a wait makes later work on a stream
depend on it.  From the resulting happens-before graph the test checks, for two
back-to-back calls with caller work before and after each:
  - every two accesses of one device slot, one of them a write, are ordered;
  - each chunk's copy-in precedes its contraction, which precedes its copy-out;
  - the copies start after the work queued on the caller's stream before the
    call, and the caller's later work follows every copy-out;
  - the second call's work follows the first call's.
Then each wait is dropped in turn: all but the copy-out stream's initial wait
(implied by its per-chunk waits on the contractions) must be needed."""
from __future__ import annotations

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "vlm_vision_patch_b200", "csrc")

PROGRAM = r"""
#include <cstdio>
#include <vector>
#include "pe_host_plan.h"
using namespace pe_plan;

enum Kind { kBefore, kAfter, kWaitOp, kCopyInOp, kComputeOp, kCopyOutOp };
struct Node { int stream, kind, call, chunk, slot; std::vector<int> deps; };
struct WaitInfo { int stream, event, call; };

struct Model {
    std::vector<Node> nodes;
    std::vector<WaitInfo> waits;
    int last[3] = {-1, -1, -1};
    int ev[kNumPipeEvents];
    int call = 0, drop = -1;
    Model() { for (int &e : ev) e = -1; }
    int add(int s, int kind, int chunk = -1, int slot = -1) {
        Node n{s, kind, call, chunk, slot, {}};
        if (last[s] >= 0) n.deps.push_back(last[s]);
        nodes.push_back(n);
        return last[s] = (int)nodes.size() - 1;
    }
    bool record(int e, int s) { ev[e] = last[s]; return true; }
    bool wait(int s, int e) {
        const int w = add(s, kWaitOp);
        if ((int)waits.size() != drop && ev[e] >= 0) nodes[w].deps.push_back(ev[e]);
        waits.push_back(WaitInfo{s, e, call});
        return true;
    }
    int copy_in(int c, int s) { add(kCopyIn, kCopyInOp, c, s); return 0; }
    int compute(int c, int s) { add(kCaller, kComputeOp, c, s); return 0; }
    int copy_out(int c, int s) { add(kCopyOut, kCopyOutOp, c, s); return 0; }
};

/* Two calls of n0 and n1 chunks; returns the number of violated requirements. */
static int check(int n0, int n1, int drop, std::vector<WaitInfo> *waits_out) {
    Model m;
    m.drop = drop;
    int ncalls = 0;
    for (int n : {n0, n1}) {
        m.add(kCaller, kBefore);
        if (run_pipeline(m, n) != 0) return 1000;
        m.add(kCaller, kAfter);
        ++m.call;
        ++ncalls;
    }
    if (waits_out) *waits_out = m.waits;
    const int N = (int)m.nodes.size();
    std::vector<std::vector<char>> anc(N, std::vector<char>(N, 0));   /* anc[b][a]: a happens before b */
    for (int b = 0; b < N; ++b)
        for (int d : m.nodes[b].deps) {
            anc[b][d] = 1;
            for (int a = 0; a < N; ++a) anc[b][a] |= anc[d][a];
        }
    int bad = 0;
    auto before = [&](int a, int b) { return a < b && anc[b][a]; };
    /* slot accesses: copy-in writes IN[s]; compute reads IN[s], writes OUT[s]; copy-out reads OUT[s] */
    for (int a = 0; a < N; ++a)
        for (int b = a + 1; b < N; ++b) {
            const Node &x = m.nodes[a], &y = m.nodes[b];
            if (x.slot < 0 || y.slot < 0 || x.slot != y.slot) continue;
            const bool x_in = x.kind == kCopyInOp || x.kind == kComputeOp;
            const bool y_in = y.kind == kCopyInOp || y.kind == kComputeOp;
            const bool x_out = x.kind == kComputeOp || x.kind == kCopyOutOp;
            const bool y_out = y.kind == kComputeOp || y.kind == kCopyOutOp;
            const bool in_conflict = x_in && y_in && (x.kind == kCopyInOp || y.kind == kCopyInOp);
            const bool out_conflict = x_out && y_out && (x.kind == kComputeOp || y.kind == kComputeOp);
            if ((in_conflict || out_conflict) && !before(a, b)) ++bad;
        }
    for (int call = 0; call < ncalls; ++call) {
        int bef = -1, aft = -1;
        std::vector<int> ci, cp, co;
        for (int i = 0; i < N; ++i) {
            const Node &x = m.nodes[i];
            if (x.call != call) continue;
            if (x.kind == kBefore) bef = i;
            if (x.kind == kAfter) aft = i;
            if (x.kind == kCopyInOp) ci.push_back(i);
            if (x.kind == kComputeOp) cp.push_back(i);
            if (x.kind == kCopyOutOp) co.push_back(i);
        }
        for (size_t c = 0; c < ci.size(); ++c) {
            if (!before(ci[c], cp[c]) || !before(cp[c], co[c])) ++bad;
            if (!before(bef, ci[c]) || !before(bef, co[c]) || !before(co[c], aft)) ++bad;
        }
        if (call > 0) {   /* the second call follows the first */
            int prev_aft = -1;
            for (int i = 0; i < N; ++i)
                if (m.nodes[i].call == call - 1 && m.nodes[i].kind == kAfter) prev_aft = i;
            for (int i : ci) if (!before(prev_aft, i)) ++bad;
            for (int i : co) if (!before(prev_aft, i)) ++bad;
        }
    }
    return bad;
}

int main() {
    const int sizes[] = {1, 2, 3, 5};
    int cases = 0;
    for (int n0 : sizes)
        for (int n1 : sizes) {
            std::vector<WaitInfo> waits;
            if (check(n0, n1, -1, &waits) != 0) { std::printf("race: %d %d\n", n0, n1); return 1; }
            for (size_t d = 0; d < waits.size(); ++d) {
                const bool needed = check(n0, n1, (int)d, nullptr) != 0;
                const bool implied = waits[d].stream == kCopyOut && waits[d].event == kEvStart;
                if (needed == implied) {
                    std::printf("wait %zu (stream %d, event %d, call %d) of %d/%d: %s\n", d, waits[d].stream,
                                waits[d].event, waits[d].call, n0, n1, needed ? "needed" : "not needed");
                    return 1;
                }
                ++cases;
            }
        }
    std::printf("ok %d\n", cases);
    return 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None, reason="g++ not available")
def test_host_pipeline_protocol_has_no_races(tmp_path):
    src = tmp_path / "races.cpp"
    src.write_text(PROGRAM)
    exe = tmp_path / "races"
    cc = subprocess.run(["g++", "-std=c++17", "-O1", "-Wall", "-Wextra", "-Werror", "-I", CSRC, str(src),
                         "-o", str(exe)], capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0 and run.stdout.startswith("ok"), run.stdout + run.stderr
