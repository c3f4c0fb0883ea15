"""Row partition of a grouped batch across ranks (vlm_vision_patch_b200.shard),
on the CPU.

  - The ranks' row ranges are contiguous, disjoint, in rank order and cover
    [0, N); every temporal patch of every item lands on exactly one rank, with
    its global row offset; each piece's frame range and grid satisfy the
    library's ceil(T / tp) == gt; the shares differ by at most one unit.
  - Two gloo ranks (127.0.0.1 rendezvous) each compute their pieces with the
    CPU oracle, as grouped calls of their own, and gather them: the
    reassembled rows equal the oracle's single-call result exactly.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
from vlm_vision_patch_b200.shard import shard_rows, rank_rows  # noqa: E402


def _check(T, grids, tp, world):
    parts = shard_rows(T, grids, tp, world)
    assert len(parts) == world
    N = sum(g[0] * g[1] * g[2] for g in grids)
    seen = {}
    pos = 0
    shares = []
    for r, pieces in enumerate(parts):
        a, b = rank_rows(pieces)
        if pieces:
            assert a == pos, f"rank {r} starts at {a}, expected {pos}"
            pos = b
        shares.append(b - a)
        row = a
        for pc in pieces:
            assert pc.row0 == row
            gt, gh, gw = pc.grid
            assert gt == pc.t1 - pc.t0 and pc.rows == gt * gh * gw
            assert (gh, gw) == tuple(grids[pc.item][1:])
            assert 0 <= pc.f0 < pc.f1 <= T[pc.item]
            assert -(-(pc.f1 - pc.f0) // tp) == gt, "the piece is a valid item of its own"
            item_row0 = sum(g[0] * g[1] * g[2] for g in grids[:pc.item])
            assert pc.row0 == item_row0 + pc.t0 * gh * gw
            for k in range(pc.t0, pc.t1):
                assert (pc.item, k) not in seen
                seen[(pc.item, k)] = r
            row += pc.rows
    assert pos == N
    assert len(seen) == sum(g[0] for g in grids)
    unit = max(g[1] * g[2] for g in grids)
    assert max(shares) - min(shares) <= 2 * unit or N < world * unit


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_partition_invariants(world):
    rng = np.random.default_rng(world)
    for _ in range(200):
        n = int(rng.integers(1, 12))
        T = [int(rng.integers(1, 9)) for _ in range(n)]
        tp = int(rng.integers(1, 4))
        grids = [(-(-t // tp), int(2 * rng.integers(1, 5)), int(2 * rng.integers(1, 5))) for t in T]
        _check(T, grids, tp, world)


def test_partition_of_the_16_image_group_and_the_long_video():
    import workloads
    grids = workloads.grid_draw(16 * 8, 10)
    for world in (2, 4, 8):
        _check([1] * len(grids), grids, 2, world)
        parts = shard_rows([1] * len(grids), grids, 2, world)
        assert all(pc.t0 == 0 and pc.t1 == 1 for ps in parts for pc in ps)   # images stay whole
    parts = shard_rows([64], [(32, 64, 64)], 2, 8)                             # one video: 4 temporal patches each
    assert [rank_rows(p)[1] - rank_rows(p)[0] for p in parts] == [16384] * 8
    assert [(p[0].f0, p[0].f1) for p in parts] == [(8 * r, 8 * r + 8) for r in range(8)]


def test_partition_rejects_inconsistent_items():
    with pytest.raises(ValueError):
        shard_rows([3], [(1, 2, 2)], 2, 2)     # 3 frames need 2 temporal patches
    with pytest.raises(ValueError):
        shard_rows([1], [(1, 2, 2)], 2, 0)


# ------------------------------------------------------------ two gloo ranks

C, TP, P, E = 3, 2, 2, 8
GRIDS = [(1, 4, 6), (3, 2, 4), (2, 6, 2), (1, 2, 2), (4, 4, 4)]
TS = [1, 5, 4, 2, 7]


def _inputs():
    import workloads
    frames = [workloads.uniform01((t, C, g[1] * P, g[2] * P), 900 + i) for i, (t, g) in enumerate(zip(TS, GRIDS))]
    w = workloads.normal((E, C, TP, P, P), 950, std=0.3)
    b = workloads.normal((E,), 951, std=0.1)
    return frames, w, b


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    import oracle
    import workloads
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        frames, w, b = _inputs()
        pieces = shard_rows(TS, GRIDS, TP, world)[rank]
        items = [(frames[pc.item][pc.f0:pc.f1], pc.grid) for pc in pieces]
        if items:
            out, _ = oracle.conv3d_grouped(items, 2, workloads.CLIP_MEAN, workloads.CLIP_STD, w, b, C, TP, P)
        else:
            out = np.zeros((0, E))
        got = [None] * world
        dist.all_gather_object(got, (rank_rows(pieces), out))
        if rank == 0:
            full, _ = oracle.conv3d_grouped(list(zip(frames, GRIDS)), 2, workloads.CLIP_MEAN, workloads.CLIP_STD,
                                            w, b, C, TP, P)
            asm = np.concatenate([o for (_, o) in got if o.shape[0]], 0)
            q.put(("ok", bool(np.array_equal(asm, full)), [r for (r, _) in got], full.shape[0]))
        dist.barrier()
    except Exception as e:   # reported to the test instead of hanging it
        q.put(("error", repr(e), None, None))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_two_gloo_ranks_reassemble_the_single_call_result(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    status, equal, ranges, N = q.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert status == "ok", equal
    assert ranges[0][0] == 0 and ranges[-1][1] == N and ranges[0][1] == ranges[1][0]
    assert equal, "the ranks' rows, concatenated, differ from the single-call oracle result"
