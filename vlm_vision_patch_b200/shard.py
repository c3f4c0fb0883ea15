"""Row partition of one grouped batch across ranks (one process per GPU).

Every output row of the PatchEmbed is independent of every other, so a grouped
batch shards across GPUs with no exchange on the data path: each rank embeds a
contiguous range of the batch's output rows with its own copy of the weight,
and its rows are that slice of the single-GPU output.

The unit of the cut is one temporal patch of one item.  Inside an item the
rows of temporal patch g_t come before those of g_t + 1 for merge 1 and merge 2
alike (the merge windows are row-major over (t, h/m, w/m)), so a run of
temporal patches [t0, t1) of an item is a contiguous run of gh*gw*(t1 - t0)
output rows; it reads frames [t0*tp, min(t1*tp, T)) only, the last frame
repeated as usual where the run reaches past T.  Items are concatenated in list
order (the packed sequence of the vision forward with grid_thw of shape
(num_images_or_videos, 3)).
"""
from __future__ import annotations

import dataclasses
from typing import List, Sequence, Tuple


@dataclasses.dataclass(frozen=True)
class Piece:
    """Temporal patches [t0, t1) of item `item`, which read frames [f0, f1)
    and fill global output rows [row0, row0 + rows)."""
    item: int
    t0: int
    t1: int
    f0: int
    f1: int
    grid: Tuple[int, int, int]    # (t1 - t0, gh, gw): the piece as an item of its own
    row0: int
    rows: int


def shard_rows(T: Sequence[int], grid_thw: Sequence[Sequence[int]], tp: int, world: int) -> List[List[Piece]]:
    """Split the items' output rows into `world` contiguous ranges, cut only
    between temporal patches, each range as close to an equal share of the
    rows as those cuts allow.  Returns, per rank, the pieces of its range in
    row order (a rank may get none when there are fewer units than ranks)."""
    if world < 1:
        raise ValueError("world must be >= 1")
    if len(T) != len(grid_thw):
        raise ValueError("one frame count per grid")
    units = []                       # (item, g_t, row0, rows) in output-row order
    row = 0
    for i, (t, g) in enumerate(zip(T, grid_thw)):
        gt, gh, gw = (int(v) for v in g)
        if gt < 1 or gh < 1 or gw < 1 or -(-int(t) // tp) != gt:
            raise ValueError(f"item {i}: grid {tuple(g)} does not match {t} frames at temporal patch {tp}")
        for k in range(gt):
            units.append((i, k, row, gh * gw))
            row += gh * gw
    N = row
    # unit u goes to the rank whose share [r*N/world, (r+1)*N/world) holds the
    # unit's middle row: contiguous, balanced to within one unit
    owner = [min(world - 1, (2 * r0 + n) * world // (2 * N)) for (_, _, r0, n) in units] if N else []
    out: List[List[Piece]] = [[] for _ in range(world)]
    u = 0
    while u < len(units):
        i, k0, r0, _ = units[u]
        rank = owner[u]
        v = u
        while v + 1 < len(units) and owner[v + 1] == rank and units[v + 1][0] == i:
            v += 1
        k1 = units[v][1] + 1
        gh, gw = int(grid_thw[i][1]), int(grid_thw[i][2])
        f0, f1 = k0 * tp, min(k1 * tp, int(T[i]))
        out[rank].append(Piece(i, k0, k1, f0, f1, (k1 - k0, gh, gw), r0, (k1 - k0) * gh * gw))
        u = v + 1
    return out


def rank_rows(pieces: Sequence[Piece]) -> Tuple[int, int]:
    """The [start, end) global row range a rank's pieces cover (empty: (0, 0))."""
    if not pieces:
        return (0, 0)
    return (pieces[0].row0, pieces[-1].row0 + pieces[-1].rows)
