// Chunk planning for the host-buffer calls (pe_forward_frames_grouped_host,
// pe_forward_patches_host).  Pure host C++: no CUDA, so the invariants can be
// checked by a plain g++ program.
//
// A grouped call's output rows are the items' rows concatenated in list order.
// Inside one item the temporal patch g_t is the outermost index of the row
// order, for merge 1 (raster) as for merge m (windows row-major over
// (t, h/m, w/m)), so temporal patches [t0, t0 + k) of an item are output rows
// [t0*gh*gw, (t0 + k)*gh*gw) of that item.  They are computed from frames
// [t0*tp, min((t0 + k)*tp, T)) alone: a sub-item with those frames and grid
// (k, gh, gw) yields exactly those rows, with the same last-frame repetition.
// The planner cuts the call into chunks of consecutive sub-items of about
// `target_rows` rows each.
#pragma once

#include <cstdint>
#include <vector>

namespace pe_plan {

constexpr int64_t kSlotAlign = 256;   // byte alignment of every sub-item inside an input slot

inline int64_t align_up(int64_t v, int64_t a) { return (v + a - 1) / a * a; }

struct SubItem {
    int item;          // index of the item in the call
    int t0, gt;        // temporal patches [t0, t0 + gt) of that item
    int f0, T;         // its frames [f0, f0 + T)
    int64_t row0;      // first output row, counted over the whole call
    int64_t rows;      // gt * gh * gw
    int64_t in_off;    // byte offset of the frames inside the chunk's input slot
    int64_t in_bytes;  // T * frame_bytes
};

struct Chunk {
    int first, count;  // sub-items [first, first + count)
    int64_t row0, rows;
    int64_t in_bytes;  // input slot bytes the chunk needs (sub-items at kSlotAlign offsets)
};

struct Plan {
    std::vector<SubItem> subs;
    std::vector<Chunk> chunks;
    int64_t max_in = 0;    // largest chunk input
    int64_t max_rows = 0;  // largest chunk output, in rows
};

// THW and grid: [n, 3] each, already validated (gt == ceil(T / tp), every
// entry >= 1).  frame_bytes[i]: bytes of one frame of item i (C * H * W * esize).
inline Plan plan_frames(int n, const int32_t *THW, const int32_t *grid, int tp, const int64_t *frame_bytes,
                        int64_t target_rows) {
    Plan pl;
    if (target_rows < 1) target_rows = 1;
    Chunk cur{0, 0, 0, 0, 0};
    int64_t row = 0;
    auto close = [&]() {
        if (cur.count == 0) return;
        pl.chunks.push_back(cur);
        if (cur.in_bytes > pl.max_in) pl.max_in = cur.in_bytes;
        if (cur.rows > pl.max_rows) pl.max_rows = cur.rows;
        cur = Chunk{(int)pl.subs.size(), 0, row, 0, 0};
    };
    for (int i = 0; i < n; ++i) {
        const int T = THW[3 * i], gt = grid[3 * i];
        const int64_t slab = (int64_t)grid[3 * i + 1] * grid[3 * i + 2];
        int t = 0;
        while (t < gt) {
            const int64_t need = target_rows - cur.rows;   // > 0 while the chunk is open
            int64_t k = (need + slab - 1) / slab;
            if (k < 1) k = 1;
            if (k > gt - t) k = gt - t;
            SubItem s;
            s.item = i;
            s.t0 = t;
            s.gt = (int)k;
            s.f0 = t * tp;
            const int64_t f1 = (int64_t)(t + k) * tp < T ? (int64_t)(t + k) * tp : T;
            s.T = (int)(f1 - s.f0);
            s.row0 = row;
            s.rows = k * slab;
            s.in_off = cur.in_bytes;
            s.in_bytes = (int64_t)s.T * frame_bytes[i];
            cur.in_bytes = align_up(s.in_off + s.in_bytes, kSlotAlign);
            if (cur.count == 0) cur.row0 = row;
            cur.rows += s.rows;
            ++cur.count;
            pl.subs.push_back(s);
            row += s.rows;
            t += (int)k;
            if (cur.rows >= target_rows) close();
        }
    }
    close();
    return pl;
}

// Rows per chunk for a call of N rows: about an eighth of the call (eight
// chunks keep the copy engines busy in both directions), at least `min_rows`,
// a multiple of 256 (one pair tile).
inline int64_t chunk_rows(int64_t N, int64_t min_rows = 8192) {
    int64_t r = (N + 7) / 8;
    if (r < min_rows) r = min_rows;
    return align_up(r, 256);
}

// The event protocol of the host-buffer calls, written once over an abstract
// stream/event interface so that the same code runs on CUDA and in a model
// that checks it for races.  Three streams: the caller's (contractions), a
// copy-in and a copy-out stream.  Chunk c uses input and output slot c % 2.
//   copy-in of c      waits for the contraction of c - 2 (input slot free)
//   contraction of c  waits for copy-in of c and copy-out of c - 2 (output slot free)
//   copy-out of c     waits for the contraction of c
// Both copy streams first wait for the work queued on the caller's stream, and
// the caller's stream finally waits for the last copy-out (the copy-out stream
// is in order).  `ops` provides
//   bool record(int event, int stream)   capture the stream's queued work
//   bool wait(int stream, int event)     later work on `stream` waits for it
//   int copy_in(int chunk, int slot), compute(int chunk, int slot),
//   int copy_out(int chunk, int slot)    queue the chunk's work (0: ok)
// Returns 0, the first non-zero status of a queueing call, or -1 when a record
// or wait fails.
enum PipeStream { kCaller = 0, kCopyIn = 1, kCopyOut = 2 };
enum PipeEvent { kEvStart = 0, kEvIn0 = 1, kEvComp0 = 3, kEvOut0 = 5, kNumPipeEvents = 7 };

template <class Ops>
int run_pipeline(Ops &ops, int nchunks) {
    if (!ops.record(kEvStart, kCaller) || !ops.wait(kCopyIn, kEvStart) || !ops.wait(kCopyOut, kEvStart)) return -1;
    for (int c = 0; c < nchunks; ++c) {
        const int s = c & 1;
        if (c >= 2 && !ops.wait(kCopyIn, kEvComp0 + s)) return -1;
        int r = ops.copy_in(c, s);
        if (r != 0) return r;
        if (!ops.record(kEvIn0 + s, kCopyIn) || !ops.wait(kCaller, kEvIn0 + s)) return -1;
        if (c >= 2 && !ops.wait(kCaller, kEvOut0 + s)) return -1;
        r = ops.compute(c, s);
        if (r != 0) return r;
        if (!ops.record(kEvComp0 + s, kCaller) || !ops.wait(kCopyOut, kEvComp0 + s)) return -1;
        r = ops.copy_out(c, s);
        if (r != 0) return r;
        if (!ops.record(kEvOut0 + s, kCopyOut)) return -1;
    }
    if (!ops.record(kEvStart, kCopyOut) || !ops.wait(kCaller, kEvStart)) return -1;
    return 0;
}

}  // namespace pe_plan
