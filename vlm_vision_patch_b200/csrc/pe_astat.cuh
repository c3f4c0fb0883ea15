// Resident-A frames kernel: the fused frames -> embedding path for groups of
// single images (every item T = 1, duplicated to tp = 2 frames), bf16 frames.
//
// The Conv3d cuts and projects in one step (patch详解 §4.3); for a single image
// both temporal slices of the kernel multiply the same pixels (patch详解 §4.5:
// ceil(1/2) = 1 temporal patch), so one output row is
//     out[r, e] = bias[e] + sum_k x̂[r, k] * (Ŵ[e, 0, k] + Ŵ[e, 1, k]),
// k over the C*p*p in-slice columns, with both products issued separately on
// the tensor cores (no folded weight, no extra rounding).
//
// Each CTA pair owns a contiguous range of passes; a pass is one 256-row
// M-block times one BN-wide weight tile.  The A block of an M-block (this
// CTA's 128 rows x Kh in-slice columns, gathered from the raw frames,
// normalised and placed in merge order) is built ONCE in shared memory and
// stays resident while the weight tiles of every pass over that M-block
// stream through a ring.  The patch matrix [N, K] never exists in global
// memory, and each pixel is gathered once per M-block instead of once per
// weight tile.
//
//   warps 0, 2, 3  TMA issuers of the weight ring (slice-interleaved tiles)
//   warp 1         TMEM owner; in the leader CTA one thread issues the MMAs
//   warps 4-7      epilogue: TMEM -> registers, + bias (+ position table),
//                  cast, swizzled staging, TMA stores
//   warps 8-19     A producers: gather + normalise into the resident A
//
// The resident A is stored as the MMA's 128-byte-swizzled K-major tiles (64
// columns x 128 rows, 16 KB each), the layout the tensor core reads at full
// rate (a no-swizzle layout ran the MMAs at about half rate on B200).  It is
// split into chunks of 8 image-row segments (8p columns, p/2 k-steps), each
// with a full and an empty barrier.  The first pass over an M-block waits for
// each chunk as it arrives; the last pass releases each chunk once its MMAs
// are done, so the next M-block's gather overlaps the end of the previous
// block's last pass.  Every wait is bounded (FwdParams::wait_ns, default
// kWaitTimeoutNs); after an abort the kernel drains its MMAs and weight loads
// (bounded), frees the TMEM and records PE_ERR_DEVICE_TIMEOUT.
#pragma once

#include "pe_kernels.cuh"

namespace pe {

constexpr int kAsThreads = 640;                  // 20 warps
constexpr int kAsProdWarp0 = 8;                  // warps 8..19 build A
constexpr int kAsProdWarps = 12;
constexpr int kAsProdThreads = 32 * kAsProdWarps;
constexpr int kAsChunkSegs = 8;                  // image-row segments (c, i) per A chunk: 8p columns
constexpr int kAsStageSegs = 4;                  // segments loaded together per producer stage
constexpr int kAsMaxChunks = 16;
constexpr int kAsTileBytes = kBM * 128;          // one 64-column swizzled tile of 128 rows
constexpr int kAsWTiles = 2;                     // weight tiles (64 columns each) per ring stage: 8 MMAs
constexpr uint64_t kAsDrainNs = 20000000ull;     // 20 ms: teardown waits after an abort

// mbar_wait with a run-time limit (0: kWaitTimeoutNs).
__device__ __forceinline__ bool mbar_wait_lim(uint32_t bar, uint32_t parity, volatile int *abort, uint64_t lim) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    const uint64_t limit = lim ? lim : kWaitTimeoutNs;
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if (global_timer_ns() - t0 > limit) {
            *abort = 1;
            return false;
        }
    }
}

// The same wait for the A producers, which wait for most of a block's passes:
// after a failed test the thread naps `ns` nanoseconds between tests, leaving
// the issue slots of its SM sub-partition to the roles on the critical path
// (the weight issuers and the epilogue keep testing, since a late wake-up
// there delays the next weight stage or accumulator).
__device__ __forceinline__ bool mbar_wait_nap(uint32_t bar, uint32_t parity, volatile int *abort, uint64_t lim,
                                              uint32_t ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    const uint64_t limit = lim ? lim : kWaitTimeoutNs;
    while (true) {
        __nanosleep(ns);
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if (global_timer_ns() - t0 > limit) {
            *abort = 1;
            return false;
        }
    }
}

constexpr uint32_t kAsNapNs = 100;
// One 32-column chunk of an epilogue warp's 32 rows: + bias (+ position
// table), cast, staged through a swizzled box, stored by TMA (rows past N and
// columns past E are clipped by the tensor map).
template <bool HAS_POS>
__device__ __forceinline__ void as_emit(const FwdParams &P, const CUtensorMap *tmap_out, const uint32_t (&v)[32],
                                        int col0, int64_t row0, uint8_t *stage_buf, int &nbuf, int lane) {
    if (row0 >= P.N || col0 >= P.E) return;   // whole box outside: nothing to store
    uint4 pq[8];
    if constexpr (HAS_POS) {
        const int64_t r = row0 + lane;
        const int nq = P.pos_f32 ? 8 : 4;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            pq[q] = make_uint4(0u, 0u, 0u, 0u);
            const int c0 = col0 + q * (P.pos_f32 ? 4 : 8);
            if (q < nq && r < P.N && c0 < P.E) {
                const char *a = reinterpret_cast<const char *>(P.pos) + (r * P.E + c0) * (int64_t)(P.pos_f32 ? 4 : 2);
                const char *plo = reinterpret_cast<const char *>(P.pos);
                if (PE_IN(a, 16, plo, plo + P.N * (int64_t)P.E * (P.pos_f32 ? 4 : 2), P.err))
                    asm volatile("ld.global.nc.v4.b32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(pq[q].x), "=r"(pq[q].y), "=r"(pq[q].z), "=r"(pq[q].w)
                                 : "l"(a));
            }
        }
    }
    float f[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(v[e]);
    if (P.bias) {
#pragma unroll
        for (int e = 0; e < 32; ++e)
            if (col0 + e < P.E) f[e] += __ldg(P.bias + col0 + e);
    }
    // the buffer must be free of the store issued epi_bufs boxes ago
    if (lane == 0) {
        if (P.epi_bufs >= 2) bulk_wait_read<1>(); else bulk_wait_read<0>();
    }
    __syncwarp();
    if constexpr (HAS_POS) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const uint32_t w4[4] = {pq[q].x, pq[q].y, pq[q].z, pq[q].w};
            if (P.pos_f32) {
#pragma unroll
                for (int u = 0; u < 4; ++u) f[4 * q + u] += __uint_as_float(w4[u]);
            } else if (q < 4) {
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    f[8 * q + 2 * u] += bf16lo_to_f32(w4[u]);
                    f[8 * q + 2 * u + 1] += bf16hi_to_f32(w4[u]);
                }
            }
        }
    }
    uint8_t *buf = stage_buf + (size_t)nbuf * (P.out_f32 ? 4096 : 2048);
    if (P.out_f32) {
        // 128-byte rows, 128-byte swizzle: chunk c of row r at (c ^ (r & 7))
#pragma unroll
        for (int c = 0; c < 8; ++c)
            *reinterpret_cast<float4 *>(buf + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                make_float4(f[4 * c], f[4 * c + 1], f[4 * c + 2], f[4 * c + 3]);
    } else {
        // 64-byte rows, 64-byte swizzle: chunk c of row r at (c ^ ((r >> 1) & 3))
#pragma unroll
        for (int c = 0; c < 4; ++c)
            *reinterpret_cast<uint4 *>(buf + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4)) =
                make_uint4(pack_bf16x2(f[8 * c], f[8 * c + 1]), pack_bf16x2(f[8 * c + 2], f[8 * c + 3]),
                           pack_bf16x2(f[8 * c + 4], f[8 * c + 5]), pack_bf16x2(f[8 * c + 6], f[8 * c + 7]));
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        tma_store_2d(tmap_out, smem_addr(buf), col0, (int32_t)row0);
        bulk_commit();
    }
    if (++nbuf == P.epi_bufs) nbuf = 0;
}

// The same chunk stored straight from registers: lane = row, 64 (bf16) or
// 128 (fp32) contiguous bytes per lane in 16-byte stores.  Used when the
// staging boxes do not fit beside the resident A and the weight ring.
template <bool HAS_POS>
__device__ __forceinline__ void as_emit_direct(const FwdParams &P, const uint32_t (&v)[32], int col0, int64_t row0,
                                               int lane) {
    const int64_t r = row0 + lane;
    if (r >= P.N || col0 >= P.E) return;
    const int osz = P.out_f32 ? 4 : 2;
    const char *olo = static_cast<const char *>(P.out), *ohi = olo + P.N * (int64_t)P.E * osz;
    const char *plo = static_cast<const char *>(P.pos), *phi = plo + P.N * (int64_t)P.E * (P.pos_f32 ? 4 : 2);
    (void)olo; (void)ohi; (void)plo; (void)phi;
    float f[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(v[e]);
    if (P.bias) {
#pragma unroll
        for (int e = 0; e < 32; ++e)
            if (col0 + e < P.E) f[e] += __ldg(P.bias + col0 + e);
    }
    if constexpr (HAS_POS) {
        if (P.pos_f32) {
            const float4 *pr = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(P.pos) + r * P.E + col0);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                if (col0 + 4 * q >= P.E) break;
                if (!PE_IN(pr + q, 16, plo, phi, P.err)) continue;
                const float4 a = __ldg(pr + q);
                f[4 * q] += a.x; f[4 * q + 1] += a.y; f[4 * q + 2] += a.z; f[4 * q + 3] += a.w;
            }
        } else {
            const uint4 *pr = reinterpret_cast<const uint4 *>(reinterpret_cast<const uint16_t *>(P.pos) + r * P.E + col0);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if (col0 + 8 * q >= P.E) break;
                if (!PE_IN(pr + q, 16, plo, phi, P.err)) continue;
                const uint4 a = __ldg(pr + q);
                const uint32_t w4[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    f[8 * q + 2 * u] += bf16lo_to_f32(w4[u]);
                    f[8 * q + 2 * u + 1] += bf16hi_to_f32(w4[u]);
                }
            }
        }
    }
    if (P.out_f32) {
        float *o = reinterpret_cast<float *>(P.out) + r * P.E + col0;
#pragma unroll
        for (int q = 0; q < 8; ++q)
            if (col0 + 4 * q < P.E && PE_IN(o + 4 * q, 16, olo, ohi, P.err))
                st_global_v4(o + 4 * q, __float_as_uint(f[4 * q]), __float_as_uint(f[4 * q + 1]),
                             __float_as_uint(f[4 * q + 2]), __float_as_uint(f[4 * q + 3]));
    } else {
        uint16_t *o = reinterpret_cast<uint16_t *>(P.out) + r * P.E + col0;
#pragma unroll
        for (int q = 0; q < 4; ++q)
            if (col0 + 8 * q < P.E && PE_IN(o + 8 * q, 16, olo, ohi, P.err))
                st_global_v4(o + 8 * q, pack_bf16x2(f[8 * q], f[8 * q + 1]), pack_bf16x2(f[8 * q + 2], f[8 * q + 3]),
                             pack_bf16x2(f[8 * q + 4], f[8 * q + 5]), pack_bf16x2(f[8 * q + 6], f[8 * q + 7]));
    }
}

// Byte offset of element (r, k) of the resident A: 128-byte-swizzled K-major
// tiles of 64 columns; row r of a tile at r * 128, its 16-byte chunk c at
// (c ^ (r % 8)) * 16.
__device__ __forceinline__ uint32_t as_a_off(int k, int r) {
    return (uint32_t)(k >> 6) * (uint32_t)kAsTileBytes + (uint32_t)r * 128u +
           ((uint32_t)(((k >> 3) & 7) ^ (r & 7)) << 4) + (uint32_t)(k & 7) * 2u;
}

// A producers (warps 8..19 of both CTAs).  Each thread owns up to MAXIT fixed
// units (tile row r, word jw): word jw (pixels 2jw, 2jw+1) of the row's p-pixel
// segment in every image row (c, i) of the patch.  Units are numbered so that
// consecutive threads read consecutive words of one image row (patches of a
// merge window, then the next window), so every warp load is one contiguous
// run.  A gather is done in stages of kAsStageSegs segments: all of a stage's
// words are loaded (one stage ahead of the one being normalised and stored),
// normalised with the segment's channel constants (uniform across the
// warp), and stored as 4-byte words into the swizzled tiles.  A chunk (two
// stages, 8 segments) is released to the MMA with one arrival per warp.
// Columns from C*p*p up to the tile edge are written as zeros.
template <int PT, int NORM>
__device__ __forceinline__ void as_produce(const FwdParams &P, uint8_t *a_buf, uint64_t *empty_a,
                                           uint32_t full_a_leader, volatile int *abort, int q0, int q1, int pt,
                                           int lane, uint32_t rank) {
    const int p = PT ? PT : P.P;
    const int ws = p / 2;                              // words per segment row
    const int units = kBM * ws;
    constexpr int MAXIT = (kBM * ((PT ? PT : PE_MAX_PATCH) / 2) + kAsProdThreads - 1) / kAsProdThreads;
    const int ntn = P.n_tiles_n;
    const int nseg = P.C * p;                          // (c, i) segments of a row
    const int kend = ((P.Kh + 63) >> 6) << 6;          // columns the tiles hold
    const int nstage = (nseg + kAsStageSegs - 1) / kAsStageSegs;
    constexpr int kStagesPerChunk = kAsChunkSegs / kAsStageSegs;
    if (q0 >= q1) return;
    const int mfirst = q0 / ntn, mlast = (q1 - 1) / ntn;
    const uint32_t abase = smem_addr(a_buf);

    int rr[MAXIT], jw2[MAXIT];
    bool uok[MAXIT];
#pragma unroll
    for (int v = 0; v < MAXIT; ++v) {
        const int u = pt + kAsProdThreads * v;
        uok[v] = u < units;
        int r = 0, jw = 0;
        if (uok[v]) unit_to_row_word(u, ws, P.merge, r, jw);
        rr[v] = r;
        jw2[v] = 2 * jw;
    }
    const char *src[MAXIT];
    const char *dlo[MAXIT], *dhi[MAXIT];   // frame buffers (bounds-checking build)
    int32_t sW[MAXIT], sHW[MAXIT];   // bytes
    uint32_t raw[2][kAsStageSegs][MAXIT];

    auto rows_of = [&](int mb, const char *(&sp)[MAXIT], int32_t (&w)[MAXIT], int32_t (&hw)[MAXIT]) {
#pragma unroll
        for (int v = 0; v < MAXIT; ++v) {
            const int64_t R = (int64_t)mb * (2 * kBM) + rank * kBM + rr[v];
            sp[v] = nullptr;
            dlo[v] = dhi[v] = nullptr;
            w[v] = hw[v] = 0;
            if (uok[v] && R < P.N) {
                const RowSrc rs = locate_row(P, R, 2);
                dlo[v] = rs.lo;
                dhi[v] = rs.hi;
                sp[v] = rs.base + jw2[v] * 2;
                w[v] = rs.W * 2;
                hw[v] = rs.HW * 2;
            }
        }
    };
    // L2 prefetch of a block's pixels: the first and the last word of every
    // segment row (a 2p-byte run spans at most two 32-byte sectors)
    auto prefetch_block = [&](int mb) {
#pragma unroll
        for (int v = 0; v < MAXIT; ++v) {
            const int64_t R = (int64_t)mb * (2 * kBM) + rank * kBM + rr[v];
            if (!uok[v] || R >= P.N || (jw2[v] != 0 && jw2[v] != p - 2)) continue;
            const RowSrc rs = locate_row(P, R, 2);
            const char *sp = rs.base + jw2[v] * 2;
            for (int seg = 0; seg < nseg; ++seg) {
                const int c = seg / p, i = seg - c * p;
                prefetch_l2(sp + ((int64_t)c * rs.HW + (int64_t)i * rs.W) * 2);
            }
        }
    };
    // loads of stage st of block mb into buffer b (the block's rows set up at st == 0)
    auto load = [&](const int mb, const int st, const int b) {
        if (st == 0) {
            rows_of(mb, src, sW, sHW);
            if (mb == mfirst) prefetch_block(mb);
            if (mb < mlast) prefetch_block(mb + 1);
        }
#pragma unroll
        for (int qq = 0; qq < kAsStageSegs; ++qq) {
            const int seg = kAsStageSegs * st + qq;
            const int c = seg / p, i = seg - c * p;
#pragma unroll
            for (int v = 0; v < MAXIT; ++v) {
                raw[b][qq][v] = 0u;
                if (seg < nseg && src[v]) {
                    const char *a = src[v] + (int64_t)c * sHW[v] + (int64_t)i * sW[v];
                    if (PE_IN(a, 4, dlo[v], dhi[v], P.err))
                        asm volatile("ld.global.nc.b32 %0, [%1];" : "=r"(raw[b][qq][v]) : "l"(a));
                }
            }
        }
    };
    // normalise and store stage st of gather G from buffer b; false after an abort
    auto store = [&](const int G, const int st, const int b) -> bool {
        const int h = st / kStagesPerChunk;
        if (st % kStagesPerChunk == 0 &&
            !mbar_wait_nap(smem_addr(&empty_a[h]), (G & 1) ^ 1, abort, P.wait_ns, kAsNapNs))
            return false;
#pragma unroll
        for (int qq = 0; qq < kAsStageSegs; ++qq) {
            const int seg = kAsStageSegs * st + qq;
            const bool live = seg < nseg;
            const NormConst nc = norm_const(P, live ? seg / p : 0);
#pragma unroll
            for (int v = 0; v < MAXIT; ++v) {
                const int k = seg * p + jw2[v];
                if (!uok[v] || k >= kend || (!live && k < P.Kh)) continue;
                const uint32_t w = live ? norm_word<NORM>(raw[b][qq][v], nc) : 0u;
                sts32(abase + as_a_off(k, rr[v]), w);
            }
        }
        if (st % kStagesPerChunk == kStagesPerChunk - 1 || st == nstage - 1) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(full_a_leader + 8u * (uint32_t)h);
        }
        return true;
    };

    // The columns between C*p*p and Kh meet zero weight columns but are read by
    // the last k-step: zero them once (no gather writes them).
    {
        const int npw = (P.Kh - P.cpp) / 2;   // pad words per row
        for (int idx = pt; idx < kBM * npw; idx += kAsProdThreads) {
            const int r = idx / npw;
            sts32(abase + as_a_off(P.cpp + 2 * (idx - r * npw), r), 0u);
        }
    }

    // One stage of loads in flight ahead of the stage being stored, across
    // block boundaries: the next block's first stage is loaded while the
    // producer waits for the previous block's chunks to be released.
    const int total = (mlast - mfirst + 1) * nstage;
    load(mfirst, 0, 0);
    for (int idx = 0; idx < total; idx += 2) {
        if (idx + 1 < total) load(mfirst + (idx + 1) / nstage, (idx + 1) % nstage, 1);
        if (!store(idx / nstage, idx % nstage, 0)) return;
        if (idx + 1 >= total) break;
        if (idx + 2 < total) load(mfirst + (idx + 2) / nstage, (idx + 2) % nstage, 0);
        if (!store((idx + 1) / nstage, (idx + 1) % nstage, 1)) return;
    }
}

template <int PT, int NORM>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kAsThreads, 1)
    pe_astat_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_out,
                    const __grid_constant__ FwdParams P) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *w_ring = smem;
    uint8_t *a_buf = smem + P.a_offset;
    uint8_t *epi = smem + P.epi_offset;
    const int nb = P.nb, nch = P.n_achunks;
    uint64_t *full_w = reinterpret_cast<uint64_t *>(smem + P.bar_offset);
    uint64_t *empty_w = full_w + nb;
    uint64_t *full_a = empty_w + nb;
    uint64_t *empty_a = full_a + nch;
    uint64_t *tfull = empty_a + nch;
    uint64_t *tempty = tfull + 2;
    uint64_t *mma_done = tempty + 2;
    uint32_t *posted_w = reinterpret_cast<uint32_t *>(mma_done + 1);   // leader: per issuer, 1 + its last posted stage
    uint32_t *consumed_w = posted_w + nb;                               // leader: weight stages the MMA consumed
    uint32_t *tmem_holder = consumed_w + nb;
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int q0 = (int)((int64_t)P.num_tiles * pair / npairs);
    const int q1 = (int)((int64_t)P.num_tiles * (pair + 1) / npairs);
    const int ntn = P.n_tiles_n;

    if (threadIdx.x == 0) {
        for (int s = 0; s < nb; ++s) {
            mbar_init(smem_addr(&full_w[s]), 1);
            mbar_init(smem_addr(&empty_w[s]), 1);
            posted_w[s] = 0u;
            consumed_w[s] = 0u;
        }
        for (int h = 0; h < nch; ++h) {
            mbar_init(smem_addr(&full_a[h]), 2 * kAsProdWarps);
            mbar_init(smem_addr(&empty_a[h]), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_addr(&tfull[s]), 1);
            mbar_init(smem_addr(&tempty[s]), 8);
        }
        mbar_init(smem_addr(mma_done), 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmap_w);
        prefetch_tmap(&tmap_out);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_addr(tmem_holder), 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    const int iss = (warp == 0) ? 0 : (warp == 2 || warp == 3) ? warp - 1 : -1;
    if (iss >= 0) {
        // ---------------- weight TMA issuers (both CTAs; bytes complete on the leader's barriers)
        if (lane == 0 && iss < P.n_iss) {
            const uint64_t pol_w = l2_policy_evict_last();
            const uint32_t fb0 = mapa_shared(smem_addr(&full_w[0]), 0);
            const uint32_t slot = (uint32_t)P.b_slot_bytes;
            const uint32_t tile = slot / kAsWTiles;   // this CTA's half of one 64-column weight tile
            const int nst = P.n_b_stages, n_iss = P.n_iss;
            int g = 0;
            bool ok = true;
            for (int q = q0; q < q1 && ok; ++q) {
                const int n_blk = q % ntn;
                const int wrow = n_blk * P.bn + (int)rank * (P.bn / 2);
                for (int j = 0; j < nst; ++j, ++g) {
                    if (g % n_iss != iss) continue;
                    const int s = g % nb;
                    if (!mbar_wait_lim(smem_addr(&empty_w[s]), ((g / nb) & 1) ^ 1, abort, P.wait_ns)) {
                        ok = false;
                        break;
                    }
                    // stage j: weight tiles 2j and 2j + 1 (k-steps 4j .. 4j + 3); a
                    // tile wholly past the last k-step is not loaded
                    const int ntl = (P.num_ksteps - 4 * j) >= 3 ? kAsWTiles : 1;
                    if (leader) {
                        mbar_arrive_expect_tx(smem_addr(&full_w[s]), 2u * (uint32_t)ntl * tile);
                        posted_w[iss] = (uint32_t)g + 1u;   // stages this issuer posted: its g below this
                    }
                    for (int t = 0; t < ntl; ++t)
                        tma_load_2d_pair(smem_addr(w_ring + (size_t)s * slot + (size_t)t * tile), &tmap_w,
                                         fb0 + 8u * (uint32_t)s, 64 * (kAsWTiles * j + t), wrow, pol_w);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (leader CTA only)
        // Lean on purpose: one thread must issue a pair MMA every 128 cycles,
        // so descriptors advance by constant adds and each weight stage costs
        // one barrier wait, four MMAs and one commit.
        if (leader && lane == 0) {
            constexpr uint16_t kPair = 0x3;
            const uint32_t idesc = idesc_bf16_f32(2 * kBM, P.bn);
            const uint64_t a0 = smem_desc(smem_addr(a_buf), 16, 1024, kLayoutSw128);
            const uint64_t b0 = smem_desc(smem_addr(w_ring), 16, 1024, kLayoutSw128);
            const uint32_t a_lo0 = (uint32_t)a0, b_lo0 = (uint32_t)b0;
            const uint32_t w_slot = (uint32_t)P.b_slot_bytes >> 4;
            const uint32_t w_tile = w_slot / kAsWTiles;
            constexpr uint32_t kTile = (uint32_t)kAsTileBytes >> 4;
            const int nks = P.num_ksteps, nst = P.n_b_stages;
            const int cks = (kAsChunkSegs * P.P) / 16;          // k-steps per A chunk
            const uint32_t full_w0 = smem_addr(&full_w[0]), empty_w0 = smem_addr(&empty_w[0]);
            const uint32_t full_a0 = smem_addr(&full_a[0]), empty_a0 = smem_addr(&empty_a[0]);
            int ws = 0, acc = 0, g_cons = 0;
            uint32_t wph = 0, accph = 0, aph = 0;
            const int nch = P.n_achunks;
            bool ok = true;
            for (int q = q0; q < q1 && ok; ++q) {
                const int n = q % ntn;
                const bool newA = (q == q0) || n == 0;
                const bool lastA = (q == q1 - 1) || n == ntn - 1;
                if (!mbar_wait_lim(smem_addr(&tempty[acc]), accph ^ 1, abort, P.wait_ns)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)acc * kMaxBN;
                int hw = newA ? 0 : nch;    // next A chunk to await (first pass over a block)
                int hr = lastA ? 0 : nch;   // next A chunk to release (last pass over a block)
                uint32_t a_lo = a_lo0;
                for (int j = 0; j < nst; ++j) {
                    const int s0 = 4 * j;
                    const int slast = (s0 + 3 < nks) ? s0 + 3 : nks - 1;
                    // every A chunk this stage reads has arrived
                    while (hw < nch && hw * cks <= slast) {
                        if (!mbar_wait_lim(full_a0 + 8u * (uint32_t)hw, aph, abort, P.wait_ns)) { ok = false; break; }
                        ++hw;
                    }
                    if (!ok) break;
                    if (!mbar_wait_lim(full_w0 + 8u * (uint32_t)ws, wph, abort, P.wait_ns)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t b_lo = b_lo0 + (uint32_t)ws * w_slot;
                    // stage j holds k-steps 4j .. 4j + 3 = A tile j (32-byte steps
                    // inside it); weight tile t holds k-steps 4j + 2t, 4j + 2t + 1,
                    // slice 0 at +0 and slice 1 at +64 bytes of each 128-byte row
                    const uint64_t ad0 = desc_with_lo(a0, a_lo), ad1 = desc_with_lo(a0, a_lo + 2u);
                    mma_bf16_pair(d_tmem, ad0, desc_with_lo(b0, b_lo), idesc, j > 0 ? 1u : 0u);
                    mma_bf16_pair(d_tmem, ad0, desc_with_lo(b0, b_lo + 4u), idesc, 1u);
                    if (slast > s0) {
                        mma_bf16_pair(d_tmem, ad1, desc_with_lo(b0, b_lo + 2u), idesc, 1u);
                        mma_bf16_pair(d_tmem, ad1, desc_with_lo(b0, b_lo + 6u), idesc, 1u);
                    }
                    if (slast > s0 + 1) {
                        const uint64_t ad2 = desc_with_lo(a0, a_lo + 4u);
                        mma_bf16_pair(d_tmem, ad2, desc_with_lo(b0, b_lo + w_tile), idesc, 1u);
                        mma_bf16_pair(d_tmem, ad2, desc_with_lo(b0, b_lo + w_tile + 4u), idesc, 1u);
                    }
                    if (slast > s0 + 2) {
                        const uint64_t ad3 = desc_with_lo(a0, a_lo + 6u);
                        mma_bf16_pair(d_tmem, ad3, desc_with_lo(b0, b_lo + w_tile + 2u), idesc, 1u);
                        mma_bf16_pair(d_tmem, ad3, desc_with_lo(b0, b_lo + w_tile + 6u), idesc, 1u);
                    }
                    mma_commit_pair(empty_w0 + 8u * (uint32_t)ws, kPair);
                    // A chunks whose last k-step is issued go back to the producers
                    while (hr < nch && ((hr + 1) * cks < nks ? (hr + 1) * cks : nks) - 1 <= slast) {
                        mma_commit_pair(empty_a0 + 8u * (uint32_t)hr, kPair);
                        ++hr;
                    }
                    ++g_cons;
                    if (++ws == nb) { ws = 0; wph ^= 1; }
                    a_lo += kTile;
                }
                if (!ok) break;
                mma_commit_pair(smem_addr(&tfull[acc]), kPair);
                if (++acc == 2) { acc = 0; accph ^= 1; }
                if (lastA) aph ^= 1;
            }
            *consumed_w = (uint32_t)g_cons;
            // Every MMA issued so far completes before the pair frees its TMEM,
            // also after an aborted wait.
            mma_drain(smem_addr(mma_done));
        }
    } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + 4) {
        // ---------------- epilogue (both CTAs)
        const int wq = warp & 3;   // TMEM lane quarter this warp may access
        const uint32_t tempty0 = mapa_shared(smem_addr(&tempty[0]), 0);
        uint8_t *stage_buf = epi + (size_t)wq * P.epi_bufs * (P.out_f32 ? 4096 : 2048);
        const int nchk = P.bn / 32;   // 2, 4 or 8
        int acc = 0, nbuf = 0;
        uint32_t accph = 0;
        auto passes = [&](auto kPos) {
            constexpr bool has_pos = decltype(kPos)::value;
            for (int q = q0; q < q1; ++q) {
                const int m_blk = q / ntn, n_blk = q - m_blk * ntn;
                if (!mbar_wait_lim(smem_addr(&tfull[acc]), accph, abort, P.wait_ns)) break;
                tc_fence_after();
                const int64_t row0 = (int64_t)m_blk * (2 * kBM) + rank * kBM + wq * 32;
                const uint32_t tbase = tmem_base + ((uint32_t)(wq * 32) << 16) + (uint32_t)(acc * kMaxBN);
                const int col_base = n_blk * P.bn;
                // one TMEM chunk at a time (640 threads leave no registers for a second buffer)
                uint32_t va[32];
                for (int cc = 0; cc < nchk; ++cc) {
                    tmem_ld_32x32b_x32(tbase + (uint32_t)cc * 32, va);
                    tmem_ld_wait();
                    if (P.epi_bufs > 0)
                        as_emit<has_pos>(P, &tmap_out, va, col_base + cc * 32, row0, stage_buf, nbuf, lane);
                    else
                        as_emit_direct<has_pos>(P, va, col_base + cc * 32, row0, lane);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(tempty0 + 8u * (uint32_t)acc);
                if (++acc == 2) { acc = 0; accph ^= 1; }
            }
        };
        if (P.pos) passes(std::true_type{}); else passes(std::false_type{});
        if (lane == 0) bulk_wait<0>();
        __syncwarp();
    } else if (warp >= kAsProdWarp0 && warp < kAsProdWarp0 + kAsProdWarps) {
        // ---------------- A producers (both CTAs)
        as_produce<PT, NORM>(P, a_buf, empty_a, mapa_shared(smem_addr(&full_a[0]), 0), abort, q0, q1,
                             (int)threadIdx.x - 32 * kAsProdWarp0, lane, rank);
    }

    tc_fence_before();
    __syncthreads();
    if (*abort) {
        // Weight loads already issued must land before the CTA exits: the
        // leader waits (bounded) for every posted phase the MMA did not
        // consume; the peer's loads complete on the leader's barriers too.
        if (leader && threadIdx.x == 0) {
            // stages g >= consumed were posted by issuer g % n_iss if g is
            // below its count; at most nb of them can be in flight
            const uint32_t g0 = *consumed_w;
            for (uint32_t g = g0; g < g0 + (uint32_t)nb; ++g) {
                if (g >= posted_w[g % (uint32_t)P.n_iss]) continue;
                const uint32_t bar = smem_addr(&full_w[g % (uint32_t)nb]);
                const uint32_t par = (g / (uint32_t)nb) & 1u;
                const uint64_t t0 = global_timer_ns();
                while (!mbar_try_wait(bar, par) && global_timer_ns() - t0 < kAsDrainNs) {
                }
            }
        }
        // a load a CTA issued without a posted phase: a short grace period
        if (threadIdx.x == 0) {
            const uint64_t t0 = global_timer_ns();
            while (global_timer_ns() - t0 < 20000ull) __nanosleep(1000);
        }
        __syncthreads();
    }
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, 512);
    }
    if (threadIdx.x == 0 && *abort) atomicExch(P.err, (int)PE_ERR_DEVICE_TIMEOUT);
}

}  // namespace pe
