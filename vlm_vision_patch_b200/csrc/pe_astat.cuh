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
//   warps 8-15     A producers: gather + normalise into the resident A
//
// The resident A is split into chunks of kAsChunkKs k-steps, each with a
// full and an empty barrier.  The first pass over an M-block waits for each
// chunk as it arrives; the last pass releases each chunk once its MMAs are
// done, so the next M-block's gather overlaps the end of the previous block's
// last pass.  Every wait is bounded (FwdParams::wait_ns, default
// kWaitTimeoutNs); after an abort the kernel drains its MMAs and weight
// loads (bounded), frees the TMEM and records PE_ERR_DEVICE_TIMEOUT.
#pragma once

#include "pe_kernels.cuh"

namespace pe {

constexpr int kAsThreads = 512;                  // 16 warps
constexpr int kAsProdWarp0 = 8;                  // warps 8..15 build A
constexpr int kAsProdWarps = 8;
constexpr int kAsChunkKs = 4;                    // k-steps per A chunk: 64 columns, 16 KB for 128 rows
constexpr int kAsChunkGroups = 2 * kAsChunkKs;   // 8-column groups per chunk
constexpr int kAsMaxChunks = 16;                 // resident A of at most 1024 columns
constexpr int kAsDepth = 3;                      // chunks of pixel loads in flight per producer thread
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

__device__ __forceinline__ void prefetch_l2(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

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

// Source of one output row for the producers: the byte address of pixel
// (c = 0, y = g_h*p, x = g_w*p) of the row's single frame, and the row and
// plane strides in elements.
struct AsRow {
    const char *base;
    int32_t W, HW;
    bool ok;
};

__device__ __forceinline__ AsRow as_row(const FwdParams &P, int64_t R) {
    AsRow s;
    s.ok = R < P.N;
    s.base = nullptr;
    s.W = s.HW = 0;
    if (s.ok) {
        const RowSrc rs = locate_row(P, R, 2);
        s.base = rs.base;
        s.W = rs.W;
        s.HW = rs.HW;
    }
    return s;
}

// Element offset of in-slice column k = (c*p + i)*p + j of a row.
template <int PT>
__device__ __forceinline__ int64_t as_col_off(int k, int p, const AsRow &s) {
    const int pp = PT ? PT : p;
    const int seg = k / pp, j = k - seg * pp, c = seg / pp, i = seg - c * pp;
    return (int64_t)c * s.HW + (int64_t)i * s.W + j;
}

// A producers (warps 8..15 of both CTAs).  Resident A layout: no-swizzle
// K-major, element (r, k) at (k / 8) * 2048 + r * 16 + (k % 8) * 2, i.e. one
// 2 KB block of 128 rows x 16 bytes per 8-column group.  Lane L of producer
// warp pw owns rows 8*pw + L/4 and 64 + 8*pw + L/4 and word L%4 of every
// 8-column group, so a warp's 32 four-byte stores of one group fill 128
// contiguous bytes (no bank conflict) and its loads touch the 16 bytes of
// each of 8 patch-row segments.  Chunk h of the M-block (groups
// 8h .. 8h+7) is loaded kAsDepth - 1 chunks ahead of the one being stored, so
// pixel loads overlap the wait for the chunk's release; the next M-block's
// pixels are also prefetched into L2 when a block starts.
template <int PT, int NORM>
__device__ __forceinline__ void as_produce(const FwdParams &P, uint8_t *a_buf, uint64_t *empty_a,
                                           uint32_t full_a_leader, volatile int *abort, int q0, int q1, int pw,
                                           int lane, uint32_t rank) {
    const int p = PT ? PT : P.P;
    const int ntn = P.n_tiles_n;
    const int ngr = P.Kh >> 3;         // 8-column groups of the resident A
    const int nch = P.n_achunks;
    const int cpp = P.cpp;
    const int nseg = P.C * p;          // (c, i) image-row segments of one row
    const int ro = lane >> 2, m = lane & 3;
    const int rloc[2] = {8 * pw + ro, 64 + 8 * pw + ro};
    if (q0 >= q1) return;
    const int mfirst = q0 / ntn, mlast = (q1 - 1) / ntn;
    const int total = (mlast - mfirst + 1) * nch;
    const uint32_t abase = smem_addr(a_buf);

    AsRow src[2];
    uint32_t raw[kAsDepth][2][kAsChunkGroups];

    auto prefetch_block = [&](int mb) {
#pragma unroll
        for (int o = 0; o < 2; ++o) {
            const AsRow s = as_row(P, (int64_t)mb * (2 * kBM) + rank * kBM + rloc[o]);
            if (!s.ok) continue;
            for (int seg = m; seg < nseg; seg += 4) {
                const int c = seg / p, i = seg - c * p;
                const char *a = s.base + ((int64_t)c * s.HW + (int64_t)i * s.W) * 2;
                prefetch_l2(a);
                prefetch_l2(a + 2 * p - 1);
            }
        }
    };
    auto load = [&](const int idx, const int b) {
        const int mbi = idx / nch, h = idx - mbi * nch;
        if (h == 0) {
            const int mb = mfirst + mbi;
#pragma unroll
            for (int o = 0; o < 2; ++o) src[o] = as_row(P, (int64_t)mb * (2 * kBM) + rank * kBM + rloc[o]);
            if (idx == 0) prefetch_block(mb);
            if (mb < mlast) prefetch_block(mb + 1);
        }
#pragma unroll
        for (int gi = 0; gi < kAsChunkGroups; ++gi) {
            const int g = kAsChunkGroups * h + gi;
            const int k = 8 * g + 2 * m;
            const bool live = g < ngr && k < cpp;
#pragma unroll
            for (int o = 0; o < 2; ++o) {
                raw[b][o][gi] = 0u;
                if (live && src[o].ok) {
                    const char *a = src[o].base + as_col_off<PT>(k, p, src[o]) * 2;
                    asm volatile("ld.global.nc.b32 %0, [%1];" : "=r"(raw[b][o][gi]) : "l"(a));
                }
            }
        }
    };
    auto store = [&](const int idx, const int b) -> bool {
        const int G = idx / nch, h = idx - G * nch;
        if (!mbar_wait_lim(smem_addr(&empty_a[h]), (G & 1) ^ 1, abort, P.wait_ns)) return false;
#pragma unroll
        for (int gi = 0; gi < kAsChunkGroups; ++gi) {
            const int g = kAsChunkGroups * h + gi;
            if (g >= ngr) break;
            const int k = 8 * g + 2 * m;
            const bool live = k < cpp;
            const NormConst nc = norm_const(P, live ? k / (p * p) : 0);
            const uint32_t goff = abase + (uint32_t)g * 2048u + (uint32_t)m * 4u;
#pragma unroll
            for (int o = 0; o < 2; ++o) {
                const uint32_t w = live ? norm_word<NORM>(raw[b][o][gi], nc) : 0u;
                sts32(goff + (uint32_t)rloc[o] * 16u, w);
            }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(full_a_leader + 8u * (uint32_t)h);
        return true;
    };

    // Software pipeline: chunk idx + kAsDepth - 1 is loaded before chunk idx
    // is stored; the register buffers rotate with a period of kAsDepth.
    static_assert(kAsDepth == 3, "the rotation below is written for three buffers");
    load(0, 0);
    if (total > 1) load(1, 1);
    for (int idx = 0; idx < total; idx += 3) {
        if (idx + 2 < total) load(idx + 2, 2);
        if (!store(idx, 0)) return;
        if (idx + 1 >= total) break;
        if (idx + 3 < total) load(idx + 3, 0);
        if (!store(idx + 1, 1)) return;
        if (idx + 2 >= total) break;
        if (idx + 4 < total) load(idx + 4, 1);
        if (!store(idx + 2, 2)) return;
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
    uint32_t *posted_w = reinterpret_cast<uint32_t *>(mma_done + 1);   // leader: weight phases posted per slot
    uint32_t *consumed_w = posted_w + nb;                               // leader: weight phases consumed per slot
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
                    if (leader) {
                        mbar_arrive_expect_tx(smem_addr(&full_w[s]), 2u * slot);
                        atomicAdd(&posted_w[s], 1u);
                    }
                    tma_load_2d_pair(smem_addr(w_ring + (size_t)s * slot), &tmap_w, fb0 + 8u * (uint32_t)s, 64 * j,
                                     wrow, pol_w);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (leader CTA only)
        if (leader && lane == 0) {
            constexpr uint16_t kPair = 0x3;
            const uint32_t idesc = idesc_bf16_f32(2 * kBM, P.bn);
            const uint64_t a0 = smem_desc(smem_addr(a_buf), 2048, 128, kLayoutInterleave);
            const uint64_t b0 = smem_desc(smem_addr(w_ring), 16, 1024, kLayoutSw128);
            const uint32_t a_lo0 = (uint32_t)a0, b_lo0 = (uint32_t)b0;
            const uint32_t w_slot = (uint32_t)P.b_slot_bytes >> 4;
            const int nks = P.num_ksteps, nst = P.n_b_stages;
            int ws = 0, acc = 0;
            uint32_t wph = 0, accph = 0, aph = 0;
            for (int q = q0; q < q1; ++q) {
                const int n = q % ntn;
                const bool newA = (q == q0) || n == 0;
                const bool lastA = (q == q1 - 1) || n == ntn - 1;
                if (!mbar_wait_lim(smem_addr(&tempty[acc]), accph ^ 1, abort, P.wait_ns)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)acc * kMaxBN;
                int next_wait = newA ? 0 : nks;                   // k-step whose chunk is awaited next
                int next_rel = lastA ? kAsChunkKs - 1 : nks + 1;  // k-step after which a chunk is released
                int hw = 0, hr = 0;
                bool ok = true;
                for (int j = 0; j < nst && ok; ++j) {
                    if (!mbar_wait_lim(smem_addr(&full_w[ws]), wph, abort, P.wait_ns)) { ok = false; break; }
                    ++consumed_w[ws];
                    tc_fence_after();
                    const uint32_t b_lo = b_lo0 + (uint32_t)ws * w_slot;
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk) {
                        const int s = 2 * j + kk;
                        if (s < nks) {
                            if (s == next_wait) {
                                if (!mbar_wait_lim(smem_addr(&full_a[hw]), aph, abort, P.wait_ns)) { ok = false; break; }
                                tc_fence_after();
                                ++hw;
                                next_wait += kAsChunkKs;
                            }
                            const uint64_t ad = desc_with_lo(a0, a_lo0 + (uint32_t)s * (4096u >> 4));
                            // slice 0 at byte 32*kk of the tile, slice 1 at 64 + 32*kk
                            mma_bf16_pair(d_tmem, ad, desc_with_lo(b0, b_lo + 2u * kk), idesc, (j | kk) ? 1u : 0u);
                            mma_bf16_pair(d_tmem, ad, desc_with_lo(b0, b_lo + 4u + 2u * kk), idesc, 1u);
                            if (s == next_rel || (lastA && s == nks - 1)) {
                                mma_commit_pair(smem_addr(&empty_a[hr]), kPair);
                                ++hr;
                                next_rel += kAsChunkKs;
                            }
                        }
                    }
                    if (!ok) break;
                    mma_commit_pair(smem_addr(&empty_w[ws]), kPair);
                    if (++ws == nb) { ws = 0; wph ^= 1; }
                }
                if (!ok) break;
                mma_commit_pair(smem_addr(&tfull[acc]), kPair);
                if (++acc == 2) { acc = 0; accph ^= 1; }
                if (lastA) aph ^= 1;
            }
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
                if constexpr (!has_pos) {
                    // the next chunk's TMEM load overlaps this chunk's conversion and store
                    uint32_t va[32], vb[32];
                    tmem_ld_32x32b_x32(tbase, va);
                    for (int cc = 0; cc < nchk; cc += 2) {
                        tmem_ld_wait();
                        tmem_ld_32x32b_x32(tbase + (uint32_t)(cc + 1) * 32, vb);
                        as_emit<false>(P, &tmap_out, va, col_base + cc * 32, row0, stage_buf, nbuf, lane);
                        tmem_ld_wait();
                        if (cc + 2 < nchk) tmem_ld_32x32b_x32(tbase + (uint32_t)(cc + 2) * 32, va);
                        as_emit<false>(P, &tmap_out, vb, col_base + (cc + 1) * 32, row0, stage_buf, nbuf, lane);
                    }
                } else {
                    // the position rows need the registers of the second buffer
                    uint32_t va[32];
                    for (int cc = 0; cc < nchk; ++cc) {
                        tmem_ld_32x32b_x32(tbase + (uint32_t)cc * 32, va);
                        tmem_ld_wait();
                        as_emit<true>(P, &tmap_out, va, col_base + cc * 32, row0, stage_buf, nbuf, lane);
                    }
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
                             warp - kAsProdWarp0, lane, rank);
    }

    tc_fence_before();
    __syncthreads();
    if (*abort) {
        // Weight loads already issued must land before the CTA exits: the
        // leader waits (bounded) for every posted phase the MMA did not
        // consume; the peer's loads complete on the leader's barriers too.
        if (leader && threadIdx.x == 0) {
            for (int s = 0; s < nb; ++s) {
                if (posted_w[s] <= consumed_w[s]) continue;
                const uint32_t bar = smem_addr(&full_w[s]);
                const uint32_t par = (posted_w[s] - 1u) & 1u;
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
