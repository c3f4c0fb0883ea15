// sm_100a kernels of the vision PatchEmbed (and of the PatchMerger that
// consumes its rows).
//
// The PatchEmbed is a Conv3d whose kernel equals its stride, i.e. one dense
// contraction out[N, E] = A[N, K] * W[E, K]^T (+ bias) with K = C*tp*p*p
// (Qwen2.5VL-Vision Encode-PatchEmbed: the conv is a dot product of the
// flattened input and weight; mytransformer README §4.1: F.linear(x,
// w.reshape(1280, 1176))).  One persistent kernel, pe_fwd_kernel, runs the
// contraction on CTA pairs (thread-block clusters of 2) that share each
// 256 x BN output tile through the pair form of the 5th-generation MMA
// (tcgen05 cta_group::2): every CTA stages its own 128 rows of A and BN/2 rows
// of the weight, the leader CTA issues the MMAs, and each CTA accumulates its
// 128 rows x BN fp32 in its own tensor memory.
//
//   warps 0, 2, 3 (+ 8, 9 when A is TMA-fed; + 16, 17 in the streamed mode)
//               TMA issuers: weight tiles, and A tiles in the TMA-fed modes
//   warp 1      TMEM owner; in the leader CTA one thread issues the MMAs
//   warps 4-7   epilogue: TMEM -> registers, + bias (+ position table, GELU),
//               cast, TMA stores
//   warps 8-19  A producers of the thread-fed modes: fp32 / unaligned patch
//               rows converted to bf16, or the fused frames gather that builds
//               each patch row from raw [T, C, H, W] frames, normalises it and
//               places it in merge order, straight into shared memory
//               (warps 8-15 write rows to global memory in the streamed mode).
//
// The A modes (AMode below) select how A reaches shared memory.  The
// accumulator is double buffered (2 x 256 TMEM columns) so the epilogue of one
// tile overlaps the MMAs of the next.  Every pipeline wait is bounded.
//
// Around it: the staged prepare kernel (pe_prep_rows_kernel), the fp32 casts
// (pe_cast_rows_kernel, pe_round_tf32_kernel), the weight packers, the
// patchify test hook, the PatchMerger's LayerNorm (pe_layernorm_kernel) and
// the failure self-test (pe_wait_timeout_probe_kernel).
#pragma once

#include <type_traits>

#include "pe_device.cuh"
#include "../../include/pe.h"

namespace pe {

constexpr int kThreads = 640;       // 20 warps (A produced by threads)
constexpr int kThreadsTma = 320;    // 10 warps (A fetched by TMA)
__host__ __device__ constexpr int threads_for(int amode) {
    return (amode == 0 || amode == 3 || amode == 5) ? kThreadsTma : kThreads;
}
constexpr int kStreamProdWarp0 = 8;   // kAModeTmaStream: warps 8..15 produce rows
constexpr int kStreamProdWarps = 8;
constexpr int kBM = 128;           // rows per CTA (pair tile: 256 rows)
constexpr int kMaxBN = 256;        // largest pair-MMA N
constexpr int kBK = 64;            // weight K per TMA stage (one 128-byte swizzle row)
constexpr int kProdThreads = 384;  // warps 8..19
constexpr int kProdWarps = 12;
constexpr int kEpiWarp0 = 4;
constexpr int kBStageBytes = (kMaxBN / 2) * kBK * 2;   // 16 KB: this CTA's half of the weight tile

// How the A operand reaches shared memory:
//   kAModeTma          TMA tiles of bf16 rows A[N, K] (patches, or the staged frames rows)
//   kAModePatchThreads fp32 / unaligned patch rows converted by producer warps
//   kAModeFrames       the fused gather from raw frames by producer warps
//   kAModeTmaShared    TMA tiles of single-frame rows A[N, Kh] that both temporal
//                      slices share: every A tile meets the weight tiles of
//                      slice 0 and slice 1 at the same in-slice k (tp = 2).
//   kAModeTmaStream    the rows are written by producer warps of the same grid
//                      into a global buffer in the slice-major layout and read
//                      back by TMA once their M-block is complete: single-frame
//                      rows as in kAModeTmaShared (DUPALL), otherwise both
//                      slices per row against the slice-major weight.
//   kAModeTmaTf32      TMA tiles of fp32 rows (tf32-rounded) against the
//                      tf32-rounded fp32 weight, kind::tf32 MMAs (K = 8 each)
enum AMode : int {
    kAModeTma = 0, kAModePatchThreads = 1, kAModeFrames = 2, kAModeTmaShared = 3, kAModeTmaStream = 4,
    kAModeTmaTf32 = 5
};
__host__ __device__ constexpr bool tma_fed(int amode) {
    return amode == kAModeTma || amode == kAModeTmaShared || amode == kAModeTmaStream || amode == kAModeTmaTf32;
}

struct ItemDesc {
    const void *frames;  // [T, C, H, W]
    int64_t row0;        // first output row of the item
    int32_t T, H, W;
    int32_t gt, gh, gw;
};

struct FwdParams {
    int32_t E, C, TP, P, K, Kpad;
    int32_t Kh;                                     // slice length of the shared-slice weight (C*p*p rounded to 16)
    int32_t bn, n_tiles_n, num_tiles, num_ksteps;   // num_tiles counts pair tiles
    int32_t n_b_stages, n_a_stages;                 // per tile
    int32_t nb, na;                                 // ring depths
    int32_t n_iss;                                  // TMA issuer warps, <= min(nb, na)
    int32_t a_stage_bytes;
    int32_t b_slot_bytes;                           // weight ring slot: ksub * slices * 16 KB
    int32_t ksub;                                   // TMA-fed modes: 64-wide k sub-tiles per stage (1 or 2)
    int32_t epi_offset;                             // staging area offset past the rings
    int32_t merge, n_items;
    int32_t all_t1;                   // every item is a single frame (host-side kernel choice)
    int64_t N;
    const ItemDesc *items_dev;        // table in device memory when n_items > PE_INLINE_ITEMS
    ItemDesc items[PE_INLINE_ITEMS];
    float mean[4], stdv[4];           // per-channel normalisation (see NormMode)
    float nstd_s[4], rcp_s[4], scale[4];
    int32_t norm_mode[4];
    const void *x;                    // patches input
    int32_t x_f32;                    // patches dtype is fp32
    int32_t x_vec;                    // patch rows allow 16-byte vector loads
    int32_t out_f32;
    const float *bias;                // fp32 [E] or nullptr
    const void *pos;                  // [N, E] added in the epilogue, or nullptr
    int32_t pos_f32;                  // pos dtype is fp32 (else bf16)
    int32_t act;                      // epilogue activation after bias: 0 none, 1 exact GELU
    int *err;                         // device error word
    // kAModeTmaStream
    uint16_t *a_rows;                 // [N, row_elems] rows written by the producers
    int32_t row_elems;                // slices * Kh
    uint32_t *ready;                  // per M-block count of finished producer parts (this call)
    uint32_t *ready_next;             // the next call's counters, zeroed by this call
    uint32_t ready_target;            // count that marks an M-block complete
    int32_t n_mblocks;
    // pe_astat_kernel (resident A)
    int32_t a_offset, bar_offset;     // shared-memory offsets of the resident A and of the barriers
    int32_t n_achunks;                // A chunks of 8 image-row segments (p/2 k-steps)
    int32_t epi_bufs;                 // staging boxes per epilogue warp (0: stores straight from registers)
    void *out;                        // [N, E] output (the direct-store epilogue)
    int32_t cpp;                      // C*p*p: columns of one temporal slice
    uint64_t wait_ns;                 // pipeline wait limit in ns (0: kWaitTimeoutNs)
    int32_t epi_v8;                   // register-store epilogue: out and its rows are 32-byte aligned
};

// ------------------------------------------------------------ debug bounds
//
// Built with -DPE_DEBUG_BOUNDS (libpe_debug.so, vlm_vision_patch_b200.build
// --debug-bounds): each data-dependent global access of the kernels (pixel
// gathers through the item table, streamed patch-row stores, position-table
// loads, register-to-global output stores) first checks that its address
// range lies inside the buffer it indexes.  An access outside records
// PE_ERR_DEVICE_BOUNDS in the kernel's error word and is skipped (a load
// reads zero).  TMA accesses are range-checked by the hardware against their
// tensor maps; the elementwise kernels index inside their own loop bounds.
// Without the macro PE_IN is the constant true and the checks compile to
// nothing.
#ifdef PE_DEBUG_BOUNDS
__device__ __forceinline__ bool dbg_in(const void *a, int64_t bytes, const void *lo, const void *hi, int *err) {
    const char *q = static_cast<const char *>(a);
    if (q >= static_cast<const char *>(lo) && q + bytes <= static_cast<const char *>(hi)) return true;
    if (err) atomicExch(err, (int)PE_ERR_DEVICE_BOUNDS);
    return false;
}
#define PE_IN(a, n, lo, hi, err) ::pe::dbg_in((a), (n), (lo), (hi), (err))
#else
#define PE_IN(a, n, lo, hi, err) ((void)(lo), (void)(hi), true)
#endif

// ------------------------------------------------------------ row decoding

__device__ __forceinline__ const ItemDesc &item_at(const FwdParams &P, int i) {
    return P.n_items <= PE_INLINE_ITEMS ? P.items[i] : P.items_dev[i];
}

__device__ __forceinline__ int find_item(const FwdParams &P, int64_t R) {
    int lo = 0, hi = P.n_items - 1;
    while (lo < hi) {  // last item with row0 <= R
        const int mid = (lo + hi + 1) >> 1;
        if (item_at(P, mid).row0 <= R) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Output row R -> the patch it embeds.  Items are concatenated in list order;
// inside an item rows follow the spatial-merge order for merge = 2 (2x2 windows
// consecutive, windows row-major over (t, h/2, w/2), (dh, dw) row-major inside)
// or raster order (t, h, w) for merge = 1.
struct RowSrc {
    const char *base;   // byte address of pixel (frame tau0, c = 0, y = g_h*p, x = g_w*p)
    int32_t W;          // elements per image row
    int32_t HW;         // elements per channel plane
    int32_t CHW;        // elements per frame
    int32_t tmax;       // last usable temporal offset: min(t, tmax) frames past tau0
    const char *lo, *hi;  // the item's frame buffer (filled in the bounds-checking build only)
};

__device__ __forceinline__ RowSrc locate_row(const FwdParams &P, int64_t R, int esize) {
    const ItemDesc &it = item_at(P, find_item(P, R));
    const int64_t rho = R - it.row0;
    int64_t g_t, g_h, g_w;
    if (P.merge == 2) {
        const int64_t win = rho >> 2;
        const int d = (int)(rho & 3);
        const int64_t wpr = it.gw >> 1, wpt = (int64_t)(it.gh >> 1) * wpr;
        g_t = win / wpt;
        const int64_t rem = win - g_t * wpt;
        const int64_t wy = rem / wpr;
        g_h = 2 * wy + (d >> 1);
        g_w = 2 * (rem - wy * wpr) + (d & 1);
    } else {
        g_w = rho % it.gw;
        const int64_t tmp = rho / it.gw;
        g_h = tmp % it.gh;
        g_t = tmp / it.gh;
    }
    int64_t tau0 = g_t * P.TP;
    if (tau0 > it.T - 1) tau0 = it.T - 1;
    RowSrc s;
    s.W = it.W;
    s.HW = it.H * it.W;
    s.CHW = P.C * s.HW;
    s.tmax = (int32_t)(it.T - 1 - tau0);
    const int64_t el = (tau0 * P.C * it.H + g_h * P.P) * (int64_t)it.W + g_w * P.P;
    s.base = reinterpret_cast<const char *>(it.frames) + el * esize;
    s.lo = s.hi = nullptr;
#ifdef PE_DEBUG_BOUNDS
    s.lo = reinterpret_cast<const char *>(it.frames);
    s.hi = s.lo + (int64_t)it.T * P.C * it.H * it.W * esize;
#endif
    return s;
}

// ------------------------------------------------------------ normalisation

// Per-channel pixel normalisation x_hat = bf16_rne(fp32(fp32(x - mean) / std)),
// bit-identical to an IEEE fp32 subtract and divide for every finite input.
// The host picks one mode per channel:
//   kNormIdentity  mean == +0 and std == 1: x_hat = bf16_rne(x), a plain copy
//                  for bf16 frames.
//   kNormScaled    |mean| >= 2^-70 and 2^-32 <= std <= 2^32: std = s * 2^-k with
//                  s in [1, 2).  q0 = d * rcp(s), one fused multiply-add
//                  correction q = q0 + (d - q0 * s) * rcp(s) -- Markstein's
//                  final step, which returns the correctly rounded quotient when
//                  rcp(s) is correctly rounded and nothing over/underflows
//                  (P. Markstein, IBM J. Res. Dev. 34(1), 1990) -- then the
//                  exact scaling q * 2^k.  With s in [1, 2) the first product
//                  cannot overflow, and |mean| >= 2^-70 keeps d = x - mean
//                  either 0 or above 2^-93, so the residual never underflows;
//                  an overflowing quotient still rounds to +-inf in the final
//                  scaling.  Checked exhaustively against IEEE division.
//   kNormDivide    anything else: the IEEE divide itself, per element.
enum NormMode : int { kNormIdentity = 0, kNormScaled = 1, kNormDivide = 2 };

struct NormConst {
    float mean, stdv, nstd_s, rcp_s, scale;
    int mode;
};

__device__ __forceinline__ NormConst norm_const(const FwdParams &P, int c) {
    NormConst n;
    n.mean = P.mean[c];
    n.stdv = P.stdv[c];
    n.nstd_s = P.nstd_s[c];
    n.rcp_s = P.rcp_s[c];
    n.scale = P.scale[c];
    n.mode = P.norm_mode[c];
    return n;
}

// Two pixels (lo, hi) -> their normalised values packed as bf16 x 2.
__device__ __forceinline__ uint32_t norm_pair_f32(float x0, float x1, const NormConst &n) {
    if (n.mode == kNormScaled) {
        uint64_t X, M, R, NS, SC, D, Q0, Er, Q;
        asm("mov.b64 %0, {%1, %2};" : "=l"(X) : "f"(x0), "f"(x1));
        asm("mov.b64 %0, {%1, %1};" : "=l"(M) : "f"(n.mean));
        asm("mov.b64 %0, {%1, %1};" : "=l"(R) : "f"(n.rcp_s));
        asm("mov.b64 %0, {%1, %1};" : "=l"(NS) : "f"(n.nstd_s));
        asm("mov.b64 %0, {%1, %1};" : "=l"(SC) : "f"(n.scale));
        asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(D) : "l"(X), "l"(M));
        asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(Q0) : "l"(D), "l"(R));
        asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(Er) : "l"(Q0), "l"(NS), "l"(D));
        asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(Q) : "l"(Er), "l"(R), "l"(Q0));
        asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(Q) : "l"(Q), "l"(SC));
        float q0, q1;
        asm("mov.b64 {%0, %1}, %2;" : "=f"(q0), "=f"(q1) : "l"(Q));
        return pack_bf16x2(q0, q1);
    }
    if (n.mode == kNormDivide)
        return pack_bf16x2(__fdiv_rn(__fsub_rn(x0, n.mean), n.stdv), __fdiv_rn(__fsub_rn(x1, n.mean), n.stdv));
    return pack_bf16x2(x0, x1);
}

// Same for a raw bf16 x 2 word; the identity mode is then the word itself.
__device__ __forceinline__ uint32_t norm_pair_bf16(uint32_t w, const NormConst &n) {
    if (n.mode == kNormIdentity) return w;
    return norm_pair_f32(bf16lo_to_f32(w), bf16hi_to_f32(w), n);
}

// One 2-pixel word of a frame row: the raw bf16 x 2 word, or two fp32.
template <bool F32IN> struct PixPair;
template <> struct PixPair<false> {
    uint32_t w;
    __device__ __forceinline__ void load(const char *p, const char *lo, const char *hi, int *err) {
        w = 0u;
        if (PE_IN(p, 4, lo, hi, err)) asm volatile("ld.global.nc.b32 %0, [%1];" : "=r"(w) : "l"(p));
    }
    __device__ __forceinline__ void zero() { w = 0u; }
    __device__ __forceinline__ uint32_t norm(const NormConst &n) const { return norm_pair_bf16(w, n); }
};
template <> struct PixPair<true> {
    float a, b;
    __device__ __forceinline__ void load(const char *p, const char *lo, const char *hi, int *err) {
        a = b = 0.f;
        if (PE_IN(p, 8, lo, hi, err)) asm volatile("ld.global.nc.v2.f32 {%0, %1}, [%2];" : "=f"(a), "=f"(b) : "l"(p));
    }
    __device__ __forceinline__ void zero() { a = b = 0.f; }
    __device__ __forceinline__ uint32_t norm(const NormConst &n) const { return norm_pair_f32(a, b, n); }
};

// ------------------------------------------------------------- producers

// Unit u of a segment (one 2-pixel word of one tile row) -> (tile row, word).
// For merge = 2 the order walks patch-row halves of the windows so that
// consecutive u read consecutive words of one image row.
template <int RB = kBM>
__device__ __forceinline__ void unit_to_row_word(int u, int ws, int merge, int &r, int &jw) {
    jw = u % ws;
    const int t1 = u / ws;
    if (merge == 2) {
        const int dw = t1 & 1, t2 = t1 >> 1;
        const int q = t2 % (RB / 4), dh = t2 / (RB / 4);
        r = 4 * q + 2 * dh + dw;
    } else {
        r = t1;
    }
}

// Shared state of the A producers of one CTA.
struct ProdCtx {
    uint8_t *a_ring;
    uint64_t *empty_a;          // this CTA's empty barriers
    uint32_t full_a_leader;     // shared::cluster address of the leader's full_a[0]
    volatile int *abort;
    int pt, lane;
    uint32_t rank;
};

// The stage's generic-proxy writes become visible to the MMA, then one arrival
// per warp on the leader's full barrier.
__device__ __forceinline__ void producer_release(const ProdCtx &X, int stage) {
    fence_proxy_async_smem();
    __syncwarp();
    if (X.lane == 0) mbar_arrive_cluster(X.full_a_leader + 8u * (uint32_t)stage);
}

// Normalisation of one raw bf16 x 2 word for a channel whose mode the kernel
// knows at compile time: NORM 0 = identity (the word itself), 1 = the scaled
// correctly rounded quotient, 2 = decided at run time per channel.
template <int NORM>
__device__ __forceinline__ uint32_t norm_word(uint32_t w, const NormConst &n) {
    if constexpr (NORM == 0) {
        return w;
    } else if constexpr (NORM == 1) {
        uint64_t X, M, R, NS, SC, D, Q0, Er, Q;
        asm("mov.b64 %0, {%1, %2};" : "=l"(X) : "f"(bf16lo_to_f32(w)), "f"(bf16hi_to_f32(w)));
        asm("mov.b64 %0, {%1, %1};" : "=l"(M) : "f"(n.mean));
        asm("mov.b64 %0, {%1, %1};" : "=l"(R) : "f"(n.rcp_s));
        asm("mov.b64 %0, {%1, %1};" : "=l"(NS) : "f"(n.nstd_s));
        asm("mov.b64 %0, {%1, %1};" : "=l"(SC) : "f"(n.scale));
        asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(D) : "l"(X), "l"(M));
        asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(Q0) : "l"(D), "l"(R));
        asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(Er) : "l"(Q0), "l"(NS), "l"(D));
        asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(Q) : "l"(Er), "l"(R), "l"(Q0));
        asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(Q) : "l"(Q), "l"(SC));
        float q0, q1;
        asm("mov.b64 {%0, %1}, %2;" : "=f"(q0), "=f"(q1) : "l"(Q));
        return pack_bf16x2(q0, q1);
    } else {
        return norm_pair_bf16(w, n);
    }
}

// Pipelined frames producer for bf16 frames with tp = 2 and a compile-time p.
// Each producer thread owns MAXIT (tile row, word) units.  The raw words of
// stage g+1 are loaded (coalesced 32-bit loads into registers) before stage g
// is normalised and stored, so one stage of loads is always in flight behind
// the arithmetic.  A row whose item is a single frame loads its words once and
// stores the normalised word to both temporal slices.
template <int PT, int NORM, bool DUPALL>
__device__ __forceinline__ void produce_frames_reg(const FwdParams &P, const ProdCtx &X) {
    constexpr int NT = DUPALL ? 1 : 2;    // temporal slices held per (c, i)
    constexpr int p = PT;
    constexpr int ws = p / 2;
    constexpr int units = kBM * ws;
    constexpr int MAXIT = (units + kProdThreads - 1) / kProdThreads;
    const int nci = P.C * p;             // (c, i) pairs; 4 per stage
    const int nst = P.n_a_stages;

    int rr[MAXIT], kw[MAXIT];
    bool uok[MAXIT];
#pragma unroll
    for (int v = 0; v < MAXIT; ++v) {
        const int u = X.pt + kProdThreads * v;
        uok[v] = u < units;
        int r = 0, jw = 0;
        if (uok[v]) unit_to_row_word(u, ws, P.merge, r, jw);
        rr[v] = r;
        kw[v] = 2 * jw;
    }
    auto soff = [&](int q, int v) -> uint32_t {
        const int k = q * p + kw[v];
        return (uint32_t)(k >> 3) * 2048u + (uint32_t)rr[v] * 16u + (uint32_t)(k & 7) * 2u;
    };
    const uint32_t ring = smem_addr(X.a_ring);
    const int tile0 = blockIdx.x >> 1, tstride = gridDim.x >> 1;
    const int n_my_tiles = (P.num_tiles > tile0) ? (P.num_tiles - tile0 + tstride - 1) / tstride : 0;
    const int total = n_my_tiles * nst;

    // load side: row sources of the tile being loaded
    const char *src[MAXIT];
    const char *dlo[MAXIT], *dhi[MAXIT];          // frame buffers (bounds-checking build)
    int32_t sW[MAXIT], sHW[MAXIT], sT1[MAXIT];   // sT1: byte offset of the t = 1 slice (0: same frame)
    int ld_lt = 0, ld_s = 0;
    uint32_t rokb[2] = {0u, 0u}, dupb[2] = {0u, 0u};
    uint32_t raw[2][4][NT][MAXIT];
    // normalise side
    int nm_s = 0;

    auto load_stage = [&](const int b) {    // loads the next stage of the load side into buffer b
        if (ld_s == 0) {
            const int tile = tile0 + ld_lt * tstride;
            const int64_t m0 = (int64_t)(tile / P.n_tiles_n) * (2 * kBM) + X.rank * kBM;
            uint32_t rk = 0, dp = 0;
#pragma unroll
            for (int v = 0; v < MAXIT; ++v) {
                src[v] = nullptr;
                sW[v] = sHW[v] = sT1[v] = 0;
                if (!(uok[v] && m0 + rr[v] < P.N)) continue;
                const RowSrc rs = locate_row(P, m0 + rr[v], 2);
                src[v] = rs.base + (int64_t)kw[v] * 2;
                dlo[v] = rs.lo;
                dhi[v] = rs.hi;
                sW[v] = rs.W * 2;
                sHW[v] = rs.HW * 2;
                sT1[v] = rs.tmax > 0 ? rs.CHW * 2 : 0;
                rk |= 1u << v;
                if (rs.tmax == 0) dp |= 1u << v;
            }
            rokb[b] = rk;
            dupb[b] = dp;
        } else {
            rokb[b] = rokb[b ^ 1];
            dupb[b] = dupb[b ^ 1];
        }
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
            const int ci = 4 * ld_s + qq;
            const int c = ci / p, i = ci - (ci / p) * p;
#pragma unroll
            for (int v = 0; v < MAXIT; ++v) {
#pragma unroll
                for (int t = 0; t < NT; ++t) raw[b][qq][t][v] = 0u;
                if (ci < nci && (rokb[b] >> v & 1u)) {
                    const char *a = src[v] + (int64_t)c * sHW[v] + (int64_t)i * sW[v];
                    if (PE_IN(a, 4, dlo[v], dhi[v], P.err))
                        asm volatile("ld.global.nc.b32 %0, [%1];" : "=r"(raw[b][qq][0][v]) : "l"(a));
                    if constexpr (!DUPALL) {
                        if (sT1[v] != 0 && PE_IN(a + sT1[v], 4, dlo[v], dhi[v], P.err))
                            asm volatile("ld.global.nc.b32 %0, [%1];" : "=r"(raw[b][qq][NT - 1][v]) : "l"(a + sT1[v]));
                    }
                }
            }
        }
        if (++ld_s == nst) { ld_s = 0; ++ld_lt; }
    };
    auto store_stage = [&](const int g, const int b) -> bool {   // normalise buffer b into stage g's slot
        const int slot = g % P.na;
        if (!mbar_wait(smem_addr(&X.empty_a[slot]), ((g / P.na) & 1) ^ 1, X.abort)) return false;
        const uint32_t As = ring + (uint32_t)slot * (uint32_t)P.a_stage_bytes;
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
            const int ci = 4 * nm_s + qq;
            const bool live = ci < nci;
            const NormConst nc = norm_const(P, live ? ci / p : 0);
#pragma unroll
            for (int v = 0; v < MAXIT; ++v) {
                if (!(rokb[b] >> v & 1u)) continue;
                uint32_t w0 = 0u, w1 = 0u;
                if (live) {
                    w0 = norm_word<NORM>(raw[b][qq][0][v], nc);
                    w1 = (DUPALL || (dupb[b] >> v & 1u)) ? w0 : norm_word<NORM>(raw[b][qq][NT - 1][v], nc);
                }
                sts32(As + soff(2 * qq, v), w0);
                sts32(As + soff(2 * qq + 1, v), w1);
            }
        }
        producer_release(X, slot);
        if (++nm_s == nst) nm_s = 0;
        return true;
    };

    if (total > 0) load_stage(0);
    for (int g = 0; g < total; g += 2) {
        if (g + 1 < total) load_stage(1);
        if (!store_stage(g, 0)) return;
        if (g + 1 >= total) break;
        if (g + 2 < total) load_stage(0);
        if (!store_stage(g + 1, 1)) return;
    }
}

// Frames producer.  The frames path runs in the K order k' = ((c*p + i)*tp + t)*p + j
// (the weight is packed in the same order), so that one A stage holds 8 whole
// segments (c, i, t) of p pixels: 4 (c, i) pairs x both temporal slices when
// tp = 2.  Layout: no-swizzle K-major, element (r, k') at
// (k' / 8) * 2048 + r * 16 + (k' % 8) * 2 of the stage.
template <int PT, bool F32IN>
__device__ __forceinline__ void produce_frames(const FwdParams &P, const ProdCtx &X) {
    const int p = PT ? PT : P.P;
    const int ws = p >> 1;
    const int units = kBM * ws;
    constexpr int MAXIT = (kBM * ((PT ? PT : PE_MAX_PATCH) / 2) + kProdThreads - 1) / kProdThreads;
    constexpr int esize = F32IN ? 4 : 2;
    const int TP = P.TP;
    const int nseg = P.C * TP * p;
    const int nci = P.C * p;            // (c, i) pairs

    int rr[MAXIT], kw[MAXIT];
    bool uok[MAXIT];
#pragma unroll
    for (int v = 0; v < MAXIT; ++v) {
        const int u = X.pt + kProdThreads * v;
        uok[v] = u < units;
        int r = 0, jw = 0;
        if (uok[v]) unit_to_row_word(u, ws, P.merge, r, jw);
        rr[v] = r;
        kw[v] = 2 * jw;
    }
    // shared-memory byte offset of (row, k' = q*p + kw) inside a stage
    auto soff = [&](int q, int v) -> uint32_t {
        const int k = q * p + kw[v];
        return (uint32_t)(k >> 3) * 2048u + (uint32_t)rr[v] * 16u + (uint32_t)(k & 7) * 2u;
    };

    int stage = 0;
    uint32_t phase = 0;
    for (int tile = blockIdx.x >> 1; tile < P.num_tiles; tile += gridDim.x >> 1) {
        const int64_t m0 = (int64_t)(tile / P.n_tiles_n) * (2 * kBM) + X.rank * kBM;
        if (m0 >= P.N) {
            // Nothing of this CTA's half exists: release the stages untouched
            // (their rows are never stored).
            for (int s = 0; s < P.n_a_stages; ++s) {
                if (!mbar_wait(smem_addr(&X.empty_a[stage]), phase ^ 1, X.abort)) return;
                producer_release(X, stage);
                if (++stage == P.na) { stage = 0; phase ^= 1; }
            }
            continue;
        }
        const int64_t mlast = (m0 + kBM - 1 < P.N) ? m0 + kBM - 1 : P.N - 1;
        const int it0 = find_item(P, m0);
        const bool fast = (TP == 2) && (it0 == find_item(P, mlast));
        const ItemDesc &itd = item_at(P, it0);
        const bool dup = fast && itd.T == 1;     // both temporal slices are the same frame
        const int uW = itd.W, uHW = itd.H * itd.W;

        const char *src[MAXIT];
        const char *dlo[MAXIT], *dhi[MAXIT];     // frame buffers (bounds-checking build)
        int32_t sW[MAXIT], sHW[MAXIT], sCHW[MAXIT], sTm[MAXIT];
        bool rok[MAXIT];
#pragma unroll
        for (int v = 0; v < MAXIT; ++v) {
            rok[v] = uok[v] && (m0 + rr[v] < P.N);
            src[v] = nullptr;
            dlo[v] = dhi[v] = nullptr;
            sW[v] = sHW[v] = sCHW[v] = sTm[v] = 0;
            if (rok[v]) {
                const RowSrc s = locate_row(P, m0 + rr[v], esize);
                src[v] = s.base + (int64_t)kw[v] * esize;
                dlo[v] = s.lo;
                dhi[v] = s.hi;
                sW[v] = s.W;
                sHW[v] = s.HW;
                sCHW[v] = s.CHW;
                sTm[v] = s.tmax;
            }
        }
        int c = 0, i = 0;   // (c, i) of the stage's first segment pair (fast path)
        for (int s = 0; s < P.n_a_stages; ++s) {
            if (!mbar_wait(smem_addr(&X.empty_a[stage]), phase ^ 1, X.abort)) return;
            uint8_t *As = X.a_ring + (size_t)stage * P.a_stage_bytes;
            if (fast) {
                // 4 (c, i) pairs, t = 0 and t = 1 each: segment q = 2 * qq + t
                PixPair<F32IN> px[4][2][MAXIT];
                int cq[4];
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    const bool live = (4 * s + qq) < nci;
                    cq[qq] = live ? c : -1;
                    const int64_t uoff = ((int64_t)c * uHW + (int64_t)i * uW) * esize;
#pragma unroll
                    for (int v = 0; v < MAXIT; ++v) {
                        px[qq][0][v].zero();
                        px[qq][1][v].zero();
                        if (live && rok[v]) {
                            px[qq][0][v].load(src[v] + uoff, dlo[v], dhi[v], P.err);
                            if (!dup) {
                                const int64_t t1 = (sTm[v] > 0 ? (int64_t)sCHW[v] : 0) * esize;
                                px[qq][1][v].load(src[v] + uoff + t1, dlo[v], dhi[v], P.err);
                            }
                        }
                    }
                    if (++i == p) { i = 0; ++c; }
                }
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    const int ch = cq[qq];
                    const NormConst nc = norm_const(P, ch < 0 ? 0 : ch);
#pragma unroll
                    for (int v = 0; v < MAXIT; ++v) {
                        if (!rok[v]) continue;
                        const uint32_t w0 = ch >= 0 ? px[qq][0][v].norm(nc) : 0u;
                        const uint32_t w1 = dup ? w0 : (ch >= 0 ? px[qq][1][v].norm(nc) : 0u);
                        *reinterpret_cast<uint32_t *>(As + soff(2 * qq, v)) = w0;
                        *reinterpret_cast<uint32_t *>(As + soff(2 * qq + 1, v)) = w1;
                    }
                }
            } else {
                PixPair<F32IN> px[8][MAXIT];
                int cq[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int seg = 8 * s + q;
                    const bool live = seg < nseg;
                    const int t = seg % TP, ci = seg / TP;
                    const int cc = ci / p, ii = ci - cc * p;
                    cq[q] = live ? cc : -1;
#pragma unroll
                    for (int v = 0; v < MAXIT; ++v) {
                        px[q][v].zero();
                        if (live && rok[v]) {
                            const int tt = t < sTm[v] ? t : sTm[v];
                            const int64_t off = (int64_t)tt * sCHW[v] + (int64_t)cc * sHW[v] + (int64_t)ii * sW[v];
                            px[q][v].load(src[v] + off * esize, dlo[v], dhi[v], P.err);
                        }
                    }
                }
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int ch = cq[q];
                    const NormConst nc = norm_const(P, ch < 0 ? 0 : ch);
#pragma unroll
                    for (int v = 0; v < MAXIT; ++v) {
                        if (!rok[v]) continue;
                        const uint32_t w = ch >= 0 ? px[q][v].norm(nc) : 0u;
                        *reinterpret_cast<uint32_t *>(As + soff(q, v)) = w;
                    }
                }
            }
            producer_release(X, stage);
            if (++stage == P.na) { stage = 0; phase ^= 1; }
        }
    }
}

// Patch-row producer for rows the TMA cannot fetch directly (fp32 rows, or bf16
// rows whose stride is not a multiple of 16 bytes): 64 k per stage, converted
// to bf16 (RNE) into the no-swizzle K-major layout.
__device__ __forceinline__ void produce_patches(const FwdParams &P, const ProdCtx &X) {
    const int K = P.K;
    int stage = 0;
    uint32_t phase = 0;
    for (int tile = blockIdx.x >> 1; tile < P.num_tiles; tile += gridDim.x >> 1) {
        const int64_t m0 = (int64_t)(tile / P.n_tiles_n) * (2 * kBM) + X.rank * kBM;
        for (int s = 0; s < P.n_a_stages; ++s) {
            if (!mbar_wait(smem_addr(&X.empty_a[stage]), phase ^ 1, X.abort)) return;
            uint8_t *As = X.a_ring + (size_t)stage * P.a_stage_bytes;
#pragma unroll
            for (int v = 0; v < (kBM * 8 + kProdThreads - 1) / kProdThreads; ++v) {
                const int u = X.pt + kProdThreads * v;  // (row, 8-column group), 1024 of them
                if (u >= kBM * 8) break;
                const int r = u >> 3, kg = u & 7;
                const int64_t R = m0 + r;
                const int k0 = s * kBK + kg * 8;
                uint32_t w[4] = {0u, 0u, 0u, 0u};
                if (R < P.N) {
                    if (P.x_f32) {
                        const float *row = reinterpret_cast<const float *>(P.x) + R * K;
                        float f[8];
                        if (P.x_vec && k0 + 8 <= K) {
                            const float4 a = __ldg(reinterpret_cast<const float4 *>(row + k0));
                            const float4 b = __ldg(reinterpret_cast<const float4 *>(row + k0 + 4));
                            f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
                            f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
                        } else {
#pragma unroll
                            for (int e = 0; e < 8; ++e) f[e] = (k0 + e < K) ? __ldg(row + k0 + e) : 0.f;
                        }
#pragma unroll
                        for (int e = 0; e < 4; ++e) w[e] = pack_bf16x2(f[2 * e], f[2 * e + 1]);
                    } else {
                        const uint16_t *row = reinterpret_cast<const uint16_t *>(P.x) + R * K;
                        if (P.x_vec && k0 + 8 <= K) {
                            const uint4 a = __ldg(reinterpret_cast<const uint4 *>(row + k0));
                            w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
                        } else {
                            uint16_t h[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) h[e] = (k0 + e < K) ? __ldg(row + k0 + e) : (uint16_t)0;
#pragma unroll
                            for (int e = 0; e < 4; ++e) w[e] = (uint32_t)h[2 * e] | ((uint32_t)h[2 * e + 1] << 16);
                        }
                    }
                }
                *reinterpret_cast<uint4 *>(As + kg * 2048 + r * 16) = make_uint4(w[0], w[1], w[2], w[3]);
            }
            producer_release(X, stage);
            if (++stage == P.na) { stage = 0; phase ^= 1; }
        }
    }
}

// ------------------------------------------------------------- MMA issue

// Issue loop of the thread-fed modes (A written into shared memory by
// producer warps, no-swizzle K-major layout, own full barriers).  The single
// MMA-issuing thread must keep pace with the tensor core (one pair MMA of
// 256 x 256 x 16 every 128 cycles), so the loop is unrolled over a super-stage
// of lcm(KSA, 4) k-steps: waits, commits and descriptor offsets sit at
// compile-time positions, descriptors advance by constant adds, and nothing
// divides.  A stages hold KSA k-steps, weight stages 4.
//   SEP_A_COMMIT  A stages have their own empty barriers (frames path);
//                 otherwise A and weight stages coincide and share one.
__host__ __device__ constexpr int lcm4(int a) { return (a % 4 == 0) ? a : (a % 2 == 0 ? 2 * a : 4 * a); }

__device__ __forceinline__ uint64_t desc_with_lo(uint64_t d, uint32_t lo) {
    return (d & 0xFFFFFFFF00000000ull) | lo;
}

template <int KSA, bool SEP_A_COMMIT>
__device__ __forceinline__ void mma_issue(const FwdParams &P, uint8_t *a_ring, uint8_t *b_ring, uint64_t *full_a,
                                          uint64_t *empty_a, uint64_t *full_b, uint64_t *empty_b, uint64_t *tfull,
                                          uint64_t *tempty, uint64_t *mma_done, uint32_t tmem_base,
                                          volatile int *abort) {
    constexpr int KSB = kBK / 16;
    constexpr int L = lcm4(KSA);
    constexpr uint16_t kPair = 0x3;
    const uint32_t idesc = idesc_bf16_f32(2 * kBM, P.bn);
    // Descriptor templates (address field of slot 0); an A k-step adds 4096
    // bytes (no-swizzle, 2 core-matrix columns), a weight k-step 32 bytes
    // (128-byte swizzle).
    const uint64_t a0 = smem_desc(smem_addr(a_ring), 2048, 128, kLayoutInterleave);
    const uint64_t b0 = smem_desc(smem_addr(b_ring), 16, 1024, kLayoutSw128);
    constexpr uint32_t kAStep = 4096u >> 4;
    const uint32_t a_slot_step = (uint32_t)P.a_stage_bytes >> 4;
    constexpr uint32_t kBSlotStep = (uint32_t)kBStageBytes >> 4;
    const uint32_t a_lo0 = (uint32_t)a0, b_lo0 = (uint32_t)b0;
    const int nk = P.num_ksteps;

    int bs = 0, as = 0, acc = 0;
    uint32_t bph = 0, aph = 0, accph = 0;
    uint32_t a_lo = a_lo0, b_lo = b_lo0;
    for (int tile = blockIdx.x >> 1; tile < P.num_tiles; tile += gridDim.x >> 1) {
        if (!mbar_wait(smem_addr(&tempty[acc]), accph ^ 1, abort)) return;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)acc * kMaxBN;
        for (int ks0 = 0; ks0 < nk; ks0 += L) {
#pragma unroll
            for (int j = 0; j < L; ++j) {
                const int ks = ks0 + j;
                if (ks < nk) {
                    if (j % KSB == 0) {
                        if (!mbar_wait(smem_addr(&full_b[bs]), bph, abort)) return;
                        b_lo = b_lo0 + (uint32_t)bs * kBSlotStep;
                    }
                    if (j % KSA == 0) {
                        if (!mbar_wait(smem_addr(&full_a[as]), aph, abort)) return;
                        a_lo = a_lo0 + (uint32_t)(SEP_A_COMMIT ? as : bs) * a_slot_step;
                    }
                    tc_fence_after();
                    mma_bf16_pair(d_tmem, desc_with_lo(a0, a_lo + (uint32_t)(j % KSA) * kAStep),
                                  desc_with_lo(b0, b_lo + (uint32_t)(j % KSB) * 2u), idesc, ks > 0 ? 1u : 0u);
                    const bool last = ks == nk - 1;
                    if (j % KSB == KSB - 1 || last) {
                        mma_commit_pair(smem_addr(&empty_b[bs]), kPair);
                        if (++bs == P.nb) { bs = 0; bph ^= 1; }
                    }
                    if (SEP_A_COMMIT && (j % KSA == KSA - 1 || last)) {
                        mma_commit_pair(smem_addr(&empty_a[as]), kPair);
                        if (++as == P.na) { as = 0; aph ^= 1; }
                    }
                    if (!SEP_A_COMMIT && (j % KSA == KSA - 1 || last)) {
                        if (++as == P.na) { as = 0; aph ^= 1; }
                    }
                }
            }
        }
        mma_commit_pair(smem_addr(&tfull[acc]), kPair);
        if (++acc == 2) { acc = 0; accph ^= 1; }
    }
}

// Streamed frames producer (kAModeTmaStream), warps 8..15 of every CTA.
//
// Each pair tile (m, n) of this CTA carries one part of M-block m's rows: the
// M-block's 256 rows x (row_elems / 8) 16-byte chunks are enumerated chunk-
// major in warp iterations of 32 rows, and split into 2 * n_tiles_n parts, so
// that the CTAs of the tiles of an M-block produce it together.  In an
// iteration each lane assembles one 16-byte chunk (8 columns of the
// slice-major row: t*Kh + (c*p + i)*p + j) of its row from at most two image
// row segments (4-byte loads), normalises it and stores it.  After each part a
// warp adds 1 to the M-block's counter with release semantics; the TMA
// issuers wait for all 8 * 2 * n_tiles_n counts before loading the block.
// Producers wait for nothing, so all counts arrive once every CTA runs.
template <int PT, int NORM, bool DUPALL>
__device__ __forceinline__ void produce_rows_stream(const FwdParams &P, int pw, int lane, uint32_t rank) {
    constexpr int p = PT, pp = PT * PT;
    constexpr int NT = DUPALL ? 1 : 2;   // slices stored per row
    constexpr int U = 4;                 // chunks in flight per lane
    const int Kh = P.Kh, qh = Kh / 8, nq = NT * qh;
    const int C = P.C, cpp = C * pp;
    const int row_elems = P.row_elems;
    // The next call's counters: nobody touches them during this call.
    for (int i = (blockIdx.x * kStreamProdWarps + pw) * 32 + lane; i < P.n_mblocks;
         i += gridDim.x * kStreamProdWarps * 32)
        P.ready_next[i] = 0u;
    const int nparts = 2 * P.n_tiles_n;
    const int wi = 8 * nq;               // warp iterations per M-block
    for (int tile = blockIdx.x >> 1; tile < P.num_tiles; tile += gridDim.x >> 1) {
        const int m = tile / P.n_tiles_n, n = tile - m * P.n_tiles_n;
        const int part = 2 * n + (int)rank;
        const int it0 = (int)((int64_t)part * wi / nparts), it1 = (int)((int64_t)(part + 1) * wi / nparts);
        int it = it0 + pw;
        if (it < it1) {
            // iterations it, it + 8, ...: one row group of 32 rows for this warp
            const int64_t row = (int64_t)m * (2 * kBM) + (it & 7) * 32 + lane;
            const bool live = row < P.N;
            const char *base0 = nullptr, *base1 = nullptr;
            const char *dlo = nullptr, *dhi = nullptr;   // frame buffer (bounds-checking build)
            int sW = 0, sHW = 0;
            uint16_t *dst = P.a_rows;
            if (live) {
                const RowSrc rs = locate_row(P, row, 2);
                dlo = rs.lo;
                dhi = rs.hi;
                base0 = rs.base;
                base1 = rs.tmax > 0 ? rs.base + (int64_t)rs.CHW * 2 : rs.base;
                sW = rs.W * 2;
                sHW = rs.HW * 2;
                dst = P.a_rows + row * row_elems;
            }
            for (; it < it1; it += 8 * U) {
                uint32_t w[U][4];
                int col[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int itu = it + 8 * u;
                    col[u] = -1;
#pragma unroll
                    for (int k = 0; k < 4; ++k) w[u][k] = 0u;
                    if (itu >= it1) continue;
                    const int q = itu >> 3;
                    const int t = (NT == 2 && q >= qh) ? 1 : 0;
                    const int kk0 = (q - t * qh) * 8;
                    col[u] = t * Kh + kk0;
                    if (!live || kk0 >= cpp) continue;
                    const int c = kk0 / pp, r2 = kk0 - c * pp, i = r2 / p, j0 = r2 - i * p;
                    const int n1 = (p - j0) < 8 ? (p - j0) : 8;
                    const int i2 = (i + 1 < p) ? i + 1 : 0, c2 = (i + 1 < p) ? c : c + 1;
                    const char *bt = t ? base1 : base0;
                    const char *s1 = bt + (int64_t)c * sHW + (int64_t)i * sW + j0 * 2;
                    const char *s2 = bt + (int64_t)c2 * sHW + (int64_t)i2 * sW;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        if (2 * k < n1) {
                            if (PE_IN(s1 + 4 * k, 4, dlo, dhi, P.err))
                                asm volatile("ld.global.nc.b32 %0, [%1];" : "=r"(w[u][k]) : "l"(s1 + 4 * k));
                        } else if (c2 < C) {
                            if (PE_IN(s2 + (2 * k - n1) * 2, 4, dlo, dhi, P.err))
                                asm volatile("ld.global.nc.b32 %0, [%1];" : "=r"(w[u][k]) : "l"(s2 + (2 * k - n1) * 2));
                        }
                    }
                }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    if (col[u] < 0 || !live) continue;
                    const int kk0 = col[u] >= Kh ? col[u] - Kh : col[u];
                    if (kk0 < cpp) {
                        const int c = kk0 / pp, r2 = kk0 - c * pp, j0 = r2 - (r2 / p) * p;
                        const int n1 = (p - j0) < 8 ? (p - j0) : 8;
                        const NormConst n1c = norm_const(P, c);
                        const NormConst n2c = norm_const(P, c + 1 < C ? c + 1 : c);
                        const bool wrap = (r2 / p) + 1 >= p;   // second segment starts the next channel
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            if (2 * k < n1) w[u][k] = norm_word<NORM>(w[u][k], n1c);
                            else if (!wrap) w[u][k] = norm_word<NORM>(w[u][k], n1c);
                            else if (c + 1 < C) w[u][k] = norm_word<NORM>(w[u][k], n2c);
                        }
                    }
                    if (PE_IN(dst + col[u], 16, P.a_rows, P.a_rows + P.N * (int64_t)row_elems, P.err))
                        st_global_v4(dst + col[u], w[u][0], w[u][1], w[u][2], w[u][3]);
                }
            }
        }
        fence_proxy_async_global();   // this lane's rows visible to TMA readers ...
        __threadfence();              // ... and ordered before lane 0's release
        __syncwarp();
        if (lane == 0) red_release_add(P.ready + m, 1u);
    }
}

// Issue loop of the TMA-fed modes.  Ring slot s holds KSUB A tiles of 64 k
// (16 KB each) and KSUB * SLICES weight tiles; every stage is 4 * KSUB
// k-steps, each issued once per slice, unrolled so that the issuing thread
// spends a few instructions per MMA and keeps the tensor pipe fed.
//   SLICES == 2 (single-frame rows): the A tile holds in-slice k and the slot
//   also holds the weight tiles of slice 0 and slice 1 at the same k, so the
//   rows are fetched once for the two temporal slices they stand for.
//   KSUB == 2: 128 k per stage (8 MMAs per barrier round trip).
template <int SLICES, int KSUB, bool TF32 = false>
__device__ __forceinline__ void mma_issue_tma(const FwdParams &P, uint8_t *a_ring, uint8_t *b_ring, uint64_t *full_b,
                                              uint64_t *empty_b, uint64_t *tfull, uint64_t *tempty,
                                              uint64_t *mma_done, uint32_t tmem_base, volatile int *abort) {
    constexpr uint16_t kPair = 0x3;
    constexpr uint32_t kTile = (uint32_t)kBStageBytes >> 4;   // one 16 KB tile, descriptor units
    constexpr int KS = 4 * KSUB;                               // k-steps per stage
    const uint32_t idesc = TF32 ? idesc_tf32_f32(2 * kBM, P.bn) : idesc_bf16_f32(2 * kBM, P.bn);
    const uint64_t a0 = smem_desc(smem_addr(a_ring), 16, 1024, kLayoutSw128);
    const uint64_t b0 = smem_desc(smem_addr(b_ring), 16, 1024, kLayoutSw128);
    const uint32_t a_lo0 = (uint32_t)a0, b_lo0 = (uint32_t)b0;
    const uint32_t a_slot = (uint32_t)P.a_stage_bytes >> 4, b_slot = (uint32_t)P.b_slot_bytes >> 4;
    const int nk = P.num_ksteps, nst = P.n_b_stages;
    int bs = 0, acc = 0;
    uint32_t bph = 0, accph = 0;
    auto issue = [&](uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, int ks, bool first) {
        const int sub = ks / 4, j = ks % 4;
        const uint64_t ad = desc_with_lo(a0, a_lo + (uint32_t)sub * kTile + 2u * j);
        const uint32_t bl = b_lo + (uint32_t)(sub * SLICES) * kTile + 2u * j;
        if constexpr (TF32) {
            mma_tf32_pair(d_tmem, ad, desc_with_lo(b0, bl), idesc, first ? 0u : 1u);
        } else {
            mma_bf16_pair(d_tmem, ad, desc_with_lo(b0, bl), idesc, first ? 0u : 1u);
            if constexpr (SLICES == 2) mma_bf16_pair(d_tmem, ad, desc_with_lo(b0, bl + kTile), idesc, 1u);
        }
    };
    for (int tile = blockIdx.x >> 1; tile < P.num_tiles; tile += gridDim.x >> 1) {
        if (!mbar_wait(smem_addr(&tempty[acc]), accph ^ 1, abort)) return;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)acc * kMaxBN;
        for (int st = 0; st < nst; ++st) {
            if (!mbar_wait(smem_addr(&full_b[bs]), bph, abort)) return;
            tc_fence_after();
            const uint32_t a_lo = a_lo0 + (uint32_t)bs * a_slot, b_lo = b_lo0 + (uint32_t)bs * b_slot;
            const int kin = nk - KS * st;
            if (kin >= KS) {
#pragma unroll
                for (int ks = 0; ks < KS; ++ks) issue(d_tmem, a_lo, b_lo, ks, st == 0 && ks == 0);
            } else {
                for (int ks = 0; ks < kin; ++ks) issue(d_tmem, a_lo, b_lo, ks, st == 0 && ks == 0);
            }
            mma_commit_pair(smem_addr(&empty_b[bs]), kPair);
            if (++bs == P.nb) { bs = 0; bph ^= 1; }
        }
        mma_commit_pair(smem_addr(&tfull[acc]), kPair);
        if (++acc == 2) { acc = 0; accph ^= 1; }
    }
}

// Runtime-p frames path (p not 14 or 16): the same protocol, not unrolled.
__device__ __noinline__ void mma_issue_generic(const FwdParams &P, uint8_t *a_ring, uint8_t *b_ring,
                                               uint64_t *full_a, uint64_t *empty_a, uint64_t *full_b,
                                               uint64_t *empty_b, uint64_t *tfull, uint64_t *tempty,
                                               uint64_t *mma_done, uint32_t tmem_base, volatile int *abort) {
    constexpr uint16_t kPair = 0x3;
    const uint32_t idesc = idesc_bf16_f32(2 * kBM, P.bn);
    const int ks_a = P.P >> 1;
    int bs = 0, as = 0, acc = 0;
    uint32_t bph = 0, aph = 0, accph = 0;
    for (int tile = blockIdx.x >> 1; tile < P.num_tiles; tile += gridDim.x >> 1) {
        if (!mbar_wait(smem_addr(&tempty[acc]), accph ^ 1, abort)) return;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)acc * kMaxBN;
        int ka = 0, kbi = 0;
        for (int ks = 0; ks < P.num_ksteps; ++ks) {
            if (kbi == 0 && !mbar_wait(smem_addr(&full_b[bs]), bph, abort)) return;
            if (ka == 0 && !mbar_wait(smem_addr(&full_a[as]), aph, abort)) return;
            tc_fence_after();
            const uint64_t adesc =
                smem_desc(smem_addr(a_ring + (size_t)as * P.a_stage_bytes) + ka * 4096, 2048, 128, kLayoutInterleave);
            const uint64_t bdesc = smem_desc(smem_addr(b_ring + (size_t)bs * kBStageBytes) + kbi * 32, 16, 1024,
                                             kLayoutSw128);
            mma_bf16_pair(d_tmem, adesc, bdesc, idesc, ks > 0 ? 1u : 0u);
            const bool last = (ks == P.num_ksteps - 1);
            if (++kbi == kBK / 16 || last) {
                mma_commit_pair(smem_addr(&empty_b[bs]), kPair);
                kbi = 0;
                if (++bs == P.nb) { bs = 0; bph ^= 1; }
            }
            if (++ka == ks_a || last) {
                mma_commit_pair(smem_addr(&empty_a[as]), kPair);
                ka = 0;
                if (++as == P.na) { as = 0; aph ^= 1; }
            }
        }
        mma_commit_pair(smem_addr(&tfull[acc]), kPair);
        if (++acc == 2) { acc = 0; accph ^= 1; }
    }
}

// ------------------------------------------------------------- the kernel

// REGSTORE: the epilogue writes each lane's row straight from registers
// (P.out) instead of staging 32 x 32 boxes for TMA stores.  Faster only where
// the epilogue, not the MMAs, bounds a tile (the folded weight's half-K tiles).
template <int AMODE, int PT, bool F32IN, int NORM, bool DUPALL, bool REGSTORE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(threads_for(AMODE), 1)
    pe_fwd_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                  const __grid_constant__ CUtensorMap tmap_out, const __grid_constant__ FwdParams P) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *b_ring = smem;
    uint8_t *a_ring = b_ring + (size_t)P.nb * P.b_slot_bytes;
    constexpr bool kTmaA = tma_fed(AMODE);
    uint8_t *epi = smem + P.epi_offset;
    uint64_t *bars = reinterpret_cast<uint64_t *>(epi + 4 * 8192);   // 8 KB staging per epilogue warp
    uint64_t *full_b = bars;
    uint64_t *empty_b = full_b + P.nb;
    uint64_t *full_a = empty_b + P.nb;
    uint64_t *empty_a = full_a + P.na;
    uint64_t *tfull = empty_a + P.na;
    uint64_t *tempty = tfull + 2;
    uint64_t *mma_done = tempty + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < P.nb; ++s) {
            mbar_init(smem_addr(&full_b[s]), 1);
            mbar_init(smem_addr(&empty_b[s]), 1);
        }
        for (int s = 0; s < P.na; ++s) {
            mbar_init(smem_addr(&full_a[s]), kTmaA ? 1 : 2 * kProdWarps);
            mbar_init(smem_addr(&empty_a[s]), 1);
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
        if (kTmaA) prefetch_tmap(&tmap_x);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_addr(tmem_holder), 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    // Issuer warps: 0, 2, 3 and, when no warp produces A, 8 and 9.  At most
    // P.n_iss of them issue, and P.n_iss never exceeds a ring depth: an issuer
    // then can never lap a slot, so its parity waits cannot alias.
    const int iss = (warp == 0) ? 0 : (warp == 2 || warp == 3) ? warp - 1
                  : (AMODE == kAModeTmaStream) ? ((warp == 16 || warp == 17) ? warp - 13 : -1)
                  : (kTmaA && warp >= 8 && warp < 10) ? warp - 5 : -1;
    const int n_iss = P.n_iss;
    if (iss >= 0) {
        // ---------------- TMA issuers (both CTAs; bytes complete on the leader's barriers).
        // Stage g of this CTA's sequence is issued by issuer g % n_iss: one
        // thread's bulk copies are serviced one after another, so several
        // issuing warps keep several copies in flight.
        if (lane == 0 && iss < n_iss) {
            // The A rows may come from the kernel launched just before this
            // one (the staged prepare step): nothing is loaded before it ends.
            griddep_wait();
            const uint64_t pol_w = l2_policy_evict_last();
            const uint64_t pol_x = l2_policy_evict_first();
            const uint32_t b_bytes = (uint32_t)(P.bn / 2) * kBK * 2;
            const uint32_t a_bytes = kBM * kBK * 2;
            const uint32_t fb0 = mapa_shared(smem_addr(&full_b[0]), 0);
            int g = 0;
            bool ok = true;
            int ready_m = -1;
            for (int tile = blockIdx.x >> 1; tile < P.num_tiles && ok; tile += gridDim.x >> 1) {
                const int m_blk = tile / P.n_tiles_n, n_blk = tile % P.n_tiles_n;
                for (int kb = 0; kb < P.n_b_stages && ok; ++kb, ++g) {
                    if (g % n_iss != iss) continue;
                    if (AMODE == kAModeTmaStream && m_blk != ready_m) {
                        // rows of this M-block come from producer warps across the grid
                        if (!wait_count(P.ready + m_blk, P.ready_target, abort)) { ok = false; break; }
                        fence_proxy_async_global();
                        ready_m = m_blk;
                    }
                    // In the TMA-fed path A and weight share ring slot and barriers.
                    const int bs = g % P.nb;
                    if (!mbar_wait(smem_addr(&empty_b[bs]), ((g / P.nb) & 1) ^ 1, abort)) { ok = false; break; }
                    constexpr uint32_t kSlices =
                        (AMODE == kAModeTmaShared || (AMODE == kAModeTmaStream && DUPALL)) ? 2u : 1u;
                    const int ksub = kTmaA ? P.ksub : 1;
                    if (leader)
                        mbar_arrive_expect_tx(smem_addr(&full_b[bs]),
                                              2u * (uint32_t)ksub * (kSlices * b_bytes + (kTmaA ? a_bytes : 0u)));
                    const uint32_t adst = smem_addr(a_ring + (size_t)bs * P.a_stage_bytes);
                    const uint32_t bdst = smem_addr(b_ring + (size_t)bs * P.b_slot_bytes);
                    const int wrow = n_blk * P.bn + (int)rank * (P.bn / 2);
                    // k columns per 128-byte tile row: 64 bf16 or 32 fp32 (tf32)
                    constexpr int kBKe = (AMODE == kAModeTmaTf32) ? kBK / 2 : kBK;
                    for (int sub = 0; sub < ksub; ++sub) {
                        const int kx = (kb * ksub + sub) * kBKe;
                        if (kTmaA)
                            tma_load_2d_pair(adst + (uint32_t)sub * kBStageBytes, &tmap_x, fb0 + 8u * bs, kx,
                                             m_blk * (2 * kBM) + (int)rank * kBM, pol_x);
                        const uint32_t bsub = bdst + (uint32_t)(sub * (int)kSlices) * kBStageBytes;
                        tma_load_2d_pair(bsub, &tmap_w, fb0 + 8u * bs, kx, wrow, pol_w);
                        if (kSlices == 2)
                            tma_load_2d_pair(bsub + kBStageBytes, &tmap_w, fb0 + 8u * bs, P.Kh + kx, wrow, pol_w);
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (leader CTA only)
        if (leader && lane == 0) {
            constexpr int KSA = (AMODE == kAModeFrames) ? (PT ? PT / 2 : 0) : 4;
            if constexpr (kTmaA) {
                constexpr int kSl = (AMODE == kAModeTmaShared || (AMODE == kAModeTmaStream && DUPALL)) ? 2 : 1;
                if constexpr (AMODE == kAModeTmaTf32)
                    mma_issue_tma<1, 2, true>(P, a_ring, b_ring, full_b, empty_b, tfull, tempty, mma_done, tmem_base,
                                              abort);
                else if (kSl == 1 && P.ksub == 2)
                    mma_issue_tma<kSl, 2>(P, a_ring, b_ring, full_b, empty_b, tfull, tempty, mma_done, tmem_base, abort);
                else
                    mma_issue_tma<kSl, 1>(P, a_ring, b_ring, full_b, empty_b, tfull, tempty, mma_done, tmem_base, abort);
            }
            else if constexpr (KSA > 0)
                mma_issue<KSA, AMODE == kAModeFrames>(P, a_ring, b_ring, full_a, empty_a, full_b,
                                                                          empty_b, tfull, tempty, mma_done, tmem_base,
                                                                          abort);
            else
                mma_issue_generic(P, a_ring, b_ring, full_a, empty_a, full_b, empty_b, tfull, tempty, mma_done,
                                  tmem_base, abort);
            // Every MMA issued so far completes before the pair frees its TMEM, also
            // when an issue loop returned early because a wait gave up.
            mma_drain(smem_addr(mma_done));
        }
    } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + 4) {
        // ---------------- epilogue (both CTAs)
        // Each warp drains its 32 TMEM lanes in 32-column chunks, loading chunk
        // c+1 from TMEM while chunk c is converted, and hands each converted
        // 32 x 32 box to a TMA store through a ring of staging buffers.
        const int wq = warp & 3;  // TMEM lane quarter this warp may access
        const uint32_t tempty0 = mapa_shared(smem_addr(&tempty[0]), 0);
        const int nbufs = P.out_f32 ? 2 : 4;
        uint8_t *stage_buf = epi + (size_t)wq * 8192;
        const int nch = P.bn / 32;   // 2, 4 or 8
        int acc = 0, nbuf = 0;
        uint32_t accph = 0;
        // position-embedding row segment of this lane's row for chunk cc, PD = 1
        // for a bf16 table (four 16-byte pieces), 2 for fp32 (eight).  A chunk
        // wholly inside the table takes unguarded loads; at the edges E % 8 == 0
        // keeps each 16-byte piece wholly inside the row or wholly past it.
        auto load_pos = [&](auto kPD, uint4 (&pq)[8], int cc, int64_t row0, int n_blk) {
            constexpr int PD = decltype(kPD)::value;
            constexpr int NQ = PD == 2 ? 8 : 4, ES = PD == 2 ? 4 : 2;
            const int col0 = n_blk * P.bn + cc * 32;
            const int64_t r = row0 + lane;
            const char *plo = reinterpret_cast<const char *>(P.pos);
            const char *phi = plo + P.N * (int64_t)P.E * ES;
            const char *a0 = plo + (r * P.E + col0) * (int64_t)ES;
            if (r < P.N && col0 + 32 <= P.E) {
#pragma unroll
                for (int q = 0; q < NQ; ++q) {
                    pq[q] = make_uint4(0u, 0u, 0u, 0u);
                    if (PE_IN(a0 + 16 * q, 16, plo, phi, P.err))
                        asm volatile("ld.global.nc.v4.b32 {%0, %1, %2, %3}, [%4];"
                                     : "=r"(pq[q].x), "=r"(pq[q].y), "=r"(pq[q].z), "=r"(pq[q].w)
                                     : "l"(a0 + 16 * q));
                }
            } else {
#pragma unroll
                for (int q = 0; q < NQ; ++q) {
                    pq[q] = make_uint4(0u, 0u, 0u, 0u);
                    if (r < P.N && col0 + q * (16 / ES) < P.E && PE_IN(a0 + 16 * q, 16, plo, phi, P.err))
                        asm volatile("ld.global.nc.v4.b32 {%0, %1, %2, %3}, [%4];"
                                     : "=r"(pq[q].x), "=r"(pq[q].y), "=r"(pq[q].z), "=r"(pq[q].w)
                                     : "l"(a0 + 16 * q));
                }
            }
        };
        // pq holds chunk cc's table segment on entry (loaded one chunk ahead);
        // once added, it is reloaded with chunk cc + 1's while this chunk is
        // staged and stored
        auto emit = [&](auto kPos, auto kAct, const uint32_t (&v)[32], int cc, int64_t row0, int n_blk,
                        uint4 (&pq)[8]) {
            constexpr int PD = decltype(kPos)::value;
            constexpr bool has_act = decltype(kAct)::value;
            const int col0 = n_blk * P.bn + cc * 32;
            if (row0 >= P.N || col0 >= P.E) return;   // whole box outside: nothing to store
            float f[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(v[e]);
            if (P.bias) {
                if (col0 + 32 <= P.E) {   // the bias buffer is the library's own: 16-byte aligned
                    const float4 *b4 = reinterpret_cast<const float4 *>(P.bias + col0);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float4 b = __ldg(b4 + i);
                        f[4 * i] += b.x;
                        f[4 * i + 1] += b.y;
                        f[4 * i + 2] += b.z;
                        f[4 * i + 3] += b.w;
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (col0 + e < P.E) f[e] += __ldg(P.bias + col0 + e);
                }
            }
            // the buffer must be free of the store issued nbufs chunks ago
            if constexpr (!REGSTORE) {
                if (lane == 0) {
                    if (nbufs == 4) bulk_wait_read<3>(); else bulk_wait_read<1>();
                }
                __syncwarp();
            }
            if constexpr (has_act) {   // exact GELU, 0.5 x (1 + erf(x / sqrt 2)), in fp32
#pragma unroll
                for (int e = 0; e < 32; ++e) f[e] = 0.5f * f[e] * (1.0f + erff(f[e] * 0.70710678118654752f));
            }
            if constexpr (PD != 0) {   // out = acc + bias + pos, in fp32, before the output cast
#pragma unroll
                for (int q = 0; q < (PD == 2 ? 8 : 4); ++q) {
                    const uint32_t w4[4] = {pq[q].x, pq[q].y, pq[q].z, pq[q].w};
                    if constexpr (PD == 2) {
#pragma unroll
                        for (int u = 0; u < 4; ++u) f[4 * q + u] += __uint_as_float(w4[u]);
                    } else {
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            f[8 * q + 2 * u] += bf16lo_to_f32(w4[u]);
                            f[8 * q + 2 * u + 1] += bf16hi_to_f32(w4[u]);
                        }
                    }
                }
                if (cc + 1 < nch) load_pos(kPos, pq, cc + 1, row0, n_blk);
            }
            if constexpr (REGSTORE) {
                const int64_t r = row0 + lane;
                if (r >= P.N) return;
                const bool whole = col0 + 32 <= P.E;
                char *o = static_cast<char *>(P.out) + (r * P.E + col0) * (int64_t)(P.out_f32 ? 4 : 2);
                const char *olo = static_cast<const char *>(P.out);
                const char *ohi = olo + P.N * (int64_t)P.E * (P.out_f32 ? 4 : 2);
                if (!P.out_f32) {
                    uint32_t w[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c) w[c] = pack_bf16x2(f[2 * c], f[2 * c + 1]);
                    if (whole && P.epi_v8) {
                        if (PE_IN(o, 64, olo, ohi, P.err)) {
                            st_global_v8(o, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
                            st_global_v8(o + 32, w[8], w[9], w[10], w[11], w[12], w[13], w[14], w[15]);
                        }
                    } else {
#pragma unroll
                        for (int q = 0; q < 4; ++q)   // E % 8 == 0: a 16-byte piece is wholly in or past the row
                            if (col0 + 8 * q < P.E && PE_IN(o + 16 * q, 16, olo, ohi, P.err))
                                st_global_v4(o + 16 * q, w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
                    }
                } else {
                    uint32_t w[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) w[c] = __float_as_uint(f[c]);
                    if (whole && P.epi_v8) {
                        if (PE_IN(o, 128, olo, ohi, P.err)) {
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                st_global_v8(o + 32 * q, w[8 * q], w[8 * q + 1], w[8 * q + 2], w[8 * q + 3],
                                             w[8 * q + 4], w[8 * q + 5], w[8 * q + 6], w[8 * q + 7]);
                        }
                    } else {
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            if (col0 + 4 * q < P.E && PE_IN(o + 16 * q, 16, olo, ohi, P.err))
                                st_global_v4(o + 16 * q, w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
                    }
                }
                return;
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
                tma_store_2d(&tmap_out, smem_addr(buf), col0, (int32_t)row0);
                bulk_commit();
            }
            if (++nbuf == nbufs) nbuf = 0;
        };
        // the tile loop, compiled without options, with the position-embedding
        // add, and with the GELU (the PatchMerger's fc1)
        // With a position table, each lane asks L2 for its row of the table
        // for this CTA's next tile (and for the first tile) before waiting for
        // the accumulator: the MMAs of the tile hide that fetch, and the
        // per-chunk table loads below then find the rows in L2.
        auto prefetch_pos = [&](int t) {
            const int64_t r = (int64_t)(t / P.n_tiles_n) * (2 * kBM) + rank * kBM + wq * 32 + lane;
            const int c0 = (t % P.n_tiles_n) * P.bn;
            if (r >= P.N || c0 >= P.E) return;
            const int es = P.pos_f32 ? 4 : 2;
            const int nc = (P.E - c0) < P.bn ? (P.E - c0) : P.bn;
            const uintptr_t a = reinterpret_cast<uintptr_t>(P.pos) + (uintptr_t)((r * P.E + c0) * es);
            const uintptr_t end = a + (uintptr_t)nc * es;
            prefetch_l2(reinterpret_cast<const void *>(a));
            for (uintptr_t q = (a & ~(uintptr_t)127) + 128; q < end; q += 128)
                prefetch_l2(reinterpret_cast<const void *>(q));
        };
        auto tiles = [&](auto kPos, auto kAct) {
            for (int tile = blockIdx.x >> 1; tile < P.num_tiles; tile += gridDim.x >> 1) {
                const int m_blk = tile / P.n_tiles_n, n_blk = tile % P.n_tiles_n;
                if constexpr (decltype(kPos)::value != 0) {
                    if (tile == (int)(blockIdx.x >> 1)) prefetch_pos(tile);
                    if (tile + (int)(gridDim.x >> 1) < P.num_tiles) prefetch_pos(tile + (int)(gridDim.x >> 1));
                }
                if (!mbar_wait(smem_addr(&tfull[acc]), accph, abort)) break;
                tc_fence_after();
                const int64_t row0 = (int64_t)m_blk * (2 * kBM) + rank * kBM + wq * 32;
                const uint32_t tbase = tmem_base + ((uint32_t)(wq * 32) << 16) + (uint32_t)(acc * kMaxBN);
                uint4 pq[8];
                if constexpr (decltype(kPos)::value != 0) load_pos(kPos, pq, 0, row0, n_blk);
                if constexpr (kTmaA && AMODE != kAModeTmaStream && decltype(kPos)::value != 2) {
                    // registers to spare: the next chunk's TMEM load overlaps this chunk's work
                    // (not with an fp32 table, whose 32 registers of look-ahead take their place)
                    uint32_t va[32], vb[32];
                    tmem_ld_32x32b_x32(tbase, va);
                    for (int cc = 0; cc < nch; cc += 2) {
                        tmem_ld_wait();
                        tmem_ld_32x32b_x32(tbase + (uint32_t)(cc + 1) * 32, vb);
                        emit(kPos, kAct, va, cc, row0, n_blk, pq);
                        tmem_ld_wait();
                        if (cc + 2 < nch) tmem_ld_32x32b_x32(tbase + (uint32_t)(cc + 2) * 32, va);
                        emit(kPos, kAct, vb, cc + 1, row0, n_blk, pq);
                    }
                } else {
                    uint32_t va[32];
                    for (int cc = 0; cc < nch; ++cc) {
                        tmem_ld_32x32b_x32(tbase + (uint32_t)cc * 32, va);
                        tmem_ld_wait();
                        emit(kPos, kAct, va, cc, row0, n_blk, pq);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(tempty0 + 8u * (uint32_t)acc);
                if (++acc == 2) { acc = 0; accph ^= 1; }
            }
        };
        using PosNone = std::integral_constant<int, 0>;
        if (P.pos && P.pos_f32) tiles(std::integral_constant<int, 2>{}, std::false_type{});
        else if (P.pos) tiles(std::integral_constant<int, 1>{}, std::false_type{});
        else if (P.act) tiles(PosNone{}, std::true_type{});
        else tiles(PosNone{}, std::false_type{});
        if (lane == 0) bulk_wait<0>();
        __syncwarp();
    } else if (AMODE == kAModeTmaStream && warp >= kStreamProdWarp0 && warp < kStreamProdWarp0 + kStreamProdWarps) {
        // ---------------- row producers (both CTAs)
        if constexpr (AMODE == kAModeTmaStream && PT != 0)
            produce_rows_stream<PT, NORM, DUPALL>(P, warp - kStreamProdWarp0, lane, rank);
    } else if (warp >= 8 && !kTmaA) {
        // ---------------- A producers (both CTAs)
        ProdCtx X;
        X.a_ring = a_ring;
        X.empty_a = (AMODE == kAModePatchThreads) ? empty_b : empty_a;   // stages coincide
        X.full_a_leader = mapa_shared(smem_addr(&full_a[0]), 0);
        X.abort = abort;
        X.pt = threadIdx.x - 256;
        X.lane = lane;
        X.rank = rank;
        if constexpr (AMODE == kAModeFrames && PT != 0 && !F32IN) {
            if (P.TP == 2) produce_frames_reg<PT, NORM, DUPALL>(P, X);
            else produce_frames<PT, F32IN>(P, X);
        } else if constexpr (AMODE == kAModeFrames) {
            produce_frames<PT, F32IN>(P, X);
        }
        else if constexpr (AMODE == kAModePatchThreads)
            produce_patches(P, X);
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, 512);
    }
    if (threadIdx.x == 0 && *abort) atomicExch(P.err, (int)PE_ERR_DEVICE_TIMEOUT);
}

// ------------------------------------------------------------- helpers

// Weight packing.  Ŵ[e, k] = bf16_rne(W[e, k]), the bias widened exactly to
// fp32.  Row e of the packed weight holds `ld` columns, in one of three orders:
//   0  the view(-1, C, tp, p, p) order k = ((c*tp + t)*p + i)*p + j (patches
//      path), zero past K;
//   1  k' = ((c*p + i)*tp + t)*p + j, the order the frames producer fills its
//      stages in, zero past K;
//   2  slice-major: column t*Kh + (c*p + i)*p + j, slice t of the kernel in its
//      own block of Kh >= C*p*p columns (zero past C*p*p), for rows that share
//      one A row across the temporal slices;
//   3  folded: column (c*p + i)*p + j holds bf16_rne(Ŵ[e,c,0,i,j] + Ŵ[e,c,1,i,j])
//      (the two bf16-rounded slices summed in fp32, rounded once), zero past
//      C*p*p: single-frame rows meet both slices in one product (tp = 2);
//   4  slice-interleaved (tp = 2): 64-column tile s holds slice 0's in-slice
//      columns 32s..32s+31 followed by slice 1's same columns (in-slice column
//      (c*p + i)*p + j, zero past C*p*p), so one 128-byte-swizzled tile feeds
//      two k-steps of both slices against one resident single-frame A.
__global__ void pe_pack_weight_kernel(const void *w, int w_f32, const void *bias, int b_f32,
                                      uint16_t *wpack, float *bias32, int E, int C, int TP, int P,
                                      int ld, int order, int Kh) {
    const int K = C * TP * P * P;
    const int64_t total = (int64_t)E * ld;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t e = idx / ld;
        const int kd = (int)(idx - e * ld);
        int k = -1;
        if (order == 0) {
            if (kd < K) k = kd;
        } else if (order == 1) {
            if (kd < K) {
                const int j = kd % P, t = (kd / P) % TP, ci = kd / (P * TP);
                const int c = ci / P, i = ci % P;
                k = ((c * TP + t) * P + i) * P + j;
            }
        } else if (order == 2) {
            const int t = kd / Kh, kk = kd - t * Kh;
            if (t < TP && kk < C * P * P) {
                const int j = kk % P, i = (kk / P) % P, c = kk / (P * P);
                k = ((c * TP + t) * P + i) * P + j;
            }
        } else if (order == 4) {
            // 64-column tile s = [slice 0, columns 32s..32s+31 | slice 1, the same columns]
            const int s = kd >> 6, w = kd & 63, t = w >> 5, kk = 32 * s + (w & 31);
            if (t < TP && kk < C * P * P) {
                const int j = kk % P, i = (kk / P) % P, c = kk / (P * P);
                k = ((c * TP + t) * P + i) * P + j;
            }
        }
        uint16_t v = 0;
        if (order == 3) {
            k = -1;
            if (kd < C * P * P) {
                const int j = kd % P, i = (kd / P) % P, c = kd / (P * P);
                float sum = 0.f;
                for (int t = 0; t < TP; ++t) {
                    const int64_t kt = ((c * TP + t) * P + i) * P + j;
                    const float wt = w_f32 ? __bfloat162float(__float2bfloat16_rn(reinterpret_cast<const float *>(w)[e * K + kt]))
                                           : __uint_as_float((uint32_t)reinterpret_cast<const uint16_t *>(w)[e * K + kt] << 16);
                    sum = __fadd_rn(sum, wt);
                }
                const __nv_bfloat16 b = __float2bfloat16_rn(sum);
                v = *reinterpret_cast<const uint16_t *>(&b);
            }
        }
        if (k >= 0) {
            if (w_f32) {
                const __nv_bfloat16 b = __float2bfloat16_rn(reinterpret_cast<const float *>(w)[e * K + k]);
                v = *reinterpret_cast<const uint16_t *>(&b);
            } else {
                v = reinterpret_cast<const uint16_t *>(w)[e * K + k];
            }
        }
        wpack[idx] = v;
        if (kd == 0 && bias && bias32)
            bias32[e] = b_f32 ? reinterpret_cast<const float *>(bias)[e]
                              : __uint_as_float((uint32_t)reinterpret_cast<const uint16_t *>(bias)[e] << 16);
    }
}

// Staged frames path, prepare step: normalised patch rows written once for
// the TMA-fed contraction, through shared memory so that both sides of the
// copy are coalesced.  bf16 frames, or fp32 frames (F32IN, prep_unit_f32).  A CTA owns kPrepRows consecutive output rows and one
// (row, word) unit per thread; consecutive threads read consecutive words of
// one image row.  Each thread loads its word of the p image rows of every
// channel (single-frame rows: all channels at once; otherwise one channel of
// both temporal slices ahead of the one being stored), normalises them and
// writes them into the CTA's row block in shared memory; one bulk copy then
// stores the contiguous block of rows.
//   SHARED  one slice per row, A[N, Kh], column (c*p + i)*p + j, zero up to
//           Kh: single-frame rows with tp = 2 (met by the slice-major
//           weight) and every row with tp = 1 (met by the frames-order one);
//   else    A[N, K] in the frames order k' = ((c*p + i)*tp + t)*p + j, the
//           last frame repeated where a temporal patch runs past T.
constexpr int kPrepRows = 16;

// fp32 frames: one (row, word) unit of the prepare kernel.  The same rows
// as the bf16 form (two pixels per unit, 8-byte loads: an image row starts
// 56-byte aligned and a unit at 8 bytes), normalised from the fp32 values.
template <int PT, bool SHARED>
__device__ __forceinline__ void prep_unit_f32(const FwdParams &P, int64_t R, int jw, uint32_t srow, int row_elems,
                                              int nci) {
    constexpr int p = PT, NT = SHARED ? 1 : 2;
    const RowSrc rs = locate_row(P, R, 4);
    const char *src = rs.base + 8 * jw;
    const int64_t sW = (int64_t)rs.W * 4, sHW = (int64_t)rs.HW * 4;
    const int64_t sT1 = (!SHARED && rs.tmax > 0) ? (int64_t)rs.CHW * 4 : 0;
    const char *dlo = rs.lo, *dhi = rs.hi;   // frame buffer (bounds-checking build)
    PixPair<true> px[2][NT][p];
    auto load = [&](const int b, const int c) {
        const char *a = src + (int64_t)c * sHW;
#pragma unroll
        for (int i = 0; i < p; ++i) {
            px[b][0][i].load(a + (int64_t)i * sW, dlo, dhi, P.err);
            if constexpr (!SHARED) {
                px[b][NT - 1][i].zero();
                if (sT1 != 0) px[b][NT - 1][i].load(a + (int64_t)i * sW + sT1, dlo, dhi, P.err);
            }
        }
    };
    auto store = [&](const int b, const int c) {
        const NormConst nc = norm_const(P, c);
#pragma unroll
        for (int i = 0; i < p; ++i) {
            const int ci = c * p + i;
            const uint32_t w0 = px[b][0][i].norm(nc);
            if constexpr (SHARED) {
                sts32(srow + (uint32_t)((ci * p + 2 * jw) * 2), w0);
            } else {
                const uint32_t w1 = sT1 ? px[b][NT - 1][i].norm(nc) : w0;
                sts32(srow + (uint32_t)((ci * 2 * p + 2 * jw) * 2), w0);
                sts32(srow + (uint32_t)((ci * 2 * p + p + 2 * jw) * 2), w1);
            }
        }
    };
    const int C = P.C;
    load(0, 0);
    for (int c = 0; c < C; c += 2) {
        if (c + 1 < C) load(1, c + 1);
        store(0, c);
        if (c + 1 >= C) break;
        if (c + 2 < C) load(0, c + 2);
        store(1, c + 1);
    }
    if (SHARED && 2 * jw < row_elems - nci * p)   // zero columns up to Kh
        sts32(srow + (uint32_t)((nci * p + 2 * jw) * 2), 0u);
}

template <int PT, int NORM, bool SHARED, bool F32IN = false>
__global__ void __launch_bounds__(kPrepRows *PT / 2) pe_prep_rows_kernel(const __grid_constant__ FwdParams P,
                                                                        uint16_t *A, int row_elems) {
    constexpr int p = PT, ws = p / 2, NT = SHARED ? 1 : 2;
    extern __shared__ __align__(128) uint8_t prep_smem[];
    griddep_launch_dependents();   // the contraction may start its prologue
    const int64_t m0 = (int64_t)blockIdx.x * kPrepRows;
    const int64_t left = P.N - m0;
    const int rows = left < kPrepRows ? (int)left : kPrepRows;
    const int nci = P.C * p;
    int r, jw;
    unit_to_row_word<kPrepRows>((int)threadIdx.x, ws, P.merge, r, jw);
    const uint32_t srow = smem_addr(prep_smem) + (uint32_t)(r * row_elems * 2);
    if constexpr (F32IN) {
        if (r < rows) prep_unit_f32<PT, SHARED>(P, m0 + r, jw, srow, row_elems, nci);
    } else if (r < rows) {
        const RowSrc rs = locate_row(P, m0 + r, 2);
        const char *src = rs.base + 4 * jw;
        const int sW = rs.W * 2, sHW = rs.HW * 2;
        const int sT1 = (!SHARED && rs.tmax > 0) ? rs.CHW * 2 : 0;
        const char *dlo = rs.lo, *dhi = rs.hi;   // frame buffer (bounds-checking build)
        // One channel (p image rows, every temporal slice) per register buffer;
        // the loads of channel c + 1 are in flight while channel c is stored.
        uint32_t raw[2][NT][p];
        auto load = [&](const int b, const int c) {
            const char *a = src + (int64_t)c * sHW;
#pragma unroll
            for (int i = 0; i < p; ++i) {
                raw[b][0][i] = 0u;
                if (PE_IN(a + (int64_t)i * sW, 4, dlo, dhi, P.err))
                    asm volatile("ld.global.nc.b32 %0, [%1];" : "=r"(raw[b][0][i]) : "l"(a + (int64_t)i * sW));
                if constexpr (!SHARED) {
                    raw[b][NT - 1][i] = 0u;
                    if (sT1 != 0 && PE_IN(a + (int64_t)i * sW + sT1, 4, dlo, dhi, P.err))
                        asm volatile("ld.global.nc.b32 %0, [%1];"
                                     : "=r"(raw[b][NT - 1][i]) : "l"(a + (int64_t)i * sW + sT1));
                }
            }
        };
        auto store = [&](const int b, const int c) {
            const NormConst nc = norm_const(P, c);
#pragma unroll
            for (int i = 0; i < p; ++i) {
                const int ci = c * p + i;
                const uint32_t w0 = norm_word<NORM>(raw[b][0][i], nc);
                if constexpr (SHARED) {
                    sts32(srow + (uint32_t)((ci * p + 2 * jw) * 2), w0);
                } else {
                    const uint32_t w1 = sT1 ? norm_word<NORM>(raw[b][NT - 1][i], nc) : w0;
                    sts32(srow + (uint32_t)((ci * 2 * p + 2 * jw) * 2), w0);
                    sts32(srow + (uint32_t)((ci * 2 * p + p + 2 * jw) * 2), w1);
                }
            }
        };
        const int C = P.C;
        if constexpr (SHARED) {
            // one slice per row: every channel's loads in flight at once
            uint32_t all[4][p];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                if (c >= C) break;
                const char *a = src + (int64_t)c * sHW;
#pragma unroll
                for (int i = 0; i < p; ++i) {
                    all[c][i] = 0u;
                    if (PE_IN(a + (int64_t)i * sW, 4, dlo, dhi, P.err))
                        asm volatile("ld.global.nc.b32 %0, [%1];" : "=r"(all[c][i]) : "l"(a + (int64_t)i * sW));
                }
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                if (c >= C) break;
                const NormConst nc = norm_const(P, c);
#pragma unroll
                for (int i = 0; i < p; ++i)
                    sts32(srow + (uint32_t)(((c * p + i) * p + 2 * jw) * 2), norm_word<NORM>(all[c][i], nc));
            }
        } else {
            load(0, 0);
            for (int c = 0; c < C; c += 2) {
                if (c + 1 < C) load(1, c + 1);
                store(0, c);
                if (c + 1 >= C) break;
                if (c + 2 < C) load(0, c + 2);
                store(1, c + 1);
            }
        }
        if (SHARED && 2 * jw < row_elems - nci * p)   // zero columns up to Kh
            sts32(srow + (uint32_t)((nci * p + 2 * jw) * 2), 0u);
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (threadIdx.x == 0 && rows > 0) {
        bulk_store(A + m0 * row_elems, smem_addr(prep_smem), (uint32_t)(rows * row_elems * 2));
        bulk_commit();
        bulk_wait<0>();
    }
}

// LayerNorm of bf16 rows [N, E] (E % 8 == 0) into bf16 rows: one warp per row,
// fp32 statistics over the E features (mean, then the biased variance of the
// deviations), y = (x - mean) * rsqrt(var + eps) * gamma + beta, rounded to
// bf16.  The PatchMerger's first step (mytransformer README §3.2, §4.1).
__global__ void pe_layernorm_kernel(const uint16_t *__restrict__ x, int64_t N, int E, const float *__restrict__ gamma,
                                    const float *__restrict__ beta, float eps, uint16_t *__restrict__ y) {
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= N) return;
    const uint4 *xr = reinterpret_cast<const uint4 *>(x + row * E);
    const int nv = E / 8;
    float s = 0.f;
    for (int i = lane; i < nv; i += 32) {
        const uint4 v = __ldg(xr + i);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) s += bf16lo_to_f32(w[u]) + bf16hi_to_f32(w[u]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float mean = s / (float)E;
    float q = 0.f;
    for (int i = lane; i < nv; i += 32) {
        const uint4 v = __ldg(xr + i);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float d0 = bf16lo_to_f32(w[u]) - mean, d1 = bf16hi_to_f32(w[u]) - mean;
            q += d0 * d0 + d1 * d1;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
    const float inv = rsqrtf(q / (float)E + eps);
    uint4 *yr = reinterpret_cast<uint4 *>(y + row * E);
    for (int i = lane; i < nv; i += 32) {
        const uint4 v = __ldg(xr + i);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t o4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int e = 8 * i + 2 * u;
            const float a = (bf16lo_to_f32(w[u]) - mean) * inv * __ldg(gamma + e) + __ldg(beta + e);
            const float b = (bf16hi_to_f32(w[u]) - mean) * inv * __ldg(gamma + e + 1) + __ldg(beta + e + 1);
            o4[u] = pack_bf16x2(a, b);
        }
        yr[i] = make_uint4(o4[0], o4[1], o4[2], o4[3]);
    }
}

// bf16 or fp32 values -> fp32 (exact).
__global__ void pe_to_f32_kernel(const void *src, int src_f32, float *dst, int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        dst[i] = src_f32 ? reinterpret_cast<const float *>(src)[i]
                         : __uint_as_float((uint32_t)reinterpret_cast<const uint16_t *>(src)[i] << 16);
}

// fp32 patch rows -> tf32-rounded fp32 rows (nearest, ties away from zero)
// for the tf32 contraction.  4 elements per thread.
__global__ void pe_round_tf32_kernel(const float *__restrict__ x, uint32_t *__restrict__ A, int64_t n4) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(x) + i);
        *(reinterpret_cast<uint4 *>(A) + i) = make_uint4(round_tf32(a.x), round_tf32(a.y), round_tf32(a.z), round_tf32(a.w));
    }
}

// The weight for the tf32 contraction: W[e, k] (view order) rounded to tf32,
// as fp32 words, zero for K <= k < ld.
__global__ void pe_pack_weight_tf32_kernel(const void *w, int w_f32, uint32_t *wpack, int E, int K, int ld) {
    const int64_t total = (int64_t)E * ld;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t e = idx / ld;
        const int k = (int)(idx - e * ld);
        uint32_t v = 0u;
        if (k < K) {
            const float f = w_f32 ? reinterpret_cast<const float *>(w)[e * K + k]
                                  : __uint_as_float((uint32_t)reinterpret_cast<const uint16_t *>(w)[e * K + k] << 16);
            v = round_tf32(f);
        }
        wpack[idx] = v;
    }
}

// fp32 patch rows -> bf16 (round to nearest even) rows for the TMA-fed
// contraction: the same rounding the contraction applies to fp32 inputs
// everywhere.  8 elements per thread (32-byte loads, 16-byte stores).
__global__ void pe_cast_rows_kernel(const float *__restrict__ x, uint16_t *__restrict__ A, int64_t n8) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(x) + 2 * i);
        const float4 b = __ldg(reinterpret_cast<const float4 *>(x) + 2 * i + 1);
        *(reinterpret_cast<uint4 *>(A) + i) =
            make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
    }
}

// rows[R, k] for every output row R, in the view(-1, C, tp, p, p) order: the
// frames producer's gather and normalisation written to memory (bf16 or fp32
// values; bf16-exact either way).
template <bool F32IN>
__global__ void pe_patchify_kernel(const __grid_constant__ FwdParams P, void *rows, int rows_f32) {
    constexpr int esize = F32IN ? 4 : 2;
    const int p = P.P, ws = p >> 1;
    const int words = P.K >> 1;
    const int64_t total = P.N * words;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t R = idx / words;
        const int wk = (int)(idx - R * words);
        const int seg = wk / ws, jw = wk - seg * ws;
        const int i = seg % p, t = (seg / p) % P.TP, c = seg / (p * P.TP);
        const RowSrc s = locate_row(P, R, esize);
        const int tt = t < s.tmax ? t : s.tmax;
        const int64_t off = (int64_t)tt * s.CHW + (int64_t)c * s.HW + (int64_t)i * s.W + 2 * jw;
        PixPair<F32IN> px;
        px.load(s.base + off * esize, s.lo, s.hi, P.err);
        const uint32_t w = px.norm(norm_const(P, c));
        const int64_t k = 2 * (int64_t)wk;
        if (rows_f32) {
            float *o = reinterpret_cast<float *>(rows) + R * P.K + k;
            o[0] = bf16lo_to_f32(w);
            o[1] = bf16hi_to_f32(w);
        } else {
            *reinterpret_cast<uint32_t *>(reinterpret_cast<uint16_t *>(rows) + R * P.K + k) = w;
        }
    }
}

// Item-table upload without a host staging buffer: up to kItemsPerFill
// descriptors travel in the launch's parameter block (copied when the launch
// is queued) and one thread per descriptor writes it to dst[0..n).
constexpr int kItemsPerFill = 64;
struct ItemBatch {
    ItemDesc d[kItemsPerFill];
};
__global__ void pe_fill_items_kernel(const __grid_constant__ ItemBatch b, ItemDesc *dst, int n) {
    const int i = threadIdx.x;
    if (i < n) dst[i] = b.d[i];
}

// Failure-path self-test.  One warp waits, through the same bounded wait the
// pipelines use (mbar_wait, kWaitTimeoutNs), on the first phase of a freshly
// initialised shared-memory barrier that nothing ever completes.  The wait
// gives up, sets the abort flag, and the kernel records PE_ERR_DEVICE_TIMEOUT
// in the error word as pe_fwd_kernel does after an aborted wait.  The error
// word is the only global memory it touches.
__global__ void pe_wait_timeout_probe_kernel(int *err) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_addr(&bar), 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(smem_addr(&bar), 0, &abort_flag);
    __syncthreads();
    if (threadIdx.x == 0 && abort_flag) atomicExch(err, (int)PE_ERR_DEVICE_TIMEOUT);
}

}  // namespace pe
