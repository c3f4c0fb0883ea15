// C ABI of the vision PatchEmbed library (see include/pe.h for the contract of
// every entry point).  Host side: argument validation, weight packing, TMA
// tensor-map encoding, tile-shape choice and kernel launches.  Nothing here
// computes on the host; every step of the forward path runs in the kernels of
// pe_kernels.cuh.
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/pe.h"
#include "pe_host_plan.h"
#include "pe_kernels.cuh"
#include "pe_astat.cuh"

using namespace pe;

struct pe_handle {
    int dev = -1;
    int E = 0, C = 0, tp = 0, p = 0, K = 0, Kpad = 0;
    int Kh = 0;                 // C*p*p rounded up to 16: one temporal slice of the slice-major weight
    bool has_bias = false;
    bool weight_set = false;
    uint16_t *wpack = nullptr;  // dev [E, Kpad] bf16, view(-1, C, tp, p, p) k order
    uint16_t *wpack_f = nullptr; // dev [E, Kpad] bf16, k order of the frames producer
    uint16_t *wpack_t = nullptr; // dev [E, 2*Kh] bf16, slice-major (tp == 2 only)
    uint16_t *wpack_fold = nullptr; // dev [E, Kh] bf16, both slices summed (tp == 2 only)
    uint16_t *wpack_i = nullptr; // dev [E, Kw] bf16, slice-interleaved 64-column tiles (tp == 2 only)
    int Kw = 0;                 // 64 * ceil(Kh / 32)
    bool fold = false;          // pe_set_temporal_fold
    uint32_t *wpack32 = nullptr; // dev [E, Kp32] fp32 words, tf32-rounded, view order
    int Kp32 = 0;               // K rounded up to 32
    bool tf32 = false;          // pe_set_tf32
    float *bias = nullptr;      // dev [E] fp32 (has_bias)
    int *err = nullptr;         // dev error word
    float mean[4] = {0, 0, 0, 0};
    float stdv[4] = {1, 1, 1, 1};
    CUtensorMap tmap_w[3];      // weight boxes of 32, 64, 128 rows (half a pair tile)
    CUtensorMap tmap_wf[3];     // same for the frames-order weight
    CUtensorMap tmap_wt[3];     // same for the slice-major weight
    CUtensorMap tmap_wfold[3];  // same for the folded weight
    CUtensorMap tmap_wi[3];     // same for the slice-interleaved weight
    CUtensorMap tmap_w32[3];    // same for the tf32 weight (32 fp32 columns per box)
    int num_sms = 0;
    int smem_optin = 0;
    // item table for grouped calls beyond PE_INLINE_ITEMS
    ItemDesc *items_dev = nullptr;
    ItemDesc *items_pinned = nullptr;
    int items_cap = 0;
    // staged frames path: normalised patch rows [N, K] (grow-only)
    uint16_t *stage_rows = nullptr;
    size_t stage_bytes = 0;
    // streamed frames path: two arrays of per-M-block ready counters, used by
    // alternate calls (each call zeroes the other one)
    uint32_t *ready = nullptr;
    int ready_cap = 0;
    int ready_parity = 0;
    // profiling: one event pair per call around the contraction kernel
    std::vector<cudaEvent_t> prof_ev;
    int prof_cap = 0, prof_n = 0;
    int64_t prof_launches = 0;   // kernels launched by forward calls while profiling
    bool prof_on = false;
    int prof_target = 0;         // 0: the contraction kernel, 1: the kernel before it
    cudaEvent_t items_evt = nullptr;
    bool items_evt_pending = false;
    // host-buffer calls: two input and two output slots in one device buffer,
    // a copy-in and a copy-out stream, and per-slot events (created on first use)
    uint8_t *host_ws = nullptr;
    size_t host_ws_in = 0, host_ws_out = 0;   // bytes of one input / one output slot
    cudaStream_t s_in = nullptr, s_out = nullptr;
    cudaEvent_t ev_start = nullptr, ev_in[2] = {}, ev_comp[2] = {}, ev_out[2] = {};
};

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 2-D tensor [rows, cols] (cols contiguous, row stride `ld` elements) of bf16 or
// fp32, box [box_rows, box_cols]; out-of-bounds elements read as zero and are
// not written by stores.
bool make_tmap(CUtensorMap *m, const void *base, bool f32, uint64_t rows, uint64_t cols, uint64_t ld,
               uint32_t box_rows, uint32_t box_cols, CUtensorMapSwizzle swz) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const uint64_t es = f32 ? 4 : 2;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {ld * es};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
              const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_bf16(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint64_t ld,
                    uint32_t box_rows) {
    return make_tmap(m, base, false, rows, cols, ld, box_rows, 64, CU_TENSOR_MAP_SWIZZLE_128B);
}

// Output [N, E]: 32 x 32 boxes, swizzled to match the epilogue's staging layout.
bool make_out_tmap(CUtensorMap *m, void *out, bool f32, int64_t N, int E) {
    return make_tmap(m, out, f32, (uint64_t)N, (uint64_t)E, (uint64_t)E, 32, 32,
                     f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B);
}

// One NVTX range per public call, named after it: visible on Nsight timelines
// and usable as an ncu filter (--nvtx --nvtx-include); without a tool attached
// the push and pop return at once.
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

// Runs an entry point's body so that no C++ exception crosses the C ABI: a
// failed host allocation (the item tables and chunk plans are std::vectors)
// returns PE_ERR_HOST_MEMORY, anything else PE_ERR_CUDA.
template <class F>
pe_status no_throw(F &&body) {
    try {
        return body();
    } catch (const std::bad_alloc &) {
        return PE_ERR_HOST_MEMORY;
    } catch (...) {
        return PE_ERR_CUDA;
    }
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_dtype(int d) { return d == PE_F32 || d == PE_BF16; }

struct DeviceGuard {
    int prev = -1;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
        if (prev != dev) cudaSetDevice(dev);
    }
    ~DeviceGuard() {
        int cur = -1;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

int bn_override() {
    const char *s = std::getenv("PE_BN");
    if (!s) return 0;
    const int v = std::atoi(s);
    return (v == 64 || v == 128 || v == 256) ? v : 0;
}

// Tile width: the widest BN (256: the pair MMA at full rate) unless the problem
// is too small to fill the GPU in one wave at 256; then every pair runs at most
// one tile, so the narrowest BN that still fits one wave finishes first (a
// second round of narrow tiles costs more than the narrow MMAs save).
int choose_bn(int64_t N, int E, int num_pairs) {
    if (const int o = bn_override()) return o;
    const int64_t mt = (N + 2 * kBM - 1) / (2 * kBM);
    auto tiles = [&](int bn) { return mt * ((E + bn - 1) / bn); };
    if (tiles(256) >= num_pairs) return 256;
    if (tiles(64) <= num_pairs) return 64;
    if (tiles(128) <= num_pairs) return 128;
    return 256;
}

thread_local pe_handle *t_prof_handle = nullptr;   // handle of the call being launched

// `after_prep`: the kernel reads rows written by the kernel launched just
// before it on `st`; it is launched with programmatic stream serialisation so
// that its prologue overlaps that kernel's tail (its TMA issuers wait on
// griddepcontrol.wait before the first load).
// `coop`: every CTA must be resident at once (CTAs wait for rows that other
// CTAs produce): cooperative launch.
template <int AMODE, int PT, bool F32IN, int NORM = 2, bool DUPALL = false, bool REGSTORE = false>
cudaError_t launch_fwd(const CUtensorMap &tw, const FwdParams &P, const CUtensorMap &tx, const CUtensorMap &to,
                       size_t smem, int grid, cudaStream_t st, bool after_prep = false, bool coop = false) {
    auto kern = pe_fwd_kernel<AMODE, PT, F32IN, NORM, DUPALL, REGSTORE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    pe_handle *h = t_prof_handle;
    const bool prof = h && h->prof_on && h->prof_target == 0 && h->prof_n < h->prof_cap;
    if (prof) cudaEventRecord(h->prof_ev[2 * h->prof_n], st);
    // an event between the two kernels (either profiling target) serialises
    // them anyway; a window that only counts launches keeps the overlap
    const bool pdl = after_prep && !(h && h->prof_on && h->prof_cap > 0);
    if (pdl || coop) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)grid);
        cfg.blockDim = dim3((unsigned)threads_for(AMODE));
        cfg.dynamicSmemBytes = smem;
        cfg.stream = st;
        cudaLaunchAttribute at[2];
        int na = 0;
        if (pdl) {
            at[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            at[na].val.programmaticStreamSerializationAllowed = 1;
            ++na;
        }
        if (coop) {
            at[na].id = cudaLaunchAttributeCooperative;
            at[na].val.cooperative = 1;
            ++na;
        }
        cfg.attrs = at;
        cfg.numAttrs = na;
        e = cudaLaunchKernelEx(&cfg, kern, tw, tx, to, P);
    } else {
        kern<<<grid, threads_for(AMODE), smem, st>>>(tw, tx, to, P);
        e = cudaGetLastError();
    }
    if (prof) {
        cudaEventRecord(h->prof_ev[2 * h->prof_n + 1], st);
        ++h->prof_n;
    }
    if (h && h->prof_on) ++h->prof_launches;
    return e;
}

// Event pair around the kernel a call launches before its contraction, when
// the handle profiles that kernel (pe_profile_target 1).
struct PreKernelEvents {
    pe_handle *h;
    bool on;
    PreKernelEvents(pe_handle *hh, cudaStream_t st)
        : h(hh), on(hh && hh->prof_on && hh->prof_target == 1 && hh->prof_n < hh->prof_cap), s(st) {
        if (on) cudaEventRecord(h->prof_ev[2 * h->prof_n], s);
    }
    ~PreKernelEvents() {
        if (on) {
            cudaEventRecord(h->prof_ev[2 * h->prof_n + 1], s);
            ++h->prof_n;
        }
    }
    cudaStream_t s;
};

struct ProfScope {   // makes the handle's profiling events visible to launch_fwd
    explicit ProfScope(pe_handle *h) { t_prof_handle = h; }
    ~ProfScope() { t_prof_handle = nullptr; }
};

int bn_index(int bn) { return bn == 64 ? 0 : (bn == 128 ? 1 : 2); }

// Pair tiles, grid (two CTAs per pair, at most one pair per two SMs).
void plan_tiles(const pe_handle *h, FwdParams &P, int64_t N, int &grid, bool &ok) {
    const int num_pairs = h->num_sms / 2;
    P.bn = choose_bn(N, P.E, num_pairs);
    P.n_tiles_n = (P.E + P.bn - 1) / P.bn;
    const int64_t mt = (N + 2 * kBM - 1) / (2 * kBM);
    ok = mt * P.n_tiles_n <= INT32_MAX;
    P.num_tiles = ok ? (int)(mt * P.n_tiles_n) : 0;
    grid = 2 * std::min(P.num_tiles, num_pairs);
}

void fill_common(const pe_handle *h, FwdParams &P) {
    std::memset(&P, 0, sizeof(P));
    P.E = h->E;
    P.C = h->C;
    P.TP = h->tp;
    P.P = h->p;
    P.K = h->K;
    P.Kpad = h->Kpad;
    P.Kh = h->Kh;
    for (int c = 0; c < 4; ++c) {
        const float mu = h->mean[c], sd = h->stdv[c];
        uint32_t mu_bits;
        std::memcpy(&mu_bits, &mu, 4);
        P.mean[c] = mu;
        P.stdv[c] = sd;
        int e = 0;
        const float s = 2.0f * std::frexp(sd, &e);   // sd = s * 2^(e-1), s in [1, 2)
        P.nstd_s[c] = -s;
        P.rcp_s[c] = 1.0f / s;                        // IEEE division on the host: correctly rounded
        P.scale[c] = std::ldexp(1.0f, 1 - e);         // 1 / sd = (1 / s) * 2^(1-e)
        if (mu_bits == 0u && sd == 1.0f)
            P.norm_mode[c] = kNormIdentity;
        else if (std::fabs(mu) >= 0x1p-70f && sd >= 0x1p-32f && sd <= 0x1p32f)
            P.norm_mode[c] = kNormScaled;
        else
            P.norm_mode[c] = kNormDivide;
    }
    P.bias = h->has_bias ? h->bias : nullptr;
    P.err = h->err;
}

// Ring depths and per-tile stage counts; returns the dynamic shared memory size.
// `kcols`: columns of the TMA-fed A rows (default K).
size_t plan_pipeline(const pe_handle *h, FwdParams &P, int amode, int kcols = -1) {
    if (kcols < 0) kcols = P.K;
    P.num_ksteps = (kcols + 15) / 16;
    P.ksub = 1;
    P.b_slot_bytes = kBStageBytes;
    if (amode == kAModeTmaShared) {
        P.num_ksteps = P.Kh / 16;            // k-steps per slice; each is issued once per slice
        P.b_slot_bytes = 2 * kBStageBytes;   // weight tiles of both slices
    } else if (amode == kAModeTma) {
        P.ksub = 2;                          // 128 k per stage: 8 MMAs per barrier round trip
        P.b_slot_bytes = 2 * kBStageBytes;
    } else if (amode == kAModeTmaTf32) {
        P.num_ksteps = (kcols + 7) / 8;      // tf32 MMAs take 8 k each
        P.ksub = 2;                          // 64 k per stage (two 32-column fp32 tiles)
        P.b_slot_bytes = 2 * kBStageBytes;
    }
    P.n_b_stages = (P.num_ksteps + 4 * P.ksub - 1) / (4 * P.ksub);
    if (amode == kAModeFrames) {
        P.a_stage_bytes = 2048 * P.P;  // 8 segments of p pixels, 128 rows
        P.n_a_stages = (P.C * P.TP * P.P + 7) / 8;
    } else {
        P.a_stage_bytes = P.ksub * kBM * kBK * 2;
        P.n_a_stages = P.n_b_stages;
    }
    const size_t epi_bytes = (size_t)4 * 8192;   // staging ring of the 4 epilogue warps
    auto rings = [&](int nb, int na) { return (size_t)nb * P.b_slot_bytes + (size_t)na * P.a_stage_bytes; };
    auto total = [&](int nb, int na) {
        const size_t r = (rings(nb, na) + 1023) / 1024 * 1024;
        return 1024 + r + epi_bytes + (size_t)(2 * nb + 2 * na + 5) * 8 + 16;
    };
    int nb = 6, na = (amode == kAModeFrames) ? 4 : 6;
    if (amode == kAModeFrames) {
        while (total(nb, na) > (size_t)h->smem_optin) {
            if (nb > 5) --nb;
            else if (na > 3) --na;
            else if (nb > 3) --nb;
            else if (na > 2) --na;
            else if (nb > 2) --nb;
            else break;
        }
    } else {
        // A and weight stages share ring slots: equal depths
        while (total(nb, na) > (size_t)h->smem_optin && nb > 2) { --nb; --na; }
    }
    P.nb = nb;
    P.na = na;
    P.n_iss = std::min(tma_fed(amode) ? 5 : 3, std::min(nb, na));
    P.epi_offset = (int)((rings(nb, na) + 1023) / 1024 * 1024);
    return total(nb, na);
}

pe_status finish(cudaError_t e) { return e == cudaSuccess ? PE_OK : PE_ERR_CUDA; }

// Validate one frames item and fill its descriptor.  Returns PE_OK or an error.
pe_status make_item(const pe_handle *h, const void *frames, int T, int H, int W, const int32_t *g,
                    int merge, int64_t row0, ItemDesc &d) {
    if (!frames || !g) return PE_ERR_INVALID_ARG;
    if (!aligned16(frames)) return PE_ERR_ALIGN;
    if (T < 1 || H < 1 || W < 1 || g[0] < 1 || g[1] < 1 || g[2] < 1) return PE_ERR_SHAPE;
    if ((int64_t)H != (int64_t)g[1] * h->p || (int64_t)W != (int64_t)g[2] * h->p) return PE_ERR_SHAPE;
    if (((int64_t)T + h->tp - 1) / h->tp != g[0]) return PE_ERR_SHAPE;
    if (merge == 2 && ((g[1] & 1) || (g[2] & 1))) return PE_ERR_SHAPE;
    if ((int64_t)T * h->C * H * W >= (int64_t)1 << 40) return PE_ERR_UNSUPPORTED;
    if ((int64_t)h->C * H * W > INT32_MAX) return PE_ERR_UNSUPPORTED;
    d.frames = frames;
    d.row0 = row0;
    d.T = T;
    d.H = H;
    d.W = W;
    d.gt = g[0];
    d.gh = g[1];
    d.gw = g[2];
    return PE_OK;
}

// Shared front half of the frames entry points: validation + item table.
pe_status setup_frames(pe_handle *h, int n, const void *const *frames, int f_dt, const int32_t *THW,
                       const int32_t *grid, int merge, const void *out, FwdParams &P, cudaStream_t st) {
    if (!h || n < 1 || !frames || !THW || !grid || !out) return PE_ERR_INVALID_ARG;
    if (!valid_dtype(f_dt)) return PE_ERR_DTYPE;
    if (merge != 1 && merge != 2) return PE_ERR_INVALID_ARG;
    if ((h->p & 1) || h->p > PE_MAX_PATCH) return PE_ERR_UNSUPPORTED;
    if (!aligned16(out)) return PE_ERR_ALIGN;
    fill_common(h, P);
    P.merge = merge;
    P.n_items = n;
    std::vector<ItemDesc> items((size_t)n);
    int64_t row0 = 0;
    P.all_t1 = 1;
    for (int i = 0; i < n; ++i) {
        const pe_status s = make_item(h, frames[i], THW[3 * i], THW[3 * i + 1], THW[3 * i + 2], grid + 3 * i,
                                      merge, row0, items[(size_t)i]);
        if (s != PE_OK) return s;
        P.all_t1 = P.all_t1 && THW[3 * i] == 1;
        row0 += (int64_t)grid[3 * i] * grid[3 * i + 1] * grid[3 * i + 2];
    }
    P.N = row0;
    if (n <= PE_INLINE_ITEMS) {
        for (int i = 0; i < n; ++i) P.items[i] = items[(size_t)i];
        P.items_dev = nullptr;
        return PE_OK;
    }
    // Upload the table into the handle's workspace (pinned staging, stream order).
    if (h->items_evt_pending) {
        if (cudaEventSynchronize(h->items_evt) != cudaSuccess) return PE_ERR_CUDA;
        h->items_evt_pending = false;
    }
    if (n > h->items_cap) {
        if (h->items_dev) cudaFree(h->items_dev);
        if (h->items_pinned) cudaFreeHost(h->items_pinned);
        h->items_dev = nullptr;
        h->items_pinned = nullptr;
        h->items_cap = 0;
        const int cap = std::max(n, 64);
        if (cudaMalloc(&h->items_dev, sizeof(ItemDesc) * cap) != cudaSuccess) return PE_ERR_CUDA;
        if (cudaMallocHost(&h->items_pinned, sizeof(ItemDesc) * cap) != cudaSuccess) return PE_ERR_CUDA;
        h->items_cap = cap;
    }
    std::memcpy(h->items_pinned, items.data(), sizeof(ItemDesc) * (size_t)n);
    if (cudaMemcpyAsync(h->items_dev, h->items_pinned, sizeof(ItemDesc) * (size_t)n, cudaMemcpyHostToDevice,
                        st) != cudaSuccess)
        return PE_ERR_CUDA;
    if (cudaEventRecord(h->items_evt, st) != cudaSuccess) return PE_ERR_CUDA;
    h->items_evt_pending = true;
    P.items_dev = h->items_dev;
    return PE_OK;
}

// Staged frames path: prepare kernel writes A once, then the TMA-fed pair
// GEMM reads it back.  The fused producer repeats its gather for every weight
// tile of a row block; measured on B200 the staged pair is faster at every
// size (about 2x at ~1000 patches, where both are latency-bound, 3x at 59k
// patches; 6.8x for fp32 frames), so it runs whenever it can: bf16 or fp32
// frames, tp = 2, p in {14, 16}.

bool staged_eligible(const pe_handle *h, int f_dt) {
    // tp = 1 rows are one slice wide (Kh columns, a multiple of 16); tp = 2
    // video rows are K wide, so K must keep their rows 16-byte aligned
    return (f_dt == PE_BF16 || f_dt == PE_F32) && (h->p == 14 || h->p == 16) &&
           (h->tp == 1 || (h->tp == 2 && (h->K % 8) == 0));
}

// bf16 frames with tp = 2 and p in {14, 16}: 0 = fused kernel, 1 = staged
// pair (the default), 2 = streamed kernel; PE_FRAMES_PATH=fused|staged|streamed
// overrides.  Every other frames call takes the fused kernel.  The
// streamed kernel overlaps row production with the contraction but its
// producer warps' scattered loads and stores slow the contraction down more
// than the separate prepare kernel costs (measured on B200), so it is not the
// default.
int frames_path(const pe_handle *h, int f_dt) {
    if (!staged_eligible(h, f_dt)) return 0;
    const char *e = std::getenv("PE_FRAMES_PATH");
    if (e && std::strcmp(e, "fused") == 0) return 0;
    if (e && std::strcmp(e, "streamed") == 0 && f_dt == PE_BF16 && h->tp == 2) return 2;   // bf16 words, tp = 2
    return 1;
}

template <int PT, int NORM, bool SHARED, bool F32IN = false>
cudaError_t launch_prep_rows(const FwdParams &P, uint16_t *A, int row_elems, cudaStream_t st) {
    auto kern = pe_prep_rows_kernel<PT, NORM, SHARED, F32IN>;
    const int smem = kPrepRows * row_elems * 2;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = (P.N + kPrepRows - 1) / kPrepRows;
    kern<<<(unsigned)grid, kPrepRows * PT / 2, smem, st>>>(P, A, row_elems);
    return cudaGetLastError();
}

template <int PT>
cudaError_t launch_prep(const FwdParams &P, bool all_scaled, bool shared, bool f32, uint16_t *A, int row_elems,
                        cudaStream_t st) {
    if (f32)   // fp32 frames: the normalisation mode is read per channel
        return shared ? launch_prep_rows<PT, 2, true, true>(P, A, row_elems, st)
                      : launch_prep_rows<PT, 2, false, true>(P, A, row_elems, st);
    if (all_scaled)
        return shared ? launch_prep_rows<PT, 1, true>(P, A, row_elems, st)
                      : launch_prep_rows<PT, 1, false>(P, A, row_elems, st);
    return shared ? launch_prep_rows<PT, 2, true>(P, A, row_elems, st)
                  : launch_prep_rows<PT, 2, false>(P, A, row_elems, st);
}

// shared: every row is a single frame (tp == 2), so A holds one slice per row
// (A[N, Kh]) and the contraction meets it with the slice-major weight.
// wmode 1 (fold): single-frame rows against the folded weight (one product
// per pixel); wmode 2: tp = 1, whose rows are one frame's patch in the view
// order, against the frames-order weight (the same order when tp = 1).
pe_status run_frames_staged(pe_handle *h, FwdParams &P, void *out, bool all_scaled, bool shared, bool f32,
                            cudaStream_t st, int wmode = 0) {
    const int row_elems = shared ? h->Kh : h->K;
    const size_t need = (size_t)P.N * row_elems * 2;
    if (need > h->stage_bytes) {
        if (h->stage_rows) {
            if (cudaStreamSynchronize(st) != cudaSuccess) return PE_ERR_CUDA;
            cudaFree(h->stage_rows);
        }
        h->stage_rows = nullptr;
        h->stage_bytes = 0;
        if (cudaMalloc(&h->stage_rows, need) != cudaSuccess) return PE_ERR_CUDA;
        h->stage_bytes = need;
    }
    // All host-side planning first, so that the two launches leave the host
    // back to back and the contraction is queued before the prepare kernel ends.
    FwdParams G = P;
    G.x = h->stage_rows;
    G.x_f32 = 0;
    G.x_vec = 1;
    int grid = 0;
    bool ok = true;
    plan_tiles(h, G, G.N, grid, ok);
    if (!ok) return PE_ERR_UNSUPPORTED;
    const int amode = (shared && wmode == 0) ? kAModeTmaShared : kAModeTma;
    const size_t smem = plan_pipeline(h, G, amode, row_elems);
    CUtensorMap tx, to;
    if (!make_tmap_bf16(&tx, h->stage_rows, (uint64_t)G.N, (uint64_t)row_elems, (uint64_t)row_elems, kBM))
        return PE_ERR_CUDA;
    if (!make_out_tmap(&to, out, G.out_f32, G.N, G.E)) return PE_ERR_CUDA;
    cudaError_t e;
    {
        PreKernelEvents pk(h, st);
        e = (h->p == 14) ? launch_prep<14>(P, all_scaled, shared, f32, h->stage_rows, row_elems, st)
                         : launch_prep<16>(P, all_scaled, shared, f32, h->stage_rows, row_elems, st);
    }
    if (h->prof_on) ++h->prof_launches;
    if (e != cudaSuccess) return PE_ERR_CUDA;
    if (wmode == 1) {
        // the folded weight halves each tile's MMAs, so the epilogue bounds the
        // tile: its rows are stored straight from registers
        G.out = out;
        G.epi_v8 = reinterpret_cast<uintptr_t>(out) % 32 == 0 && (int64_t)G.E * (G.out_f32 ? 4 : 2) % 32 == 0;
        return finish(launch_fwd<kAModeTma, 0, false, 2, false, true>(h->tmap_wfold[bn_index(G.bn)], G, tx, to, smem,
                                                                      grid, st, true));
    }
    if (wmode == 2)
        return finish(launch_fwd<kAModeTma, 0, false>(h->tmap_wf[bn_index(G.bn)], G, tx, to, smem, grid, st, true));
    if (shared)
        return finish(
            launch_fwd<kAModeTmaShared, 0, false>(h->tmap_wt[bn_index(G.bn)], G, tx, to, smem, grid, st, true));
    return finish(launch_fwd<kAModeTma, 0, false>(h->tmap_wf[bn_index(G.bn)], G, tx, to, smem, grid, st, true));
}

// Streamed frames path: one cooperative kernel whose producer warps write the
// normalised rows (slice-major, one slice for single-frame rows, two
// otherwise) into the handle's row buffer while its TMA-fed pair GEMM consumes
// the completed M-blocks.
pe_status run_frames_streamed(pe_handle *h, FwdParams &P, void *out, bool all_scaled, bool shared, cudaStream_t st) {
    const int row_elems = (shared ? 1 : 2) * h->Kh;
    const size_t need = (size_t)P.N * row_elems * 2;
    const int64_t mt = (P.N + 2 * kBM - 1) / (2 * kBM);
    if (mt > INT32_MAX / 2) return PE_ERR_UNSUPPORTED;
    if (need > h->stage_bytes || mt > h->ready_cap) {
        if (cudaStreamSynchronize(st) != cudaSuccess) return PE_ERR_CUDA;
    }
    if (need > h->stage_bytes) {
        if (h->stage_rows) cudaFree(h->stage_rows);
        h->stage_rows = nullptr;
        h->stage_bytes = 0;
        if (cudaMalloc(&h->stage_rows, need) != cudaSuccess) return PE_ERR_CUDA;
        h->stage_bytes = need;
    }
    if (mt > h->ready_cap) {
        if (h->ready) cudaFree(h->ready);
        h->ready = nullptr;
        h->ready_cap = 0;
        const int cap = (int)std::max<int64_t>(mt, 1024);
        if (cudaMalloc(&h->ready, sizeof(uint32_t) * 2 * (size_t)cap) != cudaSuccess) return PE_ERR_CUDA;
        if (cudaMemsetAsync(h->ready, 0, sizeof(uint32_t) * 2 * (size_t)cap, st) != cudaSuccess) return PE_ERR_CUDA;
        h->ready_cap = cap;
        h->ready_parity = 0;
    }
    FwdParams G = P;
    G.x = h->stage_rows;
    G.x_f32 = 0;
    G.x_vec = 1;
    G.a_rows = h->stage_rows;
    G.row_elems = row_elems;
    G.ready = h->ready + (size_t)h->ready_parity * h->ready_cap;
    G.ready_next = h->ready + (size_t)(h->ready_parity ^ 1) * h->ready_cap;
    G.n_mblocks = (int)mt;
    int grid = 0;
    bool ok = true;
    plan_tiles(h, G, G.N, grid, ok);
    if (!ok) return PE_ERR_UNSUPPORTED;
    G.ready_target = (uint32_t)(kStreamProdWarps * 2 * G.n_tiles_n);
    // single-frame rows: one slice against both weight slices; otherwise both
    // slices of a row in sequence against the slice-major weight
    const size_t smem = plan_pipeline(h, G, shared ? kAModeTmaShared : kAModeTma, row_elems);
    CUtensorMap tx, to;
    if (!make_tmap_bf16(&tx, h->stage_rows, (uint64_t)G.N, (uint64_t)row_elems, (uint64_t)row_elems, kBM))
        return PE_ERR_CUDA;
    if (!make_out_tmap(&to, out, G.out_f32, G.N, G.E)) return PE_ERR_CUDA;
    const CUtensorMap &tw = h->tmap_wt[bn_index(G.bn)];
    h->ready_parity ^= 1;
    cudaError_t e;
#define PE_LAUNCH_STREAM(PP, NN)                                                                                    \
    (shared ? launch_fwd<kAModeTmaStream, PP, false, NN, true>(tw, G, tx, to, smem, grid, st, false, true)          \
            : launch_fwd<kAModeTmaStream, PP, false, NN, false>(tw, G, tx, to, smem, grid, st, false, true))
    if (h->p == 14)
        e = all_scaled ? PE_LAUNCH_STREAM(14, 1) : PE_LAUNCH_STREAM(14, 2);
    else
        e = all_scaled ? PE_LAUNCH_STREAM(16, 1) : PE_LAUNCH_STREAM(16, 2);
#undef PE_LAUNCH_STREAM
    return finish(e);
}

int env_int(const char *name, int dflt) {
    const char *s = std::getenv(name);
    return s ? std::atoi(s) : dflt;
}

// Resident-A kernel (pe_astat_kernel): weight ring depth, staging boxes and
// shared-memory offsets.  Returns the dynamic shared memory size, or 0 when
// the resident A does not fit beside a ring of two weight stages.
// PE_ASTAT_NB / PE_ASTAT_EPIBUFS pin the ring depth / staging boxes.
size_t plan_astat(const pe_handle *h, FwdParams &P) {
    if (P.Kh % 16 != 0 || (P.P & 1)) return 0;
    P.num_ksteps = P.Kh / 16;
    P.n_achunks = (P.C * P.P + kAsChunkSegs - 1) / kAsChunkSegs;   // chunks of 8 segments (8p columns)
    const int cks = kAsChunkSegs * P.P / 16;                          // k-steps per chunk
    if (P.n_achunks > kAsMaxChunks || cks < 1 || (P.num_ksteps + cks - 1) / cks != P.n_achunks) return 0;
    P.cpp = P.C * P.P * P.P;
    P.n_b_stages = (P.Kh + 63) / 64;           // 2 slice-interleaved tiles (4 k-steps of both slices) per stage
    P.b_slot_bytes = kAsWTiles * (P.bn / 2) * 128;   // this CTA's half of the stage's tiles
    P.ksub = 1;
    const size_t a_bytes = (size_t)((P.Kh + 63) / 64) * kAsTileBytes;   // 64-column swizzled tiles
    const size_t box = P.out_f32 ? 4096 : 2048;
    auto up = [](size_t v) { return (v + 1023) / 1024 * 1024; };
    auto bars = [&](int nb) { return (size_t)(2 * nb + 2 * P.n_achunks + 5) * 8 + (size_t)(2 * nb + 2) * 4; };
    auto total = [&](int nb, int bufs) {
        return 1024 + up((size_t)nb * P.b_slot_bytes) + up(a_bytes) + 4 * (size_t)bufs * box + bars(nb);
    };
    const int nb_pin = env_int("PE_ASTAT_NB", 0), bufs_pin = env_int("PE_ASTAT_EPIBUFS", -1);
    // staging boxes (TMA stores) when they fit beside two weight stages; else
    // the epilogue stores straight from registers (bufs = 0)
    for (int nb = 8; nb >= 2; --nb) {
        if (nb_pin && nb != nb_pin) continue;
        for (int bufs = 2; bufs >= 0; --bufs) {
            if (bufs_pin >= 0 && bufs != bufs_pin) continue;
            const size_t t = total(nb, bufs);
            if (t > (size_t)h->smem_optin) continue;
            P.nb = nb;
            P.na = 0;
            P.epi_bufs = bufs;
            P.n_iss = std::min(3, nb);
            P.a_offset = (int)up((size_t)nb * P.b_slot_bytes);
            P.epi_offset = P.a_offset + (int)up(a_bytes);
            P.bar_offset = P.epi_offset + 4 * bufs * (int)box;
            return t;
        }
    }
    return 0;
}

// Single images (every item T = 1), tp = 2, bf16 frames: the resident-A kernel
// applies when the handle has the slice-interleaved weight and A fits.
bool astat_eligible(const pe_handle *h, const FwdParams &P, int f_dt) {
    return f_dt == PE_BF16 && h->tp == 2 && P.all_t1 && h->wpack_i && (h->p & 1) == 0;
}

template <int PT, int NORM>
cudaError_t launch_astat(const CUtensorMap &tw, const CUtensorMap &to, const FwdParams &P, size_t smem, int grid,
                         cudaStream_t st) {
    auto kern = pe_astat_kernel<PT, NORM>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    pe_handle *h = t_prof_handle;
    const bool prof = h && h->prof_on && h->prof_target == 0 && h->prof_n < h->prof_cap;
    if (prof) cudaEventRecord(h->prof_ev[2 * h->prof_n], st);
    kern<<<grid, kAsThreads, smem, st>>>(tw, to, P);
    e = cudaGetLastError();
    if (prof) {
        cudaEventRecord(h->prof_ev[2 * h->prof_n + 1], st);
        ++h->prof_n;
    }
    if (h && h->prof_on) ++h->prof_launches;
    return e;
}

// One launch from raw frames to embeddings; allocates nothing.  Returns
// PE_ERR_UNSUPPORTED (nothing launched) when the resident A does not fit.
pe_status run_frames_astat(pe_handle *h, FwdParams &P, void *out, cudaStream_t st) {
    int grid = 0;
    bool ok = true;
    plan_tiles(h, P, P.N, grid, ok);
    if (!ok) return PE_ERR_UNSUPPORTED;
    const size_t smem = plan_astat(h, P);
    if (smem == 0) return PE_ERR_UNSUPPORTED;
    const uint64_t wl = (uint64_t)env_int("PE_TEST_WAIT_NS", 0);
    P.wait_ns = wl;
    P.out = out;
    CUtensorMap to;
    if (!make_out_tmap(&to, out, P.out_f32, P.N, P.E)) return PE_ERR_CUDA;
    const CUtensorMap &tw = h->tmap_wi[bn_index(P.bn)];
    bool all_scaled = true;
    for (int c = 0; c < P.C; ++c) all_scaled = all_scaled && P.norm_mode[c] == kNormScaled;
    cudaError_t e;
    if (h->p == 14)
        e = all_scaled ? launch_astat<14, 1>(tw, to, P, smem, grid, st) : launch_astat<14, 2>(tw, to, P, smem, grid, st);
    else
        e = launch_astat<0, 2>(tw, to, P, smem, grid, st);
    return finish(e);
}

pe_status run_frames(pe_handle *h, FwdParams &P, int f_dt, void *out, int out_dt, cudaStream_t st,
                     bool allow_staged = true) {
    P.out_f32 = out_dt == PE_F32;
    if (P.N == 0) return PE_OK;
    // Temporal folding (opt-in): single-frame items meet the summed slices of
    // the weight; the staged path's rows for them are already one slice wide.
    if (allow_staged && h->fold && h->wpack_fold && P.all_t1 && staged_eligible(h, f_dt)) {
        bool all_scaled = true;
        for (int c = 0; c < P.C; ++c) all_scaled = all_scaled && P.norm_mode[c] == kNormScaled;
        return run_frames_staged(h, P, out, all_scaled, true, f_dt == PE_F32, st, 1);
    }
    // Single images: the resident-A kernel when asked for (PE_FRAMES_PATH=astat)
    // and for the allocation-free call (it needs no workspace); otherwise the
    // staged pair, which measured faster on B200 (the resident A leaves the
    // weight ring too little shared memory to hide its latency).
    const char *fp = std::getenv("PE_FRAMES_PATH");
    const bool want_astat = (fp && std::strcmp(fp, "astat") == 0) || !allow_staged;
    if (want_astat && astat_eligible(h, P, f_dt)) {
        FwdParams A = P;
        const pe_status sa = run_frames_astat(h, A, out, st);
        if (sa != PE_ERR_UNSUPPORTED) return sa;
    }
    const int lp = allow_staged ? frames_path(h, f_dt) : 0;
    if (lp != 0) {
        bool all_scaled = true;
        for (int c = 0; c < P.C; ++c) all_scaled = all_scaled && P.norm_mode[c] == kNormScaled;
        const bool shared = h->tp == 2 && P.all_t1 && h->wpack_t;
        if (lp == 2) return run_frames_streamed(h, P, out, all_scaled, shared, st);
        if (h->tp == 1)   // one frame per temporal patch: one-slice rows, frames-order weight
            return run_frames_staged(h, P, out, all_scaled, true, f_dt == PE_F32, st, 2);
        return run_frames_staged(h, P, out, all_scaled, shared, f_dt == PE_F32, st);
    }
    int grid = 0;
    bool ok = true;
    plan_tiles(h, P, P.N, grid, ok);
    if (!ok) return PE_ERR_UNSUPPORTED;
    const size_t smem = plan_pipeline(h, P, kAModeFrames);
    CUtensorMap dummy, to;
    std::memset(&dummy, 0, sizeof(dummy));
    if (!make_out_tmap(&to, out, P.out_f32, P.N, P.E)) return PE_ERR_CUDA;
    const CUtensorMap &tw = h->tmap_wf[bn_index(P.bn)];
    const bool f32 = f_dt == PE_F32;
    // One normalisation mode for every channel lets the producer drop the
    // per-word mode test (1: all scaled; 2: anything else, decided per word),
    // and frames that are all single images (T = 1, tp = 2) need only one
    // temporal slice per (c, i).
    bool all_scaled = true;
    for (int c = 0; c < P.C; ++c) all_scaled = all_scaled && P.norm_mode[c] == kNormScaled;
    bool dupall = h->tp == 2;
    dupall = dupall && P.all_t1;
    cudaError_t e;
    if (!f32 && (h->p == 14 || h->p == 16)) {
#define PE_LAUNCH_FRAMES(PP)                                                                                  \
    (all_scaled ? (dupall ? launch_fwd<kAModeFrames, PP, false, 1, true>(tw, P, dummy, to, smem, grid, st)       \
                          : launch_fwd<kAModeFrames, PP, false, 1, false>(tw, P, dummy, to, smem, grid, st))     \
                : (dupall ? launch_fwd<kAModeFrames, PP, false, 2, true>(tw, P, dummy, to, smem, grid, st)       \
                          : launch_fwd<kAModeFrames, PP, false, 2, false>(tw, P, dummy, to, smem, grid, st)))
        e = (h->p == 14) ? PE_LAUNCH_FRAMES(14) : PE_LAUNCH_FRAMES(16);
#undef PE_LAUNCH_FRAMES
    } else if (h->p == 14)
        e = launch_fwd<kAModeFrames, 14, true>(tw, P, dummy, to, smem, grid, st);
    else if (h->p == 16)
        e = launch_fwd<kAModeFrames, 16, true>(tw, P, dummy, to, smem, grid, st);
    else
        e = f32 ? launch_fwd<kAModeFrames, 0, true>(tw, P, dummy, to, smem, grid, st)
                : launch_fwd<kAModeFrames, 0, false>(tw, P, dummy, to, smem, grid, st);
    return finish(e);
}

}  // namespace

extern "C" {

const char *pe_status_string(pe_status s) {
    switch (s) {
        case PE_OK: return "ok";
        case PE_ERR_INVALID_ARG: return "invalid argument";
        case PE_ERR_SHAPE: return "inconsistent shape";
        case PE_ERR_DTYPE: return "unsupported dtype";
        case PE_ERR_ALIGN: return "device pointer not 16-byte aligned";
        case PE_ERR_NO_WEIGHT: return "weight not set";
        case PE_ERR_CUDA: return "CUDA error";
        case PE_ERR_UNSUPPORTED: return "unsupported configuration";
        case PE_ERR_DEVICE_TIMEOUT: return "device pipeline wait timed out";
        case PE_ERR_HOST_MEMORY: return "host memory allocation failed";
        case PE_ERR_DEVICE_BOUNDS: return "a kernel index fell outside its buffer (bounds-checking build)";
    }
    return "unknown status";
}

int64_t pe_num_patches(const int32_t *grid_thw, int n) {
    if (n == 0) return 0;
    if (!grid_thw || n < 0) return -1;
    int64_t s = 0;
    for (int i = 0; i < n; ++i) {
        const int32_t *g = grid_thw + 3 * i;
        if (g[0] < 1 || g[1] < 1 || g[2] < 1) return -1;
        const int64_t th = (int64_t)g[0] * g[1];           // < 2^62: no overflow
        if (th > INT64_MAX / g[2]) return -1;
        const int64_t rows = th * g[2];
        if (s > INT64_MAX - rows) return -1;
        s += rows;
    }
    return s;
}

int pe_device(const pe_handle *h) { return h ? h->dev : -1; }

pe_status pe_create(int E, int C, int tp, int p, int has_bias, pe_handle **out) {
    if (!out) return PE_ERR_INVALID_ARG;
    *out = nullptr;
    if (E < 16 || E > 65535 || (E % 8) != 0 || C < 1 || C > 4 || tp < 1 || tp > 4 || p < 1)
        return PE_ERR_INVALID_ARG;
    const int64_t K = (int64_t)C * tp * p * p;
    if (K > 8192) return PE_ERR_UNSUPPORTED;
    pe_handle *h = new (std::nothrow) pe_handle();
    if (!h) return PE_ERR_CUDA;
    if (cudaGetDevice(&h->dev) != cudaSuccess) { delete h; return PE_ERR_CUDA; }
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, h->dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, h->dev);
    if (major != 10 || minor != 0) { delete h; return PE_ERR_UNSUPPORTED; }
    cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->dev);
    cudaDeviceGetAttribute(&h->smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, h->dev);
    h->E = E;
    h->C = C;
    h->tp = tp;
    h->p = p;
    h->K = (int)K;
    h->Kpad = (int)((K + 63) / 64 * 64);
    h->Kh = (C * p * p + 15) / 16 * 16;
    h->has_bias = has_bias != 0;
    bool ok = cudaMalloc(&h->wpack, sizeof(uint16_t) * (size_t)E * h->Kpad) == cudaSuccess &&
              cudaMalloc(&h->wpack_f, sizeof(uint16_t) * (size_t)E * h->Kpad) == cudaSuccess &&
              cudaMalloc(&h->err, sizeof(int)) == cudaSuccess &&
              cudaMemset(h->err, 0, sizeof(int)) == cudaSuccess &&
              cudaEventCreateWithFlags(&h->items_evt, cudaEventDisableTiming) == cudaSuccess;
    if (ok && h->has_bias) ok = cudaMalloc(&h->bias, sizeof(float) * E) == cudaSuccess;
    h->Kp32 = (int)((K + 31) / 32 * 32);
    if (ok) ok = cudaMalloc(&h->wpack32, sizeof(uint32_t) * (size_t)E * h->Kp32) == cudaSuccess;
    h->Kw = 64 * ((h->Kh + 31) / 32);
    if (ok && tp == 2) ok = cudaMalloc(&h->wpack_t, sizeof(uint16_t) * (size_t)E * 2 * h->Kh) == cudaSuccess &&
                            cudaMalloc(&h->wpack_fold, sizeof(uint16_t) * (size_t)E * h->Kh) == cudaSuccess &&
                            cudaMalloc(&h->wpack_i, sizeof(uint16_t) * (size_t)E * h->Kw) == cudaSuccess;
    if (ok) {
        const uint32_t boxes[3] = {32, 64, 128};   // half of BN = 64, 128, 256
        for (int i = 0; i < 3 && ok; ++i)
            ok = make_tmap_bf16(&h->tmap_w[i], h->wpack, (uint64_t)E, (uint64_t)h->Kpad, (uint64_t)h->Kpad,
                                boxes[i]) &&
                 make_tmap_bf16(&h->tmap_wf[i], h->wpack_f, (uint64_t)E, (uint64_t)h->Kpad, (uint64_t)h->Kpad,
                                boxes[i]) &&
                 (!h->wpack_t || make_tmap_bf16(&h->tmap_wt[i], h->wpack_t, (uint64_t)E, (uint64_t)(2 * h->Kh),
                                                (uint64_t)(2 * h->Kh), boxes[i])) &&
                 (!h->wpack_fold || make_tmap_bf16(&h->tmap_wfold[i], h->wpack_fold, (uint64_t)E, (uint64_t)h->Kh,
                                                   (uint64_t)h->Kh, boxes[i])) &&
                 (!h->wpack_i || make_tmap_bf16(&h->tmap_wi[i], h->wpack_i, (uint64_t)E, (uint64_t)h->Kw,
                                                (uint64_t)h->Kw, boxes[i])) &&
                 make_tmap(&h->tmap_w32[i], h->wpack32, true, (uint64_t)E, (uint64_t)h->Kp32, (uint64_t)h->Kp32,
                           boxes[i], 32, CU_TENSOR_MAP_SWIZZLE_128B);
    }
    if (!ok) { pe_destroy(h); return PE_ERR_CUDA; }
    *out = h;
    return PE_OK;
}

void pe_destroy(pe_handle *h) {
    if (!h) return;
    DeviceGuard g(h->dev);
    cudaDeviceSynchronize();
    if (h->wpack) cudaFree(h->wpack);
    if (h->wpack_f) cudaFree(h->wpack_f);
    if (h->wpack_t) cudaFree(h->wpack_t);
    if (h->wpack_fold) cudaFree(h->wpack_fold);
    if (h->wpack_i) cudaFree(h->wpack_i);
    if (h->wpack32) cudaFree(h->wpack32);
    if (h->bias) cudaFree(h->bias);
    if (h->err) cudaFree(h->err);
    if (h->items_dev) cudaFree(h->items_dev);
    if (h->items_pinned) cudaFreeHost(h->items_pinned);
    if (h->stage_rows) cudaFree(h->stage_rows);
    if (h->ready) cudaFree(h->ready);
    if (h->items_evt) cudaEventDestroy(h->items_evt);
    for (cudaEvent_t e : h->prof_ev) cudaEventDestroy(e);
    if (h->host_ws) cudaFree(h->host_ws);
    for (cudaStream_t s : {h->s_in, h->s_out})
        if (s) cudaStreamDestroy(s);
    for (cudaEvent_t e : {h->ev_start, h->ev_in[0], h->ev_in[1], h->ev_comp[0], h->ev_comp[1], h->ev_out[0],
                          h->ev_out[1]})
        if (e) cudaEventDestroy(e);
    delete h;
}

pe_status pe_set_weight(pe_handle *h, const void *w, pe_dtype w_dt, const void *bias, pe_dtype b_dt,
                        pe_stream_t stream) {
    NvtxRange nvtx("pe_set_weight");
    if (!h || !w) return PE_ERR_INVALID_ARG;
    if (!valid_dtype(w_dt) || (bias && !valid_dtype(b_dt))) return PE_ERR_DTYPE;
    if ((bias != nullptr) != h->has_bias) return PE_ERR_INVALID_ARG;
    if (!aligned16(w) || (bias && !aligned16(bias))) return PE_ERR_ALIGN;
    DeviceGuard g(h->dev);
    const int64_t total = (int64_t)h->E * h->Kpad;
    const int threads = 256;
    const int blocks = (int)std::min<int64_t>((total + threads - 1) / threads, (int64_t)h->num_sms * 8);
    cudaStream_t st = (cudaStream_t)stream;
    pe_pack_weight_kernel<<<blocks, threads, 0, st>>>(w, w_dt == PE_F32, bias, b_dt == PE_F32, h->wpack, h->bias,
                                                      h->E, h->C, h->tp, h->p, h->Kpad, 0, h->Kh);
    if (cudaGetLastError() != cudaSuccess) return PE_ERR_CUDA;
    pe_pack_weight_kernel<<<blocks, threads, 0, st>>>(w, w_dt == PE_F32, nullptr, b_dt == PE_F32, h->wpack_f,
                                                      nullptr, h->E, h->C, h->tp, h->p, h->Kpad, 1, h->Kh);
    if (cudaGetLastError() != cudaSuccess) return PE_ERR_CUDA;
    if (h->wpack_t) {
        pe_pack_weight_kernel<<<blocks, threads, 0, st>>>(w, w_dt == PE_F32, nullptr, b_dt == PE_F32, h->wpack_t,
                                                          nullptr, h->E, h->C, h->tp, h->p, 2 * h->Kh, 2, h->Kh);
        if (cudaGetLastError() != cudaSuccess) return PE_ERR_CUDA;
    }
    if (h->wpack_fold) {
        pe_pack_weight_kernel<<<blocks, threads, 0, st>>>(w, w_dt == PE_F32, nullptr, b_dt == PE_F32, h->wpack_fold,
                                                          nullptr, h->E, h->C, h->tp, h->p, h->Kh, 3, h->Kh);
        if (cudaGetLastError() != cudaSuccess) return PE_ERR_CUDA;
    }
    if (h->wpack_i) {
        pe_pack_weight_kernel<<<blocks, threads, 0, st>>>(w, w_dt == PE_F32, nullptr, b_dt == PE_F32, h->wpack_i,
                                                          nullptr, h->E, h->C, h->tp, h->p, h->Kw, 4, h->Kh);
        if (cudaGetLastError() != cudaSuccess) return PE_ERR_CUDA;
    }
    pe_pack_weight_tf32_kernel<<<blocks, threads, 0, st>>>(w, w_dt == PE_F32, h->wpack32, h->E, h->K, h->Kp32);
    if (cudaGetLastError() != cudaSuccess) return PE_ERR_CUDA;
    h->weight_set = true;
    return PE_OK;
}

pe_status pe_set_tf32(pe_handle *h, int enable) {
    if (!h) return PE_ERR_INVALID_ARG;
    if (enable && (h->K % 4) != 0) return PE_ERR_UNSUPPORTED;
    h->tf32 = enable != 0;
    return PE_OK;
}

pe_status pe_set_temporal_fold(pe_handle *h, int enable) {
    if (!h) return PE_ERR_INVALID_ARG;
    if (enable && h->tp != 2) return PE_ERR_UNSUPPORTED;
    h->fold = enable != 0;
    return PE_OK;
}

pe_status pe_set_norm(pe_handle *h, const float *mean, const float *std) {
    if (!h || !mean || !std) return PE_ERR_INVALID_ARG;
    for (int c = 0; c < h->C; ++c) {
        if (!(std[c] > 0.f) || !(std[c] < 3.0e38f) || !(mean[c] == mean[c]) ||
            !(mean[c] < 3.0e38f && mean[c] > -3.0e38f))
            return PE_ERR_INVALID_ARG;
    }
    for (int c = 0; c < h->C; ++c) {
        h->mean[c] = mean[c];
        h->stdv[c] = std[c];
    }
    return PE_OK;
}

}  // extern "C"

namespace {

// Shared body of pe_forward_patches and pe_forward_patches_pos.
pe_status forward_patches(pe_handle *h, const void *x, pe_dtype x_dt, int64_t N, const void *pos, int pos_dt,
                          void *out, pe_dtype out_dt, pe_stream_t stream) {
    if (!h || N < 0) return PE_ERR_INVALID_ARG;
    if (!valid_dtype(x_dt) || !valid_dtype(out_dt)) return PE_ERR_DTYPE;
    if (!h->weight_set) return PE_ERR_NO_WEIGHT;
    if (N == 0) return PE_OK;
    if (!x || !out) return PE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(out)) return PE_ERR_ALIGN;
    DeviceGuard g(h->dev);
    ProfScope ps(h);
    FwdParams P;
    fill_common(h, P);
    P.N = N;
    P.x = x;
    P.x_f32 = x_dt == PE_F32;
    P.out_f32 = out_dt == PE_F32;
    P.pos = pos;
    P.pos_f32 = pos_dt == PE_F32;
    P.merge = 1;
    const bool tma = (x_dt == PE_BF16) && (h->K % 8 == 0);
    P.x_vec = (x_dt == PE_BF16) ? (h->K % 8 == 0) : (h->K % 4 == 0);
    // fp32 rows with K % 8 == 0: cast them to bf16 once into the workspace and
    // run the TMA-fed contraction (PE_PATCHES_PATH=threads keeps the producer
    // warps converting inside the contraction kernel).
    if (x_dt == PE_F32 && h->tf32) {
        // tf32 contraction: rows rounded to tf32 once into the workspace, then
        // kind::tf32 pair MMAs against the tf32-rounded weight (K % 4 == 0).
        const size_t need = (size_t)N * h->K * 4;
        cudaStream_t st = (cudaStream_t)stream;
        if (need > h->stage_bytes) {
            if (h->stage_rows) {
                if (cudaStreamSynchronize(st) != cudaSuccess) return PE_ERR_CUDA;
                cudaFree(h->stage_rows);
            }
            h->stage_rows = nullptr;
            h->stage_bytes = 0;
            if (cudaMalloc(&h->stage_rows, need) != cudaSuccess) return PE_ERR_CUDA;
            h->stage_bytes = need;
        }
        int grid = 0;
        bool ok = true;
        plan_tiles(h, P, N, grid, ok);
        if (!ok) return PE_ERR_UNSUPPORTED;
        const size_t smem = plan_pipeline(h, P, kAModeTmaTf32);
        CUtensorMap tx, to;
        if (!make_tmap(&tx, h->stage_rows, true, (uint64_t)N, (uint64_t)h->K, (uint64_t)h->K, kBM, 32,
                       CU_TENSOR_MAP_SWIZZLE_128B))
            return PE_ERR_CUDA;
        if (!make_out_tmap(&to, out, P.out_f32, N, h->E)) return PE_ERR_CUDA;
        const int64_t n4 = (int64_t)N * h->K / 4;
        const int cb = (int)std::min<int64_t>((n4 + 255) / 256, (int64_t)h->num_sms * 8);
        {
            PreKernelEvents pk(h, st);
            pe_round_tf32_kernel<<<cb, 256, 0, st>>>(reinterpret_cast<const float *>(x),
                                                     reinterpret_cast<uint32_t *>(h->stage_rows), n4);
        }
        if (h->prof_on) ++h->prof_launches;
        if (cudaGetLastError() != cudaSuccess) return PE_ERR_CUDA;
        FwdParams G = P;
        G.x = h->stage_rows;
        G.x_f32 = 1;
        G.x_vec = 1;
        return finish(
            launch_fwd<kAModeTmaTf32, 0, false>(h->tmap_w32[bn_index(G.bn)], G, tx, to, smem, grid, st, true));
    }
    const char *pp = std::getenv("PE_PATCHES_PATH");
    if (x_dt == PE_F32 && (h->K % 8) == 0 && !(pp && std::strcmp(pp, "threads") == 0)) {
        const size_t need = (size_t)N * h->K * 2;
        cudaStream_t st = (cudaStream_t)stream;
        if (need > h->stage_bytes) {
            if (h->stage_rows) {
                if (cudaStreamSynchronize(st) != cudaSuccess) return PE_ERR_CUDA;
                cudaFree(h->stage_rows);
            }
            h->stage_rows = nullptr;
            h->stage_bytes = 0;
            if (cudaMalloc(&h->stage_rows, need) != cudaSuccess) return PE_ERR_CUDA;
            h->stage_bytes = need;
        }
        int grid = 0;
        bool ok = true;
        plan_tiles(h, P, N, grid, ok);
        if (!ok) return PE_ERR_UNSUPPORTED;
        const size_t smem = plan_pipeline(h, P, kAModeTma);
        CUtensorMap tx, to;
        if (!make_tmap_bf16(&tx, h->stage_rows, (uint64_t)N, (uint64_t)h->K, (uint64_t)h->K, kBM)) return PE_ERR_CUDA;
        if (!make_out_tmap(&to, out, P.out_f32, N, h->E)) return PE_ERR_CUDA;
        const int64_t n8 = (int64_t)N * h->K / 8;
        const int cb = (int)std::min<int64_t>((n8 + 255) / 256, (int64_t)h->num_sms * 8);
        {
            PreKernelEvents pk(h, st);
            pe_cast_rows_kernel<<<cb, 256, 0, st>>>(reinterpret_cast<const float *>(x), h->stage_rows, n8);
        }
        if (h->prof_on) ++h->prof_launches;
        if (cudaGetLastError() != cudaSuccess) return PE_ERR_CUDA;
        FwdParams G = P;
        G.x = h->stage_rows;
        G.x_f32 = 0;
        G.x_vec = 1;
        return finish(launch_fwd<kAModeTma, 0, false>(h->tmap_w[bn_index(G.bn)], G, tx, to, smem, grid, st, true));
    }
    int grid = 0;
    bool ok = true;
    plan_tiles(h, P, N, grid, ok);
    if (!ok) return PE_ERR_UNSUPPORTED;
    const size_t smem = plan_pipeline(h, P, tma ? kAModeTma : kAModePatchThreads);
    cudaStream_t st = (cudaStream_t)stream;
    CUtensorMap tx, to;
    std::memset(&tx, 0, sizeof(tx));
    if (!make_out_tmap(&to, out, P.out_f32, N, h->E)) return PE_ERR_CUDA;
    const CUtensorMap &tw = h->tmap_w[bn_index(P.bn)];
    if (tma) {
        if (!make_tmap_bf16(&tx, x, (uint64_t)N, (uint64_t)h->K, (uint64_t)h->K, kBM)) return PE_ERR_CUDA;
        return finish(launch_fwd<kAModeTma, 0, false>(tw, P, tx, to, smem, grid, st));
    }
    return finish(launch_fwd<kAModePatchThreads, 0, false>(tw, P, tx, to, smem, grid, st));
}

// Shared body of pe_forward_frames_grouped and pe_forward_frames_grouped_pos.
pe_status forward_frames_grouped(pe_handle *h, int n, const void *const *frames, pe_dtype f_dt,
                                 const int32_t *THW, const int32_t *grid_thw, int merge, const void *pos,
                                 int pos_dt, void *out, pe_dtype out_dt, pe_stream_t stream) {
    if (!h) return PE_ERR_INVALID_ARG;
    if (!valid_dtype(out_dt)) return PE_ERR_DTYPE;
    if (!h->weight_set) return PE_ERR_NO_WEIGHT;
    DeviceGuard g(h->dev);
    ProfScope ps(h);
    FwdParams P;
    const pe_status s = setup_frames(h, n, frames, f_dt, THW, grid_thw, merge, out, P, (cudaStream_t)stream);
    if (s != PE_OK) return s;
    P.pos = pos;
    P.pos_f32 = pos_dt == PE_F32;
    return run_frames(h, P, f_dt, out, out_dt, (cudaStream_t)stream);
}

pe_status check_pos(const void *pos, int pos_dt) {
    if (!pos) return PE_ERR_INVALID_ARG;
    if (!valid_dtype(pos_dt)) return PE_ERR_DTYPE;
    if (!aligned16(pos)) return PE_ERR_ALIGN;
    return PE_OK;
}

}  // namespace

extern "C" {

pe_status pe_forward_patches(pe_handle *h, const void *x, pe_dtype x_dt, int64_t N, void *out,
                             pe_dtype out_dt, pe_stream_t stream) {
    NvtxRange nvtx("pe_forward_patches");
    return forward_patches(h, x, x_dt, N, nullptr, PE_BF16, out, out_dt, stream);
}

pe_status pe_forward_patches_pos(pe_handle *h, const void *x, pe_dtype x_dt, int64_t N, const void *pos,
                                 pe_dtype pos_dt, void *out, pe_dtype out_dt, pe_stream_t stream) {
    NvtxRange nvtx("pe_forward_patches_pos");
    if (N > 0) {
        const pe_status s = check_pos(pos, pos_dt);
        if (s != PE_OK) return s;
    }
    return forward_patches(h, x, x_dt, N, pos, pos_dt, out, out_dt, stream);
}

pe_status pe_forward_frames_grouped(pe_handle *h, int n, const void *const *frames, pe_dtype f_dt,
                                    const int32_t *THW, const int32_t *grid_thw, int merge, void *out,
                                    pe_dtype out_dt, pe_stream_t stream) {
    NvtxRange nvtx("pe_forward_frames_grouped");
    return no_throw([&] {
        return forward_frames_grouped(h, n, frames, f_dt, THW, grid_thw, merge, nullptr, PE_BF16, out, out_dt, stream);
    });
}

pe_status pe_forward_frames_grouped_pos(pe_handle *h, int n, const void *const *frames, pe_dtype f_dt,
                                        const int32_t *THW, const int32_t *grid_thw, int merge, const void *pos,
                                        pe_dtype pos_dt, void *out, pe_dtype out_dt, pe_stream_t stream) {
    NvtxRange nvtx("pe_forward_frames_grouped_pos");
    const pe_status s = check_pos(pos, pos_dt);
    if (s != PE_OK) return s;
    return no_throw([&] {
        return forward_frames_grouped(h, n, frames, f_dt, THW, grid_thw, merge, pos, pos_dt, out, out_dt, stream);
    });
}

pe_status pe_forward_frames(pe_handle *h, const void *frames, pe_dtype f_dt, int T, int H, int W,
                            const int32_t grid_thw[3], int merge, void *out, pe_dtype out_dt,
                            pe_stream_t stream) {
    const int32_t thw[3] = {T, H, W};
    const void *fr[1] = {frames};
    return pe_forward_frames_grouped(h, 1, fr, f_dt, thw, grid_thw, merge, out, out_dt, stream);
}

pe_status pe_patchify(pe_handle *h, int n, const void *const *frames, pe_dtype f_dt, const int32_t *THW,
                      const int32_t *grid_thw, int merge, void *rows, pe_dtype rows_dt, pe_stream_t stream) {
    NvtxRange nvtx("pe_patchify");
    if (!h) return PE_ERR_INVALID_ARG;
    if (!valid_dtype(rows_dt)) return PE_ERR_DTYPE;
    DeviceGuard g(h->dev);
    FwdParams P;
    cudaStream_t st = (cudaStream_t)stream;
    const pe_status s = no_throw([&] { return setup_frames(h, n, frames, f_dt, THW, grid_thw, merge, rows, P, st); });
    if (s != PE_OK) return s;
    if (P.N == 0) return PE_OK;
    const int64_t total = P.N * (h->K / 2);
    const int threads = 256;
    const int blocks = (int)std::min<int64_t>((total + threads - 1) / threads, (int64_t)h->num_sms * 16);
    if (f_dt == PE_F32)
        pe_patchify_kernel<true><<<blocks, threads, 0, st>>>(P, rows, rows_dt == PE_F32);
    else
        pe_patchify_kernel<false><<<blocks, threads, 0, st>>>(P, rows, rows_dt == PE_F32);
    return finish(cudaGetLastError());
}

// ---------------------------------------------------------------------------
// pe_forward_frames_grouped_noalloc: the grouped call with its item table in
// this fixed, file-scope device array instead of the handle's workspace.  The
// array lives in every device that loads the library, for the life of the
// process.  Host code must not hand the symbol itself to a kernel (on the host
// it only names a stand-in); its device address comes from
// cudaGetSymbolAddress, looked up once per device with that device current.
static __device__ __align__(256) ItemDesc g_noalloc_items[PE_NOALLOC_MAX_ITEMS];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
ItemDesc *g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_items on the current device (set up on first use).
cudaError_t noalloc_table(int dev, ItemDesc **out) {
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *ptr = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_items);
        if (e != cudaSuccess) return e;
        g_noalloc_ptr[dev] = static_cast<ItemDesc *>(ptr);
    }
    *out = g_noalloc_ptr[dev];
    return cudaSuccess;
}
}  // namespace

pe_status pe_forward_frames_grouped_noalloc(pe_handle *h, int n, const void *const *frames, pe_dtype f_dt,
                                            const int32_t *THW, const int32_t *grid_thw, int merge, void *out,
                                            pe_dtype out_dt, pe_stream_t stream) {
    NvtxRange nvtx("pe_forward_frames_grouped_noalloc");
    if (!h || n < 1 || !frames || !THW || !grid_thw || !out) return PE_ERR_INVALID_ARG;
    if (n > PE_NOALLOC_MAX_ITEMS) return PE_ERR_UNSUPPORTED;
    if (!valid_dtype(f_dt) || !valid_dtype(out_dt)) return PE_ERR_DTYPE;
    if (merge != 1 && merge != 2) return PE_ERR_INVALID_ARG;
    if (!h->weight_set) return PE_ERR_NO_WEIGHT;
    if ((h->p & 1) || h->p > PE_MAX_PATCH) return PE_ERR_UNSUPPORTED;
    if (!aligned16(out)) return PE_ERR_ALIGN;
    DeviceGuard g(h->dev);
    ProfScope ps(h);
    cudaStream_t st = (cudaStream_t)stream;
    FwdParams P;
    fill_common(h, P);
    P.merge = merge;
    P.n_items = n;
    // Validate every item before anything is copied or launched.
    int64_t row0 = 0;
    P.all_t1 = 1;
    for (int i = 0; i < n; ++i) {
        P.all_t1 = P.all_t1 && THW[3 * i] == 1;
        ItemDesc d;
        const pe_status s = make_item(h, frames[i], THW[3 * i], THW[3 * i + 1], THW[3 * i + 2], grid_thw + 3 * i,
                                      merge, row0, d);
        if (s != PE_OK) return s;
        if (n <= PE_INLINE_ITEMS) P.items[i] = d;
        row0 += (int64_t)grid_thw[3 * i] * grid_thw[3 * i + 1] * grid_thw[3 * i + 2];
    }
    P.N = row0;
    if (n > PE_INLINE_ITEMS) {
        ItemDesc *table = nullptr;
        if (noalloc_table(h->dev, &table) != cudaSuccess) return PE_ERR_CUDA;
        // Upload in groups of kItemsPerFill descriptors, each passed by value in
        // the parameter block of a one-block kernel: stream-ordered, no host
        // staging buffer, and the host never waits.
        ItemBatch batch;
        int64_t r0 = 0;
        for (int base = 0; base < n; base += kItemsPerFill) {
            const int m = std::min(kItemsPerFill, n - base);
            std::memset(&batch, 0, sizeof(batch));
            for (int j = 0; j < m; ++j) {
                const int i = base + j;
                make_item(h, frames[i], THW[3 * i], THW[3 * i + 1], THW[3 * i + 2], grid_thw + 3 * i, merge, r0,
                          batch.d[j]);
                r0 += (int64_t)grid_thw[3 * i] * grid_thw[3 * i + 1] * grid_thw[3 * i + 2];
            }
            pe_fill_items_kernel<<<1, kItemsPerFill, 0, st>>>(batch, table + base, m);
            if (h->prof_on) ++h->prof_launches;
            if (cudaGetLastError() != cudaSuccess) return PE_ERR_CUDA;
        }
        P.items_dev = table;
    }
    return run_frames(h, P, f_dt, out, out_dt, st, /*allow_staged=*/false);   // never allocates
}

pe_status pe_profile_begin(pe_handle *h, int max_calls) {
    if (!h || max_calls < 0 || max_calls > 1000000) return PE_ERR_INVALID_ARG;
    DeviceGuard g(h->dev);
    for (cudaEvent_t e : h->prof_ev) cudaEventDestroy(e);
    h->prof_ev.clear();
    h->prof_cap = h->prof_n = 0;
    h->prof_on = false;
    try {
        h->prof_ev.assign((size_t)2 * max_calls, nullptr);
    } catch (const std::bad_alloc &) {
        return PE_ERR_HOST_MEMORY;
    }
    for (auto &e : h->prof_ev)
        if (cudaEventCreate(&e) != cudaSuccess) return PE_ERR_CUDA;
    h->prof_cap = max_calls;
    h->prof_n = 0;
    h->prof_launches = 0;
    h->prof_on = true;
    return PE_OK;
}

pe_status pe_profile_target(pe_handle *h, int target) {
    if (!h || (target != 0 && target != 1)) return PE_ERR_INVALID_ARG;
    h->prof_target = target;
    return PE_OK;
}

pe_status pe_profile_end(pe_handle *h, float *ms, int *n, int64_t *launches) {
    if (!h || !n || (*n > 0 && !ms)) return PE_ERR_INVALID_ARG;
    if (launches) *launches = h->prof_launches;
    DeviceGuard g(h->dev);
    const int cnt = std::min(h->prof_n, *n);
    pe_status st = PE_OK;
    for (int i = 0; i < cnt; ++i) {
        if (cudaEventSynchronize(h->prof_ev[2 * i + 1]) != cudaSuccess ||
            cudaEventElapsedTime(&ms[i], h->prof_ev[2 * i], h->prof_ev[2 * i + 1]) != cudaSuccess)
            st = PE_ERR_CUDA;
    }
    *n = cnt;
    for (cudaEvent_t e : h->prof_ev) cudaEventDestroy(e);
    h->prof_ev.clear();
    h->prof_cap = h->prof_n = 0;
    h->prof_on = false;
    return st;
}

pe_status pe_selftest_wait_timeout(pe_handle *h, pe_stream_t stream) {
    if (!h) return PE_ERR_INVALID_ARG;
    DeviceGuard g(h->dev);
    pe_wait_timeout_probe_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(h->err);
    return finish(cudaGetLastError());
}

pe_status pe_last_error(pe_handle *h) {
    if (!h) return PE_ERR_INVALID_ARG;
    DeviceGuard g(h->dev);
    int v = 0;
    if (cudaMemcpy(&v, h->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return PE_ERR_CUDA;
    if (v != 0 && cudaMemset(h->err, 0, sizeof(int)) != cudaSuccess) return PE_ERR_CUDA;
    return v == 0 ? PE_OK : (pe_status)v;
}

// ---------------------------------------------------------------------------
// Host-buffer calls: the call's inputs and outputs live in host memory.  The
// work is cut into chunks (pe_host_plan.h); chunk c uses input and output slot
// c % 2 of the handle's device buffer.  Its inputs are copied in on the
// handle's copy-in stream, its rows computed on the caller's stream by the
// device-pointer path, and copied out on the handle's copy-out stream, so
// that (with pinned host memory) the copies in both directions and the
// contraction of neighbouring chunks overlap.  Events order the slots:
//   copy-in of c  waits for the contraction of c - 2 (input slot free),
//   contraction of c  waits for copy-in of c and copy-out of c - 2,
//   copy-out of c  waits for the contraction of c.
// The caller's stream waits for the last copy-out before the call returns.
}  // extern "C"

namespace {

pe_status host_pipe_init(pe_handle *h) {
    bool ok = true;
    for (cudaStream_t *s : {&h->s_in, &h->s_out})
        if (ok && !*s) ok = cudaStreamCreateWithFlags(s, cudaStreamNonBlocking) == cudaSuccess;
    for (cudaEvent_t *e : {&h->ev_start, &h->ev_in[0], &h->ev_in[1], &h->ev_comp[0], &h->ev_comp[1], &h->ev_out[0],
                           &h->ev_out[1]})
        if (ok && !*e) ok = cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
    return ok ? PE_OK : PE_ERR_CUDA;   // objects already created are kept and released by pe_destroy
}

// Grow-only slots; the old buffer is freed only after every stream that may
// still use it has drained.
pe_status host_slots(pe_handle *h, int64_t in_bytes, int64_t out_bytes, cudaStream_t st) {
    const size_t in = (size_t)pe_plan::align_up(std::max<int64_t>(in_bytes, 1), pe_plan::kSlotAlign);
    const size_t out = (size_t)pe_plan::align_up(std::max<int64_t>(out_bytes, 1), pe_plan::kSlotAlign);
    if (in <= h->host_ws_in && out <= h->host_ws_out) return PE_OK;
    const size_t new_in = std::max(in, h->host_ws_in), new_out = std::max(out, h->host_ws_out);
    if (h->host_ws) {
        if (cudaStreamSynchronize(st) != cudaSuccess || cudaStreamSynchronize(h->s_in) != cudaSuccess ||
            cudaStreamSynchronize(h->s_out) != cudaSuccess)
            return PE_ERR_CUDA;
        cudaFree(h->host_ws);
    }
    h->host_ws = nullptr;
    h->host_ws_in = h->host_ws_out = 0;
    if (cudaMalloc(&h->host_ws, 2 * (new_in + new_out)) != cudaSuccess) return PE_ERR_CUDA;
    h->host_ws_in = new_in;
    h->host_ws_out = new_out;
    return PE_OK;
}

uint8_t *slot_in(const pe_handle *h, int s) { return h->host_ws + (size_t)s * h->host_ws_in; }
uint8_t *slot_out(const pe_handle *h, int s) { return h->host_ws + 2 * h->host_ws_in + (size_t)s * h->host_ws_out; }

// Chunk rows: PE_HOST_CHUNK_ROWS overrides the planner's choice (tests use it
// to force many small chunks).
int64_t host_chunk_rows(int64_t N) {
    if (const char *s = std::getenv("PE_HOST_CHUNK_ROWS")) {
        const long long v = std::atoll(s);
        if (v > 0) return (int64_t)v;
    }
    return pe_plan::chunk_rows(N);
}

// pe_plan::run_pipeline's stream/event interface on CUDA: the caller's
// stream and the handle's copy streams and events.
template <class CopyIn, class Compute, class CopyOut>
struct CudaPipeOps {
    pe_handle *h;
    cudaStream_t st;
    CopyIn &copy_in_fn;
    Compute &compute_fn;
    CopyOut &copy_out_fn;
    cudaStream_t stream(int id) const {
        return id == pe_plan::kCaller ? st : (id == pe_plan::kCopyIn ? h->s_in : h->s_out);
    }
    cudaEvent_t event(int id) const {
        if (id == pe_plan::kEvStart) return h->ev_start;
        if (id < pe_plan::kEvComp0) return h->ev_in[id - pe_plan::kEvIn0];
        if (id < pe_plan::kEvOut0) return h->ev_comp[id - pe_plan::kEvComp0];
        return h->ev_out[id - pe_plan::kEvOut0];
    }
    bool record(int e, int s) { return cudaEventRecord(event(e), stream(s)) == cudaSuccess; }
    bool wait(int s, int e) { return cudaStreamWaitEvent(stream(s), event(e), 0) == cudaSuccess; }
    int copy_in(int c, int s) { return (int)copy_in_fn(c, slot_in(h, s), h->s_in); }
    int compute(int c, int s) { return (int)compute_fn(c, slot_in(h, s), slot_out(h, s), st); }
    int copy_out(int c, int s) { return (int)copy_out_fn(c, slot_out(h, s), h->s_out); }
};

template <class CopyIn, class Compute, class CopyOut>
pe_status run_host_pipeline(pe_handle *h, int nchunks, cudaStream_t st, CopyIn copy_in, Compute compute,
                            CopyOut copy_out) {
    CudaPipeOps<CopyIn, Compute, CopyOut> ops{h, st, copy_in, compute, copy_out};
    const int r = pe_plan::run_pipeline(ops, nchunks);
    return r == 0 ? PE_OK : (r < 0 ? PE_ERR_CUDA : (pe_status)r);
}

alignas(16) const unsigned char kStandIn[16] = {};   // validation stand-in for a frames pointer

}  // namespace

extern "C" {

// Body of pe_forward_frames_grouped_host (internal linkage; the exported
// call runs it under no_throw).
static pe_status frames_grouped_host_body(pe_handle *h, int n, const void *const *frames_host, pe_dtype f_dt,
                                          const int32_t *THW, const int32_t *grid_thw, int merge, void *out_host,
                                          pe_dtype out_dt, pe_stream_t stream) {
    if (!h || n < 1 || !frames_host || !THW || !grid_thw || !out_host) return PE_ERR_INVALID_ARG;
    if (!valid_dtype(f_dt) || !valid_dtype(out_dt)) return PE_ERR_DTYPE;
    if (merge != 1 && merge != 2) return PE_ERR_INVALID_ARG;
    if (!h->weight_set) return PE_ERR_NO_WEIGHT;
    if ((h->p & 1) || h->p > PE_MAX_PATCH) return PE_ERR_UNSUPPORTED;
    // Every item is validated as the device-pointer call validates it, before
    // anything is allocated, copied or launched.
    const int64_t es = f_dt == PE_F32 ? 4 : 2;
    std::vector<int64_t> frame_bytes((size_t)n);
    int64_t N = 0;
    for (int i = 0; i < n; ++i) {
        if (!frames_host[i]) return PE_ERR_INVALID_ARG;
        ItemDesc d;
        const pe_status s = make_item(h, kStandIn, THW[3 * i], THW[3 * i + 1], THW[3 * i + 2], grid_thw + 3 * i, merge,
                                      N, d);
        if (s != PE_OK) return s;
        frame_bytes[(size_t)i] = (int64_t)h->C * THW[3 * i + 1] * THW[3 * i + 2] * es;
        N += (int64_t)grid_thw[3 * i] * grid_thw[3 * i + 1] * grid_thw[3 * i + 2];
    }
    DeviceGuard g(h->dev);
    cudaStream_t st = (cudaStream_t)stream;
    const pe_plan::Plan pl = pe_plan::plan_frames(n, THW, grid_thw, h->tp, frame_bytes.data(), host_chunk_rows(N));
    const int64_t row_bytes = (int64_t)h->E * (out_dt == PE_F32 ? 4 : 2);
    pe_status r = host_pipe_init(h);
    if (r == PE_OK) r = host_slots(h, pl.max_in, pl.max_rows * row_bytes, st);
    if (r != PE_OK) return r;
    std::vector<const void *> ptrs;
    std::vector<int32_t> thw, grid;
    auto copy_in = [&](int c, uint8_t *slot, cudaStream_t s) -> pe_status {
        const pe_plan::Chunk &ch = pl.chunks[(size_t)c];
        for (int j = ch.first; j < ch.first + ch.count; ++j) {
            const pe_plan::SubItem &sb = pl.subs[(size_t)j];
            const char *src = static_cast<const char *>(frames_host[sb.item]) + (int64_t)sb.f0 * frame_bytes[(size_t)sb.item];
            if (cudaMemcpyAsync(slot + sb.in_off, src, (size_t)sb.in_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
                return PE_ERR_CUDA;
        }
        return PE_OK;
    };
    auto compute = [&](int c, uint8_t *in, uint8_t *out, cudaStream_t s) -> pe_status {
        const pe_plan::Chunk &ch = pl.chunks[(size_t)c];
        ptrs.clear();
        thw.clear();
        grid.clear();
        for (int j = ch.first; j < ch.first + ch.count; ++j) {
            const pe_plan::SubItem &sb = pl.subs[(size_t)j];
            const int32_t *it = THW + 3 * sb.item, *gr = grid_thw + 3 * sb.item;
            ptrs.push_back(in + sb.in_off);
            thw.insert(thw.end(), {sb.T, it[1], it[2]});
            grid.insert(grid.end(), {sb.gt, gr[1], gr[2]});
        }
        return forward_frames_grouped(h, ch.count, ptrs.data(), f_dt, thw.data(), grid.data(), merge, nullptr, PE_BF16,
                                      out, out_dt, s);
    };
    auto copy_out = [&](int c, uint8_t *slot, cudaStream_t s) -> pe_status {
        const pe_plan::Chunk &ch = pl.chunks[(size_t)c];
        return cudaMemcpyAsync(static_cast<char *>(out_host) + ch.row0 * row_bytes, slot, (size_t)(ch.rows * row_bytes),
                               cudaMemcpyDeviceToHost, s) == cudaSuccess
                   ? PE_OK
                   : PE_ERR_CUDA;
    };
    return run_host_pipeline(h, (int)pl.chunks.size(), st, copy_in, compute, copy_out);
}

pe_status pe_forward_frames_grouped_host(pe_handle *h, int n, const void *const *frames_host, pe_dtype f_dt,
                                         const int32_t *THW, const int32_t *grid_thw, int merge, void *out_host,
                                         pe_dtype out_dt, pe_stream_t stream) {
    NvtxRange nvtx("pe_forward_frames_grouped_host");
    return no_throw([&] {
        return frames_grouped_host_body(h, n, frames_host, f_dt, THW, grid_thw, merge, out_host, out_dt, stream);
    });
}

pe_status pe_forward_patches_host(pe_handle *h, const void *x_host, pe_dtype x_dt, int64_t N, void *out_host,
                                  pe_dtype out_dt, pe_stream_t stream) {
    NvtxRange nvtx("pe_forward_patches_host");
    if (!h || N < 0) return PE_ERR_INVALID_ARG;
    if (!valid_dtype(x_dt) || !valid_dtype(out_dt)) return PE_ERR_DTYPE;
    if (!h->weight_set) return PE_ERR_NO_WEIGHT;
    if (N == 0) return PE_OK;
    if (!x_host || !out_host) return PE_ERR_INVALID_ARG;
    DeviceGuard g(h->dev);
    cudaStream_t st = (cudaStream_t)stream;
    const int64_t per = std::min(host_chunk_rows(N), N);
    const int64_t nch = (N + per - 1) / per;
    if (nch > INT32_MAX) return PE_ERR_UNSUPPORTED;
    const int64_t in_row = (int64_t)h->K * (x_dt == PE_F32 ? 4 : 2);
    const int64_t out_row = (int64_t)h->E * (out_dt == PE_F32 ? 4 : 2);
    pe_status r = host_pipe_init(h);
    if (r == PE_OK) r = host_slots(h, per * in_row, per * out_row, st);
    if (r != PE_OK) return r;
    auto rows_of = [&](int c) { return std::min(per, N - (int64_t)c * per); };
    auto copy_in = [&](int c, uint8_t *slot, cudaStream_t s) -> pe_status {
        const char *src = static_cast<const char *>(x_host) + (int64_t)c * per * in_row;
        return cudaMemcpyAsync(slot, src, (size_t)(rows_of(c) * in_row), cudaMemcpyHostToDevice, s) == cudaSuccess
                   ? PE_OK
                   : PE_ERR_CUDA;
    };
    auto compute = [&](int c, uint8_t *in, uint8_t *out, cudaStream_t s) -> pe_status {
        return forward_patches(h, in, x_dt, rows_of(c), nullptr, PE_BF16, out, out_dt, s);
    };
    auto copy_out = [&](int c, uint8_t *slot, cudaStream_t s) -> pe_status {
        char *dst = static_cast<char *>(out_host) + (int64_t)c * per * out_row;
        return cudaMemcpyAsync(dst, slot, (size_t)(rows_of(c) * out_row), cudaMemcpyDeviceToHost, s) == cudaSuccess
                   ? PE_OK
                   : PE_ERR_CUDA;
    };
    return run_host_pipeline(h, (int)nch, st, copy_in, compute, copy_out);
}

// ---------------------------------------------------------------------------
// PatchMerger: LayerNorm, the m*m neighbouring rows of a merge window
// concatenated (they are adjacent in merge order, so [N, E] is [V, m*m*E]
// without a copy), then fc1 + exact GELU and fc2 on the TMA-fed pair GEMM.
}  // extern "C"

struct pe_merger {
    pe_handle core;              // device properties for the shared planners (owns nothing)
    int E = 0, m2 = 0, H = 0, D = 0;
    float eps = 1e-6f;
    bool weights_set = false;
    uint16_t *w1 = nullptr;      // [D, D] bf16
    uint16_t *w2 = nullptr;      // [H, D] bf16
    float *b1 = nullptr, *b2 = nullptr, *gamma = nullptr, *beta = nullptr;
    bool has_b1 = false, has_b2 = false;
    int *err = nullptr;
    CUtensorMap tmap_w1[3], tmap_w2[3];
    uint16_t *ln_rows = nullptr;  // [N, E] bf16 workspace
    size_t ln_bytes = 0;
    uint16_t *hid = nullptr;      // [V, D] bf16 workspace
    size_t hid_bytes = 0;
};

namespace {

bool grow(uint16_t **buf, size_t *cap, size_t need, cudaStream_t st) {
    if (need <= *cap) return true;
    if (*buf) {
        if (cudaStreamSynchronize(st) != cudaSuccess) return false;
        cudaFree(*buf);
    }
    *buf = nullptr;
    *cap = 0;
    if (cudaMalloc(buf, need) != cudaSuccess) return false;
    *cap = need;
    return true;
}

// One linear layer of the merger on the pair GEMM: out[V, nout] = act(A[V, D] W^T + b).
pe_status merger_linear(pe_merger *pm, const uint16_t *A, int64_t V, const CUtensorMap *tw3, int nout,
                        const float *bias, int act, void *out, int out_dt, cudaStream_t st) {
    FwdParams G;
    std::memset(&G, 0, sizeof(G));
    G.E = nout;
    G.K = pm->D;
    G.Kpad = pm->D;
    G.C = 1;
    G.TP = 1;
    G.P = 1;
    G.N = V;
    G.x = A;
    G.x_vec = 1;
    G.bias = bias;
    G.act = act;
    G.out_f32 = out_dt == PE_F32;
    G.err = pm->err;
    int grid = 0;
    bool ok = true;
    plan_tiles(&pm->core, G, V, grid, ok);
    if (!ok) return PE_ERR_UNSUPPORTED;
    const size_t smem = plan_pipeline(&pm->core, G, kAModeTma, pm->D);
    CUtensorMap tx, to;
    if (!make_tmap_bf16(&tx, A, (uint64_t)V, (uint64_t)pm->D, (uint64_t)pm->D, kBM)) return PE_ERR_CUDA;
    if (!make_out_tmap(&to, out, G.out_f32, V, nout)) return PE_ERR_CUDA;
    return finish(launch_fwd<kAModeTma, 0, false>(tw3[bn_index(G.bn)], G, tx, to, smem, grid, st, true));
}

}  // namespace

extern "C" {

pe_status pe_merger_create(int E, int m, int H, float eps, pe_merger **out) {
    if (!out) return PE_ERR_INVALID_ARG;
    *out = nullptr;
    if (E < 8 || (E % 8) != 0 || m < 1 || m > 4 || H < 16 || (H % 8) != 0 || !(eps > 0.f)) return PE_ERR_INVALID_ARG;
    const int64_t D = (int64_t)E * m * m;
    if ((D % 64) != 0 || D > 65536) return PE_ERR_UNSUPPORTED;
    pe_merger *pm = new (std::nothrow) pe_merger();
    if (!pm) return PE_ERR_CUDA;
    if (cudaGetDevice(&pm->core.dev) != cudaSuccess) { delete pm; return PE_ERR_CUDA; }
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, pm->core.dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, pm->core.dev);
    if (major != 10 || minor != 0) { delete pm; return PE_ERR_UNSUPPORTED; }
    cudaDeviceGetAttribute(&pm->core.num_sms, cudaDevAttrMultiProcessorCount, pm->core.dev);
    cudaDeviceGetAttribute(&pm->core.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, pm->core.dev);
    pm->E = E;
    pm->m2 = m * m;
    pm->H = H;
    pm->D = (int)D;
    pm->eps = eps;
    bool ok = cudaMalloc(&pm->w1, sizeof(uint16_t) * (size_t)(D * D)) == cudaSuccess &&
              cudaMalloc(&pm->w2, sizeof(uint16_t) * (size_t)H * D) == cudaSuccess &&
              cudaMalloc(&pm->b1, sizeof(float) * (size_t)D) == cudaSuccess &&
              cudaMalloc(&pm->b2, sizeof(float) * (size_t)H) == cudaSuccess &&
              cudaMalloc(&pm->gamma, sizeof(float) * (size_t)E) == cudaSuccess &&
              cudaMalloc(&pm->beta, sizeof(float) * (size_t)E) == cudaSuccess &&
              cudaMalloc(&pm->err, sizeof(int)) == cudaSuccess && cudaMemset(pm->err, 0, sizeof(int)) == cudaSuccess;
    const uint32_t boxes[3] = {32, 64, 128};
    for (int i = 0; i < 3 && ok; ++i)
        ok = make_tmap_bf16(&pm->tmap_w1[i], pm->w1, (uint64_t)D, (uint64_t)D, (uint64_t)D, boxes[i]) &&
             make_tmap_bf16(&pm->tmap_w2[i], pm->w2, (uint64_t)H, (uint64_t)D, (uint64_t)D, boxes[i]);
    if (!ok) { pe_merger_destroy(pm); return PE_ERR_CUDA; }
    *out = pm;
    return PE_OK;
}

void pe_merger_destroy(pe_merger *pm) {
    if (!pm) return;
    DeviceGuard g(pm->core.dev);
    cudaDeviceSynchronize();
    for (void *p : {(void *)pm->w1, (void *)pm->w2, (void *)pm->b1, (void *)pm->b2, (void *)pm->gamma,
                    (void *)pm->beta, (void *)pm->err, (void *)pm->ln_rows, (void *)pm->hid})
        if (p) cudaFree(p);
    for (cudaEvent_t e : pm->core.prof_ev) cudaEventDestroy(e);   // profiling window left open
    delete pm;
}

pe_status pe_merger_set_weights(pe_merger *pm, const void *gamma, const void *beta, const void *w1, const void *b1,
                                const void *w2, const void *b2, pe_dtype dt, pe_stream_t stream) {
    if (!pm || !gamma || !beta || !w1 || !w2) return PE_ERR_INVALID_ARG;
    if (!valid_dtype(dt)) return PE_ERR_DTYPE;
    for (const void *p : {gamma, beta, w1, w2, b1, b2})
        if (p && !aligned16(p)) return PE_ERR_ALIGN;
    DeviceGuard g(pm->core.dev);
    cudaStream_t st = (cudaStream_t)stream;
    const int64_t D = pm->D, H = pm->H;
    auto to_bf16 = [&](const void *src, uint16_t *dst, int64_t n) -> bool {
        if (dt == PE_BF16) return cudaMemcpyAsync(dst, src, sizeof(uint16_t) * n, cudaMemcpyDeviceToDevice, st) == cudaSuccess;
        const int64_t n8 = n / 8;   // D % 64 == 0: whole 8-element groups
        const int cb = (int)std::min<int64_t>((n8 + 255) / 256, (int64_t)pm->core.num_sms * 8);
        pe_cast_rows_kernel<<<cb, 256, 0, st>>>(reinterpret_cast<const float *>(src), dst, n8);
        return cudaGetLastError() == cudaSuccess;
    };
    auto to_f32 = [&](const void *src, float *dst, int64_t n) -> bool {
        const int cb = (int)std::min<int64_t>((n + 255) / 256, 1024);
        pe_to_f32_kernel<<<cb, 256, 0, st>>>(src, dt == PE_F32, dst, n);
        return cudaGetLastError() == cudaSuccess;
    };
    if (!to_bf16(w1, pm->w1, D * D) || !to_bf16(w2, pm->w2, H * D) || !to_f32(gamma, pm->gamma, pm->E) ||
        !to_f32(beta, pm->beta, pm->E))
        return PE_ERR_CUDA;
    pm->has_b1 = b1 != nullptr;
    pm->has_b2 = b2 != nullptr;
    if ((b1 && !to_f32(b1, pm->b1, D)) || (b2 && !to_f32(b2, pm->b2, H))) return PE_ERR_CUDA;
    pm->weights_set = true;
    return PE_OK;
}

pe_status pe_merger_forward(pe_merger *pm, const void *x, int64_t N, void *out, pe_dtype out_dt, pe_stream_t stream) {
    NvtxRange nvtx("pe_merger_forward");
    if (!pm || N < 0) return PE_ERR_INVALID_ARG;
    if (!valid_dtype(out_dt)) return PE_ERR_DTYPE;
    if (!pm->weights_set) return PE_ERR_NO_WEIGHT;
    if (N % pm->m2 != 0) return PE_ERR_SHAPE;
    if (N == 0) return PE_OK;
    if (!x || !out) return PE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(out)) return PE_ERR_ALIGN;
    DeviceGuard g(pm->core.dev);
    ProfScope ps(&pm->core);
    cudaStream_t st = (cudaStream_t)stream;
    const int64_t V = N / pm->m2;
    if (!grow(&pm->ln_rows, &pm->ln_bytes, sizeof(uint16_t) * (size_t)N * pm->E, st) ||
        !grow(&pm->hid, &pm->hid_bytes, sizeof(uint16_t) * (size_t)V * pm->D, st))
        return PE_ERR_CUDA;
    const int64_t blocks = (N + 7) / 8;
    pe_layernorm_kernel<<<(unsigned)blocks, 256, 0, st>>>(reinterpret_cast<const uint16_t *>(x), N, pm->E, pm->gamma,
                                                         pm->beta, pm->eps, pm->ln_rows);
    if (pm->core.prof_on) ++pm->core.prof_launches;
    if (cudaGetLastError() != cudaSuccess) return PE_ERR_CUDA;
    pe_status s = merger_linear(pm, pm->ln_rows, V, pm->tmap_w1, pm->D, pm->has_b1 ? pm->b1 : nullptr, 1, pm->hid,
                                PE_BF16, st);
    if (s != PE_OK) return s;
    return merger_linear(pm, pm->hid, V, pm->tmap_w2, pm->H, pm->has_b2 ? pm->b2 : nullptr, 0, out, out_dt, st);
}

pe_status pe_merger_profile_begin(pe_merger *pm, int max_calls) {
    if (!pm) return PE_ERR_INVALID_ARG;
    return pe_profile_begin(&pm->core, max_calls);
}

pe_status pe_merger_profile_end(pe_merger *pm, float *ms, int *n, int64_t *launches) {
    if (!pm) return PE_ERR_INVALID_ARG;
    return pe_profile_end(&pm->core, ms, n, launches);
}

pe_status pe_merger_last_error(pe_merger *pm) {
    if (!pm) return PE_ERR_INVALID_ARG;
    DeviceGuard g(pm->core.dev);
    int v = 0;
    if (cudaMemcpy(&v, pm->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return PE_ERR_CUDA;
    if (v != 0 && cudaMemset(pm->err, 0, sizeof(int)) != cudaSuccess) return PE_ERR_CUDA;
    return v == 0 ? PE_OK : (pe_status)v;
}

}  // extern "C"
