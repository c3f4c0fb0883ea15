/*
 * CPU oracle for the Qwen2-VL / Qwen2.5-VL vision PatchEmbed.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is built into its own shared library and
 * is called only by the test suite, by the package's smoke check and by the
 * benchmark's CPU-baseline leg.  It shares no code, header or table with the
 * CUDA library, and the CUDA library never calls it.
 *
 * What it computes (plain, slow, obviously correct; fp64 accumulation):
 *
 *   PatchEmbed is a Conv3d with in_channels C, out_channels E, kernel size
 *   (tp, p, p) equal to its stride and no padding (Qwen2.5VL-Vision
 *   Encode-PatchEmbed, the Conv3d description and python验证; Optimize VLM
 *   PatchEmbed, Qwen3VLVisionPatchEmbed; patch详解 §4.3).  Each output voxel is
 *   the dot product of one (C, tp, p, p) block with one filter.
 *
 *   - patches form: the input rows are blocks already flattened in
 *     view(-1, C, tp, p, p) order, i.e. element k(c,t,i,j) = ((c*tp+t)*p+i)*p+j
 *     (Optimize VLM PatchEmbed, Qwen3VLVisionPatchEmbed.forward).
 *   - frames form: a direct Conv3d over the video volume [T, C, H, W]; the time
 *     axis is padded by repeating the last frame until it holds tp*grid_t
 *     frames (patch详解 §4.5 counts ceil(T/tp) temporal patches; a single image
 *     is thereby duplicated to tp frames), each pixel is normalised
 *     per channel in fp32 as (x - mean_c) / std_c and rounded to bf16, and the
 *     output row of grid cell (g_t, g_h, g_w) follows the spatial-merge order
 *     (mytransformer README §3.2/§4.1: 2x2 neighbours consecutive for the
 *     PatchMerger; Qwen2.5VL语言模型 MRoPE: merged grid row-major, h outer).
 *
 *   Compute precision: the GPU multiplies bf16 operands, so both the input
 *   values and the weights are rounded to bf16 (round to nearest even) before
 *   the fp64 multiply-accumulate; the bias is added in fp64 as given.
 *
 *   Readings taken where the pages are silent (each is listed in the design
 *   notes): row order inside a 2x2 window is (dh, dw) row-major; temporal
 *   padding repeats the last frame; normalisation is an IEEE fp32 subtract then
 *   an IEEE fp32 divide, then bf16 round-to-nearest-even.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fno-fast-math -shared -fPIC
 * (no contraction into FMA, so the fp32 normalisation is exactly two roundings).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* bf16 round-to-nearest-even of an fp32 value, returned widened to fp32.
 * Definition: keep the top 16 bits of the IEEE single after adding half an ulp
 * of bf16 (0x7fff plus the parity of the kept lsb, which gives ties-to-even).
 * NaN stays NaN (quiet bit forced); infinities stay infinite. */
float oracle_bf16_round(float v)
{
    uint32_t u;
    memcpy(&u, &v, 4);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0u) {
        u = (u | 0x00400000u) & 0xffff0000u;
    } else {
        u = (u + 0x7fffu + ((u >> 16) & 1u)) & 0xffff0000u;
    }
    float r;
    memcpy(&r, &u, 4);
    return r;
}

void oracle_bf16_round_array(const float *in, float *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_bf16_round(in[i]);
}

/* The fp32 normalisation of one pixel followed by the bf16 rounding. */
float oracle_normalize_pixel(float x, float mean, float std)
{
    volatile float d = x - mean;   /* one IEEE fp32 rounding */
    volatile float q = d / std;    /* one IEEE fp32 rounding */
    return oracle_bf16_round(q);
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Output row of grid cell (g_t, g_h, g_w) in an item with grid (t, h, w).
 * merge == 1: raster order (t, h, w).
 * merge == m > 1: windows of m x m patches are consecutive, windows ordered
 * row-major over (t, h/m, w/m), inside a window (dh, dw) row-major. */
int64_t oracle_row_index(int64_t g_t, int64_t g_h, int64_t g_w,
                         int64_t h, int64_t w, int merge)
{
    if (merge <= 1)
        return (g_t * h + g_h) * w + g_w;
    const int64_t m = merge;
    const int64_t window = (g_t * (h / m) + g_h / m) * (w / m) + g_w / m;
    return window * m * m + (g_h % m) * m + (g_w % m);
}

/*
 * Patches form: out[n, e] = bias[e] + sum_{c,t,i,j} xb[n, k(c,t,i,j)] * wb[e, c, t, i, j]
 *   x     : [N, K] fp32 host array, K = C*tp*p*p, rows in view(-1,C,tp,p,p) order
 *   w     : [E, C, tp, p, p] fp32
 *   bias  : [E] fp32 or NULL
 *   out   : [N, E] fp64;  absdot (optional): [N, E] fp64 = sum_k |xb_k * wb_k|
 *   row_mask (optional): [N] bytes; rows with 0 are skipped (left untouched).
 */
void oracle_conv3d_patches(const float *x, int64_t N, const float *w, const float *bias,
                           int E, int C, int tp, int p, const uint8_t *row_mask,
                           double *out, double *absdot)
{
    const int64_t K = (int64_t)C * tp * p * p;
    float *wb = (float *)malloc(sizeof(float) * (size_t)(E * K));
    oracle_bf16_round_array(w, wb, (int64_t)E * K);

#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t n = 0; n < N; ++n) {
        if (row_mask && !row_mask[n])
            continue;
        for (int e = 0; e < E; ++e) {
            double acc = 0.0, mag = 0.0;
            for (int c = 0; c < C; ++c)
                for (int t = 0; t < tp; ++t)
                    for (int i = 0; i < p; ++i)
                        for (int j = 0; j < p; ++j) {
                            const int64_t k = (((int64_t)c * tp + t) * p + i) * p + j;
                            const double xv = (double)oracle_bf16_round(x[n * K + k]);
                            const double wv = (double)wb[(int64_t)e * K + k];
                            acc += xv * wv;
                            mag += fabs(xv * wv);
                        }
            out[n * E + e] = acc + (bias ? (double)bias[e] : 0.0);
            if (absdot)
                absdot[n * E + e] = mag;
        }
    }
    free(wb);
}

/* Patches form on the fp32 values exactly as given (no bf16 rounding of x or
 * w): the Conv3d definition in fp64, the reference for contractions that keep
 * more than bf16 precision of fp32 inputs.  Same layout and outputs as
 * oracle_conv3d_patches. */
void oracle_conv3d_patches_fp32(const float *x, int64_t N, const float *w, const float *bias,
                                int E, int C, int tp, int p, const uint8_t *row_mask,
                                double *out, double *absdot)
{
    const int64_t K = (int64_t)C * tp * p * p;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t n = 0; n < N; ++n) {
        if (row_mask && !row_mask[n])
            continue;
        for (int e = 0; e < E; ++e) {
            double acc = 0.0, mag = 0.0;
            for (int c = 0; c < C; ++c)
                for (int t = 0; t < tp; ++t)
                    for (int i = 0; i < p; ++i)
                        for (int j = 0; j < p; ++j) {
                            const int64_t k = (((int64_t)c * tp + t) * p + i) * p + j;
                            const double xv = (double)x[n * K + k];
                            const double wv = (double)w[(int64_t)e * K + k];
                            acc += xv * wv;
                            mag += fabs(xv * wv);
                        }
            out[n * E + e] = acc + (bias ? (double)bias[e] : 0.0);
            if (absdot)
                absdot[n * E + e] = mag;
        }
    }
}

/* The normalised, time-padded volume Fh[tau, c, y, x] for tau < tp*gt:
 * Fp[tau] = F[min(tau, T-1)], Fh = bf16(fp32(fp32(Fp - mean_c) / std_c)). */
static float *normalized_volume(const float *frames, int T, int C, int H, int W,
                                int tpad, const float *mean, const float *std)
{
    const int64_t plane = (int64_t)H * W;
    float *vol = (float *)malloc(sizeof(float) * (size_t)((int64_t)tpad * C * plane));
#pragma omp parallel for schedule(static)
    for (int64_t tc = 0; tc < (int64_t)tpad * C; ++tc) {
        const int tau = (int)(tc / C), c = (int)(tc % C);
        const int src = tau < T ? tau : T - 1;
        const float *s = frames + ((int64_t)src * C + c) * plane;
        float *d = vol + tc * plane;
        for (int64_t q = 0; q < plane; ++q)
            d[q] = oracle_normalize_pixel(s[q], mean[c], std[c]);
    }
    return vol;
}

/*
 * Frames form: direct Conv3d with kernel = stride = (tp, p, p) over the
 * normalised, time-padded volume, rows placed by oracle_row_index.
 *   frames: [T, C, H, W] fp32 host (bf16 inputs are passed widened, exactly)
 *   grid  : (gt, gh, gw); requires H == gh*p, W == gw*p, ceil(T/tp) == gt
 *   out   : [gt*gh*gw, E] fp64; absdot optional; row_mask optional (by output row)
 * Returns 0 on success, -1 on inconsistent sizes.
 */
int oracle_conv3d_frames(const float *frames, int T, int H, int W,
                         int gt, int gh, int gw, int merge,
                         const float *mean, const float *std,
                         const float *w, const float *bias, int E, int C, int tp, int p,
                         const uint8_t *row_mask, double *out, double *absdot)
{
    if (H != gh * p || W != gw * p || (T + tp - 1) / tp != gt || T < 1)
        return -1;
    if (merge > 1 && (gh % merge || gw % merge))
        return -1;
    const int64_t K = (int64_t)C * tp * p * p;
    const int tpad = gt * tp;
    float *vol = normalized_volume(frames, T, C, H, W, tpad, mean, std);
    float *wb = (float *)malloc(sizeof(float) * (size_t)(E * K));
    oracle_bf16_round_array(w, wb, (int64_t)E * K);
    const int64_t ncell = (int64_t)gt * gh * gw;

#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t cell = 0; cell < ncell; ++cell) {
        const int64_t g_t = cell / ((int64_t)gh * gw);
        const int64_t g_h = (cell / gw) % gh;
        const int64_t g_w = cell % gw;
        const int64_t r = oracle_row_index(g_t, g_h, g_w, gh, gw, merge);
        if (row_mask && !row_mask[r])
            continue;
        for (int e = 0; e < E; ++e) {
            double acc = 0.0, mag = 0.0;
            for (int c = 0; c < C; ++c)
                for (int t = 0; t < tp; ++t)
                    for (int i = 0; i < p; ++i)
                        for (int j = 0; j < p; ++j) {
                            const int64_t tau = g_t * tp + t;
                            const int64_t y = g_h * p + i, xx = g_w * p + j;
                            const double fv =
                                (double)vol[((tau * C + c) * H + y) * W + xx];
                            const double wv =
                                (double)wb[(((((int64_t)e * C + c) * tp + t) * p + i) * p) + j];
                            acc += fv * wv;
                            mag += fabs(fv * wv);
                        }
            out[r * E + e] = acc + (bias ? (double)bias[e] : 0.0);
            if (absdot)
                absdot[r * E + e] = mag;
        }
    }
    free(wb);
    free(vol);
    return 0;
}

/*
 * Patchify: rows[r, k(c,t,i,j)] = Fh[g_t*tp + t, c, g_h*p + i, g_w*p + j]
 * for the output row r of cell (g_t, g_h, g_w).  rows: [gt*gh*gw, K] fp32.
 * Returns 0 on success, -1 on inconsistent sizes.
 */
int oracle_patchify(const float *frames, int T, int H, int W, int gt, int gh, int gw,
                    int merge, const float *mean, const float *std, int C, int tp, int p,
                    float *rows)
{
    if (H != gh * p || W != gw * p || (T + tp - 1) / tp != gt || T < 1)
        return -1;
    if (merge > 1 && (gh % merge || gw % merge))
        return -1;
    const int64_t K = (int64_t)C * tp * p * p;
    const int tpad = gt * tp;
    float *vol = normalized_volume(frames, T, C, H, W, tpad, mean, std);
    const int64_t ncell = (int64_t)gt * gh * gw;
#pragma omp parallel for schedule(static)
    for (int64_t cell = 0; cell < ncell; ++cell) {
        const int64_t g_t = cell / ((int64_t)gh * gw);
        const int64_t g_h = (cell / gw) % gh;
        const int64_t g_w = cell % gw;
        const int64_t r = oracle_row_index(g_t, g_h, g_w, gh, gw, merge);
        for (int c = 0; c < C; ++c)
            for (int t = 0; t < tp; ++t)
                for (int i = 0; i < p; ++i)
                    for (int j = 0; j < p; ++j) {
                        const int64_t k = (((int64_t)c * tp + t) * p + i) * p + j;
                        const int64_t tau = g_t * tp + t;
                        rows[r * K + k] =
                            vol[((tau * C + c) * H + g_h * p + i) * W + g_w * p + j];
                    }
    }
    free(vol);
    return 0;
}

/* PatchMerger (mytransformer README §3.2 and §4.1: LayerNorm, then the 2x2
 * neighbouring patch rows concatenated, 1280 x 4 = 5120, then a GELU MLP
 * 5120 -> 5120 -> hidden).  x: [N, E] fp32 rows in merge order (N = V * m*m),
 * so rows 4v .. 4v+3 form merged row v.  Compute precision mirrors a bf16
 * pipeline: the LayerNorm output and the GELU output are rounded to bf16,
 * weights are rounded to bf16, everything else is fp64.  LayerNorm:
 * (x - mean) / sqrt(var + eps) * gamma + beta with the biased variance over
 * the E features.  GELU: the exact form 0.5 * y * (1 + erf(y / sqrt(2))).
 * out: [V, H] fp64; absdot: [V, H] sum over k of |g_k * w2_k| (g = the bf16
 * GELU output), for tolerance scaling.  v_mask: optional [V] row selector. */
void oracle_patch_merger(const float *x, int64_t V, int E, int m2, const float *gamma, const float *beta,
                         double eps, const float *w1, const float *b1, const float *w2, const float *b2,
                         int H, const uint8_t *v_mask, double *out, double *absdot)
{
    const int64_t D = (int64_t)E * m2;
    float *w1b = (float *)malloc(sizeof(float) * (size_t)(D * D));
    float *w2b = (float *)malloc(sizeof(float) * (size_t)(H * D));
    oracle_bf16_round_array(w1, w1b, D * D);
    oracle_bf16_round_array(w2, w2b, (int64_t)H * D);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t v = 0; v < V; ++v) {
        if (v_mask && !v_mask[v])
            continue;
        double *hln = (double *)malloc(sizeof(double) * (size_t)D);
        double *g = (double *)malloc(sizeof(double) * (size_t)D);
        for (int q = 0; q < m2; ++q) {                 /* LayerNorm of each of the m*m rows */
            const float *row = x + (v * m2 + q) * (int64_t)E;
            double mean = 0.0, var = 0.0;
            for (int e = 0; e < E; ++e) mean += (double)row[e];
            mean /= E;
            for (int e = 0; e < E; ++e) var += ((double)row[e] - mean) * ((double)row[e] - mean);
            var /= E;
            const double inv = 1.0 / sqrt(var + eps);
            for (int e = 0; e < E; ++e) {
                const double y = ((double)row[e] - mean) * inv * (double)gamma[e] + (double)beta[e];
                hln[(int64_t)q * E + e] = (double)oracle_bf16_round((float)y);
            }
        }
        for (int64_t j = 0; j < D; ++j) {              /* fc1 + GELU */
            double acc = 0.0;
            for (int64_t k = 0; k < D; ++k) acc += hln[k] * (double)w1b[j * D + k];
            const double y = acc + (b1 ? (double)b1[j] : 0.0);
            const double gl = 0.5 * y * (1.0 + erf(y / sqrt(2.0)));
            g[j] = (double)oracle_bf16_round((float)gl);
        }
        for (int h = 0; h < H; ++h) {                  /* fc2 */
            double acc = 0.0, mag = 0.0;
            for (int64_t k = 0; k < D; ++k) {
                const double t = g[k] * (double)w2b[(int64_t)h * D + k];
                acc += t;
                mag += fabs(t);
            }
            out[v * H + h] = acc + (b2 ? (double)b2[h] : 0.0);
            if (absdot)
                absdot[v * H + h] = mag;
        }
        free(hln);
        free(g);
    }
    free(w1b);
    free(w2b);
}
