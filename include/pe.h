/*
 * pe.h -- C ABI of the B200 (sm_100a) vision PatchEmbed library (libpe.so).
 *
 * The operation.  Qwen2-VL / Qwen2.5-VL embed every video patch of C channels,
 * tp frames and p x p pixels with a Conv3d whose kernel equals its stride, so
 * each output row is the dot product of one flattened patch with one flattened
 * filter (Qwen2.5VL-Vision Encode-PatchEmbed: the Conv3d description and the
 * python验证 check; Optimize VLM PatchEmbed: Qwen3VLVisionPatchEmbed, "it's
 * actually Linear projection"; patch详解 §4.3):
 *
 *     out[n, e] = bias[e] + sum_k  x[n, k] * W[e, k],   K = C * tp * p * p,
 *
 * with k(c, t, i, j) = ((c * tp + t) * p + i) * p + j, the view(-1, C, tp, p, p)
 * order of the patch vectors and of the flattened [E, C, tp, p, p] weight.
 *
 * Arithmetic.  Operands are rounded to bf16 (round to nearest even) and
 * multiplied on the tensor cores with fp32 accumulation; the bias is added in
 * fp32; the result is stored as fp32 or rounded to bf16.  The pages cast the
 * input to the weight's dtype before the conv (Qwen3VLVisionPatchEmbed.forward).
 *
 * Conventions for every call:
 *   - All tensor arguments are raw pointers.  "dev" means CUDA device memory of
 *     the current device, "host" means ordinary host memory.  The caller owns
 *     every input and output buffer; the library owns only what a handle holds
 *     (packed weight, fp32 bias, normalisation constants, tensor-map
 *     descriptors, a small device workspace and a device error word).
 *   - Calls that take a stream are asynchronous on that stream.  They do not
 *     synchronise it, except when a grow-only workspace has to be enlarged
 *     (the old buffer is freed only after the stream drains).  Argument and
 *     shape errors are detected on the host and returned before anything is
 *     launched or written.
 *   - Dense row-major layouts only.  Device pointers must be 16-byte aligned.
 *   - No C++ exception crosses this interface.  A CUDA error maps to
 *     PE_ERR_CUDA, a failed host allocation to PE_ERR_HOST_MEMORY.
 *   - The forward calls, pe_set_weight and pe_patchify each open an NVTX
 *     range named after the call (Nsight timelines; ncu --nvtx filters);
 *     without a tool attached it costs nothing measurable.
 *   - Forward calls that use a handle's workspace must be serialised on one
 *     stream: grouped calls with more than PE_INLINE_ITEMS items (item table),
 *     frames calls on the staged or streamed path (see pe_forward_frames), and
 *     pe_forward_patches on fp32 rows.  pe_set_weight, pe_set_norm,
 *     pe_set_temporal_fold and pe_set_tf32 must not run concurrently with
 *     anything else on the same handle.
 */
#ifndef PE_H_
#define PE_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (cudaStream_t / CUstream); NULL is the legacy default stream. */
typedef struct CUstream_st *pe_stream_t;

typedef struct pe_handle pe_handle;

typedef enum {
    PE_OK = 0,
    PE_ERR_INVALID_ARG = 1,    /* NULL pointer, non-positive size, bad enum value      */
    PE_ERR_SHAPE = 2,          /* sizes inconsistent with the handle or the grid       */
    PE_ERR_DTYPE = 3,          /* dtype not supported for this argument                */
    PE_ERR_ALIGN = 4,          /* a device pointer is not 16-byte aligned              */
    PE_ERR_NO_WEIGHT = 5,      /* forward called before pe_set_weight                  */
    PE_ERR_CUDA = 6,           /* a CUDA runtime/driver call failed                    */
    PE_ERR_UNSUPPORTED = 7,    /* valid request outside what the kernels implement     */
    PE_ERR_DEVICE_TIMEOUT = 8, /* a kernel gave up waiting on its pipeline (bounded wait) */
    PE_ERR_HOST_MEMORY = 9,    /* a host allocation (item table, chunk plan) failed    */
    PE_ERR_DEVICE_BOUNDS = 10  /* the bounds-checking debug build found a kernel index
                                  outside its buffer (the access was skipped)          */
} pe_status;

typedef enum { PE_F32 = 0, PE_BF16 = 1 } pe_dtype;

/* Grouped calls with at most this many items pass their item table inside the
 * kernel launch; larger groups upload it into the handle's device workspace. */
#define PE_INLINE_ITEMS 16

/* Largest patch side the fused frames path accepts (p must also be even). */
#define PE_MAX_PATCH 32

/*
 * pe_create -- allocate a handle for a PatchEmbed with hidden size E (out
 * channels), C input channels, temporal patch tp and spatial patch p; has_bias
 * != 0 makes pe_set_weight require a bias.  The constructor arguments are the
 * module's config fields in_channels, temporal_patch_size, patch_size,
 * hidden_size and bias (Qwen2.5VL-Vision Encode-PatchEmbed, the candle
 * Qwen2_5VisionPatchEmbed::new; Optimize VLM PatchEmbed, Qwen3VLVisionPatchEmbed).
 * Requires 1 <= C <= 4, 1 <= tp <= 4, 1 <= p, 16 <= E <= 65535 and E % 8 == 0,
 * K = C*tp*p*p <= 8192.  Selects the current CUDA device; the handle must be
 * used on that device.  *out receives the handle (NULL on failure).
 * Errors: PE_ERR_INVALID_ARG, PE_ERR_UNSUPPORTED, PE_ERR_CUDA.
 */
pe_status pe_create(int E, int C, int tp, int p, int has_bias, pe_handle **out);

/*
 * pe_set_weight -- pack the Conv3d weight.
 *   w    : dev [E, C, tp, p, p], dtype w_dt (PE_F32 or PE_BF16), dense.
 *   bias : dev [E] of dtype b_dt, or NULL.  Must be non-NULL iff the handle was
 *          created with has_bias.
 * The weight is rounded to bf16 (RNE) into a handle-owned [E, Kpad] buffer
 * (Kpad = K rounded up to 64, zero padded) -- the flatten(1, 4) of the candle
 * module on Qwen2.5VL-Vision Encode-PatchEmbed -- and the bias is widened
 * exactly to fp32.  Asynchronous on `stream`; w and bias may be freed once the
 * stream has passed this point.  Errors: PE_ERR_INVALID_ARG, PE_ERR_DTYPE,
 * PE_ERR_ALIGN, PE_ERR_CUDA.
 */
pe_status pe_set_weight(pe_handle *h, const void *w, pe_dtype w_dt, const void *bias,
                        pe_dtype b_dt, pe_stream_t stream);

/*
 * pe_set_norm -- per-channel pixel normalisation used by the frames calls:
 * x_hat = bf16_rne( fp32( fp32(x - mean[c]) / std[c] ) ), IEEE fp32 subtract
 * and divide, bit-exact for every finite pixel value x (non-finite pixels give
 * NaN).  mean, std: host [C] fp32; mean[c] finite, std[c] finite and > 0.
 * Default after pe_create: mean 0, std 1 (x_hat = bf16_rne(x)).
 * Errors: PE_ERR_INVALID_ARG.
 */
pe_status pe_set_norm(pe_handle *h, const float *mean, const float *std);

/*
 * pe_set_temporal_fold -- opt-in temporal folding for single-frame items.
 * A single image is duplicated to tp = 2 frames before the Conv3d (patch详解
 * §4.5 counts ceil(1/2) = 1 temporal patch), so both temporal slices of the
 * kernel multiply the same pixels: out = x̂ · (Ŵ[:,:,0] + Ŵ[:,:,1]).  With
 * folding enabled, frames calls whose items all have T == 1 (bf16 frames,
 * p in {14, 16}) multiply by the folded weight bf16_rne(fp32(Ŵ0 + Ŵ1)) once,
 * which halves the contraction (K = C*p*p instead of C*tp*p*p).  This changes
 * the rounding of the result: each weight term carries one more bf16 rounding,
 * at most 2^-8 of |Ŵ0 + Ŵ1|, so the worst-case bound is 2^-8 * sum |x̂ ŵ|
 * rather than the unfolded path's fp32-accumulation bound.  Other calls (and
 * pe_forward_frames_grouped_noalloc, which never uses the workspace that the
 * folded path needs) are unaffected.  enable = 0 (the default) or 1.  Errors: PE_ERR_INVALID_ARG,
 * PE_ERR_UNSUPPORTED (tp != 2).
 */
pe_status pe_set_temporal_fold(pe_handle *h, int enable);

/*
 * pe_set_tf32 -- opt-in tf32 contraction for fp32 patch rows.
 * Qwen2.5VL-Vision Encode-PatchEmbed checks the Conv3d against the matmul in
 * fp32 (the python check: a max difference of about 4e-6); the default bf16
 * compute keeps 8 significant bits of each input.  With tf32 enabled,
 * pe_forward_patches on fp32 rows rounds the rows and the weight to tf32
 * (10 fraction bits, nearest with ties away from zero) and contracts with
 * kind::tf32 tensor-core MMAs accumulating in fp32: each product then carries
 * at most about 2^-10 relative error instead of 2^-7.  Half the bf16 tensor
 * rate.  Requires K % 4 == 0.  enable = 0 (default) or 1.  bf16 rows and the
 * frames calls are unaffected.  Errors: PE_ERR_INVALID_ARG, PE_ERR_UNSUPPORTED.
 */
pe_status pe_set_tf32(pe_handle *h, int enable);

/*
 * pe_forward_patches -- out = x @ W^T (+ bias) on already patchified rows.
 *   x   : dev [N, K] of dtype x_dt (PE_BF16 or PE_F32), rows in
 *         view(-1, C, tp, p, p) order as the Qwen2-VL processor emits
 *         pixel_values (mytransformer README §3.2: pixel_values [N, 1176]).
 *   out : dev [N, E] of dtype out_dt.
 * Rows are processed in the given order; N may be 0 (nothing is launched).
 * Compute dtype bf16: fp32 rows are rounded to bf16 (nearest even).  With fp32
 * rows and K % 8 == 0 a small kernel casts them once into the handle's
 * grow-only workspace and the TMA-fed contraction reads them back (calls that
 * use the workspace must be serialised on one stream); PE_PATCHES_PATH=threads
 * converts inside the contraction kernel instead.  bf16 rows are read directly.
 * Errors: PE_ERR_INVALID_ARG, PE_ERR_DTYPE, PE_ERR_ALIGN, PE_ERR_NO_WEIGHT,
 * PE_ERR_CUDA.
 */
pe_status pe_forward_patches(pe_handle *h, const void *x, pe_dtype x_dt, int64_t N,
                             void *out, pe_dtype out_dt, pe_stream_t stream);

/*
 * pe_forward_patches_pos -- pe_forward_patches with a position-embedding
 * table added in the same epilogue: out[r, e] = (x @ W^T)[r, e] + bias[e] +
 * pos[r, e], summed in fp32 before the output cast.  The vision model adds the
 * interpolated position embeddings to the patch embeddings right after the
 * PatchEmbed ("Optimize VLM PatchEmbed", the Qwen3-VL vision model forward:
 * hidden_states + pos_embeds); the table's interpolation is the caller's.
 *   pos    : dev [N, E] of dtype pos_dt (PE_F32 or PE_BF16), dense, 16-byte
 *            aligned, in the same row order as out.
 * Errors: as pe_forward_patches; a NULL or unaligned pos (with N > 0) gives
 * PE_ERR_INVALID_ARG / PE_ERR_ALIGN, a bad pos_dt PE_ERR_DTYPE.
 */
pe_status pe_forward_patches_pos(pe_handle *h, const void *x, pe_dtype x_dt, int64_t N, const void *pos,
                                 pe_dtype pos_dt, void *out, pe_dtype out_dt, pe_stream_t stream);

/*
 * pe_forward_frames -- patchify + normalise + embed of one image/video.
 *   frames   : dev [T, C, H, W] of dtype f_dt (PE_BF16 or PE_F32), dense.
 *   grid_thw : host [3] = (gt, gh, gw) in patch units.  Requires H == gh*p,
 *              W == gw*p and ceil(T / tp) == gt (patch详解 §4.5).  When T is not
 *              a multiple of tp the last frame is repeated, so a single image
 *              (T = 1) is duplicated to tp frames.
 *   merge    : 1 or 2.  With merge = m > 1 the rows come in spatial-merge order:
 *              m x m windows consecutive, windows row-major over
 *              (t, h/m, w/m), (dh, dw) row-major inside a window (mytransformer
 *              README §3.2 PatchMerger and §4.1; Qwen2.5VL语言模型 MRoPE example:
 *              merged grid row-major, h outer).  gh and gw must be multiples of m.
 *   out      : dev [gt*gh*gw, E] of dtype out_dt.
 * Requires p even and p <= PE_MAX_PATCH.  Execution paths, all within the
 * same tolerance of the exact result:
 *   staged   (default for bf16 or fp32 frames with tp in {1, 2} and p in {14, 16}) a prepare
 *            kernel writes the normalised rows once into the handle's
 *            grow-only workspace, then the TMA-fed contraction reads them back;
 *   resident A  (PE_FRAMES_PATH=astat, and the allocation-free call, when
 *            every item is a single frame, the frames are bf16, tp = 2 and the
 *            C*p*p-column A block fits in shared memory beside the weight
 *            ring) one kernel; each 256-row block's normalised patches are
 *            gathered from the frames once into shared memory, in merge order,
 *            and every weight tile streams past them; both temporal slices of
 *            the weight meet the one frame.  No workspace; the [N, K] patch
 *            matrix never exists in memory.  It issues, row by row, the same
 *            MMAs in the same order as the staged path, so the two give
 *            identical bits.  On B200 it runs slower than the staged pair (the
 *            resident A leaves the weight ring too little shared memory);
 *   fused    one kernel that gathers each A tile again for every weight tile
 *            (tp in {3, 4}, p not in {14, 16}, and the allocation-free
 *            call's other groups);
 *   streamed one cooperative kernel: producer warps write the same rows while
 *            the contraction consumes the completed row blocks (an option for
 *            bf16 frames: slower than staged on B200).
 * The environment variable PE_FRAMES_PATH=staged|astat|fused|streamed selects
 * a path instead of the default.  PE_TEST_WAIT_NS=n (a test hook) gives the
 * resident-A kernel's pipeline waits a limit of n ns instead of 2 s, so that a
 * test can make them run out and exercise the kernel's unwinding: the call
 * then leaves an incomplete output and pe_last_error reports
 * PE_ERR_DEVICE_TIMEOUT.
 * Errors: as pe_forward_patches plus PE_ERR_SHAPE, PE_ERR_UNSUPPORTED.
 */
pe_status pe_forward_frames(pe_handle *h, const void *frames, pe_dtype f_dt, int T, int H,
                            int W, const int32_t grid_thw[3], int merge, void *out,
                            pe_dtype out_dt, pe_stream_t stream);

/*
 * pe_forward_frames_grouped -- pe_forward_frames over n items in ONE launch; the
 * rows of item i follow those of items 0..i-1 (the packed sequence of the vision
 * forward with grid_thw of shape (num_images_or_videos, 3): Optimize VLM
 * PatchEmbed, the vision model's forward).
 *   frames   : host array of n dev pointers, item i is [THW[3i], C, THW[3i+1], THW[3i+2]]
 *   THW      : host [n, 3] frame dims (T, H, W) per item
 *   grid_thw : host [n, 3] patch grid per item
 *   out      : dev [sum_i gt_i*gh_i*gw_i, E]
 * All items share f_dt, merge and out_dt.  Errors: as pe_forward_frames.
 */
pe_status pe_forward_frames_grouped(pe_handle *h, int n, const void *const *frames, pe_dtype f_dt,
                                    const int32_t *THW, const int32_t *grid_thw, int merge,
                                    void *out, pe_dtype out_dt, pe_stream_t stream);

/*
 * pe_forward_frames_grouped_pos -- pe_forward_frames_grouped with a
 * position-embedding table added in the same epilogue, as in
 * pe_forward_patches_pos: out[r, e] = conv[r, e] + bias[e] + pos[r, e] in fp32
 * before the output cast.
 *   pos    : dev [N, E] of dtype pos_dt, N = the items' total patch count, rows
 *            in the output's order (items in list order, merge order inside
 *            an item), dense, 16-byte aligned.
 * Errors: as pe_forward_frames_grouped; a NULL or unaligned pos gives
 * PE_ERR_INVALID_ARG / PE_ERR_ALIGN, a bad pos_dt PE_ERR_DTYPE.
 */
pe_status pe_forward_frames_grouped_pos(pe_handle *h, int n, const void *const *frames, pe_dtype f_dt,
                                        const int32_t *THW, const int32_t *grid_thw, int merge, const void *pos,
                                        pe_dtype pos_dt, void *out, pe_dtype out_dt, pe_stream_t stream);

/* Largest item count pe_forward_frames_grouped_noalloc accepts. */
#define PE_NOALLOC_MAX_ITEMS 1024

/*
 * pe_forward_frames_grouped_noalloc -- pe_forward_frames_grouped for callers
 * that must not allocate memory while they run: serving loops that hand every
 * byte of device memory to their own pool up front and forbid cudaMalloc
 * (and its implicit device synchronisation) on the request path.  The plain
 * grouped call allocates, on its first group of more than PE_INLINE_ITEMS
 * items, a device table and a pinned host staging buffer in the handle; this
 * variant instead uses a fixed table of PE_NOALLOC_MAX_ITEMS item descriptors
 * (40 bytes each) in the library's static device memory, which every device
 * that loads the library holds until the process exits.  It never calls
 * cudaMalloc, cudaMallocHost or cudaFree.  The pages have no counterpart: this
 * is an allocation-free calling convention of this library only.
 *
 * Arguments, layouts and results are those of pe_forward_frames_grouped.
 * n > PE_NOALLOC_MAX_ITEMS returns PE_ERR_UNSUPPORTED before anything runs.
 * With more than PE_INLINE_ITEMS items the descriptors are written into the
 * table by small kernels on `stream` whose launch parameters carry them (up to
 * 64 per launch), so no host staging buffer is used and the host never waits.
 * The first call on a device (with more than PE_INLINE_ITEMS items) looks up
 * the table's device address; make that first call before any stream capture.
 * All calls share the one table and it keeps the last call's contents, so calls
 * that can overlap on the GPU (different streams) race; calls on one stream
 * are ordered and safe.  Groups of single images take the one-launch
 * resident-A kernel, which needs no workspace; other groups take the fused
 * kernel (never the staged path, whose row buffer is allocated on first use).
 */
pe_status pe_forward_frames_grouped_noalloc(pe_handle *h, int n, const void *const *frames, pe_dtype f_dt,
                                            const int32_t *THW, const int32_t *grid_thw, int merge,
                                            void *out, pe_dtype out_dt, pe_stream_t stream);

/*
 * pe_forward_frames_grouped_host -- pe_forward_frames_grouped with the frames
 * and the output in HOST memory: the call copies the frames in, embeds them
 * and copies the rows out.  It is the call for a caller whose decoded frames
 * sit in host memory and who wants the embeddings back there.  The pages have
 * no counterpart; the arithmetic is exactly that of the device-pointer call.
 *   frames_host : host array of n host pointers, item i is
 *                 [THW[3i], C, THW[3i+1], THW[3i+2]] of dtype f_dt, dense
 *   out_host    : host [sum_i gt_i*gh_i*gw_i, E] of dtype out_dt, dense
 *   Other arguments as pe_forward_frames_grouped.
 * The items are cut into chunks of about an eighth of the rows (at least 8192
 * rows; whole items, and whole temporal patches of a video, which are
 * contiguous output rows).  Each chunk is copied into one of two device input
 * slots on the handle's copy-in stream, computed on `stream` by the
 * device-pointer path, and copied out of one of two output slots on the
 * handle's copy-out stream; so one chunk's copy in, another's contraction and
 * a third's copy out overlap.  The environment variable PE_HOST_CHUNK_ROWS
 * overrides the chunk size.
 * Ordering: the copies start after the work already queued on `stream`, and
 * `stream` waits for the last copy out, so out_host is complete once `stream`
 * has drained (cudaStreamSynchronize, or an event recorded after the call).
 * The host buffers must stay valid and unchanged until then.  Pinned host
 * memory (cudaMallocHost / cudaHostRegister) gives the overlap; with pageable
 * memory the copies are staged by the CUDA driver and the call blocks the host
 * on each copy.
 * Workspace: the handle's grow-only device slots and two streams, created on
 * first use; calls on one handle must be serialised on one stream.
 * Errors: as pe_forward_frames_grouped; every item is validated before
 * anything is copied or launched.  A CUDA error after work was queued returns
 * PE_ERR_CUDA with the earlier chunks possibly done.
 */
pe_status pe_forward_frames_grouped_host(pe_handle *h, int n, const void *const *frames_host, pe_dtype f_dt,
                                         const int32_t *THW, const int32_t *grid_thw, int merge, void *out_host,
                                         pe_dtype out_dt, pe_stream_t stream);

/*
 * pe_forward_patches_host -- pe_forward_patches with x and out in HOST memory,
 * pipelined over row chunks exactly as pe_forward_frames_grouped_host.
 *   x_host   : host [N, K] of dtype x_dt, dense, rows as in pe_forward_patches
 *   out_host : host [N, E] of dtype out_dt, dense
 * Ordering, workspace and pinned-memory notes as for
 * pe_forward_frames_grouped_host.  N may be 0 (nothing is queued).
 * Errors: PE_ERR_INVALID_ARG, PE_ERR_DTYPE, PE_ERR_NO_WEIGHT, PE_ERR_CUDA.
 */
pe_status pe_forward_patches_host(pe_handle *h, const void *x_host, pe_dtype x_dt, int64_t N, void *out_host,
                                  pe_dtype out_dt, pe_stream_t stream);

/*
 * pe_patchify -- test hook: the fused producer's gather and normalisation
 * written out to memory instead of feeding the tensor cores.
 *   rows : dev [sum_i N_i, K] of dtype rows_dt (PE_BF16 or PE_F32; values are
 *          bf16-exact either way), row order and k order as in the forward calls.
 * Other arguments as pe_forward_frames_grouped.
 */
pe_status pe_patchify(pe_handle *h, int n, const void *const *frames, pe_dtype f_dt,
                      const int32_t *THW, const int32_t *grid_thw, int merge, void *rows,
                      pe_dtype rows_dt, pe_stream_t stream);

/*
 * pe_num_patches -- sum_i gt_i * gh_i * gw_i over host grid_thw [n, 3];
 * 0 for n == 0; -1 on a NULL pointer with n > 0, negative n, a
 * non-positive entry or a sum that does not fit in int64_t.
 */
int64_t pe_num_patches(const int32_t *grid_thw, int n);

/*
 * pe_profile_begin / pe_profile_end -- device time of each forward call's
 * contraction kernel (the resident-A or fused kernel, or the GEMM that follows
 * the prepare or cast kernel), recorded with a CUDA event pair on the call's stream
 * around that launch.  pe_profile_begin creates event pairs for up to
 * max_calls calls (0..1e6; 0 records no events and only counts launches) and
 * starts recording; pe_profile_end waits for the recorded events, writes the
 * elapsed milliseconds of the first min(*n, recorded) calls to host ms[] and
 * that count to *n, writes to *launches (if not NULL) how many kernels the
 * forward calls launched in the window (two per call on the staged frames
 * path and for fp32 patch rows, one otherwise, plus the item-table fills of
 * the allocation-free call), then frees the events and
 * stops recording.  Profiling is a measurement aid: it allocates events and must not
 * overlap another profiling window on the same handle.  An event recorded
 * between two kernels of one call serialises them, so a window with events
 * runs the staged path a few microseconds slower than a window without.
 * Errors: PE_ERR_INVALID_ARG, PE_ERR_CUDA.
 */
pe_status pe_profile_begin(pe_handle *h, int max_calls);
pe_status pe_profile_end(pe_handle *h, float *ms, int *n, int64_t *launches);

/*
 * pe_profile_target -- which kernel of a forward call the profiling event
 * pairs bracket from now on: 0 (the default) the contraction kernel, as
 * described above; 1 the kernel that runs before it, the prepare kernel of a
 * staged frames call or the cast / tf32-rounding kernel of an fp32 patches
 * call (calls without one record nothing).  The patchify read's achieved
 * memory throughput is the frames bytes over that time.  An event after the
 * prepare kernel keeps the contraction from starting early, as any event
 * between the two does.
 * Errors: PE_ERR_INVALID_ARG (NULL handle, target not 0 or 1).
 */
pe_status pe_profile_target(pe_handle *h, int target);

/*
 * pe_selftest_wait_timeout -- test hook for failure detection: one warp waits,
 * through the bounded wait every pipeline uses, on a shared-memory barrier
 * phase that nothing completes.  The wait gives up after its limit (2 s), and
 * the kernel records PE_ERR_DEVICE_TIMEOUT in the handle's error word exactly
 * as a contraction kernel whose pipeline stalled does; pe_last_error then
 * reports and clears it, and the handle stays usable.  Nothing faults, traps
 * or hangs.  Asynchronous on `stream`.
 * Errors: PE_ERR_INVALID_ARG (NULL handle), PE_ERR_CUDA (launch failed).
 */
pe_status pe_selftest_wait_timeout(pe_handle *h, pe_stream_t stream);

/*
 * pe_last_error -- read and clear the handle's device error word.  Call after
 * synchronising the streams the handle ran on.  Returns PE_OK, or
 * PE_ERR_DEVICE_TIMEOUT if a kernel stopped waiting on its pipeline (it then
 * wrote an incomplete output and left the device usable), or PE_ERR_CUDA if
 * the word could not be read.
 */
pe_status pe_last_error(pe_handle *h);

/* Static English text for a status code (never NULL). */
const char *pe_status_string(pe_status s);

/* Release the handle and everything it owns.  NULL is a no-op.  Synchronises
 * the device first so no launch still uses the handle's buffers. */
void pe_destroy(pe_handle *h);

/* Device this handle was created on, or -1 for NULL. */
int pe_device(const pe_handle *h);

/* ------------------------------------------------------------------------
 * PatchMerger -- the step that consumes the PatchEmbed rows in merge order
 * (mytransformer README §3.2 and §4.1): LayerNorm of each row, the m*m rows of
 * a merge window concatenated (1280 x 4 = 5120 for Qwen2-VL), then a GELU MLP
 * D -> D -> H (D = E*m*m; 5120 -> 5120 -> 1536).  Readings where the page is
 * silent: an affine LayerNorm (gamma, beta) with the biased variance and the
 * given eps (1e-6 for Qwen2-VL), the exact erf GELU, bias on both linear
 * layers optional.  Compute: bf16 operands on the tensor cores with fp32
 * accumulation; the LayerNorm output and the GELU output are stored as bf16.
 */
typedef struct pe_merger pe_merger;

/*
 * pe_merger_create -- E: rows' width (multiple of 8); m: merge size (1..4);
 * H: output width (multiple of 8, >= 16); eps > 0.  D = E*m*m must be a
 * multiple of 64 and at most 65536.  Binds to the current CUDA device.
 * Errors: PE_ERR_INVALID_ARG, PE_ERR_UNSUPPORTED, PE_ERR_CUDA.
 */
pe_status pe_merger_create(int E, int m, int H, float eps, pe_merger **out);

/*
 * pe_merger_set_weights -- device pointers, all of dtype dt (copied and packed;
 * the caller keeps ownership): gamma, beta [E]; w1 [D, D] and w2 [H, D] in the
 * nn.Linear [out, in] layout; b1 [D] and b2 [H] or NULL.  16-byte aligned.
 * Asynchronous on stream.  Errors: PE_ERR_INVALID_ARG, PE_ERR_DTYPE,
 * PE_ERR_ALIGN, PE_ERR_CUDA.
 */
pe_status pe_merger_set_weights(pe_merger *pm, const void *gamma, const void *beta, const void *w1,
                                const void *b1, const void *w2, const void *b2, pe_dtype dt,
                                pe_stream_t stream);

/*
 * pe_merger_forward -- x: dev [N, E] bf16 rows in merge order (the PatchEmbed
 * output); N a multiple of m*m (N = 0: nothing is launched).  out: dev
 * [N / (m*m), H] of dtype out_dt.  Three launches on stream: LayerNorm, fc1
 * with the GELU in its epilogue, fc2.  The intermediate rows live in the
 * merger's grow-only workspace, so calls must be serialised on one stream.
 * Errors: PE_ERR_INVALID_ARG, PE_ERR_DTYPE, PE_ERR_ALIGN, PE_ERR_NO_WEIGHT,
 * PE_ERR_SHAPE, PE_ERR_CUDA.
 */
pe_status pe_merger_forward(pe_merger *pm, const void *x, int64_t N, void *out, pe_dtype out_dt,
                            pe_stream_t stream);

/*
 * pe_merger_profile_begin / pe_merger_profile_end -- as pe_profile_begin /
 * pe_profile_end, around each of the two linear layers of every forward call
 * (so the times alternate fc1, fc2); launches counts all three kernels.
 */
pe_status pe_merger_profile_begin(pe_merger *pm, int max_calls);
pe_status pe_merger_profile_end(pe_merger *pm, float *ms, int *n, int64_t *launches);

/* pe_merger_last_error -- as pe_last_error, for the merger's kernels. */
pe_status pe_merger_last_error(pe_merger *pm);

/* pe_merger_destroy -- waits for the device, frees everything; NULL is a no-op. */
void pe_merger_destroy(pe_merger *pm);

#ifdef __cplusplus
}
#endif

#endif /* PE_H_ */
