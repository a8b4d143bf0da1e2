/*
 * moeq.h -- C ABI of the compressed-expert routed MoE layer for NVIDIA B200
 * (sm_100a).
 *
 * The layer is the routed-expert FFN of a MiMo-V2.6-Flash-shaped MoE block:
 * every token t is sent to k experts e = topk_ids[t][s] with weights
 * topk_w[t][s], and
 *
 *     out[t] = sum_s topk_w[t][s] * W_down,e ( silu(W_gate,e x[t]) * (W_up,e x[t]) )
 *
 * with silu(z) = z / (1 + e^-z).  The expert matrices stay compressed in
 * device memory and are decoded inside the matrix products.  Sources (page
 * title, section):
 *   - "MiMo-V2.6-Flash-RL GGUF for a single DGX Spark", "Architecture notes":
 *     256 routed experts, 8 active per token, no shared expert; experts stored
 *     as MXFP4, one E8M0 exponent per 32 values.
 *   - "MiMo-V2.6-Flash-RL Mixed-Quant GGUF", "Why this model needs an
 *     asymmetric layout": packed MXFP4, two weights per byte; gate/up and down
 *     projections per expert.
 *   - "MiMo-V2.6-Flash-RL UNCENSORED VQ GGUF", "Recipe" and "Why 13 bits plus
 *     an 8-bit residual": each 8 consecutive weights of an expert row are one
 *     13-bit index into the layer's 8192x8 codebook (shared by all experts and
 *     gate/up/down), times an f16 row gain; an optional second 256x8 book codes
 *     the first stage's residual with 8 more bits per 8 weights; the kernels
 *     keep the layer's whole codebook in shared memory while they decode every
 *     selected expert.
 *   - "MiMo-V2.6-Flash-RL GGUF for a single DGX Spark", "Recipe": a 32-value
 *     expert-intermediate sum can pass f16's 65504, so intermediates are kept
 *     in a type with f32's exponent range.
 *
 * Conventions
 *   - Every call returns a moeq_status; no exception or signal crosses the ABI.
 *   - Projection p: MOEQ_GATE [inter][hidden], MOEQ_UP [inter][hidden],
 *     MOEQ_DOWN [hidden][inter].  Rows are output features; the reduction axis
 *     K is contiguous in memory.
 *   - A "stream" argument is a cudaStream_t passed as void* (NULL = the legacy
 *     default stream).  Device pointers must be on the layer's device.
 *   - One layer's workspace is not re-entrant: calls on one layer must be
 *     ordered (one stream, or explicit events).  Distinct layers are
 *     independent and may be used from different host threads.
 */
#ifndef MOEQ_H
#define MOEQ_H

#include <stdint.h>

#if defined(__GNUC__)
#define MOEQ_API __attribute__((visibility("default")))
#else
#define MOEQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOEQ_OK = 0,
    MOEQ_ERR_INVALID_ARGUMENT = 1,  /* bad pointer, size, enum or weight byte  */
    MOEQ_ERR_UNSUPPORTED = 2,       /* valid but not implemented combination   */
    MOEQ_ERR_OUT_OF_MEMORY = 3,     /* a device allocation failed              */
    MOEQ_ERR_CUDA = 4,              /* a CUDA runtime call or launch failed    */
    MOEQ_ERR_NOT_UPLOADED = 5,      /* forward/dequant before upload_weights   */
    MOEQ_ERR_ROUTE_OUT_OF_RANGE = 6,/* device flag: an id outside [-1, E) seen */
    MOEQ_ERR_TIMEOUT = 7            /* device flag: a bounded wait gave up     */
} moeq_status;

typedef enum {
    MOEQ_FMT_MXFP4 = 0,
    MOEQ_FMT_VQ13 = 1,      /* 13-bit stream, bf16 books                              */
    MOEQ_FMT_VQ13_R8 = 2,   /* ... plus the 8-bit residual stage                      */
    MOEQ_FMT_GVQ1 = 3,      /* 12-bit stream + bit-12 plane, 1-byte E4M3 book entries */
    MOEQ_FMT_GVQ1_R8 = 4    /* ... plus the 8-bit residual stage                      */
} moeq_format;
typedef enum { MOEQ_ACT_F32 = 0, MOEQ_ACT_BF16 = 1 } moeq_dtype;
typedef enum { MOEQ_GATE = 0, MOEQ_UP = 1, MOEQ_DOWN = 2 } moeq_proj;
/* Routing weights of the router (moeq_router_upload). */
typedef enum { MOEQ_SCORE_SIGMOID = 0, MOEQ_SCORE_SOFTMAX = 1 } moeq_score;

typedef struct {
    int32_t hidden;      /* H: model width (K of gate/up, N of down)              */
    int32_t inter;       /* I: expert intermediate width                          */
    int32_t n_experts;   /* E, 1..1024                                            */
    int32_t top_k;       /* k, 1..min(E, 64)                                      */
    int32_t max_tokens;  /* largest n_tokens any forward will pass, >= 1          */
    int32_t fmt;         /* moeq_format                                           */
    int32_t act;         /* moeq_dtype of x and out                               */
    int32_t device;      /* CUDA device ordinal                                   */
} moeq_layer_desc;

typedef struct moeq_layer *moeq_layer_t;

/*
 * Host copy of a layer's compressed weights, logical layout, one array per
 * projection p (index = moeq_proj).  N, K are the projection's rows and
 * reduction length.
 *
 * MXFP4 ("Architecture notes" above):
 *   codes[p]   uint8 [E][N][K/2]  element k of a row is the low nibble of byte
 *                                 k/2 when k is even, the high nibble when odd;
 *                                 nibble = E2M1 (sign, 2 exponent bits with
 *                                 bias 1, 1 mantissa bit)
 *   scales[p]  uint8 [E][N][K/32] E8M0 byte b: weight = e2m1 * 2^(b-127);
 *                                 b = 255 (NaN) is rejected
 * VQ13 / VQ13_R8 ("Recipe" above):
 *   idx13[p]   uint8 [E][N][K*13/64]  per row, the K/8 indices as one
 *                                 little-endian bitstream: index j is bits
 *                                 13j..13j+12, bit q of the stream is bit q%8
 *                                 of byte q/8
 *   idx8[p]    uint8 [E][N][K/8]  residual index per 8-vector (VQ13_R8 only)
 *   book13     uint16 bf16 [8192][8]  base codebook; entry dimension i is K
 *                                 offset 8j+i of group j
 *   book8      uint16 bf16 [256][8]   residual codebook (VQ13_R8 only)
 *   gain[p]    uint16 f16 [E][N] or NULL (gain 1)
 *   weight[n][8j+i] = (book13[idx13][i] + book8[idx8][i]) * gain[n], each
 *   operation IEEE f32 round-to-nearest-even, in that order.
 * GVQ1 / GVQ1_R8 (same page, "Recipe": the indices as a 12-bit code stream
 * with a separate plane of one-bit flags; "Why 13 bits plus an 8-bit
 * residual": books of 1-byte entries, 64 KiB + 2 KiB.  The byte layout and
 * the entry type are not on the page; this library reads them as follows):
 *   code12[p]  uint8 [E][N][K*3/16]  per row, the low 12 bits of the K/8
 *                                 indices as one little-endian bitstream
 *                                 (index j: bits 12j..12j+11)
 *   hi1[p]     uint8 [E][N][K/64] per row, bit 12 of index j is bit j
 *                                 (bit j%8 of byte j/8)
 *   idx8[p]    as for VQ13_R8 (GVQ1_R8 only)
 *   gbook13    uint8 [8192][8]    E4M3 entries (the OCP 8-bit float without
 *                                 infinities: sign, 4 exponent bits with
 *                                 bias 7, 3 mantissa bits); 0x7F / 0xFF
 *                                 (NaN) are rejected
 *   gbook8     uint8 [256][8]     E4M3 residual entries (GVQ1_R8 only)
 *   gscale[2]  the f32 scales of gbook13 and gbook8 (finite)
 *   gain[p]    as for VQ13
 *   weight[n][8j+i] = (e4m3(gbook13[c][i]) * gscale[0]
 *                      + e4m3(gbook8[r][i]) * gscale[1]) * gain[n],
 *   each operation IEEE f32 round-to-nearest-even, in that order.
 * Arrays not used by the format must be NULL.
 */
typedef struct {
    const uint8_t *codes[3];
    const uint8_t *scales[3];
    const uint8_t *idx13[3];
    const uint8_t *idx8[3];
    const uint16_t *book13;
    const uint16_t *book8;
    const uint16_t *gain[3];
    const uint8_t *code12[3];
    const uint8_t *hi1[3];
    const uint8_t *gbook13;
    const uint8_t *gbook8;
    float gscale[2];
} moeq_weights;

/* Create a layer on desc->device and allocate, on that device, its weight
 * storage and a workspace sized for desc->max_tokens.  The library owns all
 * of it until moeq_layer_destroy.
 * Errors: INVALID_ARGUMENT (NULL pointer; a non-positive size; top_k > E or
 * > 64; E > 1024; for MXFP4 hidden or inter not a multiple of 128, or
 * above 1024 and not a multiple of 1024; for VQ13 / GVQ1 not a multiple of
 * 64;
 * unknown fmt/act), CUDA (bad device), OUT_OF_MEMORY.  On error *out
 * is set to NULL and nothing is left allocated. */
MOEQ_API moeq_status moeq_layer_create(const moeq_layer_desc *desc, moeq_layer_t *out);

/* Copy the host arrays of w into the layer (the library may store them in a
 * different internal order).  Validates first: every array the format needs
 * is non-NULL, arrays it does not use are NULL, no E8M0 byte is 255, no
 * E4M3 book entry is NaN, the GVQ1 book scales are finite.  Uses
 * `stream` for the copies and synchronizes it before returning, so the
 * caller may free w's arrays as soon as the call returns.
 * Errors: INVALID_ARGUMENT (validation), CUDA. */
MOEQ_API moeq_status moeq_upload_weights(moeq_layer_t layer, const moeq_weights *w, void *stream);

/* out[t] for t < n_tokens, as defined at the top of this file.
 *   x         device, act dtype, [n_tokens][hidden], row-major
 *   topk_ids  device int32 [n_tokens][top_k]; -1 = no route (contributes 0);
 *             any other id outside [0, E) is skipped and raises
 *             MOEQ_ERR_ROUTE_OUT_OF_RANGE in the layer status word
 *   topk_w    device f32 [n_tokens][top_k]; any values (need not sum to 1)
 *   out       device, act dtype, [n_tokens][hidden]; overwritten
 * Asynchronous on `stream`: all pointers must stay valid until the stream
 * reaches the end of the call.  Stream order holds as usual; at decode sizes
 * the first kernel may be scheduled while the previous kernel on the stream
 * drains (programmatic dependent launch) but waits for it to complete before
 * it reads any argument or workspace.  The sum over routes is accumulated in
 * f32 and rounded once (RNE) to the output dtype; the order in which routes
 * are added is not specified.  n_tokens == 0 is a no-op.
 * Errors (synchronous): INVALID_ARGUMENT (NULL pointer, n_tokens < 0 or >
 * max_tokens), NOT_UPLOADED, CUDA (launch). */
MOEQ_API moeq_status moeq_forward(moeq_layer_t layer, const void *x, const int32_t *topk_ids,
                         const float *topk_w, int32_t n_tokens, void *out, void *stream);

/* moeq_forward with HOST buffers (same shapes and dtypes): copies x,
 * topk_ids and topk_w to the layer's device staging area, runs the forward
 * and copies out back, all on `stream`, and synchronizes the stream before
 * returning.  Host buffers may be pageable or pinned.
 * Errors: as moeq_forward, and CUDA for a failed copy or synchronize. */
MOEQ_API moeq_status moeq_forward_host(moeq_layer_t layer, const void *x_host, const int32_t *topk_ids_host,
                              const float *topk_w_host, int32_t n_tokens, void *out_host,
                              void *stream);

/* The route/bucket step of moeq_forward on its own: groups the routes of
 * topk_ids (device int32 [n_tokens][top_k]) by expert.
 *   offsets_out  device int32 [E+1]: offsets_out[e] = number of valid routes
 *                whose expert is below e (valid: id in [0, E))
 *   perm_out     device int32 [n_tokens*top_k]: its first offsets_out[E]
 *                entries are the valid route ids r = t*top_k + s, expert by
 *                expert, ascending r within an expert (a stable sort)
 * Ids of -1 are skipped; other ids outside [0, E) are skipped and raise
 * MOEQ_ERR_ROUTE_OUT_OF_RANGE in the status word.  Asynchronous on
 * `stream`; uses the layer's workspace (ordered like moeq_forward).
 * Source: "MiMo-V2.6-Flash-RL GGUF for a single DGX Spark", "Speed" (each
 * expert's tokens are gathered into one matmul) and "Architecture notes"
 * (k of E experts per token).
 * Errors: INVALID_ARGUMENT (NULL pointer, n_tokens < 1 or > max_tokens),
 * CUDA. */
MOEQ_API moeq_status moeq_route(moeq_layer_t layer, const int32_t *topk_ids, int32_t n_tokens,
                                int32_t *offsets_out, int32_t *perm_out, void *stream);

/* moeq_route for callers that cannot allocate device memory: no layer
 * handle, and no cudaMalloc, cudaFree or other allocating call, ever.
 * Meant for code that runs where allocation is not allowed or not wanted:
 * inside another framework's memory pool that owns the whole device, under
 * a hard memory budget, or in a context where a device allocation would
 * synchronize or fail.  No passage of the paper corresponds to it: it is a
 * packaging of the route/bucket step, not part of the method.
 *
 * Arguments and results are those of moeq_route, on the current device:
 * topk_ids (device int32 [n_tokens][top_k]) in, offsets_out (device int32
 * [n_experts+1]) and perm_out (device int32 [n_tokens*top_k]) out, all
 * owned by the caller; asynchronous on `stream`.  Ids of -1 are skipped;
 * other ids outside [0, n_experts) are skipped too, and this entry point
 * does not report them (offsets_out[n_experts] counts the valid routes
 * only; moeq_route reports them through its layer).
 *
 * The kernel's scratch (the list of active experts and a status word, 4104
 * bytes) is one fixed array inside the library, one copy per device that
 * loads it, held until the process exits.  Limits that follow from it:
 * n_experts <= 1024; beyond that the call returns MOEQ_ERR_UNSUPPORTED and
 * launches nothing.  Every call on a device shares that array and it keeps
 * the last call's contents (the status word is cleared on `stream` before
 * each launch): calls that overlap on the GPU, from different streams or
 * threads, race on it and must be ordered by the caller.  The first call on
 * each device sets up (looks up the array's device address and sets the
 * kernel's shared-memory limit); make that first call before any stream
 * capture on that device.  The library itself makes no allocating call
 * here, but under the CUDA runtime's lazy module loading the first call on
 * a device may be what makes the runtime load this module, which places
 * the module's code and the scratch array in device memory: one more
 * reason to make the first call early, before the device's memory is
 * handed to another pool.
 * Errors: INVALID_ARGUMENT (NULL pointer, n_tokens < 1, top_k outside
 * [1, 64], n_experts < 1, n_tokens*top_k > 2^30), UNSUPPORTED (n_experts >
 * 1024), CUDA. */
MOEQ_API moeq_status moeq_route_noalloc(const int32_t *topk_ids, int32_t n_tokens, int32_t top_k,
                                        int32_t n_experts, int32_t *offsets_out, int32_t *perm_out,
                                        void *stream);

/* The router that produces a forward's routing ("MiMo-V2.6-Flash-RL GGUF for
 * a single DGX Spark", "Architecture notes": sigmoid routing, 8 of 256
 * routed experts per token, no shared expert).  For token t:
 *   z[t][e] = sum_h x[t][h] wr[e][h]                        (the logits)
 *   topk_ids[t] = the top_k experts of largest z, in descending z, equal z
 *                 to the lower expert id first
 *   topk_w[t][j] = s_j / sum_i s_i over the selected experts, where
 *                 s = 1 / (1 + e^-z) (MOEQ_SCORE_SIGMOID, the pages' router)
 *                 or s = e^(z - z_max) (MOEQ_SCORE_SOFTMAX, a softmax over
 *                 the selected logits)
 * The pages give no more: the matrix shape, the selection on z (the sigmoid
 * is increasing) and the normalisation over the selected experts are this
 * library's readings.
 *
 * moeq_router_upload: copies the router matrix, host f32 [n_experts][hidden]
 * row-major (every value finite and of magnitude <= 3.38e38), into the
 * layer and fixes the weighting `score` (moeq_score).  The library stores it
 * in its own layout and allocates, on first upload, the router's workspace
 * (sized by max_tokens); the caller may free wr when the call returns (it
 * synchronizes `stream`).  May be called again to replace the matrix.
 * Errors: INVALID_ARGUMENT (NULL, unknown score, a non-finite or too large
 * value), OUT_OF_MEMORY, CUDA. */
MOEQ_API moeq_status moeq_router_upload(moeq_layer_t layer, const float *wr, int32_t score, void *stream);

/* Run the router on x (device, the layer's act dtype, [n_tokens][hidden],
 * 4-byte aligned) into topk_ids (device int32 [n_tokens][top_k]) and topk_w
 * (device f32 [n_tokens][top_k]), and, when `logits` is not NULL, the logits
 * themselves (device f32 [n_tokens][n_experts]).  The logits are accumulated
 * in f32 from the exact f32 products of x and wr (for bf16 x the router
 * matrix is held as three bf16 terms whose sum is wr to 24 bits); the sum
 * over a row is split into K slices added in a fixed order, so results do
 * not depend on timing.  The selection is taken on those f32 logits, the
 * weights are computed in f32.  Asynchronous on `stream`; uses the router's
 * workspace (calls on one layer must be ordered).
 * Errors: INVALID_ARGUMENT (NULL, n_tokens outside [1, max_tokens],
 * misaligned x), NOT_UPLOADED (no router matrix), CUDA. */
MOEQ_API moeq_status moeq_router(moeq_layer_t layer, const void *x, int32_t n_tokens, int32_t *topk_ids,
                                 float *topk_w, float *logits, void *stream);

/* moeq_router followed by moeq_forward on the routing it produced: out =
 * the layer output of x (both device, act dtype, [n_tokens][hidden]);
 * topk_ids / topk_w are caller-owned device buffers that receive the
 * routing.  n_tokens == 0 is a no-op.  Errors: as moeq_router and
 * moeq_forward. */
MOEQ_API moeq_status moeq_forward_routed(moeq_layer_t layer, const void *x, int32_t n_tokens, int32_t *topk_ids,
                                         float *topk_w, void *out, void *stream);

/* VQ encoder: the indices that store a matrix in the VQ13 / VQ13_R8 format
 * ("MiMo-V2.6-Flash-RL UNCENSORED VQ GGUF", "Recipe": each 8-weight vector
 * of an expert row is replaced by the index of a codebook entry, the row
 * scaled by an f16 gain; a second, 256-entry book encodes the remainder the
 * first stage leaves, without changing the first stage's indices; the
 * assignment minimises an error weighted per column by importance).  The codebooks, gains and column weights are given; training
 * them is not part of this library.
 *   w           device f32 [n_rows][n_cols], row-major, 16-byte aligned;
 *               n_cols a multiple of 64
 *   gain        device f16 [n_rows] row gains, or NULL (gain 1)
 *   col_weight  device f32 [n_cols] importance of each column (>= 0), or
 *               NULL (all 1)
 *   book13      device bf16 [8192][8], 16-byte aligned
 *   book8       device bf16 [256][8], 16-byte aligned, or NULL (no residual
 *               stage; then idx8_out must be NULL too)
 *   idx13_out   device uint8 [n_rows][n_cols*13/64]: per row, the 13-bit
 *               indices as the little-endian bitstream of moeq_weights
 *   idx8_out    device uint8 [n_rows][n_cols/8], 8-byte aligned: residual
 *               indices, or NULL
 * For vector j of row n (columns 8j..8j+7) the base index c minimises
 * sum_i col_weight_i (w_i - g book13[c][i])^2 (g the row's gain); then, for
 * that c, the residual index r minimises sum_i col_weight_i
 * (w_i - g (book13[c][i] + book8[r][i]))^2.  The errors are evaluated in f32
 * in the expanded form g^2 sum cw b^2 - 2 g sum (cw w) b; ties go to the
 * lowest index; the base index does not depend on the residual stage.
 * Every output byte of the rows is written; the call allocates nothing and
 * is asynchronous on `stream` (current device).  Errors: INVALID_ARGUMENT
 * (NULL, sizes, alignment, book8 without idx8_out or the reverse), CUDA. */
MOEQ_API moeq_status moeq_vq_encode(const float *w, int32_t n_rows, int32_t n_cols, const uint16_t *gain,
                                    const float *col_weight, const uint16_t *book13, const uint16_t *book8,
                                    uint8_t *idx13_out, uint8_t *idx8_out, void *stream);

/* moeq_forward that also records five caller-created CUDA events (passed
 * as cudaEvent_t cast to void*) on `stream` at its phase boundaries:
 * events[0] before the first launch, [1] after route/bucket, [2] after the
 * gate/up + SwiGLU kernel, [3] after the down projection and combine, [4]
 * after the final cast.  Where a phase is fused into another, its two
 * events are recorded back to back.  For measuring kernel durations; the
 * results are those of moeq_forward.  Errors: as moeq_forward, and
 * INVALID_ARGUMENT for a NULL events array. */
MOEQ_API moeq_status moeq_forward_profiled(moeq_layer_t layer, const void *x, const int32_t *topk_ids,
                                           const float *topk_w, int32_t n_tokens, void *out, void *stream,
                                           void *const *events);

/* Decode projection `proj` of expert `expert` into out, device f32 [N][K],
 * logical layout.  Bit-exact: every element equals the f32 weight defined
 * by the format above (signed zeros, f32 subnormals and +-inf overflow of
 * an E8M0 x E2M1 product included).  Asynchronous on `stream`.
 * Errors: INVALID_ARGUMENT (expert or proj out of range, NULL out),
 * NOT_UPLOADED, CUDA. */
MOEQ_API moeq_status moeq_dequant(moeq_layer_t layer, int32_t expert, int32_t proj, float *out, void *stream);

/* The layer's device status word, read after synchronizing the device:
 * MOEQ_OK, or the first-raised device flag (MOEQ_ERR_ROUTE_OUT_OF_RANGE,
 * MOEQ_ERR_TIMEOUT).  clear != 0 resets it.
 * MOEQ_ERR_TIMEOUT means that a kernel's bounded wait on another part of
 * the same kernel (about a second; never expected in normal operation)
 * gave up: the kernel stopped issuing work, waited for its own copies and
 * tensor-core operations in flight, released its on-chip memory and
 * returned, so the device stays usable, but that forward's output is
 * undefined.  Clearing the status after a timeout also resets the grid
 * barrier of the one-launch MXFP4 decode step, which a forward that gave up
 * part-way can leave behind; until the status is cleared, later MXFP4
 * decode forwards on the layer are undefined too.  Errors:
 * INVALID_ARGUMENT, CUDA. */
MOEQ_API moeq_status moeq_layer_status(moeq_layer_t layer, int32_t clear);

/* Number of kernels the layer has launched so far (a launch captured into
 * a CUDA graph counts once, at capture); -1 for a NULL layer.  Lets a caller
 * check that the work ran in this library's kernels. */
MOEQ_API int64_t moeq_kernel_launches(moeq_layer_t layer);

/* Static description of a status code; never NULL. */
MOEQ_API const char *moeq_status_string(moeq_status s);

/* Free everything the layer owns (synchronizes its device first).
 * NULL is a no-op. */
MOEQ_API void moeq_layer_destroy(moeq_layer_t layer);

#ifdef __cplusplus
}
#endif

#endif /* MOEQ_H */
