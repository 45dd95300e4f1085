/*
 * vggt_attn.h -- C ABI of the B200 (sm_100a) hot path of VGGT's
 * alternating-attention trunk: frame attention, global attention and
 * AVGGT's training-free Subsampled Global Attention (SGA).
 *
 * Sources (web pages, cited by title and section):
 *  [VGGT]  "VGGT CVPR25 Best Paper" notes, section "Alternating-Attention":
 *          frame-wise self-attention (tokens of one view attend within that
 *          view) alternates with global self-attention (the tokens of all N
 *          views form one sequence); no cross-attention.
 *  [AVGGT] "AVGGT: Rethinking Global Attention for Accelerating VGGT",
 *          technical summary section 3 (Methodology): step one turns early
 *          global layers into frame attention; step two, SGA, keeps every
 *          query, keeps K/V for all special tokens plus the patch tokens on a
 *          fixed s_h x s_w grid (one per window), restores each token's own
 *          (diagonal) term, replaces all dropped K/V columns by one mean key
 *          and one mean value, and lets the three parts share one softmax
 *          normalisation.
 *  [DISSECT] "Vggt cvpr2025 dissection", section 2.5: 518x518 views with
 *          14x14 patches give a 37x37 patch grid.
 *
 * Token layout.  Q, K, V and O are bf16, contiguous [N, L, H, d]
 * (= [S, H, d] with S = N * L; the global view needs no copy).  Each frame
 * holds L = n_special + patch_h * patch_w tokens: the special tokens first,
 * then the patch grid row-major, so token t = n*L + p and patch (r, c) is
 * p = n_special + r*patch_w + c.  d must be 64.
 *
 * SGA, exactly (per head, scale s, logits s_ij = s * q_i . k_j):
 *   kept set K: every special token, and patch (r, c) when r is the centre
 *   row of its stride-s_h window and c the centre column of its stride-s_w
 *   window (windows [a*s, min((a+1)*s, n)), shorter last window included,
 *   centre = a*s + (len-1)/2); D = the other patch tokens; M_i = |D| - [i in D];
 *   kbar, vbar = means of k_j, v_j over j in D;
 *   O_i = ( sum_{j in K} e^{s_ij} v_j + [i in D] e^{s_ii} v_i
 *           + M_i e^{s q_i.kbar} vbar ) / (same with every v replaced by 1),
 *   i.e. the mean column enters with logit s*q_i.kbar + ln M_i; when
 *   M_i = 0 it is absent.
 *
 * Conventions for every call:
 *  - Device pointers are caller-owned and must stay valid until the work
 *    queued on `stream` has finished.  The library never allocates or frees
 *    memory and keeps no state between calls except a per-device flag that
 *    records kernel attributes and a 4-byte device error word.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  All
 *    work is queued asynchronously on it; no call synchronises.
 *  - Bad arguments are rejected before anything is queued: the call returns
 *    VGGT_ERR_INVALID_ARG / VGGT_ERR_UNSUPPORTED / VGGT_ERR_WORKSPACE.
 *    A failed launch returns VGGT_ERR_CUDA.  Every wait inside a kernel is
 *    bounded; a wait that runs out sets the device error word, the kernel
 *    returns early, and vggt_check() reports VGGT_ERR_TIMEOUT.
 *  - Device pointers to bf16 data must be 16-byte aligned; O must not
 *    overlap Q, K or V.
 */
#ifndef VGGT_ATTN_H
#define VGGT_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define VGGT_ABI_VERSION 3

typedef enum {
    VGGT_OK = 0,
    VGGT_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, overlap, bad scale or stride */
    VGGT_ERR_UNSUPPORTED = 2, /* head_dim != 64, n_heads > 64, or S too large for 32-bit indices */
    VGGT_ERR_WORKSPACE = 3,   /* SGA workspace smaller than vggt_sga_workspace_bytes() */
    VGGT_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed */
    VGGT_ERR_TIMEOUT = 5,     /* a bounded in-kernel wait ran out (see vggt_check) */
    VGGT_ERR_BOUNDS = 6       /* debug builds only: a device index check failed (see vggt_check) */
} vggt_status;

typedef struct {
    int32_t n_frames;  /* N >= 1 */
    int32_t n_special; /* special tokens per frame, >= 0 (VGGT: 5) */
    int32_t patch_h;   /* patch rows h >= 0 (518x518 views: 37) */
    int32_t patch_w;   /* patch columns w >= 0 */
    int32_t n_heads;   /* H, 1..64 */
    int32_t head_dim;  /* d, must be 64 */
} vggt_shape;

/* Human-readable name of a status code; never NULL. */
const char *vggt_status_string(vggt_status status);

/* VGGT_ABI_VERSION of the loaded library. */
int32_t vggt_abi_version(void);

/* S = N * (n_special + h*w), or -1 if the shape is invalid. */
int64_t vggt_num_tokens(vggt_shape shape);

/* Closed-form SGA counts [AVGGT section 3, step two]: kept tokens
 * N * (n_special + ceil(h/s_h) * ceil(w/s_w)) and dropped tokens
 * N * h*w - N * ceil(h/s_h)*ceil(w/s_w).  -1 if shape or stride is invalid. */
int64_t vggt_sga_num_kept(vggt_shape shape, int32_t s_h, int32_t s_w);
int64_t vggt_sga_num_dropped(vggt_shape shape, int32_t s_h, int32_t s_w);

/* Bytes of device workspace vggt_attn_sga() needs for this shape and stride
 * (0 if invalid).  Layout, from the start of the workspace (offsets in bytes,
 * HD = n_heads * 64):
 *   [0, 4*HD)          kbar, float [H][64]   (written when |D| > 0)
 *   [4*HD, 8*HD)       vbar, float [H][64]
 *   then, 256-aligned: per-block partial sums, float [640][2][HD]
 *   then, 256-aligned: gathered kept keys,   bf16 [n_kept][H][64]
 *   then, 256-aligned: gathered kept values, bf16 [n_kept][H][64]
 * The contents after a call are informative only (tests read kbar/vbar). */
size_t vggt_sga_workspace_bytes(vggt_shape shape, int32_t s_h, int32_t s_w);

/* SGA index [AVGGT section 3, step two: uniform grid K/V sampling].
 * kept_idx: int32 [n_kept], device, written with the kept token indices in
 *           ascending order (n_kept = vggt_sga_num_kept()).
 * mult:     int32 [S], device, written with M_t = |D| - [t in D].
 * The index depends only on (shape without H/d, s_h, s_w) and can be reused
 * across heads and layers.  One kernel launch. */
vggt_status vggt_sga_build_index(vggt_shape shape, int32_t s_h, int32_t s_w,
                                 int32_t *kept_idx, int32_t *mult, void *stream);

/* Frame attention [VGGT "Alternating-Attention"; AVGGT section 3 step one]:
 * O_i = softmax_j(scale * q_i . k_j) v_j over the keys j of i's own frame.
 * q, k, v: bf16 [N, L, H, 64], device, read-only.  o: bf16 [N, L, H, 64],
 * device, written.  lse: optional float [S, H] (NULL to skip), written with
 * the natural log of sum_j exp(scale * q_i . k_j).  scale > 0 (1/sqrt(64) is
 * the usual choice).  One kernel launch. */
vggt_status vggt_attn_frame(const void *q, const void *k, const void *v, void *o, float *lse,
                            vggt_shape shape, float scale, void *stream);

/* Global attention [VGGT "Alternating-Attention"]: as vggt_attn_frame but j
 * runs over all S tokens of all frames.  One kernel launch. */
vggt_status vggt_attn_global(const void *q, const void *k, const void *v, void *o, float *lse,
                             vggt_shape shape, float scale, void *stream);

/* Subsampled Global Attention [AVGGT section 3, step two], defined at the top
 * of this file.  kept_idx and mult must be the output of
 * vggt_sga_build_index() for the same shape and stride (device, read-only).
 * workspace: device, >= vggt_sga_workspace_bytes() bytes, 256-byte aligned,
 * overwritten.  lse as for vggt_attn_frame (the diagonal and mean terms
 * included).  Three kernel launches (gather + mean-fill partial sums, mean
 * finalisation (skipped when |D| = 0), attention). */
vggt_status vggt_attn_sga(const void *q, const void *k, const void *v, void *o, float *lse,
                          vggt_shape shape, int32_t s_h, int32_t s_w,
                          const int32_t *kept_idx, const int32_t *mult,
                          void *workspace, size_t workspace_bytes, float scale, void *stream);

/* Row blocks of global attention and SGA, for query-row (sequence)
 * sharding.  The pages describe no parallelism; these are the building
 * blocks of the split where each GPU owns a block of query rows (whole
 * frames, e.g.), gathers every key/value into its own memory and computes
 * only its rows.  The arithmetic per row is exactly that of the full call.
 *
 * vggt_attn_global_rows: rows 0..n_rows-1 of q_rows / o_rows / lse_rows are
 * n_rows query tokens of a sequence of S = vggt_num_tokens(shape) tokens
 * [VGGT "Alternating-Attention", global attention]; k, v hold all S tokens
 * ([S, H, 64] bf16, device, read-only).  q_rows, o_rows: bf16
 * [n_rows, H, 64]; lse_rows: optional float [n_rows, H].  1 <= n_rows <= S.
 * Global attention does not depend on where the rows sit in the sequence.
 * One kernel launch.
 *
 * vggt_attn_sga_rows: the same for SGA [AVGGT section 3, step two]: the
 * rows are tokens row0 .. row0 + n_rows - 1 of the sequence (needed for the
 * multiplicity M_i and the diagonal term, which reads k and v at row
 * row0 + i); kept_idx and mult are the index of the whole sequence; the
 * workspace is as for vggt_attn_sga (the mean-fill runs over all S tokens of
 * k and v).  0 <= row0, row0 + n_rows <= S.  Three kernel launches. */
vggt_status vggt_attn_global_rows(const void *q_rows, int32_t n_rows, const void *k, const void *v, void *o_rows,
                                  float *lse_rows, vggt_shape shape, float scale, void *stream);
vggt_status vggt_attn_sga_rows(const void *q_rows, int32_t row0, int32_t n_rows, const void *k, const void *v,
                               void *o_rows, float *lse_rows, vggt_shape shape, int32_t s_h, int32_t s_w,
                               const int32_t *kept_idx, const int32_t *mult, void *workspace,
                               size_t workspace_bytes, float scale, void *stream);

/* SGA with the query rows split across GPUs and only the kept rows
 * exchanged [AVGGT section 3, step two: the attention of a query needs the
 * kept keys/values of every frame, its own key/value, and the mean of the
 * dropped ones].  Each GPU holds the Q, K, V rows of a contiguous block of
 * frames; the kept rows of a frame depend only on that frame, so:
 *
 *   1. vggt_sga_gather_partial on each GPU's own frames (local_shape: the
 *      shape with n_frames = its frame count) writes their kept K and V rows
 *      (kept_k, kept_v: bf16 [vggt_sga_num_kept(local_shape, s_h, s_w), H,
 *      64], in sequence order) and the fp32 sums of K and of V over their
 *      dropped tokens (dropped_sums: float [2][H * 64], K first; zeros when
 *      the stride drops nothing).  workspace: device, 256-byte aligned,
 *      vggt_sga_partial_workspace_bytes(local_shape) bytes (per-block sums;
 *      0 means an invalid shape).  Two kernel launches.
 *   2. The caller concatenates every GPU's kept rows in frame order (an
 *      all-gather; they are the kept rows of the whole sequence in sequence
 *      order) and adds the dropped sums (an all-reduce of 2 * H * 64 floats).
 *   3. vggt_attn_sga_gathered for this GPU's query rows row0 .. row0 + n_rows
 *      - 1 of the whole sequence (shape: all frames): q_rows, k_rows, v_rows
 *      are those rows' Q, K, V ([n_rows, H, 64] bf16; k_rows / v_rows give
 *      the diagonal term), kept_k / kept_v the gathered kept rows, dropped_sums
 *      the summed dropped sums, mult the multiplicities of the whole sequence
 *      (vggt_sga_build_index).  means (float [2][H * 64], device, 16-byte
 *      aligned) receives k-bar and v-bar (dropped_sums / |D|).  o_rows,
 *      lse_rows as in vggt_attn_sga_rows.  Two kernel launches (one when the
 *      stride drops nothing).
 *
 * The kept-row exchange is vggt_sga_num_kept(shape) rows of K and of V
 * (150 MB at N = 100, stride 2) instead of all S rows (563 MB).  The result
 * equals vggt_attn_sga_rows' up to the order of the fp32 sums behind
 * k-bar and v-bar.  Invalid arguments (shapes, strides, scale, null or
 * misaligned pointers, overlapping outputs) return VGGT_ERR_INVALID_ARG
 * before any launch; a workspace below the size, VGGT_ERR_WORKSPACE. */
size_t vggt_sga_partial_workspace_bytes(vggt_shape local_shape);
vggt_status vggt_sga_gather_partial(const void *k, const void *v, vggt_shape local_shape, int32_t s_h, int32_t s_w,
                                    void *kept_k, void *kept_v, float *dropped_sums, void *workspace,
                                    size_t workspace_bytes, void *stream);
vggt_status vggt_attn_sga_gathered(const void *q_rows, int32_t row0, int32_t n_rows, const void *k_rows,
                                   const void *v_rows, const void *kept_k, const void *kept_v,
                                   const float *dropped_sums, const int32_t *mult, float *means, void *o_rows,
                                   float *lse_rows, vggt_shape shape, int32_t s_h, int32_t s_w, float scale,
                                   void *stream);

/* Register attention [VGGT-Omega notes, improvement one "Register
 * Attention"]: in a quarter of the global layers VGGT-Omega restricts
 * cross-frame attention to the register tokens (16 per frame) plus the
 * camera token; image tokens take no part in it.  Here: global attention
 * whose queries and keys are the n_special special tokens of all N frames,
 * O_i = softmax_j(scale * q_i . k_j) v_j for special tokens i, j.
 * Only the special-token rows of o (and of lse, when not NULL) are written;
 * every patch-token row is left untouched.  1 <= n_special <= 128
 * (VGGT_ERR_INVALID_ARG below, VGGT_ERR_UNSUPPORTED above).  The special
 * tokens are read in place (no copy, no workspace): one kernel launch. */
vggt_status vggt_attn_register(const void *q, const void *k, const void *v, void *o, float *lse,
                               vggt_shape shape, float scale, void *stream);

/* SGA without a caller-provided workspace.  The pages have no counterpart:
 * this entry point exists for callers that cannot allocate device memory at
 * the point of the call -- e.g. code running under a fixed, pre-planned
 * memory budget, inside a runtime that owns every allocation, or in a
 * region where cudaMalloc is not allowed (it can synchronise the device).
 * It computes exactly what vggt_attn_sga() computes, with the same
 * arguments minus the workspace; the scratch it needs (the per-head means,
 * the per-block partial sums and the gathered kept K/V) lives in one
 * file-scope device array of VGGT_SGA_STATIC_SCRATCH_BYTES (16 MiB) built
 * into the library.  Every GPU on which the library's device code is loaded
 * holds that array until the process exits.
 *  - Size limit: returns VGGT_ERR_WORKSPACE, before queuing anything, when
 *    vggt_sga_workspace_bytes(shape, s_h, s_w) > VGGT_SGA_STATIC_SCRATCH_BYTES
 *    (e.g. with H = 16 about 2,800 kept tokens: N = 4 at stride 2x2 fits).
 *  - Set-up: the first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current) and caches it with
 *    the context's unique ID; make that first call before any stream
 *    capture.  A context destroyed by cudaDeviceReset and created again has
 *    a new ID, so the next call looks the address up again (make that call
 *    before any capture too).  No call allocates or frees memory (no
 *    cudaMalloc, cudaFree or allocating library routine).
 *  - Argument checks: the size limit first, then the same pointer, scale and
 *    index checks as vggt_attn_sga(), all before the device is touched.
 *  - Sharing: all calls on a device use the same array, which keeps the last
 *    call's contents.  Nothing in it has to start at zero (every byte a call
 *    reads was written earlier in that same call), but calls whose work
 *    overlaps on the GPU (different streams, no ordering between them) race
 *    on the array and give wrong results: order them on one stream. */
#define VGGT_SGA_STATIC_SCRATCH_BYTES ((size_t)16 << 20)
vggt_status vggt_attn_sga_noalloc(const void *q, const void *k, const void *v, void *o, float *lse,
                                  vggt_shape shape, int32_t s_h, int32_t s_w,
                                  const int32_t *kept_idx, const int32_t *mult, float scale, void *stream);

/* Fused QKV projection with a 2D rotary position embedding.  [Feed-forward
 * optimization in Visual Geometry Grounded and 3DGS, Cut3R part, section
 * 3.5 "position encoding"]: RoPE is applied to Q and K before every
 * attention; the pages give no formula, so this 2D form is a reading:
 *   y[t] = W x[t] + b (C = H*64 inputs, 3C outputs);
 *   Q = y[0:C], K = y[C:2C], V = y[2C:3C], each written as [S, H, 64];
 *   in Q and K, a patch token at grid (r, c) is rotated by position r in
 *   the first 32 dimensions of every head and by c in the last 32; within
 *   a 32-dimension half, dimensions i and i + 16 (i < 16) form a pair
 *   (a, b) -> (a cos - b sin, b cos + a sin) at angle pos * base^(-i/16);
 *   special tokens are not rotated.
 * x: bf16 [S, C] device, read-only.  w: bf16 [3C, C] device, read-only (the
 * out x in layout of a linear layer).  bias: float [3C] device or NULL.
 * q, k, v: bf16 [S, H, 64] device, written; they must not overlap each
 * other or the inputs.  rope_base > 0 (100 is the usual choice for 2D
 * grids).  n_heads must be even and patch_h, patch_w <= 128
 * (VGGT_ERR_UNSUPPORTED otherwise).  One kernel launch. */
vggt_status vggt_qkv_rope(const void *x, const void *w, const float *bias, void *q, void *k, void *v,
                          vggt_shape shape, float rope_base, void *stream);

/* Output projection of an attention layer: y[t] = W o[t] + b, the same
 * tensor-core GEMM as vggt_qkv_rope without the rotation.  o: bf16 [S, H,
 * 64] (= [S, C], C = H*64) device, read-only, e.g. an attention output.
 * w: bf16 [C, C] device (out x in).  bias: float [C] device or NULL.
 * y: bf16 [S, C] device, written; it must not overlap the inputs.
 * n_heads must be even.  One kernel launch. */
vggt_status vggt_out_proj(const void *o, const void *w, const float *bias, void *y, vggt_shape shape,
                          void *stream);

/* Layer schedule of an alternating-attention trunk.  [VGGT
 * "Alternating-Attention"] frame and global layers alternate; [AVGGT section
 * 3] step one turns the early global layers into frame attention and step
 * two runs SGA in the remaining ones; [VGGT-Omega, improvement one] a
 * quarter of the global layers become register attention.  A schedule lists
 * the attention layers of a trunk in order, one descriptor each. */
typedef enum {
    VGGT_LAYER_FRAME = 0,
    VGGT_LAYER_GLOBAL = 1,
    VGGT_LAYER_SGA = 2,     /* stride s_h x s_w */
    VGGT_LAYER_REGISTER = 3 /* needs n_special >= 1; writes only special-token rows of o */
} vggt_layer_kind;

typedef struct {
    int32_t kind; /* vggt_layer_kind */
    int32_t s_h;  /* SGA stride, >= 1; ignored for the other kinds */
    int32_t s_w;
} vggt_layer;

#define VGGT_MAX_LAYERS 1024      /* layers per schedule */
#define VGGT_MAX_SGA_STRIDES 8    /* distinct SGA strides per schedule */

/* Bytes of device workspace vggt_attn_schedule() needs (0 when no layer
 * needs any), -1 if the shape or a descriptor is invalid.  Layout (every part 256-byte aligned): for each
 * distinct SGA stride, in order of first use, its index (kept_idx int32
 * [n_kept], then mult int32 [S]); then one SGA workspace as large as the
 * largest vggt_sga_workspace_bytes() of those strides, shared by the SGA
 * layers in turn.  Frame, global and register layers need none. */
int64_t vggt_schedule_workspace_bytes(vggt_shape shape, const vggt_layer *layers, int32_t n_layers);

/* Runs n_layers attention layers in order on `stream`.
 * q, k, v, o: host arrays of n_layers device pointers; layer i reads q[i],
 * k[i], v[i] and writes o[i] with the same layout and rules as the
 * single-layer calls (layers may share buffers, e.g. to time a trunk on one
 * set of inputs).  layers: host array of n_layers descriptors,
 * 0 <= n_layers <= VGGT_MAX_LAYERS.  workspace: device, 256-byte aligned,
 * >= vggt_schedule_workspace_bytes(), overwritten; it must not overlap any
 * layer's buffers (may be NULL when that size is 0: no SGA layer).
 * The SGA index of each distinct stride is built once per call (one launch)
 * and reused by every SGA layer with that stride: it depends only on the
 * token layout and the stride.  Every argument of every layer is checked
 * before anything is queued.  Launches: one per distinct stride, plus each
 * layer's own (frame, global, register 1; SGA 2 or 3). */
vggt_status vggt_attn_schedule(const void *const *q, const void *const *k, const void *const *v,
                               void *const *o, vggt_shape shape, const vggt_layer *layers, int32_t n_layers,
                               float scale, void *workspace, size_t workspace_bytes, void *stream);

/* Test hook for the failure path (the pages have no counterpart): runs
 * vggt_attn_global with the first scores of query rows 0..127 of every CTA
 * never signalled, and with every in-kernel wait bounded by wait_limit_ns
 * (1 ms .. 4 s) instead of the default 4 s.  The waits that depend on the
 * missing signal run out, every role of the kernel unwinds (copies and
 * UMMAs in flight are drained, TMEM is freed), the kernel returns, and the
 * next vggt_check() reports VGGT_ERR_TIMEOUT; o is left incomplete.  The
 * CUDA context stays usable.  Nothing faults, traps or hangs. */
vggt_status vggt_test_attn_global_stall(const void *q, const void *k, const void *v, void *o,
                                        vggt_shape shape, float scale, uint64_t wait_limit_ns, void *stream);

/* Synchronises `stream`, then reads and clears this device's error word.
 * Returns VGGT_ERR_TIMEOUT if a bounded wait ran out in any kernel since the
 * last check, VGGT_ERR_BOUNDS if (debug build) a device index check failed,
 * VGGT_ERR_CUDA if the stream reports an error, else VGGT_OK.  detail, if
 * not NULL, receives the raw word: bit 0 = timeout, bits 8..15 = the code of
 * the first wait site that gave up, bit 1 = index check, bits 16..23 = the
 * code of the first check site that failed. */
vggt_status vggt_check(void *stream, uint32_t *detail);

/* Debug builds (the pages have no counterpart).  The library built with
 * -DVGGT_DEBUG (libvggt_attn_debug.so, `python -m
 * feed_forward_view_vggt_b200.build --debug`) checks the computed indices of
 * its kernels on the device before each guarded access -- the output row and
 * head of the attention epilogue, the SGA seed rows, the mean-fill's token
 * rows and gathered slots, the kept token ids of the index build, the token
 * rows and the QKV projection's output rows.  A
 * failed check skips that access and records its site in the error word, so
 * the next vggt_check() returns VGGT_ERR_BOUNDS; nothing traps.  Returns 1
 * for such a build, 0 for the release library (where the checks compile
 * away). */
int32_t vggt_debug_checks(void);

#ifdef __cplusplus
}
#endif

#endif /* VGGT_ATTN_H */
