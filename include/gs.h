/*
 * gs.h -- C ABI of a differentiable, tile-binned 3D Gaussian splatting
 * rasterizer for NVIDIA B200 (sm_100a).  Library: libgs.so.
 *
 * The hot path is four calls, made in this order on one CUDA stream:
 *
 *   gs_project       raw parameters -> per-Gaussian projected records
 *   gs_bin_and_sort  records -> (tile, Gaussian) pairs sorted by tile, then
 *                    by depth, plus each tile's [start, end) range
 *   gs_render_fwd    front-to-back alpha blend of every 16x16 tile
 *   gs_render_bwd    back-to-front gradient of the blend, then the chain rule
 *                    to the raw parameters
 *
 * Around them: gs_render_features_fwd/bwd (feature channels blended with the
 * forward's weights), gs_train_step (a training step over several cameras,
 * run as concurrent lanes, ending in gs_adam_step), gs_l1_loss_grad, the
 * work counter gs_render_stats, and host-side size, carve, status, error and
 * profiling calls.
 *
 * Sources (cited by page title and section):
 *   [GSP]  "Gaussian splatting in PyTorch" (coderigor.dev), s1-s8
 *   [WEEK] "SplatRs: The Week the Gap Closed", "Throughput: the tile
 *          rasterizer" (project, count, emit, sort, range, blend)
 *   [PIX4] "SplatRs: We Gave the Model 4x More Pixels and It Got Worse",
 *          "Lesson 2 -- Your GPU will lie by omission" (pair-list size,
 *          pre-flight guards, errors that must not be silent)
 *   [BLOG] 3D Gaussian Splatting course blog index (a backward pass that
 *          recomputes the blend weights instead of storing them)
 *   [DIST] "The backward pass I deleted trained the model the Nano runs",
 *          "Training a smaller scene" (a student optimised against the
 *          teacher's renders from sixty cameras)
 *
 * Conventions shared by every call
 *   - All floating point is IEEE single precision.
 *   - Every pointer inside gs_params, gs_grads, gs_projected and gs_bins,
 *     and every array argument, is DEVICE memory owned by the caller, unless
 *     the comment says "host".  The library never allocates or frees device
 *     memory; size queries tell the caller how much to allocate.
 *   - Arrays of 4-vectors must be 16-byte aligned; all others 4-byte aligned
 *     (GS_ERR_ALIGNMENT otherwise).
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *     call only enqueues work on it and returns, except where a comment says
 *     it synchronizes.
 *   - Return value: GS_OK (0), or a negative GS_ERR_* code.  No call aborts
 *     the process, throws, or fails silently ([PIX4] Lesson 2).  Arguments
 *     are checked before anything is launched; on an argument error nothing
 *     is enqueued.
 *   - The library holds no per-call state between calls; calls on different
 *     streams with disjoint buffers may run concurrently.
 */
#ifndef GS_H_
#define GS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GS_TILE 16 /* tile edge in pixels */

enum {
    GS_OK = 0,
    GS_ERR_INVALID_ARG = -1,    /* a size, pointer or camera value is out of range */
    GS_ERR_CAPACITY = -2,       /* the pair list needs more than max_pairs entries */
    GS_ERR_TOO_LARGE = -3,      /* N or max_pairs at or above 2^30 */
    GS_ERR_ALIGNMENT = -4,      /* a pointer is not aligned as documented */
    GS_ERR_CUDA = -5,           /* a CUDA runtime call or launch failed */
    GS_ERR_DEVICE_TIMEOUT = -6, /* a bounded device-side wait gave up (reserved:
                                   no kernel of this version waits on another) */
    GS_ERR_BOUNDS = -7          /* a kernel index was out of its array's range and the
                                   access was skipped; only libgs_check.so (built with
                                   GS_CHECK) tests indices, into bins->status */
};

/* Pinhole camera ([GSP] s3).  Host struct, passed by pointer. */
typedef struct gs_camera {
    float viewmat[16];    /* row-major 4x4 world-to-camera [R | t; 0 0 0 1], OpenCV
                             axes: +x right, +y down, +z forward */
    float fx, fy, cx, cy; /* intrinsics in pixels; pixel (row i, col j) is sampled
                             at (j + 0.5, i + 0.5) ([GSP] s5) */
    int32_t width, height;/* image size in pixels, each in [1, 65536] */
    float near_z;         /* Gaussians with camera z <= near_z are culled (0.01,
                             [GSP] s6) */
    float bg[3];          /* background colour, weighted by the final
                             transmittance ([GSP] s5) */
    uint32_t flags;       /* GS_FLAG_* bits; 0 = the pages' plain method.
                             Unknown bits are rejected (GS_ERR_INVALID_ARG). */
} gs_camera;

/* gs_camera.flags: opacity-aware tile cut ([GSP] s4, gsplat's extent of
 * sqrt(2 ln(255 o)) standard deviations).  gs_project narrows each tile
 * rectangle to the tile columns and rows where some pixel centre can still
 * pass the alpha >= 1/255 test of the blend: with the record's conic
 * (A, B, C) and opacity o, ell = ln(255 o) + 0.01 and q = A C - B^2, the
 * largest alpha on the pixel-centre column at horizontal offset dx is
 * o exp(-dx^2 q / (2 C)), so columns whose nearest centre is farther than
 * D_x = sqrt(2 ell C / q) from the mean are cut (rows likewise with
 * D_y = sqrt(2 ell A / q)); ell <= 0 cuts everything.  The cut is skipped
 * when A C > 1024 q (an ill-conditioned conic).  Every pixel of a cut tile
 * has alpha below 0.99 / 255, so the image, the final transmittance and the
 * gradients are those of the 3-sigma rectangle (up to alpha tests that
 * single-precision rounding leaves undecided within that 1 %), while the
 * pair count, the sort and the blend work shrink.  `last` (an index into a
 * tile's list) refers to the shorter lists. */
#define GS_FLAG_TIGHT_TILES 1u

/* gs_camera.flags: variants of the method the pages describe ([GSP] s4-s6).
 * GS_FLAG_ANTIALIASED: gs_project multiplies the opacity by
 *   sqrt(det S' / det S'') (0 when det S' <= 0), S' the 2D covariance before
 *   and S'' after the 0.3 dilation; gs_render_bwd differentiates through it.
 * GS_FLAG_STOP_INCLUSIVE: a pixel stops once T (1 - alpha) <= 1e-4 (gsplat)
 *   instead of < 1e-4 (3DGS).
 * GS_FLAG_CAP_0999: alpha = min(0.999, o G) (older gsplat) instead of 0.99.
 * GS_FLAG_RADII_AXIS: the tile rectangle uses gsplat's per-axis radii
 *   ceil(3.33 sqrt(S''_xx)), ceil(3.33 sqrt(S''_yy)) instead of 3DGS's
 *   ceil(3 sqrt(lambda_max)); the record's radius is the larger one.
 * GS_FLAG_RADII_OPACITY (with GS_FLAG_RADII_AXIS): the extent is
 *   min(3.33, sqrt(2 ln(255 o))) standard deviations (o the opacity the
 *   blend uses); a Gaussian with 255 o <= 1 touches no tile.
 * The render calls take the flags of the camera they are given, which must
 * be the camera the records were projected with. */
#define GS_FLAG_ANTIALIASED 2u
#define GS_FLAG_STOP_INCLUSIVE 4u
#define GS_FLAG_CAP_0999 8u
#define GS_FLAG_RADII_AXIS 16u
#define GS_FLAG_RADII_OPACITY 32u
/* GS_FLAG_DEPTH ([GSP] s5: channels of any kind blend alike): a fourth
 * channel, each Gaussian's camera z, blended with the colours' weights and
 * no background term: image and dL_dimage are [H][W][4] (R, G, B,
 * sum_i w_i z_i; divide by 1 - T_final for the expected depth), and the
 * backward carries the fourth channel's gradient into the means.  rgb[3] of
 * the projected record holds z. */
#define GS_FLAG_DEPTH 64u
#define GS_FLAGS_ALL 127u

/* Raw (unconstrained) parameters of N Gaussians ([GSP] s1), fp32, C-contiguous. */
typedef struct gs_params {
    const float *means;          /* [N][3] world-space centres */
    const float *log_scales;     /* [N][3] scale = exp(log_scale) per axis */
    const float *quats;          /* [N][4] (w, x, y, z), any norm; normalised with
                                    max(|q|, 1e-12) so zero gives the identity */
    const float *opacity_logits; /* [N]    opacity = sigmoid(logit) */
    const float *colors;         /* [N][3] RGB used directly (SH degree 0) */
} gs_params;

/* Gradients of a scalar loss with respect to gs_params, same layouts.
 * Overwritten (not accumulated) by gs_render_bwd. */
typedef struct gs_grads {
    float *means, *log_scales, *quats, *opacity_logits, *colors;
} gs_grads;

/* Projected records of N Gaussians, written by gs_project ([GSP] s1-s4).
 * The layout is public so that records computed elsewhere can be binned and
 * rendered.  gs_projected_carve lays all arrays out in one buffer. */
typedef struct gs_projected {
    float *xy_opacity_depth; /* [N][4]: mean2d x, y (px); opacity in (0,1); camera z */
    float *conic_radius;     /* [N][4]: A, B, C with sigma = 1/2 (A dx^2 + C dy^2) + B dx dy
                                ([GSP] s4); radius in px (an integer value) */
    float *rgb;              /* [N][4]: r, g, b, 0 */
    int32_t *rect;           /* [N][4]: tile x0, y0, x1, y1, inclusive, clamped to the
                                tile grid; x0 > x1 or y0 > y1 when nothing is touched */
    uint32_t *count;         /* [N]: tiles touched = rectangle area; 0 when culled */
} gs_projected;

/* Bytes of one buffer holding every gs_projected array for n Gaussians. */
size_t gs_projected_bytes(int64_t n);
/* Points the fields of *out into `base` (device, 256-byte aligned, at least
 * gs_projected_bytes(n) bytes).  Host-only arithmetic; launches nothing. */
int gs_projected_carve(void *base, int64_t n, gs_projected *out);

/* Binning state: the sorted pair list, per-tile ranges, status words and the
 * sort's scratch, all in one caller-owned device buffer carved by
 * gs_bins_carve.  A gs_bins carved for (n, max_pairs, width, height) serves
 * any call with at most n Gaussians and an image of at most that many tiles. */
typedef struct gs_bins {
    uint32_t *pair_tile;  /* [max_pairs] tile id (ty * tiles_x + tx) of each pair, ascending */
    uint32_t *pair_gid;   /* [max_pairs] Gaussian id of each pair; within a tile, ordered by
                             (float bits of camera z, id): the order of the 64-bit key
                             (tile << 32 | depth bits) of [WEEK] with ties by id */
    uint32_t *ranges;     /* [tiles][2] start, end of each tile's pairs; [0, 0) when empty */
    uint64_t *n_pairs;    /* [1] total pairs K of the last gs_bin_and_sort (also when
                             K > max_pairs) */
    int32_t *status;      /* [1] 0, or the GS_ERR_* code a kernel of the last
                             gs_bin_and_sort recorded (GS_ERR_CAPACITY) */
    int64_t max_pairs;    /* capacity of pair_tile / pair_gid */
    int64_t max_n;        /* largest N this buffer was carved for */
    int32_t max_tiles;    /* largest tile count this buffer was carved for */
    int32_t strategy;     /* GS_BIN_*: how gs_bin_and_sort sorts (0, automatic,
                             after gs_bins_carve); every strategy gives the same
                             pairs, ranges and K */
    void *scratch;        /* sort and scan scratch (internal layout) */
    size_t scratch_bytes;
} gs_bins;

/* gs_bins.strategy.  GS_BIN_PER_TILE groups the pairs by tile through
 * counts and scans and sorts every tile's list on its own by (depth bits,
 * id); GS_BIN_GLOBAL orders the Gaussians by depth once, emits the pairs in
 * that order and groups them by tile with stable radix passes over the tile
 * id only; both give the order of the key (tile << 32 | depth bits) with
 * ties by id.  GS_BIN_AUTO takes the global strategy when the capacity
 * holds at least 1024 pairs per tile of the frame (long lists, where the
 * per-tile sorts cost the most) and at least n, else the per-tile one. */
#define GS_BIN_AUTO 0
#define GS_BIN_PER_TILE 1
#define GS_BIN_GLOBAL 2

/* Bytes of one buffer holding a gs_bins for at most n Gaussians, max_pairs
 * pairs and a width x height image.  [PIX4] Lesson 2: 400k Gaussians at full
 * resolution needed > 16.7M pairs; size max_pairs from a first call's K. */
size_t gs_bins_bytes(int64_t n, int64_t max_pairs, int32_t width, int32_t height);
/* Carves *out from `base` (device, 256-byte aligned, gs_bins_bytes bytes).
 * Host-only arithmetic.  GS_ERR_TOO_LARGE if n or max_pairs >= 2^30. */
int gs_bins_carve(void *base, int64_t n, int64_t max_pairs, int32_t width, int32_t height,
                  gs_bins *out);

/* Projection ([GSP] s1-s4, s6), one thread per Gaussian: activations;
 * Sigma = R S S^T R^T; t = W mu + tv; cull if z <= near_z or any projected
 * value (the colour included) is not finite; J from x/z, y/z clamped to the
 * frustum widened by 0.3 of the half-FoV tangent;
 * Sigma' = J W Sigma W^T J^T + 0.3 I; det clamped
 * at 1e-10; conic = (c, -b, a)/det; radius = ceil(3 sqrt(lambda_max)) with
 * the root term floored at 0.1; mean2d = (fx x/z + cx, fy y/z + cy);
 * tile rectangle per axis floor((m -+ r)/16) in single precision, clamped
 * to the grid, narrowed by the opacity-aware cut when cam->flags has
 * GS_FLAG_TIGHT_TILES.  Culled Gaussians get count 0 and an empty rectangle.
 * n may be 0.  Errors: INVALID_ARG (n < 0, null pointer with n > 0, bad
 * camera), TOO_LARGE (n >= 2^30), ALIGNMENT, CUDA. */
int gs_project(const gs_camera *cam, int64_t n, const gs_params *params, const gs_projected *out,
               void *stream);

/* Binning and sorting ([WEEK] count, emit, sort, range): counts the pairs
 * of every tile, scans the counts into per-tile ranges, emits one entry per
 * (tile, drawable Gaussian) at its tile's range, and sorts each tile's list
 * by (float bits of camera z, Gaussian id).  The result is the pair order of
 * the 64-bit key (tile << 32 | depth bits) with ties by id.
 * It also leaves in bins->scratch the order in which the blend kernels take
 * the tiles (longest list first); the render calls need bins filled by this
 * call.
 * Uses `proj` from gs_project (or any records in that layout): binning reads
 * each record's depth and its rectangle (clamped to the tile grid; `count` is
 * not read), so no record can produce a tile id outside the grid.
 * If n_pairs_host (HOST pointer) is non-NULL the call synchronizes `stream`,
 * stores K there, and returns GS_ERR_CAPACITY if K > bins->max_pairs (the
 * caller may regrow and retry) or the status a kernel recorded.  If it is
 * NULL nothing synchronizes: K and any error land in bins->n_pairs and
 * bins->status (read them with gs_read_status); on an error every tile's
 * range is left empty, so the render draws only background.
 * Errors: INVALID_ARG, TOO_LARGE, ALIGNMENT, CUDA, CAPACITY. */
int gs_bin_and_sort(const gs_camera *cam, int64_t n, const gs_projected *proj,
                    const gs_bins *bins, int64_t *n_pairs_host, void *stream);

/* Forward blend ([GSP] s5; [WEEK] blend), one CTA per 16x16 tile (tiles
 * taken in the order gs_bin_and_sort left in bins->scratch): for each
 * pixel, its tile's pairs in order, sigma as above at (j + 0.5, i + 0.5),
 * alpha = min(0.99, o exp(-sigma)); skip if sigma < 0 or alpha < 1/255;
 * stop (without adding) once T (1 - alpha) < 1e-4; C += c alpha T (the cap,
 * the stop test and a depth channel per the camera's flags).
 * Outputs (device, caller-owned, fully overwritten):
 *   image   [H][W][3]  C + T_final bg ([H][W][4] with GS_FLAG_DEPTH)
 *   T_final [H][W]     final transmittance
 *   last    [H][W]     one past the index (into pair_gid) of the last entry the
 *                      pixel added; the tile's start when it added none
 * Errors: INVALID_ARG, ALIGNMENT, CUDA. */
int gs_render_fwd(const gs_camera *cam, int64_t n, const gs_projected *proj, const gs_bins *bins,
                  float *image, float *T_final, uint32_t *last, void *stream);

/* gs_render_fwd with the training step's L1 loss ([GSP] s7) taken in the
 * same kernel, after each pixel's blend: loss = mean |image - target| over
 * every value, dL/dimage = sign(image - target) / count with sign(0) = 0 and
 * count = width x height x channels (the values gs_l1_loss_grad writes for
 * the same image, bit for bit; the loss is summed per CTA, so its last bits
 * depend on the order of the atomic adds).
 *   image, T_final, last  as gs_render_fwd
 *   target     [H][W][channels]  device, 4-byte aligned, read
 *   dL_dimage  [H][W][channels]  device, 4-byte aligned, written
 *   loss       [1]               device, nullable; zeroed, then the loss
 * Errors: INVALID_ARG, ALIGNMENT, CUDA. */
int gs_render_fwd_l1(const gs_camera *cam, int64_t n, const gs_projected *proj, const gs_bins *bins,
                     float *image, float *T_final, uint32_t *last, const float *target, float *dL_dimage,
                     float *loss, void *stream);

/* Backward ([GSP] s6; [BLOG]): one CTA per tile walks each pixel's added
 * entries back to front from `last`, recovering T_i = T_{i+1} / (1 - alpha_i)
 * instead of storing weights; dL/dalpha_i = T_i <c_i - R_i, g> with
 * R_last = bg, R_{i-1} = alpha_i c_i + (1 - alpha_i) R_i; no gradient through
 * a capped alpha; per-pixel terms are reduced across the warp before global
 * atomics.  Then the chain rule to the raw parameters, one thread per
 * Gaussian.  Culled Gaussians get exact zeros.
 *   dL_dimage [H][W][3]  gradient of the loss with respect to `image`
 *                        ([H][W][4] with GS_FLAG_DEPTH)
 *   grad2d    [N][12]    caller scratch, 16-byte aligned; overwritten.  On
 *                        return holds per Gaussian dL/d(mean2d x, y), dL/dA,
 *                        dL/dB, dL/dC, dL/dopacity, dL/d(r, g, b), dL/d of
 *                        the depth channel's value (0 without the flag), 0, 0
 *   grads                raw-parameter gradients, overwritten
 * `proj`, `bins`, T_final and last must be those of the forward call.
 * Errors: INVALID_ARG, ALIGNMENT, CUDA. */
int gs_render_bwd(const gs_camera *cam, int64_t n, const gs_params *params,
                  const gs_projected *proj, const gs_bins *bins, const float *T_final,
                  const uint32_t *last, const float *dL_dimage, float *grad2d,
                  const gs_grads *grads, void *stream);

/* Feature channels ([GSP] s5: the final weighted sum costs the same for
 * channels of any kind, RGB, depth or features).  Each Gaussian carries F
 * feature values; the forward's weights w_i = alpha_i T_i blend them with
 * no background: out[p][f] = sum_i w_i features[g_i][f].  The walk is the
 * forward's (same tests, same stop, same rounding), run once per chunk of
 * eight channels (and once for a last chunk of four when F is not a
 * multiple of 8).
 *   features [N][F]  F a positive multiple of 4 (at most 1024), 16-byte aligned
 *   out      [H][W][F], overwritten
 * `proj` and `bins` must be those gs_render_fwd used for this camera.
 * Errors: INVALID_ARG, ALIGNMENT, CUDA. */
int gs_render_features_fwd(const gs_camera *cam, int64_t n, const gs_projected *proj,
                           const gs_bins *bins, const float *features, int32_t F, float *out,
                           void *stream);

/* Backward of the feature channels: dL/dfeatures, and the features' share
 * of the blend gradient (through alpha: dL/dalpha_i = T_i <f_i - R_i, g>,
 * the colours' formula with the features' dL/dout as g and no background)
 * mapped to the raw parameters and ADDED into grads.  Call it after
 * gs_render_bwd (which overwrites grads with the colours' share).
 *   dL_dout      [H][W][F]  gradient of the loss with respect to out
 *   grad2d       [N][12]    caller scratch, 16-byte aligned
 *   dL_dfeatures [N][F]     overwritten
 *   grads                   raw-parameter gradients, accumulated into
 * T_final and last must be gs_render_fwd's for the same proj and bins.
 * Errors: INVALID_ARG, ALIGNMENT, CUDA. */
int gs_render_features_bwd(const gs_camera *cam, int64_t n, const gs_params *params,
                           const gs_projected *proj, const gs_bins *bins, const float *T_final,
                           const uint32_t *last, const float *features, int32_t F,
                           const float *dL_dout, float *grad2d, float *dL_dfeatures,
                           const gs_grads *grads, void *stream);

/* Work counts of one forward frame, for roofline arithmetic (not part of the
 * rendering path; it re-walks the blend with counters and is slower).
 * counts (device, [4] uint64, overwritten):
 *   [0] entries visited by the forward: per pixel, its tile's entries up to
 *       and including the one that stopped it (all of them if none did)
 *   [1] entries added (contributing) over all pixels
 *   [2] entries the backward walks: per pixel, last - tile start
 *   [3] pixels
 * `last` must be the forward's output for the same proj and bins.
 * Errors: INVALID_ARG, ALIGNMENT, CUDA. */
int gs_render_stats(const gs_camera *cam, int64_t n, const gs_projected *proj,
                    const gs_bins *bins, const uint32_t *last, uint64_t *counts, void *stream);

/* L1 photometric loss of the training step: loss = mean |image - target| over
 * `count` values; dL_dimage = sign(image - target) / count (sign(0) = 0).
 * loss (device, nullable) receives the mean.  Errors: INVALID_ARG, CUDA. */
int gs_l1_loss_grad(const float *image, const float *target, int64_t count, float *dL_dimage,
                    float *loss, void *stream);

/* ------------------------------------------------------------- training
 * The optimisation loop of [GSP] s7 (render, L1 loss against the target,
 * backward, one Adam step over the raw parameters with a learning rate per
 * parameter group), batched over several cameras as in [DIST] (a student
 * fitted to the teacher's renders from sixty cameras, so that it becomes a
 * 3D model rather than one memorised view). */

/* Five writable arrays in the gs_params layout: the parameters Adam
 * updates, its two moments, a gradient slot. */
typedef gs_grads gs_param_set;

/* Adam hyperparameters ([GSP] s7: torch.optim.Adam with per-parameter
 * learning rates; the pages name 1.6e-4 x scene extent for means (decayed),
 * 5e-3 for scales, 2.5e-2 for opacities and 1e-3 for quaternions). */
typedef struct gs_adam_config {
    float lr[5];   /* means, log_scales, quats, opacity_logits, colors; finite, >= 0 */
    float eps;     /* > 0, usually 1e-8 (Kingma & Ba; torch's default) */
    double beta1;  /* [0, 1), usually 0.9 */
    double beta2;  /* [0, 1), usually 0.999.  The bias corrections use the
                      betas in double precision; the moment updates use
                      beta and 1 - beta each rounded once to single */
} gs_adam_config;

/* One Adam step over the raw parameters, fused with the sum of gradient
 * slots (Kingma & Ba's algorithm in the form torch.optim.Adam evaluates it):
 *   g = grad_scale * sum_s slots[s]      (summed in slot order)
 *   t = *step + 1
 *   m = beta1 m + (1 - beta1) g
 *   v = beta2 v + (1 - beta2) g^2
 *   p = p - (lr / (1 - beta1^t)) m / (sqrt(v) / sqrt(1 - beta2^t) + eps)
 * with lr the learning rate of p's group; then *step = t.  The step count
 * lives on the device so that a captured CUDA graph replays correctly; the
 * bias corrections are evaluated in double precision.
 *   params    parameters, updated in place
 *   slots     HOST array of n_slots (1..16) gradient sets (device arrays)
 *   m, v      moments, updated in place (zero before the first step)
 *   step      DEVICE int64: steps taken so far; incremented by the call
 *   grad_out  nullable: receives g
 * Arrays of quaternions must be 16-byte aligned.  n may be 0 (only the
 * counter moves).  Errors: INVALID_ARG (n < 0, n_slots out of range, a null
 * array with n > 0, a learning rate or beta out of range), TOO_LARGE,
 * ALIGNMENT, CUDA. */
int gs_adam_step(int64_t n, const gs_param_set *params, const gs_param_set *slots, int32_t n_slots,
                 float grad_scale, const gs_param_set *m, const gs_param_set *v,
                 const gs_adam_config *cfg, int64_t *step, const gs_param_set *grad_out,
                 void *stream);

/* The buffers one camera chain of gs_train_step runs in: the render state of
 * its current camera, and the lane's gradient slot (the sum of its
 * cameras' raw-parameter gradients).  All device arrays are caller-owned. */
typedef struct gs_train_lane {
    gs_projected proj;   /* records of N Gaussians */
    gs_bins bins;        /* pair list: max_pairs must hold every camera's K */
    float *image;        /* [H][W][C] */
    float *T_final;      /* [H][W] */
    uint32_t *last;      /* [H][W] */
    float *dL_dimage;    /* [H][W][C] */
    float *grad2d;       /* [N][12], 16-byte aligned */
    gs_param_set grads;  /* gradient slot, overwritten */
    void *stream;        /* cudaStream_t the lane's cameras run on; may be the
                            step's own stream (then no event is needed) */
    void *done;          /* cudaEvent_t recorded on the lane's stream after its
                            last camera (ignored when stream is the step's) */
} gs_train_lane;

/* One training step over n_cams cameras.  Camera b runs on lane
 * b mod n_lanes, after the lane's previous camera: gs_project,
 * gs_bin_and_sort (asynchronous), gs_render_fwd, the L1 loss of camera b's
 * image against targets[b] (loss_b = mean |image - target| over H W C values),
 * and gs_render_bwd, whose raw-parameter gradients are written (first camera
 * of the lane) or added (the others) into the lane's slot.  Lanes run
 * concurrently: each waits on `fork` (recorded on `stream` by the call) and
 * `stream` waits on each lane's `done`.  Then, on `stream`, gs_adam_step
 * with the lanes' slots and grad_scale = 1 / n_cams, i.e. the gradient of
 * the mean of the cameras' losses.
 *   cams      HOST array; all of one width, height and channel count (C = 3,
 *             or 4 with GS_FLAG_DEPTH)
 *   params    raw parameters, updated in place by Adam
 *   targets   [n_cams][H][W][C]
 *   lanes     HOST array of n_lanes (1..16) lanes with disjoint buffers
 *   fork      cudaEvent_t (needed when a lane has its own stream)
 *   cfg       Adam hyperparameters; NULL skips Adam (and `m`, `v`, `step`):
 *             the step then only writes the mean gradient to grad_out,
 *             e.g. for an all-reduce across GPUs before gs_adam_step
 *   losses    nullable, DEVICE [n_cams] float: loss_b
 *   cam_stats nullable, DEVICE [n_cams][2] int64: camera b's binning status
 *             (GS_OK or GS_ERR_CAPACITY, the pair list then left empty and
 *             the camera's image background only) and its pair count K
 *   grad_out  nullable (required when cfg is NULL): the mean gradient
 * Nothing synchronizes; read cam_stats to detect an overflowed pair list.
 * The call may be captured in a CUDA graph (the lanes' streams join the
 * capture through `fork`).  Errors: INVALID_ARG, TOO_LARGE, ALIGNMENT,
 * CUDA. */
int gs_train_step(const gs_camera *cams, int32_t n_cams, int64_t n, const gs_param_set *params,
                  const float *targets, const gs_train_lane *lanes, int32_t n_lanes, void *fork,
                  const gs_param_set *m, const gs_param_set *v, const gs_adam_config *cfg,
                  int64_t *step, float *losses, int64_t *cam_stats, const gs_param_set *grad_out,
                  void *stream);

/* gs_bin_and_sort for callers that cannot allocate device memory.
 *
 * There is no counterpart in the source pages: this is a deployment variant.
 * gs_bin_and_sort needs a caller-allocated scratch buffer (gs_bins) for its
 * per-tile binning stages: the [CTA][tile] count matrix, the per-tile totals
 * and ranges, the tile order, the emitted sort keys and the long-list sort's
 * ping-pong arrays.  Some callers cannot allocate it:
 * a real-time viewer's frame loop that must never call cudaMalloc/cudaFree
 * (both can synchronize the whole device and stall a frame), or a plug-in
 * whose host application owns all device memory and hands it no allocator.
 * This call keeps that scratch in one fixed-size array inside libgs.so
 * instead, so the caller passes only its inputs and outputs.
 *
 * Limits (GS_ERR_TOO_LARGE beyond them, nothing launched): n <= 262,144
 * Gaussians, max_pairs <= 1,048,576 pairs, at most 65,536 tiles.  The array
 * (about 33 MB) is part of the library's device image: every GPU on which
 * the library is used holds it until the process exits.
 *
 * Inputs: cam, n, proj as for gs_bin_and_sort.  Outputs (device, caller-owned):
 *   pair_tile [max_pairs], pair_gid [max_pairs]  the sorted pair list, the same
 *                                                values gs_bin_and_sort writes
 *   ranges    [tiles][2]                         each tile's [start, end)
 *   *n_pairs_host (HOST, required)               K, the total pair count
 * The call synchronizes `stream` to read K and the kernels' status back, and
 * returns GS_ERR_CAPACITY when K > max_pairs (the pair arrays are then left
 * undefined and the ranges empty), as gs_bin_and_sort does.  It calls no allocating routine.
 *
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  Every call, on every stream, shares the one
 * array per device and clears the parts that must start at zero itself;
 * calls whose work overlaps on the GPU (two streams, or two host threads)
 * race on it and must be serialized by the caller. */
int gs_bin_and_sort_static(const gs_camera *cam, int64_t n, const gs_projected *proj,
                           uint32_t *pair_tile, uint32_t *pair_gid, uint32_t *ranges,
                           int64_t max_pairs, int64_t *n_pairs_host, void *stream);

/* Synchronizes `stream`, then returns bins->status and stores K in
 * *n_pairs_host (HOST, nullable).  GS_ERR_CUDA if the copy fails. */
int gs_read_status(const gs_bins *bins, int64_t *n_pairs_host, void *stream);

/* Synchronizes `stream` and returns the device error word the kernels of
 * the last gs_bin_and_sort on `bins` recorded: GS_OK, or the GS_ERR_* code
 * (GS_ERR_CAPACITY).  The word lives in the caller's bins buffer, not in the
 * library (which holds no per-call state), so the call takes `bins`.  Same
 * as gs_read_status without the pair count.  GS_ERR_CUDA if the copy fails;
 * GS_ERR_INVALID_ARG for a NULL or incomplete bins. */
int gs_last_device_error(const gs_bins *bins, void *stream);

/* Bytes of the scratch one bin-and-sort needs for max_pairs pairs and
 * `tiles` tiles: gs_bins_bytes for any n (the layout does not depend on N)
 * and a grid of `tiles` tiles.  0 if max_pairs < 0 or tiles < 1. */
size_t gs_sort_bytes(int64_t max_pairs, int32_t tiles);

/* Static, human-readable text for a return code. */
const char *gs_error_string(int code);

/* Per-stage timing.  Between gs_profile_begin and gs_profile_end the library
 * records a CUDA event pair around each stage it launches (one kernel, or a
 * few back to back: the count and column scan of binning, the per-tile
 * sorts), on the stream it launches it on.  gs_profile_end synchronizes
 * those events and fills at most max_stats entries (one per stage name:
 * `launches` counts the kernels, `total_ms` the time); returns how many.
 * Not thread-safe; meant for benchmarks. */
typedef struct gs_profile_stat {
    char name[32];
    int32_t launches;
    float total_ms;
} gs_profile_stat;
int gs_profile_begin(int32_t max_launches);
int gs_profile_end(gs_profile_stat *out, int32_t max_stats);

/* ABI version of this header. */
int gs_version(void);

#ifdef __cplusplus
}
#endif
#endif /* GS_H_ */
