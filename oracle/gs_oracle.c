/*
 * gs_oracle.c -- plain, slow CPU oracle for the differentiable tile-binned
 * 3D Gaussian Splatting rasterizer.
 *
 * TEST INFRASTRUCTURE ONLY.  This library exists to check the CUDA path.
 * Only the test suite, the smoke check and the benchmark's CPU-baseline leg
 * may load it.  It shares no code, header, table or constant with the CUDA
 * library, and the CUDA library never calls it.
 *
 * What it computes, and where the pages define it (cited by page title and
 * section; abbreviations used below):
 *   [GSP]  "Gaussian splatting in PyTorch"
 *            s1 "What the optimiser stores: raw parameters and activations"
 *            s2 "Sigma = R S S^T R^T, by broadcasting"
 *            s3 "Into the camera and onto the screen"
 *            s4 "The low-pass filter, the conic and the radius"
 *            s5 "Compositing as tensor ops"
 *            s6 "Differentiable end to end -- and NaN-free"
 *            s8 "Dense vs tiled, and what to say in an interview"
 *   [WEEK] "SplatRs: The Week the Gap Closed", "Throughput: the tile
 *          rasterizer" (project, count, emit, sort, range, blend; a naive
 *          O(pixels x gaussians) renderer as the oracle)
 *
 * Arithmetic: IEEE double throughout, compiled without FMA contraction and
 * without fast-math.  The pages state the blend's thresholds as single
 * precision literals ([GSP] s5 listing: 0.99f, 1.f/255.f, 1e-4f); every
 * integer-valued decision (radius ceiling, tile rectangle, the three blend
 * tests, depth order) is therefore taken on the double value rounded once to
 * float, against those float constants.  Values themselves stay double.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - pixel (row i, col j) is sampled at (j + 0.5, i + 0.5)          [GSP] s5
 *   - stop test is strict: next_T < 1e-4 stops, the stopping entry is
 *     not added                                                  [GSP] s5 (3DGS)
 *   - radius = ceil(3 sqrt(lambda_max)), lambda from the dilated matrix,
 *     root term floored at 0.1                                   [GSP] s4 (3DGS)
 *   - tile rectangle of a splat: per axis lo = floor((m - r)/16),
 *     hi = floor((m + r)/16), clamped to the tile grid, in float.
 *     A pixel is considered by a splat only if its tile is inside this
 *     rectangle: this is the tiled method's cutoff, applied to the naive
 *     render so that both compute the same function.
 *   - optional opacity-aware tile cut ([GSP] s4, gsplat's extent of
 *     sqrt(2 ln(255 o)) standard deviations), taken per tile column and row
 *     against pixel centres so that it only removes tiles in which no pixel
 *     can pass the alpha >= 1/255 test (see opacity_cut)
 *   - colour parameter used directly as RGB (SH degree 0, no offset)
 *   - a Gaussian is culled (no tiles, exactly zero gradient) if its camera
 *     z <= near_z, or if any projected value (its colour included) is not
 *     finite                                                     [GSP] s6
 */
#include <math.h>
#include <float.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_TILE 16

/* Camera: row-major world-to-camera 4x4, OpenCV axes (+x right, +y down,
 * +z forward), pinhole intrinsics in pixels.                    [GSP] s3 */
typedef struct {
    double viewmat[16];
    double fx, fy, cx, cy;
    int32_t width, height;
    double near_z;
    double bg[3];
    int32_t flags;        /* ORC_FLAG_* bits: the variants below */
} orc_camera;

/* Variants of the method the pages describe, as camera flag bits (the values
 * the library's camera uses for the same options). */
#define ORC_FLAG_TIGHT_TILES    1  /* opacity-aware tile cut (opacity_cut)            */
#define ORC_FLAG_ANTIALIASED    2  /* [GSP] s4: opacity x sqrt(det S' / det S'')      */
#define ORC_FLAG_STOP_INCLUSIVE 4  /* [GSP] s5, gsplat: stop once next_T <= 1e-4      */
#define ORC_FLAG_CAP_0999       8  /* [GSP] s6, older gsplat: alpha cap 0.999         */
#define ORC_FLAG_RADII_AXIS    16  /* [GSP] s4, gsplat: radii ceil(3.33 sqrt(S''_xx)), */
                                   /* ceil(3.33 sqrt(S''_yy)) per axis                */
#define ORC_FLAG_RADII_OPACITY 32  /* with RADII_AXIS: min(3.33, sqrt(2 ln(255 o)))   */
                                   /* standard deviations; 255 o <= 1 touches nothing */
#define ORC_FLAG_DEPTH         64  /* [GSP] s5: a fourth channel, camera z, blended */
                                   /* with the colours' weights ("C channels of any */
                                   /* kind cost the same"); no background term      */
#define ORC_GSPLAT_SIGMAS 3.33
#define ORC_MAX_CH 4
static int orc_channels(const orc_camera *cam) { return (cam->flags & ORC_FLAG_DEPTH) ? 4 : 3; }
#define ORC_ALPHA_CAP_0999_F 0.999f

/* Single-precision decision constants, as the [GSP] s5 listing writes them. */
#define ORC_ALPHA_CAP_F   0.99f
#define ORC_ALPHA_MIN_F   (1.f / 255.f)
#define ORC_T_MIN_F       1e-4f

/* Constants of the projection ([GSP] s2-s4, s6). */
#define ORC_QUAT_EPS      1e-12
#define ORC_EPS2D         0.3
#define ORC_DET_MIN       1e-10
#define ORC_LAMBDA_FLOOR  0.1
#define ORC_RADIUS_SIGMAS 3.0
#define ORC_FRUSTUM_WIDEN 0.3

/* ------------------------------------------------------------------ */
/* [GSP] s2: unit quaternion (w, x, y, z) -> 3x3 rotation, normalising with
 * max(|q|, 1e-12) so that the zero quaternion gives the identity.          */
void orc_quat_to_rotmat(const double *q, double *R)
{
    double norm = sqrt(q[0] * q[0] + q[1] * q[1] + q[2] * q[2] + q[3] * q[3]);
    if (norm < ORC_QUAT_EPS) norm = ORC_QUAT_EPS;
    double w = q[0] / norm, x = q[1] / norm, y = q[2] / norm, z = q[3] / norm;
    R[0] = 1.0 - 2.0 * (y * y + z * z);
    R[1] = 2.0 * (x * y - w * z);
    R[2] = 2.0 * (x * z + w * y);
    R[3] = 2.0 * (x * y + w * z);
    R[4] = 1.0 - 2.0 * (x * x + z * z);
    R[5] = 2.0 * (y * z - w * x);
    R[6] = 2.0 * (x * z - w * y);
    R[7] = 2.0 * (y * z + w * x);
    R[8] = 1.0 - 2.0 * (x * x + y * y);
}

/* [GSP] s2: Sigma = M M^T with M = R diag(s), s = exp(log_scale)
 * (column j of R scaled by s_j). */
void orc_covariance3d(const double *q, const double *log_scale, double *Sigma)
{
    double R[9], M[9];
    orc_quat_to_rotmat(q, R);
    for (int i = 0; i < 3; i++)
        for (int j = 0; j < 3; j++) M[3 * i + j] = R[3 * i + j] * exp(log_scale[j]);
    for (int i = 0; i < 3; i++)
        for (int j = 0; j < 3; j++) {
            double acc = 0.0;
            for (int k = 0; k < 3; k++) acc += M[3 * i + k] * M[3 * j + k];
            Sigma[3 * i + j] = acc;
        }
}

/* Everything the projection of one Gaussian computes, kept for the
 * backward pass (which re-derives it rather than storing it). */
typedef struct {
    int valid;
    double q[4], qnorm, qhat[4];
    double R[9], s[3], M[9], Sigma[9];
    double W[9], tv[3];
    double t[3];
    double Sc[9];
    double lim_x_lo, lim_x_hi, lim_y_lo, lim_y_hi;
    int clamped_x, clamped_y;
    double jx, jy;
    double J[6];
    double a, b, c;        /* dilated 2D covariance entries (00, 01, 11) */
    double det;
    int det_clamped;
    double conic[3];       /* A, B, C */
    double mean2d[2];
    double opacity;
    double lambda_max;
    double radius_value;   /* 3 sqrt(lambda) before the ceiling */
    double opacity_raw;    /* sigmoid(logit) */
    double det_orig;       /* det of the undilated 2D covariance */
    double comp;           /* antialiasing compensation (1 without the flag) */
    double rx_value, ry_value;  /* per-axis radii before the ceiling */
    int extent_empty;      /* RADII_OPACITY and 255 o <= 1: no tiles */
} orc_proj;

static void project_one(const double *mean, const double *log_scale, const double *quat,
                        double opacity_logit, const orc_camera *cam, orc_proj *P)
{
    memset(P, 0, sizeof(*P));
    /* [GSP] s1: activations. */
    for (int k = 0; k < 4; k++) P->q[k] = quat[k];
    double qn = sqrt(quat[0] * quat[0] + quat[1] * quat[1] + quat[2] * quat[2] + quat[3] * quat[3]);
    P->qnorm = qn;
    double qd = qn < ORC_QUAT_EPS ? ORC_QUAT_EPS : qn;
    for (int k = 0; k < 4; k++) P->qhat[k] = quat[k] / qd;
    orc_quat_to_rotmat(quat, P->R);
    for (int j = 0; j < 3; j++) P->s[j] = exp(log_scale[j]);
    P->opacity = 1.0 / (1.0 + exp(-opacity_logit));
    P->opacity_raw = P->opacity;
    P->comp = 1.0;

    /* [GSP] s2: Sigma = (R S)(R S)^T. */
    for (int i = 0; i < 3; i++)
        for (int j = 0; j < 3; j++) P->M[3 * i + j] = P->R[3 * i + j] * P->s[j];
    for (int i = 0; i < 3; i++)
        for (int j = 0; j < 3; j++) {
            double acc = 0.0;
            for (int k = 0; k < 3; k++) acc += P->M[3 * i + k] * P->M[3 * j + k];
            P->Sigma[3 * i + j] = acc;
        }

    /* [GSP] s3: world to camera, t = W mu + tv, Sigma_c = W Sigma W^T. */
    for (int i = 0; i < 3; i++) {
        for (int j = 0; j < 3; j++) P->W[3 * i + j] = cam->viewmat[4 * i + j];
        P->tv[i] = cam->viewmat[4 * i + 3];
    }
    for (int i = 0; i < 3; i++) {
        double acc = P->tv[i];
        for (int j = 0; j < 3; j++) acc += P->W[3 * i + j] * mean[j];
        P->t[i] = acc;
    }
    double WS[9];
    for (int i = 0; i < 3; i++)
        for (int j = 0; j < 3; j++) {
            double acc = 0.0;
            for (int k = 0; k < 3; k++) acc += P->W[3 * i + k] * P->Sigma[3 * k + j];
            WS[3 * i + j] = acc;
        }
    for (int i = 0; i < 3; i++)
        for (int j = 0; j < 3; j++) {
            double acc = 0.0;
            for (int k = 0; k < 3; k++) acc += WS[3 * i + k] * P->W[3 * j + k];
            P->Sc[3 * i + j] = acc;
        }

    double tx = P->t[0], ty = P->t[1], tz = P->t[2];
    /* [GSP] s6: cull z <= near; nothing below divides by a culled z. */
    if (!(tz > cam->near_z)) { P->valid = 0; return; }

    /* [GSP] s3: x/z and y/z clamped to the frustum widened by 0.3 of the
     * half-FoV tangent on each side, for J only. */
    double tan_fovx = 0.5 * cam->width / cam->fx;
    double tan_fovy = 0.5 * cam->height / cam->fy;
    P->lim_x_lo = -(cam->cx / cam->fx + ORC_FRUSTUM_WIDEN * tan_fovx);
    P->lim_x_hi = (cam->width - cam->cx) / cam->fx + ORC_FRUSTUM_WIDEN * tan_fovx;
    P->lim_y_lo = -(cam->cy / cam->fy + ORC_FRUSTUM_WIDEN * tan_fovy);
    P->lim_y_hi = (cam->height - cam->cy) / cam->fy + ORC_FRUSTUM_WIDEN * tan_fovy;
    double xz = tx / tz, yz = ty / tz;
    double cxz = xz, cyz = yz;
    P->clamped_x = 0;
    P->clamped_y = 0;
    if (xz < P->lim_x_lo) { cxz = P->lim_x_lo; P->clamped_x = 1; }
    if (xz > P->lim_x_hi) { cxz = P->lim_x_hi; P->clamped_x = 1; }
    if (yz < P->lim_y_lo) { cyz = P->lim_y_lo; P->clamped_y = 1; }
    if (yz > P->lim_y_hi) { cyz = P->lim_y_hi; P->clamped_y = 1; }
    P->jx = tz * cxz;
    P->jy = tz * cyz;

    /* [GSP] s3: J = [[fx/z, 0, -fx x/z^2], [0, fy/z, -fy y/z^2]]. */
    P->J[0] = cam->fx / tz;
    P->J[1] = 0.0;
    P->J[2] = -cam->fx * P->jx / (tz * tz);
    P->J[3] = 0.0;
    P->J[4] = cam->fy / tz;
    P->J[5] = -cam->fy * P->jy / (tz * tz);

    /* Sigma' = J Sigma_c J^T. */
    double JS[6];
    for (int i = 0; i < 2; i++)
        for (int j = 0; j < 3; j++) {
            double acc = 0.0;
            for (int k = 0; k < 3; k++) acc += P->J[3 * i + k] * P->Sc[3 * k + j];
            JS[3 * i + j] = acc;
        }
    double cov[4];
    for (int i = 0; i < 2; i++)
        for (int j = 0; j < 2; j++) {
            double acc = 0.0;
            for (int k = 0; k < 3; k++) acc += JS[3 * i + k] * P->J[3 * j + k];
            cov[2 * i + j] = acc;
        }

    /* [GSP] s4: dilate by 0.3 I, clamp det at 1e-10, conic = (c, -b, a)/det. */
    P->a = cov[0] + ORC_EPS2D;
    P->b = cov[1];
    P->c = cov[3] + ORC_EPS2D;
    double det = P->a * P->c - P->b * P->b;
    P->det_clamped = 0;
    if (det < ORC_DET_MIN) { det = ORC_DET_MIN; P->det_clamped = 1; }
    P->det = det;
    P->conic[0] = P->c / det;
    P->conic[1] = -P->b / det;
    P->conic[2] = P->a / det;

    /* [GSP] s4, 3DGS rule: lambda_max = mid + sqrt(max(mid^2 - det, 0.1)). */
    double mid = 0.5 * (P->a + P->c);
    double disc = mid * mid - det;
    if (disc < ORC_LAMBDA_FLOOR) disc = ORC_LAMBDA_FLOOR;
    P->lambda_max = mid + sqrt(disc);
    P->radius_value = ORC_RADIUS_SIGMAS * sqrt(P->lambda_max);

    /* [GSP] s4, antialiased mode: the opacity is scaled by
     * sqrt(det Sigma' / det Sigma'') (0 when det Sigma' <= 0), which keeps a
     * small splat's total energy instead of fattening it. */
    P->det_orig = cov[0] * cov[3] - cov[1] * cov[1];
    if (cam->flags & ORC_FLAG_ANTIALIASED) {
        P->comp = P->det_orig > 0.0 ? sqrt(P->det_orig / det) : 0.0;
        P->opacity = P->opacity_raw * P->comp;
    }
    /* [GSP] s4, gsplat radii: the 3.33-sigma extent of the ellipse along x
     * and y, optionally shrunk to where the (compensated) opacity fades
     * below 1/255. */
    P->rx_value = P->ry_value = P->radius_value;
    P->extent_empty = 0;
    if (cam->flags & ORC_FLAG_RADII_AXIS) {
        double e = ORC_GSPLAT_SIGMAS;
        if (cam->flags & ORC_FLAG_RADII_OPACITY) {
            double l = log(255.0 * P->opacity);
            if (l > 0.0) {
                double ee = sqrt(2.0 * l);
                if (ee < e) e = ee;
            } else {
                e = 0.0;
                P->extent_empty = 1;
            }
        }
        P->rx_value = e * sqrt(P->a);
        P->ry_value = e * sqrt(P->c);
    }

    /* [GSP] s3: the 2D mean is not clamped. */
    P->mean2d[0] = cam->fx * tx / tz + cam->cx;
    P->mean2d[1] = cam->fy * ty / tz + cam->cy;

    P->valid = isfinite(P->mean2d[0]) && isfinite(P->mean2d[1]) && isfinite(P->conic[0]) &&
               isfinite(P->conic[1]) && isfinite(P->conic[2]) && isfinite(P->radius_value) &&
               isfinite(P->opacity);
}

static double dist_to_int(double v) { return fabs(v - nearbyint(v)); }

/* Slack of the opacity-aware cut, in ln(alpha): a tile is cut only where
 * every pixel has alpha below e^-0.01 / 255 (1 % under the threshold). */
#define ORC_CUT_SLACK    0.01
/* Largest A C / (A C - B^2) at which the cut is taken. */
#define ORC_CUT_MAX_COND 1024.0

/* Opacity-aware tile cut ([GSP] s4: gsplat shrinks a splat's extent to where
 * it fades below 1/255, sqrt(2 ln(255 o)) standard deviations).  Taken per
 * tile column and row against pixel centres:
 *   on the vertical line at horizontal offset dx from the mean, sigma is
 *   smallest at dy = -B dx / C, where it is dx^2 (A C - B^2) / (2 C); so every
 *   pixel of a tile column whose nearest centre is farther than
 *   D_x = sqrt(2 ell C / (A C - B^2)), ell = ln(255 o) + slack, from mx has
 *   alpha < e^-slack / 255 and fails the 1/255 test.  Rows likewise with
 *   D_y = sqrt(2 ell A / (A C - B^2)).
 * Column tx holds centres 16 tx + 0.5 ... 16 tx + 15.5, so it is kept iff
 *   16 tx + 0.5 <= mx + D_x and 16 tx + 15.5 >= mx - D_x,
 * i.e. tx in [ceil((mx - D_x - 15.5)/16), floor((mx + D_x - 0.5)/16)].
 * ell <= 0 (o <= e^-slack / 255): no pixel can pass, nothing is kept.
 * Not taken (all four bounds infinite) when A C - B^2 <= 0 or
 * A C > 1024 (A C - B^2): there the rounding of a single-precision sigma
 * near the threshold can exceed the slack.
 * Writes cut = {lo x, hi x, lo y, hi y} (tiles, integral or infinite).
 * Returns how far its decisions sit from flipping, as the smallest relative
 * perturbation of the conic (or, for ell, of the opacity) that could flip
 * one, to first order: |cond - 1024| / (2 cond^2) for the condition test
 * (cond moves by about 2 cond^2 per unit relative change of A, B, C), |ell|
 * for the ell test, and for each of the four bounds the pixel distance of
 * m -+ D from the nearest flip divided by (1 + D cond) (D moves by about
 * D cond). */
static double opacity_cut(double mx, double my, double A, double B, double C, double o,
                          double cut[4])
{
    cut[0] = cut[2] = -INFINITY;
    cut[1] = cut[3] = INFINITY;
    double q = A * C - B * B;
    if (!(q > 0.0)) return INFINITY;
    double cond = A * C / q;
    double margin = fabs(cond - ORC_CUT_MAX_COND) / (2.0 * cond * cond);
    if (!(cond <= ORC_CUT_MAX_COND)) return margin;
    double ell = log(255.0 * o) + ORC_CUT_SLACK;
    if (fabs(ell) < margin) margin = fabs(ell);
    if (ell <= 0.0) {
        cut[0] = cut[2] = INFINITY;
        cut[1] = cut[3] = -INFINITY;
        return margin;
    }
    const double D[2] = {sqrt(2.0 * ell * C / q), sqrt(2.0 * ell * A / q)};
    const double m[2] = {mx, my};
    for (int axis = 0; axis < 2; axis++) {
        double lo = (m[axis] - D[axis] - (ORC_TILE - 0.5)) / ORC_TILE;
        double hi = (m[axis] + D[axis] - 0.5) / ORC_TILE;
        cut[2 * axis] = ceil(lo);
        cut[2 * axis + 1] = floor(hi);
        double d0 = ORC_TILE * dist_to_int(lo) / (1.0 + D[axis] * cond);
        double d1 = ORC_TILE * dist_to_int(hi) / (1.0 + D[axis] * cond);
        if (d0 < margin) margin = d0;
        if (d1 < margin) margin = d1;
    }
    return margin;
}

/* Tile rectangle of a splat, in float (a pixel grid decision taken in single
 * precision), from per-axis radii (equal under the 3DGS rule).  With cut
 * (from opacity_cut) the bounds are narrowed to it before clamping.  Returns the tile count; writes x0, y0, x1, y1
 * (inclusive), with x0 > x1 or y0 > y1 when nothing is touched. */
static int32_t tile_rect_f32(float mx, float my, float rx, float ry, int32_t tiles_x, int32_t tiles_y,
                             const double *cut, int32_t *rect)
{
    float lx = floorf((mx - rx) * (1.0f / ORC_TILE));
    float hx = floorf((mx + rx) * (1.0f / ORC_TILE));
    float ly = floorf((my - ry) * (1.0f / ORC_TILE));
    float hy = floorf((my + ry) * (1.0f / ORC_TILE));
    if (cut) {
        lx = fmaxf(lx, (float)cut[0]);
        hx = fminf(hx, (float)cut[1]);
        ly = fmaxf(ly, (float)cut[2]);
        hy = fminf(hy, (float)cut[3]);
    }
    lx = fminf(fmaxf(lx, 0.0f), (float)tiles_x);
    ly = fminf(fmaxf(ly, 0.0f), (float)tiles_y);
    hx = fmaxf(fminf(hx, (float)(tiles_x - 1)), -1.0f);
    hy = fmaxf(fminf(hy, (float)(tiles_y - 1)), -1.0f);
    rect[0] = (int32_t)lx;
    rect[1] = (int32_t)ly;
    rect[2] = (int32_t)hx;
    rect[3] = (int32_t)hy;
    if (rect[0] > rect[2] || rect[1] > rect[3]) return 0;
    return (rect[2] - rect[0] + 1) * (rect[3] - rect[1] + 1);
}


/* Projection of n Gaussians ([GSP] s1-s4, s6).  Outputs, per Gaussian:
 *   mean2d[2], conic[3] (A, B, C), cov2d[3] (dilated a, b, c), opacity,
 *   depth (camera z), color[3] (passed through), radius (float, integral:
 *   the larger of the two radii), radius_xy[2] (per-axis radii, equal under
 *   the 3DGS rule), rect[4] (tile x0, y0, x1, y1), count (tiles touched),
 *   valid (0/1), radius_margin (smallest |radius before the ceiling -
 *   nearest integer|, px),
 *   rect_margin (min over the four rectangle edges of |(m +- r)/16 - nearest
 *   integer|, in tiles), cut_margin (what opacity_cut returns with
 *   ORC_FLAG_TIGHT_TILES, and |ln(255 o)| with the opacity-aware radii;
 *   else infinity).  The margins say how close an
 *   integer decision came to flipping.  Returns 0, or -1 on bad arguments. */
int orc_project(int64_t n, const double *means, const double *log_scales, const double *quats,
                const double *opacity_logits, const double *colors, const orc_camera *cam,
                double *mean2d, double *conic, double *cov2d, double *opacity, double *depth,
                double *color, float *radius, float *radius_xy, int32_t *rect, int32_t *count,
                uint8_t *valid, double *radius_margin, double *rect_margin, double *cut_margin)
{
    if (n < 0 || cam->width <= 0 || cam->height <= 0) return -1;
    int32_t tiles_x = (cam->width + ORC_TILE - 1) / ORC_TILE;
    int32_t tiles_y = (cam->height + ORC_TILE - 1) / ORC_TILE;
    for (int64_t g = 0; g < n; g++) {
        orc_proj P;
        project_one(means + 3 * g, log_scales + 3 * g, quats + 4 * g, opacity_logits[g], cam, &P);
        const int nc = orc_channels(cam);
        for (int k = 0; k < 3; k++) color[nc * g + k] = colors[3 * g + k];
        if (nc == 4) color[4 * g + 3] = P.t[2];  /* the depth channel: camera z */
        depth[g] = P.t[2];
        opacity[g] = P.opacity;
        /* the colour is a projected value too: not finite -> culled ([GSP] s6) */
        P.valid = P.valid && isfinite(colors[3 * g]) && isfinite(colors[3 * g + 1]) &&
                  isfinite(colors[3 * g + 2]);
        valid[g] = (uint8_t)P.valid;
        if (!P.valid) {
            mean2d[2 * g] = mean2d[2 * g + 1] = 0.0;
            conic[3 * g] = conic[3 * g + 1] = conic[3 * g + 2] = 0.0;
            cov2d[3 * g] = cov2d[3 * g + 1] = cov2d[3 * g + 2] = 0.0;
            radius[g] = 0.0f;
            radius_xy[2 * g] = radius_xy[2 * g + 1] = 0.0f;
            rect[4 * g] = 0; rect[4 * g + 1] = 0; rect[4 * g + 2] = -1; rect[4 * g + 3] = -1;
            count[g] = 0;
            radius_margin[g] = INFINITY;
            rect_margin[g] = INFINITY;
            cut_margin[g] = INFINITY;
            continue;
        }
        mean2d[2 * g] = P.mean2d[0];
        mean2d[2 * g + 1] = P.mean2d[1];
        for (int k = 0; k < 3; k++) conic[3 * g + k] = P.conic[k];
        cov2d[3 * g] = P.a;
        cov2d[3 * g + 1] = P.b;
        cov2d[3 * g + 2] = P.c;
        /* radii: ceiling taken on the float-rounded values */
        const float rxy[2] = {ceilf((float)P.rx_value), ceilf((float)P.ry_value)};
        radius[g] = rxy[0] > rxy[1] ? rxy[0] : rxy[1];
        radius_xy[2 * g] = rxy[0];
        radius_xy[2 * g + 1] = rxy[1];
        radius_margin[g] = fmin(dist_to_int(P.rx_value), dist_to_int(P.ry_value));
        const int tight = (cam->flags & ORC_FLAG_TIGHT_TILES) != 0;
        double cut[4];
        cut_margin[g] = INFINITY;
        if (tight)
            cut_margin[g] = opacity_cut(P.mean2d[0], P.mean2d[1], P.conic[0], P.conic[1],
                                        P.conic[2], P.opacity, cut);
        if (cam->flags & ORC_FLAG_RADII_OPACITY && cam->flags & ORC_FLAG_RADII_AXIS) {
            double l = fabs(log(255.0 * P.opacity));
            if (l < cut_margin[g]) cut_margin[g] = l;
        }
        if (P.extent_empty) {
            rect[4 * g] = 0; rect[4 * g + 1] = 0; rect[4 * g + 2] = -1; rect[4 * g + 3] = -1;
            count[g] = 0;
        } else {
            count[g] = tile_rect_f32((float)P.mean2d[0], (float)P.mean2d[1], rxy[0], rxy[1], tiles_x,
                                     tiles_y, tight ? cut : NULL, rect + 4 * g);
        }
        double m = INFINITY;
        for (int axis = 0; axis < 2; axis++) {
            double e0 = (P.mean2d[axis] - (double)rxy[axis]) / ORC_TILE;
            double e1 = (P.mean2d[axis] + (double)rxy[axis]) / ORC_TILE;
            double d0 = dist_to_int(e0), d1 = dist_to_int(e1);
            if (d0 < m) m = d0;
            if (d1 < m) m = d1;
        }
        rect_margin[g] = m;
    }
    return 0;
}

/* Rectangle rule alone, for callers that already hold float records (used
 * to bin records that are given in single precision): radius_xy [n][2] per
 * axis.  conic [n][3] and opacity [n] are read only when tight_tiles is set;
 * the cut is then taken on their values as given.  Records whose radii are
 * both 0 and whose opacity-aware extent was empty must be marked invalid by
 * the caller. */
int orc_tile_rects(int64_t n, const float *mean2d, const float *radius_xy, const float *conic,
                   const float *opacity, const uint8_t *valid, int32_t width, int32_t height,
                   int32_t tight_tiles, int32_t *rect, int32_t *count)
{
    if (n < 0 || width <= 0 || height <= 0) return -1;
    int32_t tiles_x = (width + ORC_TILE - 1) / ORC_TILE;
    int32_t tiles_y = (height + ORC_TILE - 1) / ORC_TILE;
    for (int64_t g = 0; g < n; g++) {
        if (!valid[g]) {
            rect[4 * g] = 0; rect[4 * g + 1] = 0; rect[4 * g + 2] = -1; rect[4 * g + 3] = -1;
            count[g] = 0;
            continue;
        }
        double cut[4];
        if (tight_tiles)
            (void)opacity_cut(mean2d[2 * g], mean2d[2 * g + 1], conic[3 * g], conic[3 * g + 1],
                              conic[3 * g + 2], opacity[g], cut);
        count[g] = tile_rect_f32(mean2d[2 * g], mean2d[2 * g + 1], radius_xy[2 * g], radius_xy[2 * g + 1],
                                 tiles_x, tiles_y, tight_tiles ? cut : NULL, rect + 4 * g);
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Binning by brute force ([WEEK]: count, emit, sort, range).
 * Every (Gaussian, tile) pair is tested for membership of the tile in the
 * Gaussian's rectangle.  A pair's key is (tile id << 32) | float bits of
 * the Gaussian's depth; pairs are ordered by (key, Gaussian id).  ranges[t]
 * = [start, end) of tile t in the ordered list, [0, 0) when empty.
 * counts[g] = number of pairs of g.  Returns the number of pairs, or -1 if
 * it exceeds max_pairs (then only counts are valid). */
typedef struct { uint64_t key; uint32_t gid; } orc_pair;

static int cmp_pair(const void *pa, const void *pb)
{
    const orc_pair *a = (const orc_pair *)pa, *b = (const orc_pair *)pb;
    if (a->key != b->key) return a->key < b->key ? -1 : 1;
    if (a->gid != b->gid) return a->gid < b->gid ? -1 : 1;
    return 0;
}

static uint32_t float_bits(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    return u;
}

int64_t orc_bin(int64_t n, const int32_t *rect, const uint8_t *valid, const float *depth32,
                int32_t width, int32_t height, int64_t max_pairs, int32_t *counts,
                uint64_t *keys, uint32_t *gids, uint32_t *ranges)
{
    int32_t tiles_x = (width + ORC_TILE - 1) / ORC_TILE;
    int32_t tiles_y = (height + ORC_TILE - 1) / ORC_TILE;
    int64_t tiles = (int64_t)tiles_x * tiles_y;
    int64_t total = 0;
    for (int64_t g = 0; g < n; g++) {
        int32_t c = 0;
        if (valid[g]) {
            const int32_t *r = rect + 4 * g;
            for (int64_t t = 0; t < tiles; t++) {
                int32_t tx = (int32_t)(t % tiles_x), ty = (int32_t)(t / tiles_x);
                if (tx >= r[0] && tx <= r[2] && ty >= r[1] && ty <= r[3]) c++;
            }
        }
        counts[g] = c;
        total += c;
    }
    if (total > max_pairs) return -1;
    orc_pair *pairs = (orc_pair *)malloc(sizeof(orc_pair) * (size_t)(total > 0 ? total : 1));
    if (!pairs) return -2;
    int64_t k = 0;
    for (int64_t g = 0; g < n; g++) {
        if (!valid[g]) continue;
        const int32_t *r = rect + 4 * g;
        for (int64_t t = 0; t < tiles; t++) {
            int32_t tx = (int32_t)(t % tiles_x), ty = (int32_t)(t / tiles_x);
            if (tx >= r[0] && tx <= r[2] && ty >= r[1] && ty <= r[3]) {
                pairs[k].key = ((uint64_t)t << 32) | (uint64_t)float_bits(depth32[g]);
                pairs[k].gid = (uint32_t)g;
                k++;
            }
        }
    }
    qsort(pairs, (size_t)total, sizeof(orc_pair), cmp_pair);
    for (int64_t t = 0; t < tiles; t++) { ranges[2 * t] = 0; ranges[2 * t + 1] = 0; }
    for (int64_t i = 0; i < total; i++) {
        keys[i] = pairs[i].key;
        gids[i] = pairs[i].gid;
        uint64_t t = pairs[i].key >> 32;
        if (i == 0 || (pairs[i - 1].key >> 32) != t) ranges[2 * t] = (uint32_t)i;
        if (i == total - 1 || (pairs[i + 1].key >> 32) != t) ranges[2 * t + 1] = (uint32_t)(i + 1);
    }
    free(pairs);
    return total;
}

/* ------------------------------------------------------------------ */
/* Global depth order of the drawable Gaussians: valid ones with a non-empty
 * rectangle, sorted by (float bits of depth, id).  [GSP] s5: one global sort
 * replaces the per-tile ones. */
typedef struct { uint32_t bits; int64_t gid; } orc_dkey;

static int cmp_dkey(const void *pa, const void *pb)
{
    const orc_dkey *a = (const orc_dkey *)pa, *b = (const orc_dkey *)pb;
    if (a->bits != b->bits) return a->bits < b->bits ? -1 : 1;
    if (a->gid != b->gid) return a->gid < b->gid ? -1 : 1;
    return 0;
}

int64_t orc_depth_order(int64_t n, const float *depth32, const int32_t *rect, const uint8_t *valid,
                        int64_t *order)
{
    orc_dkey *d = (orc_dkey *)malloc(sizeof(orc_dkey) * (size_t)(n > 0 ? n : 1));
    if (!d) return -1;
    int64_t m = 0;
    for (int64_t g = 0; g < n; g++) {
        const int32_t *r = rect + 4 * g;
        if (!valid[g] || r[0] > r[2] || r[1] > r[3]) continue;
        d[m].bits = float_bits(depth32[g]);
        d[m].gid = g;
        m++;
    }
    qsort(d, (size_t)m, sizeof(orc_dkey), cmp_dkey);
    for (int64_t i = 0; i < m; i++) order[i] = d[i].gid;
    free(d);
    return m;
}

/* ------------------------------------------------------------------ */
/* Naive render ([WEEK] naive oracle; [GSP] s5 loop).  For each pixel, walk
 * every drawable Gaussian in the global depth order, keeping those whose
 * rectangle holds the pixel's tile (the pixel's tile list, in order):
 *   sigma = 1/2 (A dx^2 + C dy^2) + B dx dy,  dx = mx - x, dy = my - y
 *   alpha = min(0.99, o exp(-sigma));  skip if sigma < 0 or alpha < 1/255
 *   next_T = T (1 - alpha);            stop (without adding) if next_T < 1e-4
 *   C += c alpha T;  T = next_T
 * and output C + T bg ([GSP] s5 final paragraph).                          */
typedef struct {
    int32_t g;
    double alpha, T, G, dx, dy;
    int clamped;
} orc_hit;

typedef struct {
    int64_t n_order;
    const int64_t *order;
    const double *mean2d, *conic, *opacity, *color;
    const int32_t *rect;
    const orc_camera *cam;
    const uint8_t *tile_mask;
    int32_t tiles_x;
    /* forward outputs */
    double *image, *T_final;
    int32_t *n_walk;
    int64_t *e_visit, *e_contrib;
    double *margin_alpha, *margin_T, *margin_clamp;
    /* backward */
    const double *dL_dimage;
    double *grad2d, *grad2d_abs; /* per-thread slices, [nthreads][n][9] */
    int64_t n;
    int nthreads;
} orc_render_ctx;

typedef struct {
    orc_render_ctx *ctx;
    int tid;
} orc_thread_arg;

static double rel_margin(double v, double thr) { return fabs(v - thr) / thr; }

/* Walks one pixel.  If hits != NULL, records every added entry (growing the
 * buffer as needed).  Returns the number of added entries. */
static int64_t walk_pixel(const orc_render_ctx *c, int32_t i, int32_t j, orc_hit **hits,
                          int64_t *cap, double rgb[ORC_MAX_CH], double *T_out, int32_t *n_walk,
                          int64_t *e_visit, int64_t *e_contrib, double *m_alpha, double *m_T,
                          double *m_clamp)
{
    const double x = j + 0.5, y = i + 0.5;
    const int32_t tx = j / ORC_TILE, ty = i / ORC_TILE;
    double T = 1.0;
    const int nc = orc_channels(c->cam);
    for (int ch = 0; ch < ORC_MAX_CH; ch++) rgb[ch] = 0.0;
    int32_t pos = 0, last_pos = 0;
    int64_t visits = 0, nh = 0;
    double ma_min = INFINITY, mt_min = INFINITY, mc = INFINITY;
    for (int64_t k = 0; k < c->n_order; k++) {
        int64_t g = c->order[k];
        const int32_t *r = c->rect + 4 * g;
        if (tx < r[0] || tx > r[2] || ty < r[1] || ty > r[3]) continue;
        pos++;
        visits++;
        double dx = c->mean2d[2 * g] - x;
        double dy = c->mean2d[2 * g + 1] - y;
        double A = c->conic[3 * g], B = c->conic[3 * g + 1], C = c->conic[3 * g + 2];
        double sigma = 0.5 * (A * dx * dx + C * dy * dy) + B * dx * dy;
        double G = exp(-sigma);
        double oG = c->opacity[g] * G;
        const float acap = (c->cam->flags & ORC_FLAG_CAP_0999) ? ORC_ALPHA_CAP_0999_F : ORC_ALPHA_CAP_F;
        int clamped = (float)oG > acap;
        double alpha = clamped ? (double)acap : oG;
        if (sigma < 0.0) continue;
        double ma = rel_margin(alpha, (double)ORC_ALPHA_MIN_F);
        if (ma < ma_min) ma_min = ma;
        if ((float)alpha < ORC_ALPHA_MIN_F) continue;
        double mcl = rel_margin(oG, (double)acap);
        if (mcl < mc) mc = mcl;
        double next_T = T * (1.0 - alpha);
        double mt = rel_margin(next_T, (double)ORC_T_MIN_F);
        if (mt < mt_min) mt_min = mt;
        /* 3DGS stops when next_T < 1e-4; gsplat when next_T <= 1e-4 */
        if ((c->cam->flags & ORC_FLAG_STOP_INCLUSIVE) ? (float)next_T <= ORC_T_MIN_F
                                                      : (float)next_T < ORC_T_MIN_F)
            break;
        for (int ch = 0; ch < nc; ch++) rgb[ch] += c->color[nc * g + ch] * alpha * T;
        if (hits) {
            if (nh == *cap) {
                *cap = *cap ? 2 * *cap : 64;
                *hits = (orc_hit *)realloc(*hits, sizeof(orc_hit) * (size_t)*cap);
            }
            orc_hit *h = &(*hits)[nh];
            h->g = (int32_t)g; h->alpha = alpha; h->T = T; h->G = G; h->dx = dx; h->dy = dy;
            h->clamped = clamped;
        }
        nh++;
        T = next_T;
        last_pos = pos;
    }
    *T_out = T;
    *n_walk = last_pos;
    *e_visit = visits;
    *e_contrib = nh;
    *m_alpha = ma_min;
    *m_T = mt_min;
    *m_clamp = mc;
    return nh;
}

static int pixel_selected(const orc_render_ctx *c, int32_t i, int32_t j)
{
    if (!c->tile_mask) return 1;
    return c->tile_mask[(i / ORC_TILE) * c->tiles_x + j / ORC_TILE] != 0;
}

static void *render_worker(void *arg)
{
    orc_thread_arg *a = (orc_thread_arg *)arg;
    orc_render_ctx *c = a->ctx;
    const orc_camera *cam = c->cam;
    for (int32_t i = a->tid; i < cam->height; i += c->nthreads) {
        for (int32_t j = 0; j < cam->width; j++) {
            if (!pixel_selected(c, i, j)) continue;
            int64_t p = (int64_t)i * cam->width + j;
            double rgb[ORC_MAX_CH], T;
            walk_pixel(c, i, j, NULL, NULL, rgb, &T, &c->n_walk[p], &c->e_visit[p],
                       &c->e_contrib[p], &c->margin_alpha[p], &c->margin_T[p], &c->margin_clamp[p]);
            const int nc = orc_channels(cam);
            for (int ch = 0; ch < nc; ch++)  /* the depth channel has no background */
                c->image[nc * p + ch] = rgb[ch] + (ch < 3 ? T * cam->bg[ch] : 0.0);
            c->T_final[p] = T;
        }
    }
    return NULL;
}

static int run_threads(orc_render_ctx *c, void *(*fn)(void *))
{
    int nt = c->nthreads < 1 ? 1 : c->nthreads;
    c->nthreads = nt;
    pthread_t th[256];
    orc_thread_arg args[256];
    if (nt > 256) nt = c->nthreads = 256;
    for (int t = 0; t < nt; t++) {
        args[t].ctx = c;
        args[t].tid = t;
        if (pthread_create(&th[t], NULL, fn, &args[t]) != 0) return -1;
    }
    for (int t = 0; t < nt; t++) pthread_join(th[t], NULL);
    return 0;
}

/* Forward render of the projected records (any precision the caller chose,
 * given here as double).  tile_mask (nullable, [tiles]) restricts the work to
 * the selected tiles; other pixels are left untouched.
 * Outputs per pixel: image[3], T_final, n_walk (position in the pixel's tile
 * list one past the last added entry), e_visit (entries visited, up to and
 * including the stopping one), e_contrib (entries added), margin_alpha (least
 * relative distance of an alpha to 1/255), margin_T (least relative distance
 * of a next_T to 1e-4), margin_clamp (least relative distance of o G to the
 * 0.99 cap). */
int orc_render(int64_t n, const double *mean2d, const double *conic, const double *opacity,
               const double *color, const float *depth32, const int32_t *rect,
               const uint8_t *valid, const orc_camera *cam, const uint8_t *tile_mask, int nthreads,
               double *image, double *T_final, int32_t *n_walk, int64_t *e_visit,
               int64_t *e_contrib, double *margin_alpha, double *margin_T, double *margin_clamp)
{
    if (n < 0 || cam->width <= 0 || cam->height <= 0) return -1;
    int64_t *order = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n > 0 ? n : 1));
    if (!order) return -2;
    int64_t m = orc_depth_order(n, depth32, rect, valid, order);
    orc_render_ctx c;
    memset(&c, 0, sizeof(c));
    c.n_order = m; c.order = order;
    c.mean2d = mean2d; c.conic = conic; c.opacity = opacity; c.color = color; c.rect = rect;
    c.cam = cam; c.tile_mask = tile_mask;
    c.tiles_x = (cam->width + ORC_TILE - 1) / ORC_TILE;
    c.image = image; c.T_final = T_final; c.n_walk = n_walk; c.e_visit = e_visit;
    c.e_contrib = e_contrib; c.margin_alpha = margin_alpha; c.margin_T = margin_T;
    c.margin_clamp = margin_clamp;
    c.n = n;
    c.nthreads = nthreads;
    int rc = run_threads(&c, render_worker);
    free(order);
    return rc;
}

/* ------------------------------------------------------------------ */
/* Analytic backward of the blend ([GSP] s6: back to front, weights
 * recomputed).  For the entries a pixel added, from the back:
 *   R_last = bg;  dL/dc_i = alpha_i T_i g;
 *   dL/dalpha_i = T_i <c_i - R_i, g>;  R_{i-1} = alpha_i c_i + (1-alpha_i) R_i
 *   unless o G was capped: dalpha/do = G, dalpha/dsigma = -o G
 *   dsigma/dA = dx^2/2, dsigma/dB = dx dy, dsigma/dC = dy^2/2,
 *   dsigma/dmx = A dx + B dy, dsigma/dmy = B dx + C dy.
 * The pixel's own T_i are those of its forward walk.  Per Gaussian the nine
 * sums (dmx, dmy, dA, dB, dC, dopacity, dr, dg, db, and d of the depth
 * channel when it is on) and the sums of their absolute contributions are
 * accumulated. */
static void *backward_worker(void *arg)
{
    orc_thread_arg *a = (orc_thread_arg *)arg;
    orc_render_ctx *c = a->ctx;
    const orc_camera *cam = c->cam;
    const int nc = orc_channels(cam), ng = 6 + nc;
    double *acc = c->grad2d + (size_t)a->tid * (size_t)c->n * ng;
    double *acc_abs = c->grad2d_abs + (size_t)a->tid * (size_t)c->n * ng;
    orc_hit *hits = NULL;
    int64_t cap = 0;
    for (int32_t i = a->tid; i < cam->height; i += c->nthreads) {
        for (int32_t j = 0; j < cam->width; j++) {
            if (!pixel_selected(c, i, j)) continue;
            int64_t p = (int64_t)i * cam->width + j;
            double rgb[ORC_MAX_CH], T, ma, mt, mc;
            int32_t nw;
            int64_t ev, ec;
            int64_t nh = walk_pixel(c, i, j, &hits, &cap, rgb, &T, &nw, &ev, &ec, &ma, &mt, &mc);
            const double *gp = c->dL_dimage + nc * p;
            double R[ORC_MAX_CH] = {cam->bg[0], cam->bg[1], cam->bg[2], 0.0};
            for (int64_t h = nh - 1; h >= 0; h--) {
                const orc_hit *e = &hits[h];
                int64_t g = e->g;
                double *d = acc + ng * g, *da = acc_abs + ng * g;
                const double *col = c->color + nc * g;
                double w = e->alpha * e->T;
                double dl_dalpha = 0.0;
                for (int ch = 0; ch < nc; ch++) {
                    double v = w * gp[ch];
                    d[6 + ch] += v;
                    da[6 + ch] += fabs(v);
                    dl_dalpha += (col[ch] - R[ch]) * gp[ch];
                }
                dl_dalpha *= e->T;
                for (int ch = 0; ch < nc; ch++) R[ch] = e->alpha * col[ch] + (1.0 - e->alpha) * R[ch];
                if (e->clamped) continue;
                double o = c->opacity[g];
                double dl_dsigma = dl_dalpha * (-o * e->G);
                double dl_do = dl_dalpha * e->G;
                double A = c->conic[3 * g], B = c->conic[3 * g + 1], C = c->conic[3 * g + 2];
                double v[6];
                v[0] = dl_dsigma * (A * e->dx + B * e->dy);
                v[1] = dl_dsigma * (B * e->dx + C * e->dy);
                v[2] = dl_dsigma * 0.5 * e->dx * e->dx;
                v[3] = dl_dsigma * e->dx * e->dy;
                v[4] = dl_dsigma * 0.5 * e->dy * e->dy;
                v[5] = dl_do;
                for (int k = 0; k < 6; k++) {
                    d[k] += v[k];
                    da[k] += fabs(v[k]);
                }
            }
        }
    }
    free(hits);
    return NULL;
}

int orc_render_bwd(int64_t n, const double *mean2d, const double *conic, const double *opacity,
                   const double *color, const float *depth32, const int32_t *rect,
                   const uint8_t *valid, const orc_camera *cam, const uint8_t *tile_mask,
                   int nthreads, const double *dL_dimage, double *grad2d, double *grad2d_abs)
{
    if (n < 0 || cam->width <= 0 || cam->height <= 0) return -1;
    int nt = nthreads < 1 ? 1 : (nthreads > 256 ? 256 : nthreads);
    const int ng = 6 + orc_channels(cam);
    int64_t *order = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n > 0 ? n : 1));
    double *acc = (double *)calloc((size_t)nt * (size_t)(n > 0 ? n : 1) * ng, sizeof(double));
    double *acc_abs = (double *)calloc((size_t)nt * (size_t)(n > 0 ? n : 1) * ng, sizeof(double));
    if (!order || !acc || !acc_abs) { free(order); free(acc); free(acc_abs); return -2; }
    int64_t m = orc_depth_order(n, depth32, rect, valid, order);
    orc_render_ctx c;
    memset(&c, 0, sizeof(c));
    c.n_order = m; c.order = order;
    c.mean2d = mean2d; c.conic = conic; c.opacity = opacity; c.color = color; c.rect = rect;
    c.cam = cam; c.tile_mask = tile_mask;
    c.tiles_x = (cam->width + ORC_TILE - 1) / ORC_TILE;
    c.dL_dimage = dL_dimage;
    c.grad2d = acc; c.grad2d_abs = acc_abs;
    c.n = n;
    c.nthreads = nt;
    int rc = run_threads(&c, backward_worker);
    /* sum the per-thread partials in thread order */
    for (int64_t k = 0; k < n * ng; k++) {
        double s = 0.0, sa = 0.0;
        for (int t = 0; t < nt; t++) {
            s += acc[(size_t)t * (size_t)n * ng + (size_t)k];
            sa += acc_abs[(size_t)t * (size_t)n * ng + (size_t)k];
        }
        grad2d[k] = s;
        grad2d_abs[k] = sa;
    }
    free(order); free(acc); free(acc_abs);
    return rc;
}

/* ------------------------------------------------------------------ */
/* Chain rule from the nine per-Gaussian 2D gradients to the raw parameters
 * ([GSP] s6: through the conic inverse, the 0.3 dilation, J and its clamp,
 * the view rotation, R S, the quaternion normalisation, exp and sigmoid; the
 * radius and the sort give none).  Culled Gaussians get exact zeros. */
static void quat_rotmat_vjp(const double *qh, const double *G, double *dq)
{
    double w = qh[0], x = qh[1], y = qh[2], z = qh[3];
    dq[0] = 2.0 * (-z * G[1] + y * G[2] + z * G[3] - x * G[5] - y * G[6] + x * G[7]);
    dq[1] = 2.0 * (y * G[1] + z * G[2] + y * G[3] - 2.0 * x * G[4] - w * G[5] + z * G[6] +
                   w * G[7] - 2.0 * x * G[8]);
    dq[2] = 2.0 * (-2.0 * y * G[0] + x * G[1] + w * G[2] + x * G[3] + z * G[5] - w * G[6] +
                   z * G[7] - 2.0 * y * G[8]);
    dq[3] = 2.0 * (-2.0 * z * G[0] - w * G[1] + x * G[2] + w * G[3] - 2.0 * z * G[4] +
                   y * G[5] + x * G[6] + y * G[7]);
}

int orc_project_bwd(int64_t n, const double *means, const double *log_scales, const double *quats,
                    const double *opacity_logits, const orc_camera *cam, const double *grad2d,
                    double *d_means, double *d_log_scales, double *d_quats,
                    double *d_opacity_logits, double *d_colors)
{
    if (n < 0) return -1;
    for (int64_t g = 0; g < n; g++) {
        double *dm = d_means + 3 * g, *dls = d_log_scales + 3 * g, *dq = d_quats + 4 * g;
        double *dc = d_colors + 3 * g;
        for (int k = 0; k < 3; k++) { dm[k] = 0.0; dls[k] = 0.0; dc[k] = 0.0; }
        for (int k = 0; k < 4; k++) dq[k] = 0.0;
        d_opacity_logits[g] = 0.0;
        orc_proj P;
        project_one(means + 3 * g, log_scales + 3 * g, quats + 4 * g, opacity_logits[g], cam, &P);
        if (!P.valid) continue;
        const int ng = 6 + orc_channels(cam);
        const double *gg = grad2d + ng * g;
        double d_mx = gg[0], d_my = gg[1], d_A = gg[2], d_B = gg[3], d_C = gg[4], d_o = gg[5];
        /* colour passes through */
        for (int k = 0; k < 3; k++) dc[k] = gg[6 + k];
        /* opacity = sigmoid(logit) x comp; comp = sqrt(D1 / D2) with D1 the
         * undilated and D2 the dilated determinant (antialiased mode) */
        d_opacity_logits[g] = d_o * P.comp * P.opacity_raw * (1.0 - P.opacity_raw);
        double d_comp = (cam->flags & ORC_FLAG_ANTIALIASED) && P.det_orig > 0.0 ? d_o * P.opacity_raw : 0.0;

        /* conic (A, B, C) = (c, -b, a) / det, det = a c - b^2 (no gradient
         * through det when it was clamped) */
        double det = P.det;
        double dl_ddet = 0.0;
        if (!P.det_clamped)
            dl_ddet = -(d_A * P.c - d_B * P.b + d_C * P.a) / (det * det);
        double d_a = d_C / det + dl_ddet * P.c;
        double d_b = -d_B / det + dl_ddet * (-2.0 * P.b);
        double d_c = d_A / det + dl_ddet * P.a;
        if (d_comp != 0.0) {
            /* d comp = comp/2 (dD1/D1 - dD2/D2); D1 = (a - e)(c - e) - b^2,
             * D2 = a c - b^2 (no D2 term when the det was clamped) */
            const double h = 0.5 * P.comp * d_comp, D1 = P.det_orig;
            const double k2 = P.det_clamped ? 0.0 : 1.0 / det;
            d_a += h * ((P.c - ORC_EPS2D) / D1 - k2 * P.c);
            d_c += h * ((P.a - ORC_EPS2D) / D1 - k2 * P.a);
            d_b += h * (-2.0 * P.b / D1 + k2 * 2.0 * P.b);
        }
        /* Sigma' = Sigma'' - 0.3 I has the same gradient; Sigma' = J Sc J^T */
        double Gp[4] = {d_a, 0.5 * d_b, 0.5 * d_b, d_c};
        /* dL/dSc = J^T Gp J */
        double GJ[6];
        for (int i = 0; i < 2; i++)
            for (int j = 0; j < 3; j++)
                GJ[3 * i + j] = Gp[2 * i] * P.J[j] + Gp[2 * i + 1] * P.J[3 + j];
        double dSc[9];
        for (int i = 0; i < 3; i++)
            for (int j = 0; j < 3; j++)
                dSc[3 * i + j] = P.J[i] * GJ[j] + P.J[3 + i] * GJ[3 + j];
        /* dL/dJ = 2 Gp J Sc */
        double dJ[6];
        for (int i = 0; i < 2; i++)
            for (int j = 0; j < 3; j++) {
                double acc = 0.0;
                for (int k = 0; k < 3; k++) acc += GJ[3 * i + k] * P.Sc[3 * k + j];
                dJ[3 * i + j] = 2.0 * acc;
            }
        /* J -> camera-space mean t */
        double tx = P.t[0], ty = P.t[1], tz = P.t[2];
        double fx = cam->fx, fy = cam->fy;
        double dt[3] = {0.0, 0.0, 0.0};
        dt[2] += dJ[0] * (-fx / (tz * tz));
        dt[2] += dJ[4] * (-fy / (tz * tz));
        if (!P.clamped_x) {
            dt[0] += dJ[2] * (-fx / (tz * tz));
            dt[2] += dJ[2] * (2.0 * fx * tx / (tz * tz * tz));
        } else {
            double lim = P.jx / tz;
            dt[2] += dJ[2] * (fx * lim / (tz * tz));
        }
        if (!P.clamped_y) {
            dt[1] += dJ[5] * (-fy / (tz * tz));
            dt[2] += dJ[5] * (2.0 * fy * ty / (tz * tz * tz));
        } else {
            double lim = P.jy / tz;
            dt[2] += dJ[5] * (fy * lim / (tz * tz));
        }
        /* the depth channel's colour is the camera z */
        if (ng == 10) dt[2] += gg[9];
        /* mean2d = (fx x/z + cx, fy y/z + cy) */
        dt[0] += d_mx * fx / tz;
        dt[1] += d_my * fy / tz;
        dt[2] += d_mx * (-fx * tx / (tz * tz)) + d_my * (-fy * ty / (tz * tz));
        /* t = W mu + tv */
        for (int j = 0; j < 3; j++) {
            double acc = 0.0;
            for (int i = 0; i < 3; i++) acc += P.W[3 * i + j] * dt[i];
            dm[j] = acc;
        }
        /* Sc = W Sigma W^T -> dSigma = W^T dSc W */
        double tmp[9], dS[9];
        for (int i = 0; i < 3; i++)
            for (int j = 0; j < 3; j++) {
                double acc = 0.0;
                for (int k = 0; k < 3; k++) acc += P.W[3 * k + i] * dSc[3 * k + j];
                tmp[3 * i + j] = acc;
            }
        for (int i = 0; i < 3; i++)
            for (int j = 0; j < 3; j++) {
                double acc = 0.0;
                for (int k = 0; k < 3; k++) acc += tmp[3 * i + k] * P.W[3 * k + j];
                dS[3 * i + j] = acc;
            }
        /* Sigma = M M^T -> dM = (dS + dS^T) M */
        double dM[9];
        for (int i = 0; i < 3; i++)
            for (int j = 0; j < 3; j++) {
                double acc = 0.0;
                for (int k = 0; k < 3; k++) acc += (dS[3 * i + k] + dS[3 * k + i]) * P.M[3 * k + j];
                dM[3 * i + j] = acc;
            }
        /* M = R diag(s) */
        double dR[9];
        for (int i = 0; i < 3; i++)
            for (int j = 0; j < 3; j++) dR[3 * i + j] = dM[3 * i + j] * P.s[j];
        for (int j = 0; j < 3; j++) {
            double acc = 0.0;
            for (int i = 0; i < 3; i++) acc += dM[3 * i + j] * P.R[3 * i + j];
            dls[j] = acc * P.s[j]; /* s = exp(log s) */
        }
        /* R(qhat) -> qhat -> q (normalisation with the 1e-12 clamp) */
        double dqh[4];
        quat_rotmat_vjp(P.qhat, dR, dqh);
        if (P.qnorm >= ORC_QUAT_EPS) {
            double dot = 0.0;
            for (int k = 0; k < 4; k++) dot += P.qhat[k] * dqh[k];
            for (int k = 0; k < 4; k++) dq[k] = (dqh[k] - P.qhat[k] * dot) / P.qnorm;
        } else {
            for (int k = 0; k < 4; k++) dq[k] = dqh[k] / ORC_QUAT_EPS;
        }
    }
    return 0;
}

/* Intermediates of one Gaussian's projection, for tests that pin single
 * steps to the pages' worked examples.  out[0..39]:
 *   0 valid, 1 clamped x/z, 2 clamped y/z, 3..8 J (2x3 row-major),
 *   9..11 undilated Sigma' (a, b, c), 12..14 dilated (a, b, c), 15 det,
 *   16..18 conic, 19 lambda_max, 20 3 sqrt(lambda), 21..22 mean2d,
 *   23..25 camera-space mean, 26..34 Sigma (world), 35 opacity,
 *   36 clamped_x flag, 37 clamped_y flag, 38 det clamped flag, 39 unused */
int orc_project_debug(const double *mean, const double *log_scale, const double *quat,
                      double opacity_logit, const orc_camera *cam, double *out)
{
    orc_proj P;
    project_one(mean, log_scale, quat, opacity_logit, cam, &P);
    memset(out, 0, sizeof(double) * 40);
    out[0] = P.valid;
    for (int k = 0; k < 9; k++) out[26 + k] = P.Sigma[k];
    for (int k = 0; k < 3; k++) out[23 + k] = P.t[k];
    out[35] = P.opacity;
    if (!(P.t[2] > cam->near_z)) return 0;
    out[1] = P.jx / P.t[2];
    out[2] = P.jy / P.t[2];
    for (int k = 0; k < 6; k++) out[3 + k] = P.J[k];
    out[9] = P.a - ORC_EPS2D; out[10] = P.b; out[11] = P.c - ORC_EPS2D;
    out[12] = P.a; out[13] = P.b; out[14] = P.c;
    out[15] = P.det;
    for (int k = 0; k < 3; k++) out[16 + k] = P.conic[k];
    out[19] = P.lambda_max;
    out[20] = P.radius_value;
    out[21] = P.mean2d[0]; out[22] = P.mean2d[1];
    out[36] = P.clamped_x; out[37] = P.clamped_y; out[38] = P.det_clamped;
    return 0;
}

/* Version tag so a loader can check it is talking to this library. */
int orc_version(void) { return 1; }
