// gs_project.cu -- projection of raw Gaussian parameters to screen-space
// records, and its backward (the chain rule from the 2D gradients to the raw
// parameters).  One thread per Gaussian; fp32 throughout.
//
// Source: "Gaussian splatting in PyTorch" (cited [GSP]), s1 activations,
// s2 covariance R S S^T R^T, s3 world-to-camera and the EWA Jacobian with its
// widened-frustum clamp, s4 dilation, conic and radius, s6 culling without
// ever dividing by a culled depth.
#include "gs_internal.cuh"

namespace gs {
namespace {

constexpr float kQuatEps = 1e-12f;
constexpr float kEps2d = 0.3f;        // [GSP] s4 low-pass dilation, px^2
constexpr float kDetMin = 1e-10f;     // [GSP] s3 det clamp
constexpr float kLambdaFloor = 0.1f;  // [GSP] s4 floor under the root
constexpr float kRadiusSigmas = 3.f;  // [GSP] s4 3DGS radius rule
constexpr float kGsplatSigmas = 3.33f;  // [GSP] s4 gsplat per-axis radii
// Opacity-aware tile cut: slack in ln(alpha) (cut tiles stay below
// e^-0.01 / 255) and the largest conic condition A C / (A C - B^2) it is
// taken at (beyond it single-precision sigma near the threshold can stray
// by more than the slack).
constexpr float kCutSlack = 0.01f;
constexpr float kCutMaxCond = 1024.f;

// Everything the forward computes for one Gaussian; the backward re-derives
// it from the raw parameters instead of storing it.
struct Proj {
    float qn, qh[4];     // |q| and the unit quaternion
    float R[9], s[3];    // rotation, scales
    float M[9];          // R diag(s)
    float Sc[6];         // camera-space covariance (xx, xy, xz, yy, yz, zz)
    float t[3];          // camera-space mean
    float J[4];          // J00, J02, J11, J12 (J01 = J10 = 0)
    float a, b, c;       // dilated 2D covariance
    float det;
    bool det_clamped, clamped_x, clamped_y;
    float A, B, C;       // conic
    float mx, my;
    float opacity;       // the opacity the blend uses (compensated in antialiased mode)
    float opacity_raw;   // sigmoid(logit)
    float det_orig;      // det of the undilated 2D covariance
    float comp;          // antialiasing compensation, 1 without the flag
    float lambda;
    bool valid;
};

__device__ __forceinline__ void project_one(const CamConst &cam, const float *mu, const float *ls,
                                            const float *q, float logit, Proj &P) {
    // [GSP] s1: activations
    float qn = sqrtf(q[0] * q[0] + q[1] * q[1] + q[2] * q[2] + q[3] * q[3]);
    P.qn = qn;
    float inv_q = 1.f / fmaxf(qn, kQuatEps);
    float w = q[0] * inv_q, x = q[1] * inv_q, y = q[2] * inv_q, z = q[3] * inv_q;
    P.qh[0] = w; P.qh[1] = x; P.qh[2] = y; P.qh[3] = z;
    P.R[0] = 1.f - 2.f * (y * y + z * z);
    P.R[1] = 2.f * (x * y - w * z);
    P.R[2] = 2.f * (x * z + w * y);
    P.R[3] = 2.f * (x * y + w * z);
    P.R[4] = 1.f - 2.f * (x * x + z * z);
    P.R[5] = 2.f * (y * z - w * x);
    P.R[6] = 2.f * (x * z - w * y);
    P.R[7] = 2.f * (y * z + w * x);
    P.R[8] = 1.f - 2.f * (x * x + y * y);
    P.s[0] = expf(ls[0]); P.s[1] = expf(ls[1]); P.s[2] = expf(ls[2]);
    P.opacity = 1.f / (1.f + expf(-logit));
    P.opacity_raw = P.opacity;
    P.comp = 1.f;

    // [GSP] s2: M = R diag(s); Sigma = M M^T.  Then [GSP] s3: the camera
    // sees V = W M, and Sigma_c = V V^T = W Sigma W^T.
#pragma unroll
    for (int i = 0; i < 3; i++)
#pragma unroll
        for (int j = 0; j < 3; j++) P.M[3 * i + j] = P.R[3 * i + j] * P.s[j];
    float V[9];
#pragma unroll
    for (int i = 0; i < 3; i++)
#pragma unroll
        for (int j = 0; j < 3; j++)
            V[3 * i + j] = cam.R[3 * i] * P.M[j] + cam.R[3 * i + 1] * P.M[3 + j] +
                           cam.R[3 * i + 2] * P.M[6 + j];
    P.Sc[0] = V[0] * V[0] + V[1] * V[1] + V[2] * V[2];
    P.Sc[1] = V[0] * V[3] + V[1] * V[4] + V[2] * V[5];
    P.Sc[2] = V[0] * V[6] + V[1] * V[7] + V[2] * V[8];
    P.Sc[3] = V[3] * V[3] + V[4] * V[4] + V[5] * V[5];
    P.Sc[4] = V[3] * V[6] + V[4] * V[7] + V[5] * V[8];
    P.Sc[5] = V[6] * V[6] + V[7] * V[7] + V[8] * V[8];

    // [GSP] s3: t = W mu + tv
#pragma unroll
    for (int i = 0; i < 3; i++)
        P.t[i] = cam.R[3 * i] * mu[0] + cam.R[3 * i + 1] * mu[1] + cam.R[3 * i + 2] * mu[2] + cam.t[i];
    const float tx = P.t[0], ty = P.t[1], tz = P.t[2];
    P.valid = tz > cam.near_z;  // [GSP] s6: nothing below divides by a culled z
    const float tzs = P.valid ? tz : 1.f;

    // [GSP] s3: J at x/z, y/z clamped to the widened frustum (for J only)
    const float inv_z = 1.f / tzs;
    const float xz = tx * inv_z, yz = ty * inv_z;
    P.clamped_x = xz < cam.lim_x_lo || xz > cam.lim_x_hi;
    P.clamped_y = yz < cam.lim_y_lo || yz > cam.lim_y_hi;
    const float cxz = fminf(fmaxf(xz, cam.lim_x_lo), cam.lim_x_hi);
    const float cyz = fminf(fmaxf(yz, cam.lim_y_lo), cam.lim_y_hi);
    P.J[0] = cam.fx * inv_z;
    P.J[1] = -cam.fx * cxz * inv_z;
    P.J[2] = cam.fy * inv_z;
    P.J[3] = -cam.fy * cyz * inv_z;

    // Sigma' = J Sigma_c J^T with J = [[J0, 0, J1], [0, J2, J3]]
    const float r0x = P.J[0] * P.Sc[0] + P.J[1] * P.Sc[2];
    const float r0y = P.J[0] * P.Sc[1] + P.J[1] * P.Sc[4];
    const float r0z = P.J[0] * P.Sc[2] + P.J[1] * P.Sc[5];
    const float r1y = P.J[2] * P.Sc[3] + P.J[3] * P.Sc[4];
    const float r1z = P.J[2] * P.Sc[4] + P.J[3] * P.Sc[5];
    const float a0 = r0x * P.J[0] + r0z * P.J[1];  // undilated
    const float c0 = r1y * P.J[2] + r1z * P.J[3];
    P.a = a0 + kEps2d;  // [GSP] s4 dilation
    P.b = r0y * P.J[2] + r0z * P.J[3];
    P.c = c0 + kEps2d;
    P.det_orig = a0 * c0 - P.b * P.b;
    float det = P.a * P.c - P.b * P.b;
    P.det_clamped = det < kDetMin;
    det = fmaxf(det, kDetMin);
    P.det = det;
    P.A = P.c / det;
    P.B = -P.b / det;
    P.C = P.a / det;
    if (cam.flags & GS_FLAG_ANTIALIASED) {
        // [GSP] s4, antialiased mode: opacity x sqrt(det S' / det S'')
        P.comp = P.det_orig > 0.f ? sqrtf(P.det_orig / det) : 0.f;
        P.opacity = P.opacity_raw * P.comp;
    }
    const float mid = 0.5f * (P.a + P.c);
    P.lambda = mid + sqrtf(fmaxf(mid * mid - det, kLambdaFloor));
    P.mx = cam.fx * tx * inv_z + cam.cx;
    P.my = cam.fy * ty * inv_z + cam.cy;
    P.valid = P.valid && isfinite(P.mx) && isfinite(P.my) && isfinite(P.A) && isfinite(P.B) &&
              isfinite(P.C) && isfinite(P.lambda) && isfinite(P.opacity);
}

// Parameter loads: consecutive threads read consecutive Gaussians, so each
// warp's loads of an [N][3] or [N][4] array cover one contiguous span.
__global__ void __launch_bounds__(256)
k_project(CamConst cam, int n, const float *__restrict__ means, const float *__restrict__ log_scales,
          const float *__restrict__ quats, const float *__restrict__ logits,
          const float *__restrict__ colors, float4 *__restrict__ xyod, float4 *__restrict__ conr,
          float4 *__restrict__ rgb, int4 *__restrict__ rect, uint32_t *__restrict__ count) {
    const int g = blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= n) return;
    float mu[3] = {means[3 * g], means[3 * g + 1], means[3 * g + 2]};
    float ls[3] = {log_scales[3 * g], log_scales[3 * g + 1], log_scales[3 * g + 2]};
    const float4 q4 = reinterpret_cast<const float4 *>(quats)[g];
    float q[4] = {q4.x, q4.y, q4.z, q4.w};
    Proj P;
    project_one(cam, mu, ls, q, logits[g], P);
    // with GS_FLAG_DEPTH the fourth colour is the camera z ([GSP] s5: any channel blends alike)
    const float4 col = make_float4(colors[3 * g], colors[3 * g + 1], colors[3 * g + 2],
                                   (cam.flags & GS_FLAG_DEPTH) ? P.t[2] : 0.f);
    rgb[g] = col;
    // the colour is a projected value too: not finite -> culled ([GSP] s6)
    if (!P.valid || !isfinite(col.x) || !isfinite(col.y) || !isfinite(col.z)) {
        xyod[g] = make_float4(0.f, 0.f, P.opacity, P.t[2]);
        conr[g] = make_float4(0.f, 0.f, 0.f, 0.f);
        rect[g] = make_int4(0, 0, -1, -1);
        count[g] = 0;
        return;
    }
    // radii: 3DGS ceil(3 sqrt(lambda_max)); gsplat per axis ceil(e sqrt(S''_ii)),
    // e = 3.33 or min(3.33, sqrt(2 ln(255 o))) ([GSP] s4)
    float rx = ceilf(kRadiusSigmas * sqrtf(P.lambda)), ry = rx;
    bool none = false;
    if (cam.flags & GS_FLAG_RADII_AXIS) {
        float e = kGsplatSigmas;
        if (cam.flags & GS_FLAG_RADII_OPACITY) {
            const float l = logf(255.f * P.opacity);
            none = !(l > 0.f);
            e = none ? 0.f : fminf(e, sqrtf(2.f * l));
        }
        rx = ceilf(e * sqrtf(P.a));
        ry = ceilf(e * sqrtf(P.c));
    }
    const float r = fmaxf(rx, ry);
    xyod[g] = make_float4(P.mx, P.my, P.opacity, P.t[2]);
    conr[g] = make_float4(P.A, P.B, P.C, r);
    if (none) {  // fades below 1/255 everywhere: no tiles
        rect[g] = make_int4(0, 0, -1, -1);
        count[g] = 0;
        return;
    }
    // Tile rectangle: floor((m -+ r) / 16) per axis, optionally narrowed by
    // the opacity-aware cut, clamped to the grid in float before any integer
    // conversion.
    const float inv_tile = 1.f / kTile;
    float lx = floorf((P.mx - rx) * inv_tile), hx = floorf((P.mx + rx) * inv_tile);
    float ly = floorf((P.my - ry) * inv_tile), hy = floorf((P.my + ry) * inv_tile);
    if (cam.flags & GS_FLAG_TIGHT_TILES) {
        // Opacity-aware cut ([GSP] s4, gsplat's sqrt(2 ln(255 o)) extent),
        // per pixel-centre column and row.  On the column at horizontal
        // offset dx from the mean, sigma is smallest at dy = -B dx / C, where
        // it is dx^2 q / (2 C), q = A C - B^2: columns whose nearest centre is
        // farther than D_x = sqrt(2 ell C / q), ell = ln(255 o) + slack, hold
        // no pixel that passes alpha >= 1/255.  Column tx (centres 16 tx + 0.5
        // ... 16 tx + 15.5) is kept iff tx lies in
        // [ceil((mx - D_x - 15.5) / 16), floor((mx + D_x - 0.5) / 16)].
        const float q = P.A * P.C - P.B * P.B;
        if (q > 0.f && P.A * P.C <= kCutMaxCond * q) {
            const float ell = logf(255.f * P.opacity) + kCutSlack;
            if (ell <= 0.f) {  // o too small for any pixel to pass
                lx = (float)cam.tiles_x;
                hx = -1.f;
                ly = (float)cam.tiles_y;
                hy = -1.f;
            } else {
                const float s2 = 2.f * ell / q;
                const float dx = sqrtf(s2 * P.C), dy = sqrtf(s2 * P.A);
                lx = fmaxf(lx, ceilf((P.mx - dx - 15.5f) * inv_tile));
                hx = fminf(hx, floorf((P.mx + dx - 0.5f) * inv_tile));
                ly = fmaxf(ly, ceilf((P.my - dy - 15.5f) * inv_tile));
                hy = fminf(hy, floorf((P.my + dy - 0.5f) * inv_tile));
            }
        }
    }
    lx = fminf(fmaxf(lx, 0.f), (float)cam.tiles_x);
    ly = fminf(fmaxf(ly, 0.f), (float)cam.tiles_y);
    hx = fmaxf(fminf(hx, (float)(cam.tiles_x - 1)), -1.f);
    hy = fmaxf(fminf(hy, (float)(cam.tiles_y - 1)), -1.f);
    const int x0 = (int)lx, y0 = (int)ly, x1 = (int)hx, y1 = (int)hy;
    rect[g] = make_int4(x0, y0, x1, y1);
    count[g] = (x0 > x1 || y0 > y1) ? 0u : (uint32_t)((x1 - x0 + 1) * (y1 - y0 + 1));
}

// Backward of R(q) for a unit quaternion: dL/dq given G = dL/dR (row-major).
__device__ __forceinline__ void rotmat_vjp(const float *qh, const float *G, float *dq) {
    const float w = qh[0], x = qh[1], y = qh[2], z = qh[3];
    dq[0] = 2.f * (-z * G[1] + y * G[2] + z * G[3] - x * G[5] - y * G[6] + x * G[7]);
    dq[1] = 2.f * (y * G[1] + z * G[2] + y * G[3] - 2.f * x * G[4] - w * G[5] + z * G[6] +
                   w * G[7] - 2.f * x * G[8]);
    dq[2] = 2.f * (-2.f * y * G[0] + x * G[1] + w * G[2] + x * G[3] + z * G[5] - w * G[6] +
                   z * G[7] - 2.f * y * G[8]);
    dq[3] = 2.f * (-2.f * z * G[0] - w * G[1] + x * G[2] + w * G[3] - 2.f * z * G[4] + y * G[5] +
                   x * G[6] + y * G[7]);
}

// grad2d per Gaussian arrives holding the blend backward's sums over pixels:
//   sum v, sum v dx, sum v dy, sum v dx^2, sum v dx dy, sum v dy^2, dL/d(r, g, b)
// with v = alpha dL/dalpha and dx, dy = mean - pixel.  With sigma =
// 1/2 (A dx^2 + C dy^2) + B dx dy and dL/dsigma = -v, dL/do = v / o:
//   dL/dmx = -(A sum v dx + B sum v dy), dL/dmy = -(B sum v dx + C sum v dy),
//   dL/dA = -sum v dx^2 / 2, dL/dB = -sum v dx dy, dL/dC = -sum v dy^2 / 2.
// Those values are written back: on return grad2d holds
// dL/d(mx, my, A, B, C, opacity, r, g, b, depth channel, 0, 0) (the depth
// channel's entry is 0 without GS_FLAG_DEPTH).
// Stores (or, with kAcc, adds) one raw-parameter gradient value.
template <bool kAcc>
__device__ __forceinline__ void put(float *a, int i, float x) {
    if (kAcc) a[i] += x;
    else a[i] = x;
}

template <bool kAcc>
__global__ void __launch_bounds__(256)
k_project_bwd(CamConst cam, int n, const float *__restrict__ means,
              const float *__restrict__ log_scales, const float *__restrict__ quats,
              const float *__restrict__ logits, const float4 *__restrict__ xyod,
              const float4 *__restrict__ conr, float4 *__restrict__ grad2d,
              float *__restrict__ d_means, float *__restrict__ d_log_scales,
              float *__restrict__ d_quats, float *__restrict__ d_logits,
              float *__restrict__ d_colors) {
    const int g = blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= n) return;
    float mu[3] = {means[3 * g], means[3 * g + 1], means[3 * g + 2]};
    float ls[3] = {log_scales[3 * g], log_scales[3 * g + 1], log_scales[3 * g + 2]};
    const float4 q4 = reinterpret_cast<const float4 *>(quats)[g];
    float q[4] = {q4.x, q4.y, q4.z, q4.w};
    Proj P;
    project_one(cam, mu, ls, q, logits[g], P);
    const float4 s0 = grad2d[3 * g], s1 = grad2d[3 * g + 1], s2 = grad2d[3 * g + 2];
    // Conic and opacity as the blend used them: the projected records.
    const float4 cr = conr[g];
    const float op = xyod[g].z;
    const float4 g0 = make_float4(-(cr.x * s0.y + cr.y * s0.z), -(cr.y * s0.y + cr.z * s0.z),
                                  -0.5f * s0.w, -s1.x);
    const float4 g1 = make_float4(-0.5f * s1.y, op > 0.f ? s0.x / op : 0.f, s1.z, s1.w);
    const float4 g2 = make_float4(s2.x, s2.y, 0.f, 0.f);  // b, depth channel
    grad2d[3 * g] = g0;
    grad2d[3 * g + 1] = g1;
    grad2d[3 * g + 2] = g2;
    if (!P.valid) {  // [GSP] s6: culled Gaussians get exact zeros
        if (kAcc) return;
        for (int k = 0; k < 3; k++) {
            d_means[3 * g + k] = 0.f;
            d_log_scales[3 * g + k] = 0.f;
            d_colors[3 * g + k] = 0.f;
        }
        reinterpret_cast<float4 *>(d_quats)[g] = make_float4(0.f, 0.f, 0.f, 0.f);
        d_logits[g] = 0.f;
        return;
    }
    const float d_mx = g0.x, d_my = g0.y, d_A = g0.z, d_B = g0.w;
    const float d_C = g1.x, d_o = g1.y;
    put<kAcc>(d_colors, 3 * g, g1.z);
    put<kAcc>(d_colors, 3 * g + 1, g1.w);
    put<kAcc>(d_colors, 3 * g + 2, g2.x);
    // opacity = sigmoid(logit) x comp
    put<kAcc>(d_logits, g, d_o * P.comp * P.opacity_raw * (1.f - P.opacity_raw));

    // conic = (c, -b, a) / det; no gradient through a clamped det
    const float inv_det = 1.f / P.det;
    float dl_ddet = 0.f;
    if (!P.det_clamped) dl_ddet = -(d_A * P.c - d_B * P.b + d_C * P.a) * inv_det * inv_det;
    float d_a = d_C * inv_det + dl_ddet * P.c;
    float d_b = -d_B * inv_det - 2.f * dl_ddet * P.b;
    float d_c = d_A * inv_det + dl_ddet * P.a;
    if ((cam.flags & GS_FLAG_ANTIALIASED) && P.det_orig > 0.f) {
        // comp = sqrt(D1 / D2), D1 = (a - e)(c - e) - b^2, D2 = a c - b^2:
        // d comp = comp / 2 (dD1 / D1 - dD2 / D2)
        const float h = 0.5f * P.comp * d_o * P.opacity_raw, i1 = 1.f / P.det_orig;
        const float i2 = P.det_clamped ? 0.f : inv_det;
        d_a += h * ((P.c - kEps2d) * i1 - P.c * i2);
        d_c += h * ((P.a - kEps2d) * i1 - P.a * i2);
        d_b += h * 2.f * P.b * (i2 - i1);
    }
    // Sigma' (undilated) has the same gradient.  Sigma' = J Sc J^T:
    //   dL/dSc = J^T Gp J,  dL/dJ = 2 Gp J Sc,  Gp = [[d_a, d_b/2], [d_b/2, d_c]]
    const float hb = 0.5f * d_b;
    const float J0 = P.J[0], J1 = P.J[1], J2 = P.J[2], J3 = P.J[3];
    // Gp J (2x3): rows [d_a J0, hb J2, d_a J1 + hb J3], [hb J0, d_c J2, hb J1 + d_c J3]
    const float GJ00 = d_a * J0, GJ01 = hb * J2, GJ02 = d_a * J1 + hb * J3;
    const float GJ10 = hb * J0, GJ11 = d_c * J2, GJ12 = hb * J1 + d_c * J3;
    // dSc = J^T (Gp J), J^T rows: [J0, 0], [0, J2], [J1, J3]
    float dSc[9];
    dSc[0] = J0 * GJ00;             dSc[1] = J0 * GJ01;             dSc[2] = J0 * GJ02;
    dSc[3] = J2 * GJ10;             dSc[4] = J2 * GJ11;             dSc[5] = J2 * GJ12;
    dSc[6] = J1 * GJ00 + J3 * GJ10; dSc[7] = J1 * GJ01 + J3 * GJ11; dSc[8] = J1 * GJ02 + J3 * GJ12;
    // dJ = 2 (Gp J) Sc, Sc symmetric
    const float *S = P.Sc;  // xx, xy, xz, yy, yz, zz
    const float dJ00 = 2.f * (GJ00 * S[0] + GJ01 * S[1] + GJ02 * S[2]);
    const float dJ02 = 2.f * (GJ00 * S[2] + GJ01 * S[4] + GJ02 * S[5]);
    const float dJ11 = 2.f * (GJ10 * S[1] + GJ11 * S[3] + GJ12 * S[4]);
    const float dJ12 = 2.f * (GJ10 * S[2] + GJ11 * S[4] + GJ12 * S[5]);
    // J -> t (the clamp passes no gradient to x, y outside its range)
    const float tx = P.t[0], ty = P.t[1], tz = P.t[2];
    const float iz = 1.f / tz, iz2 = iz * iz, iz3 = iz2 * iz;
    float dt0 = 0.f, dt1 = 0.f, dt2 = 0.f;
    dt2 -= (dJ00 * cam.fx + dJ11 * cam.fy) * iz2;
    if (!P.clamped_x) {
        dt0 -= dJ02 * cam.fx * iz2;
        dt2 += dJ02 * 2.f * cam.fx * tx * iz3;
    } else {
        const float lim = tx * iz < cam.lim_x_lo ? cam.lim_x_lo : cam.lim_x_hi;
        dt2 += dJ02 * cam.fx * lim * iz2;
    }
    if (!P.clamped_y) {
        dt1 -= dJ12 * cam.fy * iz2;
        dt2 += dJ12 * 2.f * cam.fy * ty * iz3;
    } else {
        const float lim = ty * iz < cam.lim_y_lo ? cam.lim_y_lo : cam.lim_y_hi;
        dt2 += dJ12 * cam.fy * lim * iz2;
    }
    // the depth channel's colour is the camera z
    if (cam.flags & GS_FLAG_DEPTH) dt2 += g2.y;
    // mean2d = (fx x/z + cx, fy y/z + cy)
    dt0 += d_mx * cam.fx * iz;
    dt1 += d_my * cam.fy * iz;
    dt2 -= (d_mx * cam.fx * tx + d_my * cam.fy * ty) * iz2;
    // t = W mu + tv
#pragma unroll
    for (int j = 0; j < 3; j++)
        put<kAcc>(d_means, 3 * g + j, cam.R[j] * dt0 + cam.R[3 + j] * dt1 + cam.R[6 + j] * dt2);
    // Sc = W Sigma W^T -> dSigma = W^T dSc W
    float T1[9], dS[9];
#pragma unroll
    for (int i = 0; i < 3; i++)
#pragma unroll
        for (int j = 0; j < 3; j++)
            T1[3 * i + j] = cam.R[i] * dSc[j] + cam.R[3 + i] * dSc[3 + j] + cam.R[6 + i] * dSc[6 + j];
#pragma unroll
    for (int i = 0; i < 3; i++)
#pragma unroll
        for (int j = 0; j < 3; j++)
            dS[3 * i + j] = T1[3 * i] * cam.R[j] + T1[3 * i + 1] * cam.R[3 + j] + T1[3 * i + 2] * cam.R[6 + j];
    // Sigma = M M^T -> dM = (dS + dS^T) M
    float dM[9];
#pragma unroll
    for (int i = 0; i < 3; i++)
#pragma unroll
        for (int j = 0; j < 3; j++)
            dM[3 * i + j] = (dS[3 * i] + dS[i]) * P.M[j] + (dS[3 * i + 1] + dS[3 + i]) * P.M[3 + j] +
                            (dS[3 * i + 2] + dS[6 + i]) * P.M[6 + j];
    // M = R diag(s), s = exp(log_scale)
    float dR[9];
#pragma unroll
    for (int i = 0; i < 3; i++)
#pragma unroll
        for (int j = 0; j < 3; j++) dR[3 * i + j] = dM[3 * i + j] * P.s[j];
#pragma unroll
    for (int j = 0; j < 3; j++)
        put<kAcc>(d_log_scales, 3 * g + j,
                  (dM[j] * P.R[j] + dM[3 + j] * P.R[3 + j] + dM[6 + j] * P.R[6 + j]) * P.s[j]);
    // R(q_hat) -> q_hat -> q through the normalisation with its clamp
    float dqh[4];
    rotmat_vjp(P.qh, dR, dqh);
    float4 dq;
    if (P.qn >= kQuatEps) {
        const float dot = P.qh[0] * dqh[0] + P.qh[1] * dqh[1] + P.qh[2] * dqh[2] + P.qh[3] * dqh[3];
        const float iq = 1.f / P.qn;
        dq = make_float4((dqh[0] - P.qh[0] * dot) * iq, (dqh[1] - P.qh[1] * dot) * iq,
                         (dqh[2] - P.qh[2] * dot) * iq, (dqh[3] - P.qh[3] * dot) * iq);
    } else {
        const float iq = 1.f / kQuatEps;
        dq = make_float4(dqh[0] * iq, dqh[1] * iq, dqh[2] * iq, dqh[3] * iq);
    }
    if (kAcc) {
        const float4 o = reinterpret_cast<const float4 *>(d_quats)[g];
        dq = make_float4(o.x + dq.x, o.y + dq.y, o.z + dq.z, o.w + dq.w);
    }
    reinterpret_cast<float4 *>(d_quats)[g] = dq;
}

}  // namespace

cudaError_t launch_project(const CamConst &c, int64_t n, const gs_params &p, const gs_projected &o,
                           cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    const int threads = 256;
    const int blocks = (int)((n + threads - 1) / threads);
    prof_before("project", s);
    k_project<<<blocks, threads, 0, s>>>(c, (int)n, p.means, p.log_scales, p.quats, p.opacity_logits,
                                         p.colors, reinterpret_cast<float4 *>(o.xy_opacity_depth),
                                         reinterpret_cast<float4 *>(o.conic_radius),
                                         reinterpret_cast<float4 *>(o.rgb),
                                         reinterpret_cast<int4 *>(o.rect), o.count);
    prof_after(s);
    return cudaGetLastError();
}

cudaError_t launch_project_bwd(const CamConst &c, int64_t n, const gs_params &p,
                               const gs_projected &proj, float *grad2d, const gs_grads &g,
                               cudaStream_t s, bool accumulate) {
    if (n == 0) return cudaSuccess;
    const int threads = 256;
    const int blocks = (int)((n + threads - 1) / threads);
    prof_before("project_bwd", s);
    (accumulate ? k_project_bwd<true> : k_project_bwd<false>)<<<blocks, threads, 0, s>>>(c, (int)n, p.means, p.log_scales, p.quats,
                                             p.opacity_logits,
                                             reinterpret_cast<const float4 *>(proj.xy_opacity_depth),
                                             reinterpret_cast<const float4 *>(proj.conic_radius),
                                             reinterpret_cast<float4 *>(grad2d), g.means,
                                             g.log_scales, g.quats, g.opacity_logits, g.colors);
    prof_after(s);
    return cudaGetLastError();
}

}  // namespace gs
