// gs_render.cu -- per-tile alpha blending (forward) and its back-to-front
// gradient (backward), plus the L1 photometric loss of a training step.
//
// Source: "Gaussian splatting in PyTorch" s5 (the per-pixel loop:
// sigma = 1/2 (A dx^2 + C dy^2) + B dx dy, alpha = min(0.99, o exp(-sigma)),
// skip sigma < 0 or alpha < 1/255, stop once T (1 - alpha) < 1e-4,
// C += c alpha T; pixel centres at +0.5; background weighted by the final T),
// s6 (the CUDA backward recovers T_i by dividing by 1 - alpha_j back to front;
// no gradient through the 0.99 cap) and s8 (16 x 16 tiles, each pixel walks
// only its tile's list); the course blog index (a backward that recomputes
// the blend weights rather than storing them).
//
// One CTA per tile, one thread per pixel.  The tile's list is staged through
// shared memory in batches of 256 entries, each entry converted once per tile
// to the form the inner loop wants: the conic pre-scaled by -log2(e)/2 (and
// -log2(e) for B) and log2(opacity), so that
//     log2(o exp(-sigma)) = log2 o + cA dx^2 + cB dx dy + cC dy^2
// costs five FP32 instructions and one MUFU ex2.  The forward and backward
// share that evaluation code and use explicitly rounded intrinsics, so the
// backward re-takes every skip decision bit-identically.
#include "gs_internal.cuh"

namespace gs {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kAlphaCap = 0.99f;
constexpr float kAlphaMin = 1.f / 255.f;
constexpr float kTMin = 1e-4f;
constexpr int kBlendThreads = kTilePixels;  // 256
constexpr int kBatch = kBlendThreads;

// PTX ex2.approx / rcp.approx (MUFU instructions).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Per-tile staged form of one list entry.
struct __align__(16) Staged {
    float4 geo;   // mean2d x, y; cA = -log2e A / 2; cB = -log2e B
    float2 geo2;  // cC = -log2e C / 2; log2(opacity)
};

__device__ __forceinline__ void stage_entry(const float4 xyod, const float4 conr, float4 &geo,
                                            float2 &geo2) {
    geo = make_float4(xyod.x, xyod.y, (-0.5f * kLog2e) * conr.x, -kLog2e * conr.y);
    geo2 = make_float2((-0.5f * kLog2e) * conr.z, log2f(xyod.z));
}

// Alpha of one entry at pixel centre (px, py).  Returns false when the entry
// is skipped (sigma < 0 or alpha < 1/255).  dx, dy = mean - pixel.
__device__ __forceinline__ bool eval_alpha(const float4 geo, const float2 geo2, float px, float py,
                                           float &dx, float &dy, float &alpha, bool &capped) {
    dx = __fsub_rn(geo.x, px);
    dy = __fsub_rn(geo.y, py);
    const float t = __fmaf_rn(geo.z, dx, __fmul_rn(geo.w, dy));          // cA dx + cB dy
    const float q = __fmaf_rn(t, dx, __fmul_rn(__fmul_rn(geo2.x, dy), dy));  // -sigma log2 e
    const float a = ex2_approx(__fadd_rn(q, geo2.y));                    // o exp(-sigma)
    capped = a > kAlphaCap;
    alpha = fminf(a, kAlphaCap);
    return !(q > 0.f) && alpha >= kAlphaMin;
}

__global__ void __launch_bounds__(kBlendThreads)
k_render_fwd(CamConst cam, const float4 *__restrict__ xyod, const float4 *__restrict__ conr,
             const float4 *__restrict__ rgb, const uint32_t *__restrict__ pair_gid,
             const uint2 *__restrict__ ranges, float *__restrict__ image,
             float *__restrict__ T_final, uint32_t *__restrict__ last) {
    __shared__ float4 s_geo[kBatch];
    __shared__ float2 s_geo2[kBatch];
    __shared__ float4 s_col[kBatch];

    const int tile = blockIdx.x;
    const int tx = tile % cam.tiles_x, ty = tile / cam.tiles_x;
    const int px = tx * kTile + (threadIdx.x & (kTile - 1));
    const int py = ty * kTile + (threadIdx.x >> 4);
    const bool inside = px < cam.width && py < cam.height;
    const float fx = (float)px + 0.5f, fy = (float)py + 0.5f;
    const uint2 range = ranges[tile];

    float T = 1.f, C0 = 0.f, C1 = 0.f, C2 = 0.f;
    uint32_t last_idx = range.x;
    bool done = !inside;
    for (uint32_t b = range.x; b < range.y; b += kBatch) {
        if (__syncthreads_count(done) == kBlendThreads) break;
        const uint32_t j = b + threadIdx.x;
        if (j < range.y) {
            const uint32_t g = pair_gid[j];
            float4 geo;
            float2 geo2;
            stage_entry(xyod[g], conr[g], geo, geo2);
            s_geo[threadIdx.x] = geo;
            s_geo2[threadIdx.x] = geo2;
            s_col[threadIdx.x] = rgb[g];
        }
        __syncthreads();
        const int cnt = (int)min((uint32_t)kBatch, range.y - b);
        if (!done) {
            for (int k = 0; k < cnt; k++) {
                float dx, dy, a;
                bool capped;
                if (!eval_alpha(s_geo[k], s_geo2[k], fx, fy, dx, dy, a, capped)) continue;
                const float nT = __fmaf_rn(-T, a, T);
                if (nT < kTMin) { done = true; break; }
                const float w = __fmul_rn(a, T);
                const float4 c = s_col[k];
                C0 = __fmaf_rn(w, c.x, C0);
                C1 = __fmaf_rn(w, c.y, C1);
                C2 = __fmaf_rn(w, c.z, C2);
                T = nT;
                last_idx = b + k + 1;
            }
        }
    }
    if (inside) {
        const size_t p = (size_t)py * cam.width + px;
        image[3 * p] = __fmaf_rn(T, cam.bg[0], C0);
        image[3 * p + 1] = __fmaf_rn(T, cam.bg[1], C1);
        image[3 * p + 2] = __fmaf_rn(T, cam.bg[2], C2);
        T_final[p] = T;
        last[p] = last_idx;
    }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__global__ void __launch_bounds__(kBlendThreads)
k_render_bwd(CamConst cam, const float4 *__restrict__ xyod, const float4 *__restrict__ conr,
             const float4 *__restrict__ rgb, const uint32_t *__restrict__ pair_gid,
             const uint2 *__restrict__ ranges, const float *__restrict__ T_final,
             const uint32_t *__restrict__ last, const float *__restrict__ dL_dimage,
             float *__restrict__ grad2d) {
    __shared__ float4 s_geo[kBatch];
    __shared__ float2 s_geo2[kBatch];
    __shared__ float4 s_col[kBatch];
    __shared__ float4 s_raw[kBatch];  // A, B, C, 1/opacity
    __shared__ uint32_t s_gid[kBatch];
    __shared__ uint32_t s_max_last;

    const int tile = blockIdx.x;
    const int tx = tile % cam.tiles_x, ty = tile / cam.tiles_x;
    const int px = tx * kTile + (threadIdx.x & (kTile - 1));
    const int py = ty * kTile + (threadIdx.x >> 4);
    const bool inside = px < cam.width && py < cam.height;
    const float fx = (float)px + 0.5f, fy = (float)py + 0.5f;
    const uint2 range = ranges[tile];
    const int lane = threadIdx.x & 31;

    float T = 1.f, g0 = 0.f, g1 = 0.f, g2 = 0.f;
    uint32_t my_last = range.x;
    if (inside) {
        const size_t p = (size_t)py * cam.width + px;
        T = T_final[p];
        my_last = min(max(last[p], range.x), range.y);  // never walk outside the tile's list
        g0 = dL_dimage[3 * p];
        g1 = dL_dimage[3 * p + 1];
        g2 = dL_dimage[3 * p + 2];
    }
    float R0 = cam.bg[0], R1 = cam.bg[1], R2 = cam.bg[2];
    if (threadIdx.x == 0) s_max_last = range.x;
    __syncthreads();
    atomicMax(&s_max_last, my_last);
    __syncthreads();
    const uint32_t max_last = s_max_last;

    for (uint32_t bend = max_last; bend > range.x;) {
        const uint32_t bstart = bend - range.x > (uint32_t)kBatch ? bend - kBatch : range.x;
        const uint32_t cnt = bend - bstart;
        if (threadIdx.x < cnt) {
            const uint32_t j = bend - 1 - threadIdx.x;  // slot 0 = back-most entry
            const uint32_t g = pair_gid[j];
            const float4 xo = xyod[g], cr = conr[g];
            float4 geo;
            float2 geo2;
            stage_entry(xo, cr, geo, geo2);
            s_geo[threadIdx.x] = geo;
            s_geo2[threadIdx.x] = geo2;
            s_col[threadIdx.x] = rgb[g];
            s_raw[threadIdx.x] = make_float4(cr.x, cr.y, cr.z, 1.f / xo.z);
            s_gid[threadIdx.x] = g;
        }
        __syncthreads();
        for (uint32_t k = 0; k < cnt; k++) {
            const uint32_t j = bend - 1 - k;
            float v = 0.f, gx = 0.f, gy = 0.f, gxx = 0.f, gxy = 0.f, gyy = 0.f;
            float cr0 = 0.f, cr1 = 0.f, cr2 = 0.f;
            bool contrib = false;
            if (j < my_last) {
                float dx, dy, a;
                bool capped;
                if (eval_alpha(s_geo[k], s_geo2[k], fx, fy, dx, dy, a, capped)) {
                    contrib = true;
                    const float Ti = __fmul_rn(T, rcp_approx(__fsub_rn(1.f, a)));
                    const float w = __fmul_rn(a, Ti);
                    const float4 c = s_col[k];
                    cr0 = w * g0;
                    cr1 = w * g1;
                    cr2 = w * g2;
                    const float d0 = c.x - R0, d1 = c.y - R1, d2 = c.z - R2;
                    const float dLda = Ti * (d0 * g0 + d1 * g1 + d2 * g2);
                    R0 = __fmaf_rn(a, d0, R0);
                    R1 = __fmaf_rn(a, d1, R1);
                    R2 = __fmaf_rn(a, d2, R2);
                    v = capped ? 0.f : dLda * a;  // dL/dsigma = -v, dL/do = v / o
                    gx = v * dx;
                    gy = v * dy;
                    gxx = gx * dx;
                    gxy = gx * dy;
                    gyy = gy * dy;
                    T = Ti;
                }
            }
            if (__any_sync(0xffffffffu, contrib)) {
                v = warp_sum(v);
                gx = warp_sum(gx);
                gy = warp_sum(gy);
                gxx = warp_sum(gxx);
                gxy = warp_sum(gxy);
                gyy = warp_sum(gyy);
                cr0 = warp_sum(cr0);
                cr1 = warp_sum(cr1);
                cr2 = warp_sum(cr2);
                if (lane == 0) {
                    const float4 raw = s_raw[k];
                    float *dst = grad2d + 12 * (size_t)s_gid[k];
                    atomicAdd(reinterpret_cast<float4 *>(dst),
                              make_float4(-(raw.x * gx + raw.y * gy), -(raw.y * gx + raw.z * gy),
                                          -0.5f * gxx, -gxy));
                    atomicAdd(reinterpret_cast<float4 *>(dst + 4),
                              make_float4(-0.5f * gyy, v * raw.w, cr0, cr1));
                    atomicAdd(dst + 8, cr2);
                }
            }
        }
        __syncthreads();
        bend = bstart;
    }
}

// Same walk as k_render_fwd, counting instead of blending.
__global__ void __launch_bounds__(kBlendThreads)
k_render_stats(CamConst cam, const float4 *__restrict__ xyod, const float4 *__restrict__ conr,
               const uint32_t *__restrict__ pair_gid, const uint2 *__restrict__ ranges,
               const uint32_t *__restrict__ last, unsigned long long *__restrict__ counts) {
    __shared__ float4 s_geo[kBatch];
    __shared__ float2 s_geo2[kBatch];
    __shared__ unsigned long long s_c[3];
    const int tile = blockIdx.x;
    const int tx = tile % cam.tiles_x, ty = tile / cam.tiles_x;
    const int px = tx * kTile + (threadIdx.x & (kTile - 1));
    const int py = ty * kTile + (threadIdx.x >> 4);
    const bool inside = px < cam.width && py < cam.height;
    const float fx = (float)px + 0.5f, fy = (float)py + 0.5f;
    const uint2 range = ranges[tile];
    if (threadIdx.x < 3) s_c[threadIdx.x] = 0ull;
    float T = 1.f;
    unsigned long long visits = 0, adds = 0;
    bool done = !inside;
    for (uint32_t b = range.x; b < range.y; b += kBatch) {
        if (__syncthreads_count(done) == kBlendThreads) break;
        const uint32_t j = b + threadIdx.x;
        if (j < range.y) {
            const uint32_t g = pair_gid[j];
            float4 geo;
            float2 geo2;
            stage_entry(xyod[g], conr[g], geo, geo2);
            s_geo[threadIdx.x] = geo;
            s_geo2[threadIdx.x] = geo2;
        }
        __syncthreads();
        const int cnt = (int)min((uint32_t)kBatch, range.y - b);
        if (!done) {
            for (int k = 0; k < cnt; k++) {
                float dx, dy, a;
                bool capped;
                visits++;
                if (!eval_alpha(s_geo[k], s_geo2[k], fx, fy, dx, dy, a, capped)) continue;
                const float nT = __fmaf_rn(-T, a, T);
                if (nT < kTMin) { done = true; break; }
                adds++;
                T = nT;
            }
        }
    }
    __syncthreads();
    if (inside) {
        const size_t p = (size_t)py * cam.width + px;
        atomicAdd(&s_c[0], visits);
        atomicAdd(&s_c[1], adds);
        atomicAdd(&s_c[2], (unsigned long long)(last[p] - range.x));
    }
    __syncthreads();
    if (threadIdx.x < 3) atomicAdd(&counts[threadIdx.x], s_c[threadIdx.x]);
    if (threadIdx.x == 3 && blockIdx.x == 0)
        atomicAdd(&counts[3], (unsigned long long)cam.width * cam.height);
}

__global__ void __launch_bounds__(256)
k_l1(const float *__restrict__ image, const float *__restrict__ target, int64_t count,
     float *__restrict__ dL, float *__restrict__ loss) {
    __shared__ float s_w[8];
    const float inv = 1.f / (float)count;
    float acc = 0.f;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float d = image[i] - target[i];
        dL[i] = d > 0.f ? inv : (d < 0.f ? -inv : 0.f);
        acc += fabsf(d);
    }
    if (loss) {
        acc = warp_sum(acc);
        if ((threadIdx.x & 31) == 0) s_w[threadIdx.x >> 5] = acc;
        __syncthreads();
        if (threadIdx.x == 0) {
            float s = 0.f;
            for (int w = 0; w < (int)(blockDim.x >> 5); w++) s += s_w[w];
            atomicAdd(loss, s * inv);
        }
    }
}

}  // namespace

cudaError_t launch_render_fwd(const CamConst &c, const gs_projected &proj, const gs_bins &bins,
                              float *image, float *T_final, uint32_t *last, cudaStream_t s) {
    const int tiles = c.tiles_x * c.tiles_y;
    prof_before("render_fwd", s);
    k_render_fwd<<<tiles, kBlendThreads, 0, s>>>(
        c, reinterpret_cast<const float4 *>(proj.xy_opacity_depth),
        reinterpret_cast<const float4 *>(proj.conic_radius), reinterpret_cast<const float4 *>(proj.rgb),
        bins.pair_gid, reinterpret_cast<const uint2 *>(bins.ranges), image, T_final, last);
    prof_after(s);
    return cudaGetLastError();
}

cudaError_t launch_render_bwd(const CamConst &c, const gs_projected &proj, const gs_bins &bins,
                              const float *T_final, const uint32_t *last, const float *dL_dimage,
                              float *grad2d, cudaStream_t s) {
    const int tiles = c.tiles_x * c.tiles_y;
    prof_before("render_bwd", s);
    k_render_bwd<<<tiles, kBlendThreads, 0, s>>>(
        c, reinterpret_cast<const float4 *>(proj.xy_opacity_depth),
        reinterpret_cast<const float4 *>(proj.conic_radius), reinterpret_cast<const float4 *>(proj.rgb),
        bins.pair_gid, reinterpret_cast<const uint2 *>(bins.ranges), T_final, last, dL_dimage,
        grad2d);
    prof_after(s);
    return cudaGetLastError();
}

cudaError_t launch_render_stats(const CamConst &c, const gs_projected &proj, const gs_bins &bins,
                                const uint32_t *last, uint64_t *counts, cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(counts, 0, 4 * sizeof(uint64_t), s);
    if (e != cudaSuccess) return e;
    const int tiles = c.tiles_x * c.tiles_y;
    prof_before("render_stats", s);
    k_render_stats<<<tiles, kBlendThreads, 0, s>>>(
        c, reinterpret_cast<const float4 *>(proj.xy_opacity_depth),
        reinterpret_cast<const float4 *>(proj.conic_radius), bins.pair_gid,
        reinterpret_cast<const uint2 *>(bins.ranges), last,
        reinterpret_cast<unsigned long long *>(counts));
    prof_after(s);
    return cudaGetLastError();
}

cudaError_t launch_l1(const float *image, const float *target, int64_t count, float *dL_dimage,
                      float *loss, cudaStream_t s) {
    if (loss) {
        cudaError_t e = cudaMemsetAsync(loss, 0, sizeof(float), s);
        if (e != cudaSuccess) return e;
    }
    if (count == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (count + 255) / 256;
    const int blocks = (int)(want < (int64_t)sms * 8 ? want : (int64_t)sms * 8);
    prof_before("l1_loss", s);
    k_l1<<<blocks, 256, 0, s>>>(image, target, count, dL_dimage, loss);
    prof_after(s);
    return cudaGetLastError();
}

}  // namespace gs
