// gs_render.cu -- per-tile alpha blending (forward) and its back-to-front
// gradient (backward), the frame's work counts, and the L1 loss of a training
// step.
//
// Source: "Gaussian splatting in PyTorch" s5 (the per-pixel loop:
// sigma = 1/2 (A dx^2 + C dy^2) + B dx dy, alpha = min(0.99, o exp(-sigma)),
// skip sigma < 0 or alpha < 1/255, stop once T (1 - alpha) < 1e-4 -- the
// cap 0.999 and the stop test <= 1e-4 of gsplat as camera flags,
// C += c alpha T; pixel centres at +0.5; background weighted by the final T),
// s6 (the CUDA backward recovers T_i by dividing by 1 - alpha back to front;
// no gradient through the 0.99 cap) and s8 (16 x 16 tiles, each pixel walks
// only its tile's list); the course blog index (a backward that recomputes
// the blend weights rather than storing them).
//
// Work layout.  One CTA per tile.  Each lane owns RPL vertically adjacent
// pixels of one column: lanes 0-15 the upper RPL rows of the warp's strip,
// lanes 16-31 the lower RPL rows, so a warp covers a 16 x 2RPL strip and a
// tile takes 8 / RPL warps (forward: RPL = 1, eight warps; backward: RPL = 4,
// two warps).  The tile's list is staged through shared memory in batches
// (forward 256 entries, backward 128), each entry converted once per tile to
//     geo  = (mx, my, cA, cB),  geo2 = (cC, log2 o, kx, ky)
// with cA = -log2(e) A / 2, cB = -log2(e) B, cC = -log2(e) C / 2, so that
//     log2(o exp(-sigma)) = log2 o + cA dx^2 + cB dx dy + cC dy^2;
// kx, ky serve the cull masks while staging, and geo2.z then holds the
// centre c of the range test below.
// The terms that depend only on the column (dx) are computed once per entry
// and shared by the lane's RPL pixels.
//
// Exact culling per warp.  kx = cA - cB^2 / (4 cC) and ky = cC - cB^2 / (4 cA)
// are the quadratic form's minima along a row and a column: over a strip of
// pixel centres no closer than dy_min (rows) and dx_min (columns) to the mean,
// -sigma log2(e) <= min(kx dx_min^2, ky dy_min^2).  When that bound keeps
// alpha below 1/255 with a 1 % margin at every pixel of the warp, the entry is
// skipped for the warp; each of its pixels would have skipped it anyway, so
// the result is unchanged.  The forward takes the test for all eight strips
// while staging and lets each warp walk a compacted list of its slots; the
// backward takes it per entry.
//
// The forward and backward share the evaluation code and use explicitly
// rounded intrinsics, so the backward re-takes every skip decision
// bit-identically.
#include <type_traits>

#include "gs_internal.cuh"

// Pixels per lane of the backward (a tuning knob; the default is the fastest
// measured on B200).
#ifndef GS_BWD_RPL
#define GS_BWD_RPL 4
#endif
// Backward: entries staged per round (at most 128) and resident CTAs per SM
// the register allocation targets.  Forward: resident CTAs per SM the
// register allocation targets.  (Tuning knobs; the defaults are the fastest
// measured on B200.)
#ifndef GS_FWD_MINB
#define GS_FWD_MINB 5
#endif
// Forward: issue both entries' exponentials before the alpha tests (1), or
// only in the branch of a passing entry (0).  A tuning knob.
#ifndef GS_FWD_EARLY_EX2
#define GS_FWD_EARLY_EX2 1
#endif
#ifndef GS_BWD_BATCH
#define GS_BWD_BATCH 128
#endif
#ifndef GS_BWD_MINB
#define GS_BWD_MINB (48 / GS_BWD_RPL)
#endif
// Backward entries reached by at most this many lanes of a warp add their
// sums with one atomic per lane and value instead of the warp reduce-scatter
// (0: always reduce; a tuning knob), in frames of at most
// GS_BWD_DIRECT_PAIRS pairs per Gaussian: where a Gaussian spans many tiles,
// the warps adding into its sums are many too, and the lanes' atomics on the
// same addresses queue in L2.
#ifndef GS_BWD_DIRECT
#define GS_BWD_DIRECT 8
#endif
#ifndef GS_BWD_DIRECT_PAIRS
#define GS_BWD_DIRECT_PAIRS 8
#endif

namespace gs {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
// log2(1/255) minus a margin of 0.0145 (1 % in alpha).
constexpr float kCullLog2 = -7.994353436858858f - 0.0145f;
// log2(1/255) in single precision: the alpha >= 1/255 test is taken on the
// exponent, log2(o exp(-sigma)) >= this, before the exponential.
constexpr float kLog2AlphaMin = -7.994353436858858f;
constexpr int kBatch = 256;     // forward batch (entries staged per round)
constexpr int kBwdBatch = GS_BWD_BATCH;  // backward batch: less shared memory, more CTAs per SM

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

__device__ __forceinline__ void stage_entry(const float4 xyod, const float4 conr, float4 &geo,
                                            float4 &geo2) {
    const float cA = (-0.5f * kLog2e) * conr.x;
    const float cB = -kLog2e * conr.y;
    const float cC = (-0.5f * kLog2e) * conr.z;
    // Separable bound of the exponent: max over dy of the quadratic at fixed
    // dx is kx dx^2, and likewise ky dy^2.  Not used (zero) for conics with
    // condition A C / (A C - B^2) above 1024, where single-precision rounding
    // of the exponent near the alpha threshold can exceed the cull margin.
    const float acx4 = 4.f * cA * cC, det4 = acx4 - cB * cB;  // log2(e)^2 (A C - B^2)
    const bool bounded = det4 > 0.f && acx4 <= 1024.f * det4;
    const float kx = bounded ? cA - cB * cB / (4.f * cC) : 0.f;
    const float ky = bounded ? cC - cB * cB / (4.f * cA) : 0.f;
    geo = make_float4(xyod.x, xyod.y, cA, cB);
    geo2 = make_float4(cC, log2f(xyod.z), kx, ky);
}

// Where a blend kernel reads its per-Gaussian channel values and writes its
// per-pixel and per-Gaussian channel outputs: the records' colours, or a
// chunk of four (or, with kF8, eight) feature channels.
struct ChannelIO {
    const float4 *col;  // channel values of Gaussian g at col[g * col_stride] (and the next float4 with kF8)
    int col_stride;     // in float4s
    int img_stride;     // floats per pixel of the image (forward) or dL/dimage (backward)
    float *cgrad;       // backward: the channel-gradient sums of Gaussian g at cgrad[g * cgrad_stride]
    int cgrad_stride;   // in floats
};

// The L1 loss of a training step taken in the forward's epilogue ([GSP] s7:
// loss = mean |image - target| over every value, its gradient
// sign(image - target) / count): each pixel's values against the target,
// the gradient written per value, the loss summed per CTA and added once.
// stats (nullable): [0] the bins' status word, [1] K, copied by CTA 0.
struct L1Out {
    const float *target;  // [H][W][channels]
    float *dL;            // [H][W][channels]
    float *loss;          // [1], zeroed by the caller; nullable
    float inv;            // 1 / (H W channels), rounded once
    int64_t *stats;
    const int32_t *bin_status;
    const uint64_t *bin_pairs;
};

// The blend's two skip tests (sigma < 0, alpha < 1/255) on the exponent
// q = -sigma log2(e) as one range test: a pixel takes the entry iff
// log2(1/255) - log2 o <= q <= 0, i.e. |q - c| <= -c with
// c = (log2(1/255) - log2 o) / 2, computed once per entry while staging
// (c > 0 when o < 1/255: then no pixel passes).  Every kernel that walks
// the lists stages c the same way, so their decisions agree bit for bit.
__device__ __forceinline__ float hit_center(float log2o) { return 0.5f * (kLog2AlphaMin - log2o); }

// Geometry of a lane: its column centre and first row's centre; and the
// tile's strips (2 RPL rows each): x centre and half width, y centre of the
// first strip, half height.
struct LaneGeom {
    float fx, fy0;
    float sx, hx, sy0, hy;
    int px, py0;
};

template <int kRPL>
__device__ __forceinline__ LaneGeom lane_geom(const CamConst &cam, int tile) {
    const int tx = tile % cam.tiles_x, ty = tile / cam.tiles_x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    LaneGeom L;
    L.px = tx * kTile + (lane & 15);
    L.py0 = ty * kTile + warp * 2 * kRPL + (lane >> 4) * kRPL;
    L.fx = (float)L.px + 0.5f;
    L.fy0 = (float)L.py0 + 0.5f;
    L.sx = (float)(tx * kTile) + 8.f;
    L.hx = 7.5f;
    L.sy0 = (float)(ty * kTile + kRPL);
    L.hy = (float)kRPL - 0.5f;
    return L;
}

// Bit w set unless the entry cannot reach alpha >= 1/255 anywhere in strip w
// of kStrips horizontal strips (x centre sx, half width hx; y centre
// sy0 + w step, half height hy).
template <int kStrips>
__device__ __forceinline__ uint32_t strip_mask(const float4 geo, const float4 geo2, float sx, float hx,
                                               float sy0, float step, float hy) {
    const float dxm = fmaxf(fabsf(geo.x - sx) - hx, 0.f);
    const float qx = geo2.z * dxm * dxm;
    uint32_t m = 0;
#pragma unroll
    for (int w = 0; w < kStrips; w++) {
        const float dym = fmaxf(fabsf(geo.y - (sy0 + step * (float)w)) - hy, 0.f);
        const float qb = fminf(qx, geo2.w * dym * dym);
        m |= (geo2.y + qb < kCullLog2 ? 0u : 1u) << w;
    }
    return m;
}

// Compacts the slots [k0, cnt) of a staged batch whose mask holds this
// warp's bit into list[0, n), in order (one ballot per 32 slots).  Returns n.
template <int kSlots>
__device__ __forceinline__ uint32_t compact_slots(const uint8_t *mask, uint32_t k0, uint32_t cnt, int warp,
                                                  int lane, uint8_t *list) {
    const uint32_t lt = (1u << lane) - 1u;
    uint32_t n = 0;
#pragma unroll
    for (int c = 0; c < kSlots / 32; c++) {
        const uint32_t i = c * 32 + lane;
        const bool f = i >= k0 && i < cnt && ((mask[i] >> warp) & 1u);
        const uint32_t bal = __ballot_sync(0xffffffffu, f);
        if (f) list[n + __popc(bal & lt)] = (uint8_t)i;
        n += __popc(bal);
    }
    __syncwarp();
    return n;
}

// Per-entry, per-lane terms shared by the lane's rows.
struct ColTerms {
    float dx, bdx, a0;  // mean - pixel x; cB dx; cA dx^2
};
__device__ __forceinline__ ColTerms col_terms(const float4 geo, float fx) {
    ColTerms t;
    t.dx = __fsub_rn(geo.x, fx);
    t.bdx = __fmul_rn(geo.w, t.dx);
    t.a0 = __fmul_rn(__fmul_rn(geo.z, t.dx), t.dx);
    return t;
}

// Alpha at one pixel.  q = -sigma log2(e) = cA dx^2 + dy (cB dx + cC dy);
// the entry is skipped there when sigma < 0 (q > 0) or alpha < 1/255
// (log2 o + q below log2(1/255)), both decided before the exponential.
// Returns false when skipped; else alpha = min(cap, o exp(-sigma)) and
// whether the cap applied.  dy = mean y - pixel y.
__device__ __forceinline__ bool eval_alpha(const float4 geo, const float4 geo2, const ColTerms &c, float cap,
                                           float fy, float &dy, float &alpha, bool &capped) {
    dy = __fsub_rn(geo.y, fy);
    const float u = __fmaf_rn(geo2.x, dy, c.bdx);
    const float q = __fmaf_rn(dy, u, c.a0);
    if (!(fabsf(__fsub_rn(q, geo2.z)) <= -geo2.z)) return false;  // the range test above
    const float p = __fadd_rn(q, geo2.y);              // log2(o exp(-sigma))
    const float a = ex2_approx(p);
    capped = a > cap;
    alpha = fminf(a, cap);
    return true;
}

// Forward, one pixel per thread, eight warps per tile; warp w owns the 8 x 4
// block of columns 8 (w & 1) .. + 7 and rows 4 (w >> 1) .. + 3 (an 8 x 4
// block is culled more tightly by the separable bound than a 16 x 2 strip:
// 17 % fewer walked warp-entries on 400k Gaussians at 980 x 545).  While a
// batch is staged, each entry's cull test for the eight blocks yields an
// 8-bit mask.  Each warp then takes the batch 64 slots at a time: the slots
// whose bit it holds are copied, in order, into a warp-private buffer that
// stores consecutive entries a, b side by side (mx_a, mx_b, my_a, my_b, ...),
// so that the exponents of two entries come out of one paired f32x2
// instruction each (each half rounded exactly as the scalar operation, so
// every decision equals the backward's); the walk then takes the pair's
// contributions in order.  A culled slot could not have passed the alpha
// test at any pixel of the block, so the sequence of contributions, the
// stopping entry and `last` are unchanged.
constexpr int kFwdChunk = 64;  // batch slots compacted per round
struct FwdWarpBuf {
    float4 xy[kFwdChunk / 2];   // mx_a, mx_b, my_a, my_b
    float4 ab[kFwdChunk / 2];   // cA_a, cA_b, cB_a, cB_b
    float4 cn[kFwdChunk / 2];   // cC_a, cC_b, -c_a, -c_b (c: the range test's centre)
    float2 lo[kFwdChunk / 2];   // log2 o_a, log2 o_b
    float4 col[kFwdChunk];      // channel values, entry by entry
    uint8_t slot[kFwdChunk];    // batch slot of each entry
};

// Bits of the eight 8 x 4 blocks of a tile (bit w: columns 8 (w & 1) ..,
// rows 4 (w >> 1) ..) in which the entry can reach alpha >= 1/255 (with the
// 1 % margin of the cull).  x0, y0: the tile's first pixel column and row.
__device__ __forceinline__ uint32_t block_mask(const float4 geo, const float4 geo2, float x0, float y0) {
    float qx[2], qy[4];
#pragma unroll
    for (int i = 0; i < 2; i++) {
        const float d = fmaxf(fabsf(geo.x - (x0 + 8.f * (float)i + 4.f)) - 3.5f, 0.f);
        qx[i] = geo2.z * d * d;
    }
#pragma unroll
    for (int j = 0; j < 4; j++) {
        const float d = fmaxf(fabsf(geo.y - (y0 + 4.f * (float)j + 2.f)) - 1.5f, 0.f);
        qy[j] = geo2.w * d * d;
    }
    uint32_t m = 0;
#pragma unroll
    for (int w = 0; w < 8; w++) m |= (geo2.y + fminf(qx[w & 1], qy[w >> 1]) < kCullLog2 ? 0u : 1u) << w;
    return m;
}

template <bool kDepth, bool kFeat = false, bool kL1 = false, bool kF8 = false>
__global__ void __launch_bounds__(kTilePixels, kF8 ? 4 : GS_FWD_MINB)
k_render_fwd(CamConst cam, const float4 *__restrict__ xyod, const float4 *__restrict__ conr,
             const ChannelIO io, const uint32_t *__restrict__ pair_gid,
             const uint2 *__restrict__ ranges, const uint32_t *__restrict__ order,
             float *__restrict__ image, float *__restrict__ T_final, uint32_t *__restrict__ last,
             const Bounds bd, const L1Out l1 = L1Out{}) {
    constexpr int kWarps = kTilePixels / 32;
    __shared__ float4 s_geo[kBatch];
    __shared__ float4 s_geo2[kBatch];
    __shared__ float4 s_col[kBatch];
    __shared__ uint8_t s_mask[kBatch];
    __shared__ FwdWarpBuf s_wb[kWarps];
    // kF8: channels 4-7 of a feature chunk of eight (values, then per warp)
    __shared__ float4 s_col2[kF8 ? kBatch : 1];
    __shared__ float4 s_wcol2[kF8 ? kWarps : 1][kF8 ? kFwdChunk : 1];

    const uint32_t tile_id = order[blockIdx.x];  // longest lists first
    if (!in_bounds(tile_id, bd.tiles, bd.status)) return;
    const int tile = (int)tile_id;
    const int tx = tile % cam.tiles_x, ty = tile / cam.tiles_x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int px = tx * kTile + 8 * (warp & 1) + (lane & 7);
    const int py = ty * kTile + 4 * (warp >> 1) + (lane >> 3);
    const float fx = (float)px + 0.5f, fy = (float)py + 0.5f;
    const float2 nfx = make_float2(-fx, -fx), nfy = make_float2(-fy, -fy);
    const float x0 = (float)(tx * kTile), y0 = (float)(ty * kTile);
    const uint2 range = ranges[tile];
    if (!range_in_bounds(range, bd)) return;
    FwdWarpBuf &wb = s_wb[warp];
    const uint32_t lt_mask = (1u << lane) - 1u;

    float T = 1.f, C0 = 0.f, C1 = 0.f, C2 = 0.f, C3 = 0.f;
    float C4 = 0.f, C5 = 0.f, C6 = 0.f, C7 = 0.f;  // kF8
    uint32_t lst = range.x;
    bool done = !(px < cam.width && py < cam.height);
    for (uint32_t b = range.x; b < range.y; b += kBatch) {
        if (__syncthreads_count(done) == kTilePixels) break;
        const uint32_t cnt = min((uint32_t)kBatch, range.y - b);
        if (threadIdx.x < cnt) {
            const uint32_t g = pair_gid[b + threadIdx.x];
            const bool ok = in_bounds(g, bd.n, bd.status);  // checked builds: else a slot no warp walks
            float4 geo = make_float4(0.f, 0.f, 0.f, 0.f), geo2 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (ok) stage_entry(xyod[g], conr[g], geo, geo2);
            s_geo[threadIdx.x] = geo;
            s_col[threadIdx.x] = ok ? io.col[kFeat ? (size_t)g * io.col_stride : (size_t)g] : geo;
            if (kF8) s_col2[threadIdx.x] = ok ? io.col[(size_t)g * io.col_stride + 1] : geo;
            s_mask[threadIdx.x] = ok ? (uint8_t)block_mask(geo, geo2, x0, y0) : (uint8_t)0;
            geo2.z = hit_center(geo2.y);  // kx, ky are only needed for the mask
            s_geo2[threadIdx.x] = geo2;
        }
        __syncthreads();
        for (uint32_t c0 = 0; c0 < cnt && __any_sync(0xffffffffu, !done); c0 += kFwdChunk) {
            // copy this warp's slots of [c0, c0 + 64) into the pair buffer
            uint32_t n = 0;
#pragma unroll
            for (int h = 0; h < kFwdChunk / 32; h++) {
                const uint32_t i = c0 + 32 * h + lane;
                const bool f = i < cnt && ((s_mask[i] >> warp) & 1u);
                const uint32_t bal = __ballot_sync(0xffffffffu, f);
                if (f) {
                    const uint32_t t = n + __popc(bal & lt_mask), pr = t >> 1;
                    const float4 geo = s_geo[i], geo2 = s_geo2[i];
                    float *xy = reinterpret_cast<float *>(&wb.xy[pr]);
                    float *ab = reinterpret_cast<float *>(&wb.ab[pr]);
                    float *cn = reinterpret_cast<float *>(&wb.cn[pr]);
                    const int hb = (int)(t & 1u);
                    xy[hb] = geo.x;
                    xy[2 + hb] = geo.y;
                    ab[hb] = geo.z;
                    ab[2 + hb] = geo.w;
                    cn[hb] = geo2.x;
                    cn[2 + hb] = -geo2.z;
                    reinterpret_cast<float *>(&wb.lo[pr])[hb] = geo2.y;
                    wb.col[t] = s_col[i];
                    if (kF8) s_wcol2[warp][t] = s_col2[i];
                    wb.slot[t] = (uint8_t)i;
                }
                n += __popc(bal);
            }
            if (n & 1u) {  // pad the last pair with an entry no pixel takes
                const uint32_t pr = n >> 1;
                if (lane == 0) {
                    reinterpret_cast<float *>(&wb.xy[pr])[1] = 0.f;
                    reinterpret_cast<float *>(&wb.xy[pr])[3] = 0.f;
                    reinterpret_cast<float *>(&wb.ab[pr])[1] = 0.f;
                    reinterpret_cast<float *>(&wb.ab[pr])[3] = 0.f;
                    reinterpret_cast<float *>(&wb.cn[pr])[1] = 0.f;
                    reinterpret_cast<float *>(&wb.cn[pr])[3] = -1.f;  // |q - c| <= -1 never holds
                    reinterpret_cast<float *>(&wb.lo[pr])[1] = 0.f;
                }
            }
            __syncwarp();
            int lt = -1;  // this chunk's last added entry, if any
            if (!done) {
                const uint32_t np = (n + 1u) >> 1;
                for (uint32_t k = 0; k < np; k++) {
                    const float4 xy = wb.xy[k], ab = wb.ab[k], cn = wb.cn[k];
                    const float2 dx = __fadd2_rn(make_float2(xy.x, xy.y), nfx);
                    const float2 bdx = __fmul2_rn(make_float2(ab.z, ab.w), dx);
                    const float2 a0 = __fmul2_rn(__fmul2_rn(make_float2(ab.x, ab.y), dx), dx);
                    const float2 dy = __fadd2_rn(make_float2(xy.z, xy.w), nfy);
                    const float2 u = __ffma2_rn(make_float2(cn.x, cn.y), dy, bdx);
                    const float2 q = __ffma2_rn(dy, u, a0);
                    const float2 t = __fadd2_rn(q, make_float2(cn.z, cn.w));  // q - c, as the backward
#if GS_FWD_EARLY_EX2
                    // both exponentials issued ahead of the tests, so their
                    // latency overlaps the branches (each half rounded as
                    // the scalar add, as the backward)
                    const float2 pe = __fadd2_rn(q, wb.lo[k]);
                    const float ea = ex2_approx(pe.x), eb = ex2_approx(pe.y);
#endif
                    if (fabsf(t.x) <= cn.z) {
#if GS_FWD_EARLY_EX2
                        const float a = fminf(ea, cam.alpha_cap);
#else
                        const float a = fminf(ex2_approx(__fadd_rn(q.x, wb.lo[k].x)), cam.alpha_cap);
#endif
                        const float nT = __fmaf_rn(-T, a, T);
                        if (nT < cam.t_stop) {
                            done = true;
                            break;
                        }
                        const float4 c = wb.col[2 * k];
                        const float w = __fmul_rn(a, T);
                        C0 = __fmaf_rn(w, c.x, C0);
                        C1 = __fmaf_rn(w, c.y, C1);
                        C2 = __fmaf_rn(w, c.z, C2);
                        if (kDepth) C3 = __fmaf_rn(w, c.w, C3);
                        if (kF8) {
                            const float4 c2 = s_wcol2[warp][2 * k];
                            C4 = __fmaf_rn(w, c2.x, C4);
                            C5 = __fmaf_rn(w, c2.y, C5);
                            C6 = __fmaf_rn(w, c2.z, C6);
                            C7 = __fmaf_rn(w, c2.w, C7);
                        }
                        T = nT;
                        lt = (int)(2 * k);
                    }
                    if (fabsf(t.y) <= cn.w) {
#if GS_FWD_EARLY_EX2
                        const float a = fminf(eb, cam.alpha_cap);
#else
                        const float a = fminf(ex2_approx(__fadd_rn(q.y, wb.lo[k].y)), cam.alpha_cap);
#endif
                        const float nT = __fmaf_rn(-T, a, T);
                        if (nT < cam.t_stop) {
                            done = true;
                            break;
                        }
                        const float4 c = wb.col[2 * k + 1];
                        const float w = __fmul_rn(a, T);
                        C0 = __fmaf_rn(w, c.x, C0);
                        C1 = __fmaf_rn(w, c.y, C1);
                        C2 = __fmaf_rn(w, c.z, C2);
                        if (kDepth) C3 = __fmaf_rn(w, c.w, C3);
                        if (kF8) {
                            const float4 c2 = s_wcol2[warp][2 * k + 1];
                            C4 = __fmaf_rn(w, c2.x, C4);
                            C5 = __fmaf_rn(w, c2.y, C5);
                            C6 = __fmaf_rn(w, c2.z, C6);
                            C7 = __fmaf_rn(w, c2.w, C7);
                        }
                        T = nT;
                        lt = (int)(2 * k + 1);
                    }
                }
            }
            if (lt >= 0) lst = b + wb.slot[lt] + 1;
            __syncwarp();
        }
    }
    float l1_sum = 0.f;
    if (px < cam.width && py < cam.height) {
        const size_t p = (size_t)py * cam.width + px;
        constexpr int kC = kDepth ? 4 : 3;
        float *out = image + (size_t)(kFeat ? io.img_stride : kC) * p;
        const float o[4] = {__fmaf_rn(T, cam.bg[0], C0), __fmaf_rn(T, cam.bg[1], C1),
                            __fmaf_rn(T, cam.bg[2], C2), C3};  // the fourth channel has no background
#pragma unroll
        for (int c = 0; c < kC; c++) out[c] = o[c];
        if (kF8) {  // feature chunks have no background
            out[4] = C4;
            out[5] = C5;
            out[6] = C6;
            out[7] = C7;
        }
        if (T_final) T_final[p] = T;
        if (last) last[p] = lst;
        if (kL1) {
#pragma unroll
            for (int c = 0; c < kC; c++) {
                const float d = o[c] - l1.target[kC * p + c];
                l1.dL[kC * p + c] = d > 0.f ? l1.inv : (d < 0.f ? -l1.inv : 0.f);
                l1_sum += fabsf(d);
            }
        }
    }
    if (kL1) {
        if (l1.stats && blockIdx.x == 0 && threadIdx.x == 0) {
            l1.stats[0] = (int64_t)*l1.bin_status;
            l1.stats[1] = (int64_t)*l1.bin_pairs;
        }
        if (l1.loss) {
            __shared__ float s_l1[kWarps];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) l1_sum += __shfl_xor_sync(0xffffffffu, l1_sum, o);
            if (lane == 0) s_l1[warp] = l1_sum;
            __syncthreads();
            if (threadIdx.x == 0) {
                float t = 0.f;
#pragma unroll
                for (int w = 0; w < kWarps; w++) t += s_l1[w];
                atomicAdd(l1.loss, t * l1.inv);
            }
        }
    }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Size of the kept half at xor level `level` (0: 16, 1: 8, 2: 4, 3: 2) of a
// reduce-scatter of n values.
__host__ __device__ constexpr int rs_half(int n, int level) {
    for (int i = 0; i < level; i++) n = (n + 1) / 2;
    return (n + 1) / 2;
}
// Even lanes that end a reduce-scatter of n values holding a real value (not
// the zero padding of an odd half).
__host__ __device__ constexpr uint32_t rs_valid_lanes(int n) {
    uint32_t mask = 0;
    for (int lane = 0; lane < 32; lane += 2) {
        int real = n;
        for (int level = 0; level < 4; level++) {
            const int h = rs_half(n, level);
            real = (lane & (16 >> level)) ? (real > h ? real - h : 0) : (real < h ? real : h);
        }
        if (real > 0) mask |= 1u << lane;
    }
    return mask;
}

// Warp reduce-scatter of N <= 16 values per lane.  At each xor level (16,
// 8, 4, 2) a lane keeps one half of its values and sends the other half to
// its partner, which keeps that half; the last level (1) sums the one value
// left.  A 9-value reduce takes 46 instructions instead of the 90 of nine
// full butterflies.  On return every even lane whose *idx is in [0, N)
// holds the warp total of value *idx (one lane per value).
template <int N>
__device__ __forceinline__ float reduce_scatter(const float (&v)[N], int lane, int *idx) {
    static_assert(N >= 2 && N <= 16, "2 to 16 values");
    float a[16];
#pragma unroll
    for (int i = 0; i < 16; i++) a[i] = i < N ? v[i] : 0.f;
    int m = N;  // values left per lane
#pragma unroll
    for (int off = 16; off >= 2; off >>= 1) {
        const int h = (m + 1) / 2;
        const bool up = lane & off;
#pragma unroll
        for (int i = 0; i < 8; i++) {
            if (i >= h) break;
            const float lo = a[i], hi = h + i < m ? a[h + i] : 0.f;
            a[i] = (up ? hi : lo) + __shfl_xor_sync(0xffffffffu, up ? lo : hi, off);
        }
        m = h;
    }
    const float x = a[0] + __shfl_xor_sync(0xffffffffu, a[0], 1);
    // which value the lane ended with: the halves it kept, level by level
    constexpr uint32_t kValid = rs_valid_lanes(N);
    const int base = ((lane & 16) ? rs_half(N, 0) : 0) + ((lane & 8) ? rs_half(N, 1) : 0) +
                     ((lane & 4) ? rs_half(N, 2) : 0) + ((lane & 2) ? rs_half(N, 3) : 0);
    *idx = ((kValid >> lane) & 1u) ? base : N;
    return x;
}

// Backward of the blend.  Per pixel, from the last added entry back to the
// first: with T the transmittance after entry i, r = 1 / (1 - alpha_i),
// T_i = T r, and sg = <S_i, g> where S_i = T_{i+1} R_i is the colour already
// composited behind i (S_last = T_final bg),
//     dL/dalpha_i = T_i <c_i, g> - sg / (1 - alpha_i),
//     sg <- sg + alpha_i T_i <c_i, g>,   dL/dc_i = alpha_i T_i g.
// (the same quantities as T_i <c_i - R_i, g> with R the normalised colour
// behind, carried as one scalar instead of a colour).  The nine sums
// per entry, over the warp's pixels, are
//     sum v, sum v dx, sum v dy, sum v dx^2, sum v dx dy, sum v dy^2, sum w g
// with v = alpha dL/dalpha (0 when alpha was capped), w = alpha T_i; they are
// added into grad2d, and k_project_bwd maps them to dL/d(mean2d, conic,
// opacity) with the Gaussian's own A, B, C, o.  In a frame with few pairs
// per Gaussian, an entry that at most GS_BWD_DIRECT lanes of the warp reach
// is added by those lanes directly (their atomics on the same addresses
// meet in L2); any other is summed over the warp by a reduce-scatter first,
// one atomic per value.
template <int kRPL, bool kDepth, bool kFeat = false, bool kF8 = false>
__global__ void __launch_bounds__(kTilePixels / kRPL, kF8 ? 8 : GS_BWD_MINB)
k_render_bwd(CamConst cam, const float4 *__restrict__ xyod, const float4 *__restrict__ conr,
             const ChannelIO io, const uint32_t *__restrict__ pair_gid,
             const uint2 *__restrict__ ranges, const uint32_t *__restrict__ order,
             const float *__restrict__ T_final,
             const uint32_t *__restrict__ last, const float *__restrict__ dL_dimage,
             float *__restrict__ grad2d, const Bounds bd) {
    static_assert(kRPL % 2 == 0, "the backward works on pairs of rows");
    constexpr int kThreads = kTilePixels / kRPL;
    constexpr int kWarps = kThreads / 32;
    constexpr int kPairs = kRPL / 2;
    constexpr int kB = kBwdBatch;
    __shared__ float4 s_geo[kB];
    __shared__ float4 s_geo2[kB];
    __shared__ float4 s_col[kB];
    __shared__ float4 s_col2[kF8 ? kB : 1];  // kF8: channels 4-7 of a feature chunk of eight
    __shared__ uint32_t s_gid[kB];
    __shared__ uint8_t s_mask[kB];
    __shared__ uint8_t s_list[kWarps][kB];
    __shared__ uint32_t s_max_last;

    const uint32_t tile_id = order[blockIdx.x];  // longest lists first
    if (!in_bounds(tile_id, bd.tiles, bd.status)) return;
    const int tile = (int)tile_id;
    const LaneGeom L = lane_geom<kRPL>(cam, tile);
    const uint2 range = ranges[tile];
    if (!range_in_bounds(range, bd)) return;
    const bool col_in = L.px < cam.width;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    // Per pixel state, two rows per float2 (x: row 2i, y: row 2i + 1).
    constexpr int kC = kDepth ? 4 : 3;  // image channels
    float2 T[kPairs], sg[kPairs], g0[kPairs], g1[kPairs], g2[kPairs], g3[kPairs], nfy[kPairs];
    float2 g4[kPairs], g5[kPairs], g6[kPairs], g7[kPairs];  // kF8
    uint32_t lst[kRPL];
    uint32_t lane_max = range.x;
#pragma unroll
    for (int r = 0; r < kRPL; r++) {
        float t = 1.f, d0 = 0.f, d1 = 0.f, d2 = 0.f, d3 = 0.f, d4 = 0.f, d5 = 0.f, d6 = 0.f, d7 = 0.f;
        lst[r] = range.x;
        const int py = L.py0 + r;
        if (col_in && py < cam.height) {
            const size_t p = (size_t)py * cam.width + L.px;
            t = T_final[p];
            lst[r] = min(max(last[p], range.x), range.y);  // never walk outside the tile's list
            const float *dp = dL_dimage + (size_t)(kFeat ? io.img_stride : kC) * p;
            d0 = dp[0];
            d1 = dp[1];
            d2 = dp[2];
            if (kDepth) d3 = dp[3];
            if (kF8) {
                d4 = dp[4];
                d5 = dp[5];
                d6 = dp[6];
                d7 = dp[7];
            }
        }
        const float s0 = t * (cam.bg[0] * d0 + cam.bg[1] * d1 + cam.bg[2] * d2);  // depth: no background
        const float nf = -(L.fy0 + (float)r);
        if (r & 1) {
            T[r / 2].y = t; g0[r / 2].y = d0; g1[r / 2].y = d1; g2[r / 2].y = d2; g3[r / 2].y = d3;
            sg[r / 2].y = s0; nfy[r / 2].y = nf;
            g4[r / 2].y = d4; g5[r / 2].y = d5; g6[r / 2].y = d6; g7[r / 2].y = d7;
        } else {
            T[r / 2].x = t; g0[r / 2].x = d0; g1[r / 2].x = d1; g2[r / 2].x = d2; g3[r / 2].x = d3;
            sg[r / 2].x = s0; nfy[r / 2].x = nf;
            g4[r / 2].x = d4; g5[r / 2].x = d5; g6[r / 2].x = d6; g7[r / 2].x = d7;
        }
        lane_max = max(lane_max, lst[r]);
    }
    // entries at or past every pixel's last are not walked: per warp and per CTA
    uint32_t warp_max = lane_max;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) warp_max = max(warp_max, __shfl_xor_sync(0xffffffffu, warp_max, o));
    if (threadIdx.x == 0) s_max_last = range.x;
    __syncthreads();
    if (lane == 0) atomicMax(&s_max_last, warp_max);
    __syncthreads();
    const uint32_t max_last = s_max_last;
    const bool direct = GS_BWD_DIRECT > 0 && *bd.n_pairs <= (uint64_t)GS_BWD_DIRECT_PAIRS * bd.n;

    // Sums of an entry: the six geometric ones into grad2d, the channel sums
    // after them (colours) or into io.cgrad (a feature chunk).
    constexpr int kV = 6 + kC + (kF8 ? 4 : 0);
    auto add_sums = [&](uint32_t g, int i, float x) {
        float *dst = grad2d + 12 * (size_t)g + i;
        if (kFeat && i >= 6) dst = io.cgrad + (size_t)io.cgrad_stride * g + (i - 6);
        atomicAdd(dst, x);
    };

    // The walk, compiled twice: with the direct path (frames with few pairs
    // per Gaussian) and without it, chosen once per CTA, so that frames
    // without it run the reduce-only loop.
    auto walk = [&](auto direct_tag) {
        constexpr bool kDirect = decltype(direct_tag)::value;
        for (uint32_t bend = max_last; bend > range.x;) {
            const uint32_t bstart = bend - range.x > (uint32_t)kB ? bend - kB : range.x;
            const uint32_t cnt = bend - bstart;
            // slot i holds list entry bend - 1 - i (slot 0 = back-most); each
            // thread stages two entries per round (ids first, then records), so
            // the dependent loads overlap
            for (uint32_t i0 = threadIdx.x; i0 < cnt; i0 += 2 * kThreads) {
                const uint32_t i1 = i0 + kThreads;
                uint32_t ga = pair_gid[bend - 1 - i0];
                uint32_t gb = i1 < cnt ? pair_gid[bend - 1 - i1] : ga;
                // checked builds: an id out of range is replaced by 0 and its slot
                // never walked
                const bool oka = in_bounds(ga, bd.n, bd.status), okb = i1 >= cnt || in_bounds(gb, bd.n, bd.status);
                if (kCheck && !oka) ga = 0;
                if (kCheck && !okb) gb = 0;
                const float4 xa = xyod[ga], ca = conr[ga], ra = io.col[kFeat ? (size_t)ga * io.col_stride : (size_t)ga];
                const float4 xb = xyod[gb], cb = conr[gb], rb = io.col[kFeat ? (size_t)gb * io.col_stride : (size_t)gb];
                float4 geo, geo2;
                stage_entry(xa, ca, geo, geo2);
                s_geo[i0] = geo;
                s_geo2[i0] = geo2;
                s_col[i0] = ra;
                if (kF8) s_col2[i0] = io.col[(size_t)ga * io.col_stride + 1];
                s_gid[i0] = ga;
                s_mask[i0] = oka ? (uint8_t)strip_mask<kWarps>(geo, geo2, L.sx, L.hx, L.sy0, 2.f * kRPL, L.hy) : 0;
                s_geo2[i0].z = hit_center(geo2.y);
                if (i1 < cnt) {
                    stage_entry(xb, cb, geo, geo2);
                    s_geo[i1] = geo;
                    s_geo2[i1] = geo2;
                    s_col[i1] = rb;
                    if (kF8) s_col2[i1] = io.col[(size_t)gb * io.col_stride + 1];
                    s_gid[i1] = gb;
                    s_mask[i1] = okb ? (uint8_t)strip_mask<kWarps>(geo, geo2, L.sx, L.hx, L.sy0, 2.f * kRPL, L.hy) : 0;
                    s_geo2[i1].z = hit_center(geo2.y);
                }
            }
            __syncthreads();
            // this warp's slots: reached by one of its pixels (entry below
            // warp_max) and not culled for its strip
            const uint32_t k0 = bend > warp_max ? min(bend - warp_max, cnt) : 0u;
            const uint32_t n = compact_slots<kB>(s_mask, k0, cnt, warp, lane, s_list[warp]);
            for (uint32_t t = 0; t < n; t++) {
                const uint32_t k = s_list[warp][t];
                const uint32_t j = bend - 1 - k;
                const float4 geo = s_geo[k], geo2 = s_geo2[k];
                const ColTerms ct = col_terms(geo, L.fx);
                // The exponent at the lane's rows, two rows per paired instruction
                // (each half rounded exactly as the forward's scalar evaluation,
                // so every skip decision is the same), and which rows pass.
                float2 dy[kPairs], p[kPairs];
                bool hit[kRPL];
                bool any = false;
#pragma unroll
                for (int i = 0; i < kPairs; i++) {
                    dy[i] = __fadd2_rn(make_float2(geo.y, geo.y), nfy[i]);
                    const float2 u = __ffma2_rn(make_float2(geo2.x, geo2.x), dy[i], make_float2(ct.bdx, ct.bdx));
                    const float2 q = __ffma2_rn(dy[i], u, make_float2(ct.a0, ct.a0));
                    p[i] = __fadd2_rn(q, make_float2(geo2.y, geo2.y));
                    const float2 t = __fadd2_rn(q, make_float2(-geo2.z, -geo2.z));  // q - c, as the forward
                    hit[2 * i] = j < lst[2 * i] && fabsf(t.x) <= -geo2.z;
                    hit[2 * i + 1] = j < lst[2 * i + 1] && fabsf(t.y) <= -geo2.z;
                    any |= hit[2 * i] | hit[2 * i + 1];
                }
                uint32_t hit_lanes = 0;
                if constexpr (kDirect) {
                    hit_lanes = __ballot_sync(0xffffffffu, any);
                    if (!hit_lanes) continue;
                } else if (!__any_sync(0xffffffffu, any)) {
                    continue;
                }
                // Contributions, branch-free (measured faster than skipping per
                // row, and than skipping the cap for entries that cannot reach
                // it): a skipped row has alpha 0, which zeroes w, v and every sum
                // exactly (colours of drawn Gaussians are finite) and leaves T as
                // it is (T / (1 - 0) with the approximate reciprocal of 1, which
                // is exact).
                const float4 c = s_col[k];
                const float4 c2 = kF8 ? s_col2[k] : c;
                float2 sv = make_float2(0.f, 0.f), sgy = sv, sgyy = sv, cr0 = sv, cr1 = sv, cr2 = sv, cr3 = sv;
                float2 cr4 = sv, cr5 = sv, cr6 = sv, cr7 = sv;
#pragma unroll
                for (int i = 0; i < kPairs; i++) {
                    const bool h0 = hit[2 * i], h1 = hit[2 * i + 1];
                    const float e0 = ex2_approx(p[i].x), e1 = ex2_approx(p[i].y);
                    const float2 a = make_float2(h0 ? fminf(e0, cam.alpha_cap) : 0.f, h1 ? fminf(e1, cam.alpha_cap) : 0.f);
                    // alpha for the opacity and conic gradients: 0 where the cap applied
                    const float2 av = make_float2(e0 > cam.alpha_cap ? 0.f : a.x, e1 > cam.alpha_cap ? 0.f : a.y);
                    const float2 om = __fadd2_rn(make_float2(1.f, 1.f), make_float2(-a.x, -a.y));
                    const float2 ri = make_float2(rcp_approx(om.x), rcp_approx(om.y));
                    const float2 Ti = __fmul2_rn(T[i], ri);
                    const float2 w = __fmul2_rn(a, Ti);
                    float2 cg = __ffma2_rn(make_float2(c.z, c.z), g2[i],
                                           __ffma2_rn(make_float2(c.y, c.y), g1[i],
                                                      __fmul2_rn(make_float2(c.x, c.x), g0[i])));
                    if (kDepth) cg = __ffma2_rn(make_float2(c.w, c.w), g3[i], cg);
                    if (kF8) {
                        cg = __ffma2_rn(make_float2(c2.x, c2.x), g4[i], cg);
                        cg = __ffma2_rn(make_float2(c2.y, c2.y), g5[i], cg);
                        cg = __ffma2_rn(make_float2(c2.z, c2.z), g6[i], cg);
                        cg = __ffma2_rn(make_float2(c2.w, c2.w), g7[i], cg);
                    }
                    const float2 dLda = __fmul2_rn(ri, __ffma2_rn(T[i], cg, make_float2(-sg[i].x, -sg[i].y)));
                    sg[i] = __ffma2_rn(w, cg, sg[i]);
                    cr0 = __ffma2_rn(w, g0[i], cr0);
                    cr1 = __ffma2_rn(w, g1[i], cr1);
                    cr2 = __ffma2_rn(w, g2[i], cr2);
                    if (kDepth) cr3 = __ffma2_rn(w, g3[i], cr3);
                    if (kF8) {
                        cr4 = __ffma2_rn(w, g4[i], cr4);
                        cr5 = __ffma2_rn(w, g5[i], cr5);
                        cr6 = __ffma2_rn(w, g6[i], cr6);
                        cr7 = __ffma2_rn(w, g7[i], cr7);
                    }
                    const float2 v = __fmul2_rn(dLda, av);  // dL/dsigma = -v, dL/do = v / o
                    sv = __fadd2_rn(sv, v);
                    const float2 vy = __fmul2_rn(v, dy[i]);
                    sgy = __fadd2_rn(sgy, vy);
                    sgyy = __ffma2_rn(vy, dy[i], sgyy);
                    T[i] = Ti;  // a skipped row: alpha 0, rcp.approx(1) = 1 exactly, so Ti = T
                }
                const float svs = sv.x + sv.y, sgys = sgy.x + sgy.y;
                const float sgx = svs * ct.dx;
                float vals[kV];
                vals[0] = svs;
                vals[1] = sgx;
                vals[2] = sgys;
                vals[3] = sgx * ct.dx;
                vals[4] = sgys * ct.dx;
                vals[5] = sgyy.x + sgyy.y;
                vals[6] = cr0.x + cr0.y;
                vals[7] = cr1.x + cr1.y;
                vals[8] = cr2.x + cr2.y;
                if constexpr (kDepth) vals[9] = cr3.x + cr3.y;
                if constexpr (kF8) {
                    vals[10] = cr4.x + cr4.y;
                    vals[11] = cr5.x + cr5.y;
                    vals[12] = cr6.x + cr6.y;
                    vals[13] = cr7.x + cr7.y;
                }
                if (kDirect && __popc(hit_lanes) <= GS_BWD_DIRECT) {
                    // few lanes: each adds its own sums (a lane with no row
                    // reached holds zeros and adds nothing)
                    if (any) {
                        const uint32_t g = s_gid[k];
#pragma unroll
                        for (int i = 0; i < kV; i++) add_sums(g, i, vals[i]);
                    }
                    continue;
                }
                int idx;
                const float tot = reduce_scatter<kV>(vals, lane, &idx);
                if (idx < kV) add_sums(s_gid[k], idx, tot);
            }
            __syncthreads();
            bend = bstart;
        }
    };
    if (direct)
        walk(std::true_type{});
    else
        walk(std::false_type{});
}

// The forward's walk with counters instead of blending (no culling, one pixel
// per thread): the work the method must do.
__global__ void __launch_bounds__(kTilePixels)
k_render_stats(CamConst cam, const float4 *__restrict__ xyod, const float4 *__restrict__ conr,
               const uint32_t *__restrict__ pair_gid, const uint2 *__restrict__ ranges,
               const uint32_t *__restrict__ last, unsigned long long *__restrict__ counts, const Bounds bd) {
    __shared__ float4 s_geo[kBatch];
    __shared__ float4 s_geo2[kBatch];
    __shared__ unsigned long long s_c[3];
    const int tile = blockIdx.x;
    const int tx = tile % cam.tiles_x, ty = tile / cam.tiles_x;
    const int px = tx * kTile + (threadIdx.x & (kTile - 1));
    const int py = ty * kTile + (threadIdx.x >> 4);
    const bool inside = px < cam.width && py < cam.height;
    const float fx = (float)px + 0.5f, fy = (float)py + 0.5f;
    const uint2 range = ranges[tile];
    if (!range_in_bounds(range, bd)) return;
    if (threadIdx.x < 3) s_c[threadIdx.x] = 0ull;
    float T = 1.f;
    unsigned long long visits = 0, adds = 0;
    bool done = !inside;
    for (uint32_t b = range.x; b < range.y; b += kBatch) {
        if (__syncthreads_count(done) == kTilePixels) break;
        const uint32_t j = b + threadIdx.x;
        if (j < range.y) {
            const uint32_t g = pair_gid[j];
            float4 geo = make_float4(0.f, 0.f, 0.f, 0.f), geo2 = make_float4(0.f, 0.f, 1.f, 0.f);
            if (in_bounds(g, bd.n, bd.status)) {  // checked builds: else an entry no pixel takes
                stage_entry(xyod[g], conr[g], geo, geo2);
                geo2.z = hit_center(geo2.y);
            }
            s_geo[threadIdx.x] = geo;
            s_geo2[threadIdx.x] = geo2;
        }
        __syncthreads();
        const int cnt = (int)min((uint32_t)kBatch, range.y - b);
        if (!done) {
            for (int k = 0; k < cnt; k++) {
                float dy, a;
                bool capped;
                visits++;
                const float4 geo = s_geo[k], geo2 = s_geo2[k];
                const ColTerms ct = col_terms(geo, fx);
                if (!eval_alpha(geo, geo2, ct, cam.alpha_cap, fy, dy, a, capped)) continue;
                const float nT = __fmaf_rn(-T, a, T);
                if (nT < cam.t_stop) { done = true; break; }
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

// The tile order gs_bin_and_sort left in the bins' scratch.
static const uint32_t *tile_order(const gs_bins &bins) {
    const BinsLayout L = bins_layout(bins.max_n, bins.max_pairs, bins.max_tiles);
    return reinterpret_cast<const uint32_t *>(static_cast<const char *>(bins.scratch) + L.tile_order);
}

cudaError_t launch_render_fwd(const CamConst &c, int64_t n, const gs_projected &proj, const gs_bins &bins,
                              float *image, float *T_final, uint32_t *last, cudaStream_t s, const float *target,
                              float *dL_dimage, float *loss, int64_t *stats) {
    const int tiles = c.tiles_x * c.tiles_y;
    const Bounds bd = bounds_of(bins, n, tiles);
    const bool depth = c.flags & GS_FLAG_DEPTH;
    const ChannelIO io{reinterpret_cast<const float4 *>(proj.rgb), 1, depth ? 4 : 3, nullptr, 0};
    const float4 *xy = reinterpret_cast<const float4 *>(proj.xy_opacity_depth);
    const float4 *cr = reinterpret_cast<const float4 *>(proj.conic_radius);
    const uint2 *rg = reinterpret_cast<const uint2 *>(bins.ranges);
    if (target) {  // the forward with the L1 loss in its epilogue
        if (loss) {
            const cudaError_t e = cudaMemsetAsync(loss, 0, sizeof(float), s);
            if (e != cudaSuccess) return e;
        }
        const int64_t count = (int64_t)c.width * c.height * (depth ? 4 : 3);
        const L1Out l1{target, dL_dimage, loss, 1.f / (float)count, stats, bins.status,
                       reinterpret_cast<const uint64_t *>(bins.n_pairs)};
        prof_before("render_fwd", s);
        if (depth)
            k_render_fwd<true, false, true><<<tiles, kTilePixels, 0, s>>>(c, xy, cr, io, bins.pair_gid, rg,
                                                                        tile_order(bins), image, T_final, last,
                                                                        bd, l1);
        else
            k_render_fwd<false, false, true><<<tiles, kTilePixels, 0, s>>>(c, xy, cr, io, bins.pair_gid, rg,
                                                                         tile_order(bins), image, T_final, last,
                                                                         bd, l1);
        prof_after(s);
        return cudaGetLastError();
    }
    prof_before("render_fwd", s);
    if (depth)
        k_render_fwd<true><<<tiles, kTilePixels, 0, s>>>(c, xy, cr, io, bins.pair_gid, rg, tile_order(bins), image,
                                                         T_final, last, bd);
    else
        k_render_fwd<false><<<tiles, kTilePixels, 0, s>>>(c, xy, cr, io, bins.pair_gid, rg, tile_order(bins), image,
                                                          T_final, last, bd);
    prof_after(s);
    return cudaGetLastError();
}

cudaError_t launch_render_features_fwd(const CamConst &c, int64_t n, const gs_projected &proj, const gs_bins &bins,
                                       const float *features, int F, float *out, cudaStream_t s) {
    const int tiles = c.tiles_x * c.tiles_y;
    const Bounds bd = bounds_of(bins, n, tiles);
    CamConst cf = c;  // features blend without a background
    cf.bg[0] = cf.bg[1] = cf.bg[2] = 0.f;
    prof_before("render_features_fwd", s);
    const float4 *xy = reinterpret_cast<const float4 *>(proj.xy_opacity_depth);
    const float4 *cr = reinterpret_cast<const float4 *>(proj.conic_radius);
    const uint2 *rg = reinterpret_cast<const uint2 *>(bins.ranges);
    int launched = 0;
    for (int c0 = 0; c0 < F; launched++) {  // chunks of eight channels, then one of four
        const ChannelIO io{reinterpret_cast<const float4 *>(features) + c0 / 4, F / 4, F, nullptr, 0};
        if (F - c0 >= 8) {
            k_render_fwd<true, true, false, true><<<tiles, kTilePixels, 0, s>>>(
                cf, xy, cr, io, bins.pair_gid, rg, tile_order(bins), out + c0, nullptr, nullptr, bd);
            c0 += 8;
        } else {
            k_render_fwd<true, true><<<tiles, kTilePixels, 0, s>>>(cf, xy, cr, io, bins.pair_gid, rg,
                                                                 tile_order(bins), out + c0, nullptr, nullptr, bd);
            c0 += 4;
        }
    }
    prof_after(s, launched);
    return cudaGetLastError();
}

cudaError_t launch_render_bwd(const CamConst &c, int64_t n, const gs_projected &proj, const gs_bins &bins,
                              const float *T_final, const uint32_t *last, const float *dL_dimage,
                              float *grad2d, cudaStream_t s) {
    const int tiles = c.tiles_x * c.tiles_y;
    const Bounds bd = bounds_of(bins, n, tiles);
    const bool depth = c.flags & GS_FLAG_DEPTH;
    const ChannelIO io{reinterpret_cast<const float4 *>(proj.rgb), 1, depth ? 4 : 3, grad2d + 6, 12};
    prof_before("render_bwd", s);
    if (depth)
        k_render_bwd<GS_BWD_RPL, true><<<tiles, kTilePixels / GS_BWD_RPL, 0, s>>>(
            c, reinterpret_cast<const float4 *>(proj.xy_opacity_depth),
            reinterpret_cast<const float4 *>(proj.conic_radius), io, bins.pair_gid,
            reinterpret_cast<const uint2 *>(bins.ranges), tile_order(bins), T_final, last, dL_dimage, grad2d, bd);
    else
        k_render_bwd<GS_BWD_RPL, false><<<tiles, kTilePixels / GS_BWD_RPL, 0, s>>>(
            c, reinterpret_cast<const float4 *>(proj.xy_opacity_depth),
            reinterpret_cast<const float4 *>(proj.conic_radius), io, bins.pair_gid,
            reinterpret_cast<const uint2 *>(bins.ranges), tile_order(bins), T_final, last, dL_dimage, grad2d, bd);
    prof_after(s);
    return cudaGetLastError();
}

cudaError_t launch_render_features_bwd(const CamConst &c, int64_t n, const gs_projected &proj, const gs_bins &bins,
                                       const float *T_final, const uint32_t *last, const float *features,
                                       int F, const float *dL_dout, float *grad2d, float *dL_dfeatures,
                                       cudaStream_t s) {
    const int tiles = c.tiles_x * c.tiles_y;
    const Bounds bd = bounds_of(bins, n, tiles);
    CamConst cf = c;  // features blend without a background
    cf.bg[0] = cf.bg[1] = cf.bg[2] = 0.f;
    prof_before("render_features_bwd", s);
    const float4 *xy = reinterpret_cast<const float4 *>(proj.xy_opacity_depth);
    const float4 *cr = reinterpret_cast<const float4 *>(proj.conic_radius);
    const uint2 *rg = reinterpret_cast<const uint2 *>(bins.ranges);
    int launched = 0;
    for (int c0 = 0; c0 < F; launched++) {  // chunks of eight channels, then one of four
        const ChannelIO io{reinterpret_cast<const float4 *>(features) + c0 / 4, F / 4, F, dL_dfeatures + c0, F};
        if (F - c0 >= 8) {
            k_render_bwd<GS_BWD_RPL, true, true, true><<<tiles, kTilePixels / GS_BWD_RPL, 0, s>>>(
                cf, xy, cr, io, bins.pair_gid, rg, tile_order(bins), T_final, last, dL_dout + c0, grad2d, bd);
            c0 += 8;
        } else {
            k_render_bwd<GS_BWD_RPL, true, true><<<tiles, kTilePixels / GS_BWD_RPL, 0, s>>>(
                cf, xy, cr, io, bins.pair_gid, rg, tile_order(bins), T_final, last, dL_dout + c0, grad2d, bd);
            c0 += 4;
        }
    }
    prof_after(s, launched);
    return cudaGetLastError();
}

cudaError_t launch_render_stats(const CamConst &c, int64_t n, const gs_projected &proj, const gs_bins &bins,
                                const uint32_t *last, uint64_t *counts, cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(counts, 0, 4 * sizeof(uint64_t), s);
    if (e != cudaSuccess) return e;
    const int tiles = c.tiles_x * c.tiles_y;
    const Bounds bd = bounds_of(bins, n, tiles);
    prof_before("render_stats", s);
    k_render_stats<<<tiles, kTilePixels, 0, s>>>(
        c, reinterpret_cast<const float4 *>(proj.xy_opacity_depth),
        reinterpret_cast<const float4 *>(proj.conic_radius), bins.pair_gid,
        reinterpret_cast<const uint2 *>(bins.ranges), last,
        reinterpret_cast<unsigned long long *>(counts), bd);
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
