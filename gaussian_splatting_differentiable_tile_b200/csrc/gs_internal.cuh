// gs_internal.cuh -- definitions shared by the CUDA translation units of
// libgs.so.  Not part of the public ABI (that is include/gs.h).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "gs.h"

namespace gs {

constexpr int kTile = GS_TILE;            // 16 x 16 pixel tiles
constexpr int kTilePixels = kTile * kTile;

// Radix digits of the long-list sort: 8 bits.
constexpr int kRadixBits = 8;
constexpr int kRadix = 1 << kRadixBits;

// Binning: the count matrix [CTA][tile] holds at most kBinHistCap entries
// and is split among at most kBinCTAsMax CTAs.
constexpr int kBinCTAsMax = 320;
constexpr int64_t kBinHistCap = (int64_t)1 << 22;

// Camera constants derived once on the host.
struct CamConst {
    float R[9];         // world-to-camera rotation, row-major
    float t[3];         // world-to-camera translation
    float fx, fy, cx, cy;
    float lim_x_lo, lim_x_hi, lim_y_lo, lim_y_hi;  // clamp range of x/z, y/z for J
    float near_z;
    float bg[3];
    int32_t width, height, tiles_x, tiles_y;
    uint32_t flags;     // GS_FLAG_* of the camera
    float alpha_cap;    // 0.99, or 0.999 with GS_FLAG_CAP_0999
    float t_stop;       // a pixel stops once T (1 - alpha) < t_stop
};

// Byte layout of a gs_bins buffer.  The first `zero_bytes` bytes are cleared
// by one memset at the start of every gs_bin_and_sort.
struct BinsLayout {
    size_t status, n_pairs;     // the status word and K
    size_t zero_bytes;
    size_t tile_total;          // [max_tiles] pairs per tile
    size_t ranges;              // [max_tiles][2]
    size_t tile_order;          // [max_tiles] tiles, longest list first
    size_t bin_hist;            // count matrix: per-CTA tile counts, then offsets
    size_t keys;                // u64[max_pairs] emitted sort keys
    size_t long_keys, long_ids; // u32[max_pairs] each: scratch of the long-list sort
    size_t pair_tile, pair_gid; // u32[max_pairs] each: the result
    size_t total;
};

constexpr size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

constexpr BinsLayout bins_layout(int64_t max_n, int64_t max_pairs, int32_t max_tiles) {
    (void)max_n;
    BinsLayout L{};
    size_t off = 0;
    L.status = off;       off += 8;
    L.n_pairs = off;      off += 8;
    off = align_up(off, 256);
    L.zero_bytes = off;
    const size_t tb = align_up((size_t)max_tiles * sizeof(uint32_t), 256);
    L.tile_total = off;   off += tb;
    L.ranges = off;       off += 2 * tb;
    L.tile_order = off;   off += tb;
    L.bin_hist = off;
    {
        const int64_t h = (int64_t)kBinCTAsMax * max_tiles;
        off = align_up(off + (size_t)(h < kBinHistCap ? h : kBinHistCap) * sizeof(uint32_t), 256);
    }
    const size_t pb = align_up((size_t)max_pairs * sizeof(uint32_t), 256);
    L.keys = off;      off += 2 * pb;
    L.long_keys = off; off += pb;
    L.long_ids = off;  off += pb;
    L.pair_tile = off; off += pb;
    L.pair_gid = off;  off += pb;
    L.total = off;
    return L;
}

// ---------------------------------------------------------------- device
#ifdef __CUDACC__
// A splat's tile rectangle clamped to the grid: returns the number of tiles
// it covers (0 when empty) and its first column, row and width.  Binning
// derives everything from the rectangle, so records from any source can
// never produce a tile id outside the grid.
__device__ __forceinline__ uint32_t rect_tiles(int4 r, int tiles_x, int tiles_y, int &x0, int &y0,
                                               int &w) {
    x0 = max(r.x, 0);
    y0 = max(r.y, 0);
    const int x1 = min(r.z, tiles_x - 1), y1 = min(r.w, tiles_y - 1);
    if (x0 > x1 || y0 > y1) {
        w = 0;
        return 0u;
    }
    w = x1 - x0 + 1;
    return (uint32_t)w * (uint32_t)(y1 - y0 + 1);
}
// Records the first error code only.
__device__ __forceinline__ void set_status(int32_t *status, int32_t code) {
    atomicCAS(status, 0, code);
}
#endif

// Checked builds (libgs_check.so, compiled with -DGS_CHECK) test the index of
// every gather and scatter of the blend, binning and sort kernels against its
// array's bound: an index out of range records GS_ERR_BOUNDS in the bins'
// status word and the access is skipped (no trap).  Ordinary builds compile
// the tests away.
#ifdef GS_CHECK
constexpr bool kCheck = true;
#else
constexpr bool kCheck = false;
#endif
// What a checked build tests kernel indices against.
struct Bounds {
    int32_t *status;  // where an index out of range is recorded
    uint64_t n;       // Gaussians: records, gradients
    uint64_t pairs;   // capacity of the pair list
    uint32_t tiles;   // tiles of the frame
    const uint64_t *n_pairs;  // the frame's K, on the device
};
inline Bounds bounds_of(const gs_bins &b, int64_t n, int tiles) {
    return Bounds{b.status, (uint64_t)n, (uint64_t)b.max_pairs, (uint32_t)tiles, b.n_pairs};
}
#ifdef __CUDACC__
__device__ __forceinline__ bool in_bounds(uint64_t i, uint64_t bound, int32_t *status) {
    if (!kCheck || i < bound) return true;
    set_status(status, GS_ERR_BOUNDS);
    return false;
}
// A tile's [start, end) lies inside the pair list.
__device__ __forceinline__ bool range_in_bounds(uint2 r, const Bounds &bd) {
    if (!kCheck) return true;
    return in_bounds(r.x, (uint64_t)r.y + 1, bd.status) && in_bounds(r.y, bd.pairs + 1, bd.status);
}
#endif

// Adam over the five parameter groups (gs_train.cu).
constexpr int kAdamMaxSlots = 16;
struct AdamGroup {
    float *p, *m, *v;                    // parameters and moments, updated in place
    float *out;                          // nullable: the summed, scaled gradient
    const float *slot[kAdamMaxSlots];    // gradient slots, summed in order
    int64_t count;                       // values in the group
    float lr;
    int vec;                             // every array 16-byte aligned: float4 path
};
struct AdamGroups {
    AdamGroup g[5];  // means, log_scales, quats, opacity_logits, colors
};

// ------------------------------------------------------------- launchers
// Each returns cudaGetLastError() of its launches.
cudaError_t launch_project(const CamConst &c, int64_t n, const gs_params &p, const gs_projected &o,
                           cudaStream_t s);
// accumulate: add the raw-parameter gradients into g instead of writing them
cudaError_t launch_project_bwd(const CamConst &c, int64_t n, const gs_params &p,
                               const gs_projected &proj, float *grad2d, const gs_grads &g,
                               cudaStream_t s, bool accumulate = false);
cudaError_t launch_bin_and_sort(const CamConst &c, int64_t n, const gs_projected &proj,
                                const gs_bins &bins, const BinsLayout &L, cudaStream_t s);
// With target: the L1 loss in the epilogue (dL_dimage written, *loss zeroed
// then summed when not null, stats[0..1] = the bins' status and K when not
// null).
cudaError_t launch_render_fwd(const CamConst &c, int64_t n, const gs_projected &proj, const gs_bins &bins,
                              float *image, float *T_final, uint32_t *last, cudaStream_t s,
                              const float *target = nullptr, float *dL_dimage = nullptr, float *loss = nullptr,
                              int64_t *stats = nullptr);
cudaError_t launch_render_bwd(const CamConst &c, int64_t n, const gs_projected &proj, const gs_bins &bins,
                              const float *T_final, const uint32_t *last, const float *dL_dimage,
                              float *grad2d, cudaStream_t s);
// Feature channels: passes of the blend over chunks of eight channels, then
// one of four when F is not a multiple of 8 (no background).  The backward adds the geometric sums into grad2d and
// the feature gradients into dL_dfeatures (both zeroed by the caller).
cudaError_t launch_render_features_fwd(const CamConst &c, int64_t n, const gs_projected &proj, const gs_bins &bins,
                                       const float *features, int F, float *out, cudaStream_t s);
cudaError_t launch_render_features_bwd(const CamConst &c, int64_t n, const gs_projected &proj, const gs_bins &bins,
                                       const float *T_final, const uint32_t *last, const float *features,
                                       int F, const float *dL_dout, float *grad2d, float *dL_dfeatures,
                                       cudaStream_t s);
cudaError_t launch_render_stats(const CamConst &c, int64_t n, const gs_projected &proj, const gs_bins &bins,
                                const uint32_t *last, uint64_t *counts, cudaStream_t s);
cudaError_t launch_l1(const float *image, const float *target, int64_t count, float *dL_dimage,
                      float *loss, cudaStream_t s);
// update: k_adam_tick (advances *step), then k_adam when max_count > 0;
// otherwise only the scaled slot sum is written to each group's `out`
struct AdamBetas {
    double b1, b2;   // for the bias corrections
    float b1f, b2f;  // beta rounded once, for the moment updates
    float omb1, omb2;  // 1 - beta computed in double, rounded once
};
cudaError_t launch_adam(const AdamGroups &G, int64_t max_count, const AdamBetas &betas, float eps,
                        float grad_scale, int n_slots, int64_t *step, cudaStream_t s, bool update = true);

// Profiling hooks used around every launch (gs_api.cu).
void prof_before(const char *name, cudaStream_t s);
void prof_after(cudaStream_t s, int kernels = 1);  // kernels launched since prof_before

}  // namespace gs
