// gs_internal.cuh -- definitions shared by the CUDA translation units of
// libgs.so.  Not part of the public ABI (that is include/gs.h).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "gs.h"

namespace gs {

constexpr int kTile = GS_TILE;            // 16 x 16 pixel tiles
constexpr int kTilePixels = kTile * kTile;

// Radix sort: 8-bit digits, 256 threads x 16 keys per partition.
constexpr int kRadixBits = 8;
constexpr int kRadix = 1 << kRadixBits;
constexpr int kSortThreads = 256;
constexpr int kSortItems = 16;
constexpr int kSortPart = kSortThreads * kSortItems;  // 4096 keys
constexpr int kMaxDepthPasses = 4;                    // 31 depth bits
constexpr int kMaxTilePasses = 3;                     // up to 24 tile-id bits

// Scan + emit: 256 threads x 8 Gaussians per partition.
constexpr int kScanThreads = 256;
constexpr int kScanItems = 8;
constexpr int kScanPart = kScanThreads * kScanItems;  // 2048 Gaussians

// Pair emit: 256 threads per block, 2048 pairs per block.
constexpr int kEmitThreads = 256;
constexpr int kEmitPairs = 2048;

// Bounded device-side waits: a decoupled look-back poll gives up after this
// many polls, records GS_ERR_DEVICE_TIMEOUT and lets the kernel finish.
constexpr uint32_t kSpinLimit = 1u << 21;

// Look-back words: 2 flag bits + 30 value bits (partition aggregate or
// inclusive prefix).  N and max_pairs are kept below 2^30 so values fit.
constexpr uint32_t kFlagAggregate = 1u << 30;
constexpr uint32_t kFlagInclusive = 2u << 30;
constexpr uint32_t kValueMask = (1u << 30) - 1;
constexpr uint64_t kFlag64Aggregate = 1ull << 62;
constexpr uint64_t kFlag64Inclusive = 2ull << 62;
constexpr uint64_t kValue64Mask = (1ull << 62) - 1;

// Key given to Gaussians that draw nothing: sorts after every positive float.
constexpr uint32_t kInvalidDepthKey = 0x7FFFFFFFu;

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
};

// Byte layout of a gs_bins buffer.  The first `zero_bytes` bytes are cleared
// by one memset at the start of every gs_bin_and_sort.
struct BinsLayout {
    size_t status, n_pairs, tickets, depth_hist, tile_hist;
    size_t tile_count;                              // [max_tiles] pairs per tile, then emit cursors
    size_t ranges, depth_lb, scan_lb, tile_lb;
    size_t zero_bytes;
    size_t tile_order;                              // [max_tiles] tiles, longest list first
    size_t bin_hist;                                // per-CTA tile counts, then offsets
    size_t keys_a, vals_a, keys_b, vals_b;          // depth sort, [max_n]
    size_t ptile_a, pgid_a, ptile_b, pgid_b;        // pair sort ping-pong, [max_pairs]
    size_t pair_tile, pair_gid;                     // result, [max_pairs]
    size_t total;
    int64_t depth_parts, scan_parts, tile_parts;
};

constexpr size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

constexpr BinsLayout bins_layout(int64_t max_n, int64_t max_pairs, int32_t max_tiles) {
    BinsLayout L{};
    size_t off = 0;
    L.status = off;       off += 8;
    L.n_pairs = off;      off += 8;
    off = align_up(off, 64);
    L.tickets = off;      off += 16 * sizeof(uint32_t);
    off = align_up(off, 256);
    L.depth_hist = off;   off += kMaxDepthPasses * kRadix * sizeof(uint32_t);
    L.tile_hist = off;    off += kMaxTilePasses * kRadix * sizeof(uint32_t);
    off = align_up(off, 256);
    L.tile_count = off;   off = align_up(off + (size_t)max_tiles * sizeof(uint32_t), 256);
    L.ranges = off;       off = align_up(off + (size_t)max_tiles * 2 * sizeof(uint32_t), 256);
    L.depth_parts = (max_n + kSortPart - 1) / kSortPart;
    L.scan_parts = (max_n + kScanPart - 1) / kScanPart;
    L.tile_parts = (max_pairs + kSortPart - 1) / kSortPart;
    L.depth_lb = off;
    off = align_up(off + (size_t)kMaxDepthPasses * L.depth_parts * kRadix * sizeof(uint32_t), 256);
    L.scan_lb = off;
    off = align_up(off + (size_t)L.scan_parts * sizeof(uint64_t), 256);
    L.tile_lb = off;
    off = align_up(off + (size_t)kMaxTilePasses * L.tile_parts * kRadix * sizeof(uint32_t), 256);
    L.zero_bytes = off;
    L.tile_order = off;   off = align_up(off + (size_t)max_tiles * sizeof(uint32_t), 256);
    L.bin_hist = off;
    {
        const int64_t h = (int64_t)320 * max_tiles, cap = (int64_t)1 << 22;  // per-CTA tile counts
        off = align_up(off + (size_t)(h < cap ? h : cap) * sizeof(uint32_t), 256);
    }
    size_t nb = align_up((size_t)max_n * sizeof(uint32_t), 256);
    size_t pb = align_up((size_t)max_pairs * sizeof(uint32_t), 256);
    L.keys_a = off;  off += nb;
    L.vals_a = off;  off += nb;
    L.keys_b = off;  off += nb;
    L.vals_b = off;  off += nb;
    L.ptile_a = off; off += pb;
    L.pgid_a = off;  off += pb;
    L.ptile_b = off; off += pb;
    L.pgid_b = off;  off += pb;
    L.pair_tile = off; off += pb;
    L.pair_gid = off;  off += pb;
    L.total = off;
    return L;
}

// ---------------------------------------------------------------- device
#ifdef __CUDACC__
__device__ __forceinline__ uint32_t ld_relaxed(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_relaxed(uint32_t *p, uint32_t v) {
    asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint64_t ld_relaxed64(const uint64_t *p) {
    uint64_t v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_relaxed64(uint64_t *p, uint64_t v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
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

// ------------------------------------------------------------- launchers
// Each returns cudaGetLastError() of its launches.
cudaError_t launch_project(const CamConst &c, int64_t n, const gs_params &p, const gs_projected &o,
                           cudaStream_t s);
cudaError_t launch_project_bwd(const CamConst &c, int64_t n, const gs_params &p,
                               const gs_projected &proj, float *grad2d, const gs_grads &g,
                               cudaStream_t s);
cudaError_t launch_bin_and_sort(const CamConst &c, int64_t n, const gs_projected &proj,
                                const gs_bins &bins, const BinsLayout &L, cudaStream_t s);
cudaError_t launch_render_fwd(const CamConst &c, const gs_projected &proj, const gs_bins &bins,
                              float *image, float *T_final, uint32_t *last, cudaStream_t s);
cudaError_t launch_render_bwd(const CamConst &c, const gs_projected &proj, const gs_bins &bins,
                              const float *T_final, const uint32_t *last, const float *dL_dimage,
                              float *grad2d, cudaStream_t s);
cudaError_t launch_render_stats(const CamConst &c, const gs_projected &proj, const gs_bins &bins,
                                const uint32_t *last, uint64_t *counts, cudaStream_t s);
cudaError_t launch_l1(const float *image, const float *target, int64_t count, float *dL_dimage,
                      float *loss, cudaStream_t s);

// Profiling hooks used around every launch (gs_api.cu).
void prof_before(const char *name, cudaStream_t s);
void prof_after(cudaStream_t s);

}  // namespace gs
