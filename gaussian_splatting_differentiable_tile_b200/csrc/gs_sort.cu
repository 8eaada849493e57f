// gs_sort.cu -- tile binning: count, scan, emit, per-tile sort, ranges.
//
// Source: "SplatRs: The Week the Gap Closed", "Throughput: the tile
// rasterizer" (project, count, emit, sort, range, blend).
//
// The pages key each (tile, Gaussian) pair by (tile << 32 | depth bits) and
// radix-sort all pairs on that key.  The same order is reached here without
// a global sort: pairs are grouped by tile through counts and scans, and
// each tile's short list is sorted on its own by the 64-bit key
// (depth bits << 32 | Gaussian id), which is unique, so the order inside a
// tile is by depth with ties by id -- exactly the global key order.
//
//   k_bin_count    a fixed set of CTAs splits the Gaussians into contiguous
//                  ranges; each counts its pairs per tile in shared memory
//                  and writes its row of a [CTA][tile] count matrix
//   k_bin_colscan  offsets down each tile's column, and each tile's total
//   k_tile_scan    one CTA: ranges, K (capacity check), and the order in
//                  which the sorts and the blend take the tiles (longest
//                  list first)
//   k_bin_emit     each CTA writes the keys of its pairs at its offsets,
//                  advancing shared-memory cursors
//   k_tile_sort*   per tile: one warp sorts up to 256 keys in registers; a
//                  CTA sorts up to 1024 (and a wide CTA up to 8192) as warp
//                  runs merged in shared memory; longer lists are radix
//                  sorted in global memory by one CTA each
//
// No kernel waits on another CTA, and no global atomic is contended.
#include <mutex>

#include "gs_internal.cuh"

namespace gs {
namespace {

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Lanes of the warp holding the same digit as this lane, for digits of
// `bits` (<= 8) bits or the sentinel kRadix: one ballot per digit bit (and one
// for the sentinel), each lane keeping the lanes that agree with it.  Cheaper
// than a match instruction on this hardware.
__device__ __forceinline__ uint32_t digit_peers(uint32_t d, int bits) {
    const uint32_t valid = __ballot_sync(0xffffffffu, d < kRadix);
    uint32_t peers = d < kRadix ? valid : ~valid;
#pragma unroll
    for (int b = 0; b < kRadixBits; b++) {
        if (b < bits) {
            const bool set = (d >> b) & 1u;
            const uint32_t bal = __ballot_sync(0xffffffffu, set);
            peers &= set ? bal : ~bal;
        }
    }
    return peers;
}

// ---------------------------------------------------------------------
// Per-tile binning.  A fixed set of CTAs splits the Gaussians into
// contiguous ranges; each CTA counts its pairs per tile in shared memory and
// writes its row of a [CTA][tile] count matrix (no contended global
// atomics).  A column scan gives every (CTA, tile) its offset inside the
// tile, a one-CTA scan gives the tile ranges, K and the tile order; each CTA
// then emits its pairs at its offsets through shared-memory cursors (in
// arbitrary order within the tile), and each tile's list is sorted by the
// 64-bit key (depth bits << 32 | Gaussian id).  Keys are unique, so the
// result is exactly the pair order of the global sort on
// (tile << 32 | depth bits) with ties by id.

constexpr int kBinThreads = 512;

// Rectangles of at most this many tiles are handled by their own lane; larger
// ones by the whole warp, one at a time.
constexpr uint32_t kLaneTiles = 16;
// Tile grids up to this size count in shared memory; larger ones in their
// CTA's row of the global matrix.
constexpr int kSmemTiles = 16384;
// Size classes of the per-tile sort (256 keys per warp): up to
// kTileSortShort keys (4 warps), up to kTileSortMid (32 warps, two 64 KB
// shared-memory buffers), and longer lists in global memory.
constexpr int kShortWarps = 4, kMidWarps = 32;
constexpr uint32_t kTileSortShort = 256u * kShortWarps;
constexpr uint32_t kTileSortMid = 256u * kMidWarps;

// Calls f(k, tile) for the tiles k = first, first + kStep, ... < c of a
// rectangle (row-major from column x0, row y0, w tiles wide), keeping the
// column and row by additions: kStep 1 (first 0) needs no division, kStep 32
// one per call.
template <uint32_t kStep, typename F>
__device__ __forceinline__ void rect_walk(uint32_t first, uint32_t c, int x0, int y0, uint32_t w, int tiles_x,
                                          F f) {
    uint32_t dy, dx, sq, sr;  // position, and the step in rows and columns
    if (kStep == 1) {
        dy = 0;
        dx = 0;
        sq = w == 1 ? 1u : 0u;
        sr = w == 1 ? 0u : 1u;
    } else {
        if (first >= c) return;
        dy = first / w;
        dx = first - dy * w;
        sq = kStep / w;
        sr = kStep - sq * w;
    }
    for (uint32_t k = first; k < c; k += kStep) {
        f(k, (y0 + (int)dy) * tiles_x + x0 + (int)dx);
        dx += sr;
        dy += sq;
        if (dx >= w) {
            dx -= w;
            dy++;
        }
    }
}

// Calls f(g, tile) for every pair of the Gaussians [g_begin, g_end), the
// CTA's warps striding through the range 32 Gaussians at a time, four
// groups per round (their rectangles loaded together).
template <typename F>
__device__ __forceinline__ void for_each_pair(int g_begin, int g_end, const int4 *__restrict__ rect,
                                              int tiles_x, int tiles_y, F f) {
    constexpr int kGroups = 4;
    const int lane = threadIdx.x & 31;
    for (int g0 = g_begin + (int)(threadIdx.x & ~31u); g0 < g_end; g0 += kGroups * (int)blockDim.x) {
        int4 rc[kGroups];
#pragma unroll
        for (int u = 0; u < kGroups; u++) {
            const int g = g0 + u * (int)blockDim.x + lane;
            rc[u] = g < g_end ? rect[g] : make_int4(0, 0, -1, -1);
        }
#pragma unroll
        for (int u = 0; u < kGroups; u++) {
            const int g = g0 + u * (int)blockDim.x + lane;
            int x0 = 0, y0 = 0, w = 1;
            const uint32_t c = rect_tiles(rc[u], tiles_x, tiles_y, x0, y0, w);
            if (c <= kLaneTiles) rect_walk<1>(0u, c, x0, y0, (uint32_t)w, tiles_x, [&](uint32_t, int t) { f(g, t); });
            uint32_t big = __ballot_sync(0xffffffffu, c > kLaneTiles);
            while (big) {
                const int src = __ffs(big) - 1;
                big &= big - 1;
                const int gb = __shfl_sync(0xffffffffu, g, src);
                const uint32_t cb = __shfl_sync(0xffffffffu, c, src);
                const int xb = __shfl_sync(0xffffffffu, x0, src), yb = __shfl_sync(0xffffffffu, y0, src);
                const uint32_t wb = (uint32_t)__shfl_sync(0xffffffffu, w, src);
                rect_walk<32>((uint32_t)lane, cb, xb, yb, wb, tiles_x, [&](uint32_t, int t) { f(gb, t); });
            }
        }
    }
}

__device__ __forceinline__ void cta_range(int n, int &g_begin, int &g_end) {
    const int chunk = (n + (int)gridDim.x - 1) / (int)gridDim.x;
    g_begin = min((int)blockIdx.x * chunk, n);
    g_end = min(g_begin + chunk, n);
}

// Row blockIdx of the count matrix H[CTA][tile].
__global__ void __launch_bounds__(kBinThreads, 2)
k_bin_count(int n, const int4 *__restrict__ rect, int tiles_x, int tiles_y, uint32_t *__restrict__ H,
            int32_t *__restrict__ status) {
    extern __shared__ uint32_t s_cnt[];
    const int tiles = tiles_x * tiles_y;
    uint32_t *row = H + (size_t)blockIdx.x * tiles;
    const bool smem = tiles <= kSmemTiles;
    uint32_t *cnt = smem ? s_cnt : row;
    for (int t = threadIdx.x; t < tiles; t += kBinThreads) cnt[t] = 0;
    __syncthreads();
    int g_begin, g_end;
    cta_range(n, g_begin, g_end);
    for_each_pair(g_begin, g_end, rect, tiles_x, tiles_y, [&](int, int t) {
        if (in_bounds((uint32_t)t, (uint32_t)tiles, status)) atomicAdd(&cnt[t], 1u);
    });
    __syncthreads();
    if (smem)
        for (int t = threadIdx.x; t < tiles; t += kBinThreads) row[t] = s_cnt[t];
}

// Per tile: exclusive scan down its column of H (in place) and the total.
// A CTA takes 32 tiles (lane = tile, so every row access is coalesced) and
// splits the rows among its 8 warps; each warp loads its rows at once.
constexpr int kColRows = (kBinCTAsMax + 7) / 8;
__global__ void __launch_bounds__(256)
k_bin_colscan(int tiles, int ctas, uint32_t *__restrict__ H, uint32_t *__restrict__ totals) {
    __shared__ uint32_t s_part[8][32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int t = blockIdx.x * 32 + lane;
    const int per = (ctas + 7) / 8;
    const int c0 = warp * per;
    uint32_t v[kColRows];
#pragma unroll
    for (int k = 0; k < kColRows; k++) {
        const int c = c0 + k;
        v[k] = (k < per && c < ctas && t < tiles) ? H[(size_t)c * tiles + t] : 0u;
    }
    uint32_t sum = 0;
#pragma unroll
    for (int k = 0; k < kColRows; k++) {
        const uint32_t x = v[k];
        v[k] = sum;
        sum += x;
    }
    s_part[warp][lane] = sum;
    __syncthreads();
    uint32_t base = 0, total = 0;
#pragma unroll
    for (int w = 0; w < 8; w++) {
        const uint32_t x = s_part[w][lane];
        base += w < warp ? x : 0u;
        total += x;
    }
#pragma unroll
    for (int k = 0; k < kColRows; k++) {
        const int c = c0 + k;
        if (k < per && c < ctas && t < tiles) H[(size_t)c * tiles + t] = base + v[k];
    }
    if (warp == 0 && t < tiles) totals[t] = total;
}

// One CTA: ranges from the exclusive scan of the tile totals (all empty if K
// exceeds the capacity, with GS_ERR_CAPACITY recorded), K, and the tile
// order (longest list first, by a counting sort on length in steps of 4,
// lists of 4 092 entries and more sharing the first bucket; finer or coarser
// steps measured the same).
constexpr int kScanTilesThreads = 1024;
__device__ __forceinline__ uint32_t order_bucket(uint32_t len) {
    return min(len >> 2, (uint32_t)(kScanTilesThreads - 1));
}
__global__ void __launch_bounds__(kScanTilesThreads)
k_tile_scan(int tiles, const uint32_t *__restrict__ totals, uint64_t max_pairs,
            uint32_t *__restrict__ ranges, uint32_t *__restrict__ order, uint64_t *__restrict__ n_pairs,
            int32_t *__restrict__ status) {
    __shared__ uint64_t s_w64[kScanTilesThreads / 32];
    __shared__ uint32_t s_off[kScanTilesThreads];
    __shared__ uint32_t s_w32[kScanTilesThreads / 32];
    __shared__ int s_ok;
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    const int chunk = (tiles + kScanTilesThreads - 1) / kScanTilesThreads;
    const int lo = min(t * chunk, tiles), hi = min(lo + chunk, tiles);
    uint64_t sum = 0;
    for (int i = lo; i < hi; i++) sum += totals[i];
    uint64_t x = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint64_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_w64[w] = x;
    __syncthreads();
    if (w == 0) {
        uint64_t z = s_w64[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint64_t y = __shfl_up_sync(0xffffffffu, z, o);
            if (lane >= o) z += y;
        }
        s_w64[lane] = z;
        if (lane == 31) {
            // an error recorded earlier (the global strategy's capacity check)
            // came with its K, which stays
            if (*(volatile int32_t *)status == 0) *n_pairs = z;
            const bool ok = z <= max_pairs;
            if (!ok) set_status(status, GS_ERR_CAPACITY);
            s_ok = ok && *(volatile int32_t *)status == 0;
        }
    }
    __syncthreads();
    uint64_t off = x - sum + (w > 0 ? s_w64[w - 1] : 0ull);
    const bool ok = s_ok;
    for (int i = lo; i < hi; i++) {
        const uint32_t c = totals[i];
        const bool some = ok && c > 0;  // empty tiles are [0, 0)
        ranges[2 * (size_t)i] = some ? (uint32_t)off : 0u;
        ranges[2 * (size_t)i + 1] = some ? (uint32_t)(off + c) : 0u;
        off += c;
    }
    auto bucket = [&](int i) {
        const uint32_t len = ok ? totals[i] : 0u;
        return kScanTilesThreads - 1 - (int)order_bucket(len);
    };
    s_off[t] = 0;
    __syncthreads();
    for (int i = lo; i < hi; i++) atomicAdd(&s_off[bucket(i)], 1u);
    __syncthreads();
    const uint32_t v = s_off[t];
    uint32_t y = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t z = __shfl_up_sync(0xffffffffu, y, o);
        if (lane >= o) y += z;
    }
    if (lane == 31) s_w32[w] = y;
    __syncthreads();
    if (w == 0) {
        uint32_t z = s_w32[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t q = __shfl_up_sync(0xffffffffu, z, o);
            if (lane >= o) z += q;
        }
        s_w32[lane] = z;
    }
    __syncthreads();
    s_off[t] = y - v + (w > 0 ? s_w32[w - 1] : 0u);
    __syncthreads();
    for (int i = lo; i < hi; i++) order[atomicAdd(&s_off[bucket(i)], 1u)] = (uint32_t)i;
}

__device__ __forceinline__ uint64_t pair_key(const float4 *__restrict__ xyod, uint32_t g) {
    return ((uint64_t)__float_as_uint(xyod[g].w) << 32) | g;
}

// Each CTA emits the pairs of its Gaussians as sort keys (depth bits << 32 |
// id): cursor = tile start + the CTA's column offset, advanced by
// shared-memory atomics.  Nothing is written once an error has been
// recorded.
__global__ void __launch_bounds__(kBinThreads, 2)
k_bin_emit(int n, const int4 *__restrict__ rect, const float4 *__restrict__ xyod, int tiles_x, int tiles_y,
           const uint32_t *__restrict__ ranges, uint32_t *__restrict__ H, uint64_t *__restrict__ keys,
           int32_t *__restrict__ status, uint64_t max_pairs) {
    extern __shared__ uint32_t s_cur[];
    if (*(volatile const int32_t *)status != 0) return;
    const int tiles = tiles_x * tiles_y;
    uint32_t *row = H + (size_t)blockIdx.x * tiles;
    const bool smem = tiles <= kSmemTiles;
    uint32_t *cur = smem ? s_cur : row;
    for (int t = threadIdx.x; t < tiles; t += kBinThreads) cur[t] = ranges[2 * (size_t)t] + row[t];
    __syncthreads();
    int g_begin, g_end;
    cta_range(n, g_begin, g_end);
    for_each_pair(g_begin, g_end, rect, tiles_x, tiles_y, [&](int g, int t) {
        if (!in_bounds((uint32_t)t, (uint32_t)tiles, status)) return;
        const uint32_t pos = atomicAdd(&cur[t], 1u);
        if (in_bounds(pos, max_pairs, status)) keys[pos] = pair_key(xyod, (uint32_t)g);
    });
}


// Sorts the keys of a warp ascending in registers: lane l holds elements
// 8l .. 8l + 7 in k[0..7].  Bitonic network: strides below 8 swap within the
// lane, larger strides exchange with lane ^ (stride / 8).  Stopping after
// blocks of P (a power of two) sorts the first P keys, which is all that is
// needed when the others are padding.
__device__ __forceinline__ void warp_bitonic_256(uint64_t (&k)[8], int lane, int P = 256) {
    const int l8 = lane << 3;  // element index of k[0]; k[r] is element l8 | r
#pragma unroll
    for (int kk = 2; kk <= 256; kk <<= 1) {
        if (kk > P) continue;  // the first P keys are sorted (the rest are padding)
#pragma unroll
        for (int j = kk >> 1; j > 0; j >>= 1) {
            if (j >= 8) {
                // partner in lane ^ (j / 8); directions depend on the lane only
                const bool keep_min = ((l8 & j) == 0) == ((l8 & kk) == 0);
#pragma unroll
                for (int r = 0; r < 8; r++) {
                    const uint64_t o = __shfl_xor_sync(0xffffffffu, k[r], j >> 3);
                    k[r] = ((k[r] > o) == keep_min) ? o : k[r];
                }
            } else {
#pragma unroll
                for (int r = 0; r < 8; r++) {
                    if (r & j) continue;
                    // ascending block unless bit kk of the element index is set
                    const bool asc = kk >= 8 ? (l8 & kk) == 0 : (r & kk) == 0;
                    const uint64_t x = k[r], y = k[r | j];
                    const bool sw = (x > y) == asc;
                    k[r] = sw ? y : x;
                    k[r | j] = sw ? x : y;
                }
            }
        }
    }
}

// Number of keys in the sorted run a[0, n) below x (strictly, or at most x).
template <bool kInclusive>
__device__ __forceinline__ int run_rank(const uint64_t *a, int n, uint64_t x) {
    int lo = 0, hi = n;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        const bool left = kInclusive ? a[mid] <= x : a[mid] < x;
        if (left) lo = mid + 1;
        else hi = mid;
    }
    return lo;
}

// A tile list of 1 to 256 entries sorted by one warp in registers.
__device__ __forceinline__ void warp_sort_tile(uint32_t tile, uint32_t start, uint32_t L,
                                               const uint64_t *__restrict__ keys, uint32_t *__restrict__ pair_gid,
                                               uint32_t *__restrict__ pair_tile, int lane) {
    uint64_t k[8];
#pragma unroll
    for (int r = 0; r < 8; r++) {
        const uint32_t idx = (uint32_t)(lane * 8 + r);
        k[r] = idx < L ? keys[start + idx] : ~0ull;
    }
    int P = 2;
    while ((uint32_t)P < L) P <<= 1;
    warp_bitonic_256(k, lane, P);
#pragma unroll
    for (int r = 0; r < 8; r++) {
        const uint32_t idx = (uint32_t)(lane * 8 + r);
        if (idx < L) {
            pair_gid[start + idx] = (uint32_t)k[r];
            pair_tile[start + idx] = tile;
        }
    }
}

// A tile list too long for the shared-memory sort: LSD radix sort of its
// keys in global memory by the whole CTA (8-bit digits: four passes over the
// id, then four over the depth bits; each pass stable, in chunks of kThreads
// ranked with warp ballots), ping-ponging between (ka, va) and (kb, vb) at
// the same offsets as the tile's range.  Writes the result to pair_gid and
// pair_tile.  s_wc holds kThreads / 32 rows of 256 counters.
template <int kThreads>
__device__ void global_radix_sort_tile(uint32_t start, uint32_t end, uint32_t tile,
                                       const uint64_t *__restrict__ keys, uint32_t *ka, uint32_t *va,
                                       uint32_t *kb, uint32_t *vb, uint32_t *__restrict__ pair_gid,
                                       uint32_t *__restrict__ pair_tile, uint32_t *s_base, uint32_t *s_tot,
                                       uint32_t (*s_wc)[kRadix]) {
    constexpr int kWarps = kThreads / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (uint32_t i = start + tid; i < end; i += kThreads) {
        const uint64_t key = keys[i];
        ka[i] = (uint32_t)(key >> 32);
        va[i] = (uint32_t)key;
    }
    __syncthreads();
    uint32_t *sk = ka, *sv = va, *dk = kb, *dv = vb;
    for (int pass = 0; pass < 8; pass++) {
        const bool on_id = pass < 4;
        const int shift = 8 * (pass & 3);
        for (int d = tid; d < kRadix; d += kThreads) s_base[d] = 0;
        __syncthreads();
        for (uint32_t i = start + tid; i < end; i += kThreads)
            atomicAdd(&s_base[((on_id ? sv[i] : sk[i]) >> shift) & 0xFFu], 1u);
        __syncthreads();
        if (tid == 0) {  // exclusive scan, in place
            uint32_t acc = start;
            for (int d = 0; d < kRadix; d++) {
                const uint32_t c = s_base[d];
                s_base[d] = acc;
                acc += c;
            }
        }
        __syncthreads();
        for (uint32_t c0 = start; c0 < end; c0 += kThreads) {
            const uint32_t i = c0 + tid;
            const bool in = i < end;
            const uint32_t key = in ? sk[i] : 0u, val = in ? sv[i] : 0u;
            const uint32_t d = in ? ((on_id ? val : key) >> shift) & 0xFFu : (uint32_t)kRadix;
            for (int k = tid; k < kWarps * kRadix; k += kThreads) (&s_wc[0][0])[k] = 0;
            __syncthreads();
            const uint32_t peers = digit_peers(d, 8);
            if (in && lane == __ffs(peers) - 1) s_wc[warp][d] = __popc(peers);
            __syncthreads();
            for (int dd = tid; dd < kRadix; dd += kThreads) {  // exclusive over warps
                uint32_t acc = 0;
                for (int ww = 0; ww < kWarps; ww++) {
                    const uint32_t c = s_wc[ww][dd];
                    s_wc[ww][dd] = acc;
                    acc += c;
                }
                s_tot[dd] = acc;
            }
            __syncthreads();
            if (in) {
                const uint32_t pos = s_base[d] + s_wc[warp][d] + __popc(peers & lanemask_lt());
                dk[pos] = key;
                dv[pos] = val;
            }
            __syncthreads();
            for (int dd = tid; dd < kRadix; dd += kThreads) s_base[dd] += s_tot[dd];
            __syncthreads();
        }
        uint32_t *t0 = sk, *t1 = sv;
        sk = dk; sv = dv; dk = t0; dv = t1;
        __syncthreads();
    }
    for (uint32_t i = start + tid; i < end; i += kThreads) {
        pair_gid[i] = sv[i];
        pair_tile[i] = tile;
    }
    __syncthreads();
}

// Tile lists in (lo, hi], hi = 256 kWarps: sorted by one CTA each.  Warp w
// sorts keys [256 w, 256 w + 256) in registers; the runs are then merged
// pairwise in shared memory (each key's output position is its index plus
// its rank in the other run).  Without kLong the CTA's first warp also
// sorts lists of 1 to 256 entries alone (whatever lo is), so the short and
// the mid-sized lists of a frame are sorted by one launch.  With kLong the
// CTA also takes lists above hi, by a radix sort in global memory.  With `persistent` a small grid walks the tile
// order (longest first) and stops at the first tile whose length bucket
// lies below lo's; otherwise CTA b takes the b-th tile of the order.
template <int kWarps, bool kLong>
__global__ void __launch_bounds__(kWarps * 32)
k_tile_sort(const uint32_t *__restrict__ ranges, const uint32_t *__restrict__ order, int tiles,
            const uint64_t *__restrict__ keys, uint32_t *__restrict__ pair_gid,
            uint32_t *__restrict__ pair_tile, uint32_t lo, int persistent, uint32_t *ka, uint32_t *va,
            const Bounds bd) {
    constexpr int kThreads = kWarps * 32;
    constexpr uint32_t kHi = 256u * kWarps;
    extern __shared__ uint64_t s_buf[];
    __shared__ uint32_t s_base[kLong ? kRadix : 1], s_tot[kLong ? kRadix : 1];
    __shared__ uint32_t s_wc[kLong ? kWarps : 1][kRadix];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int step = persistent ? (int)gridDim.x : tiles;
    for (int b = blockIdx.x; b < tiles; b += step) {
        const uint32_t tile = order[b];
        if (!in_bounds(tile, (uint32_t)tiles, bd.status)) break;  // uniform over the CTA
        const uint32_t start = ranges[2 * (size_t)tile], end = ranges[2 * (size_t)tile + 1];
        if (!range_in_bounds(make_uint2(start, end), bd)) break;
        const uint32_t L = end - start;
        if (persistent && order_bucket(L) < order_bucket(lo)) break;
        if (!kLong && L <= 256u) {  // a short list: one warp, in registers
            if (warp == 0 && L > 0) warp_sort_tile(tile, start, L, keys, pair_gid, pair_tile, lane);
            continue;
        }
        if (L <= lo) continue;
        if (L > kHi) {
            // longer than shared memory holds: sorted in global memory, with
            // (pair_tile, pair_gid) as the second ping-pong buffer
            if (kLong)
                global_radix_sort_tile<kThreads>(start, end, tile, keys, ka, va, pair_tile, pair_gid, pair_gid,
                                                 pair_tile, s_base, s_tot, s_wc);
            continue;
        }
        const int chunks = (int)((L + 255) / 256);
        int runs = 1;
        while (runs < chunks) runs <<= 1;
        if (warp < runs) {
            uint64_t k[8];
#pragma unroll
            for (int r = 0; r < 8; r++) {
                const uint32_t idx = (uint32_t)(warp * 256 + lane * 8 + r);
                k[r] = idx < L ? keys[start + idx] : ~0ull;
            }
            if (warp < chunks) {
                const uint32_t m = min(L - (uint32_t)warp * 256u, 256u);  // real keys of the chunk
                int P = 2;
                while ((uint32_t)P < m) P <<= 1;
                warp_bitonic_256(k, lane, P);
            }
#pragma unroll
            for (int r = 0; r < 8; r++) s_buf[warp * 256 + lane * 8 + r] = k[r];
        }
        __syncthreads();
        uint64_t *src = s_buf, *dst = s_buf + kHi;
        const int total = runs * 256;
        for (int run = 256; run < total; run <<= 1) {
            for (int i = threadIdx.x; i < total; i += kThreads) {
                const int base = i & ~(2 * run - 1), off = i - base;
                const uint64_t x = src[i];
                const int pos = off < run ? off + run_rank<false>(src + base + run, run, x)
                                          : (off - run) + run_rank<true>(src + base, run, x);
                dst[base + pos] = x;
            }
            __syncthreads();
            uint64_t *t = src;
            src = dst;
            dst = t;
        }
        for (uint32_t i = threadIdx.x; i < L; i += kThreads) {
            pair_gid[start + i] = (uint32_t)src[i];
            pair_tile[start + i] = tile;
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------
// Global binning, for frames whose tile lists are long (a thousand entries
// and more: 400k Gaussians at 1960 x 1090 give more than 2^24 pairs, about
// 2 500 per tile), where sorting each tile's list on its own costs
// L log L per tile.  The same unique order is reached with linear passes:
//   k_depth_init + LSD passes   the Gaussians ordered by the float bits of
//                               their depth (stable, so ties stay in id
//                               order); Gaussians without tiles last
//   k_rank_sums, k_rank_offsets the first pair position of each Gaussian in
//                               that order: an exclusive scan of its tile count
//   k_emit_ranked               every Gaussian writes (tile, id) for the tiles
//                               of its rectangle at its position, so the pair
//                               list comes out in (depth, id) order and is
//                               written contiguously
//   LSD passes on the tile id   stable, the id's bits split evenly into digits
//                               of at most 8 bits: the pairs grouped by
//                               tile, the (depth, id) order kept inside every
//                               tile; the last pass writes pair_tile and
//                               pair_gid
//   k_tile_bounds, k_tile_totals, k_tile_scan
//                               each tile's [start, end) read off the sorted
//                               list; the tile scan of the per-tile path then
//                               builds the tile order (longest list first)
// An LSD pass takes its elements in tiles of 4 096, one CTA per tile: a
// histogram kernel (each tile's digit counts, digit-major), an exclusive scan
// of those counts (two kernels), and a scatter kernel (each CTA ranks its
// tile's elements in input order, sorts the tile by digit in shared memory
// and writes every digit's run contiguously at its scanned offset).  The
// count matrix of the per-tile strategy is not built: K comes out of the
// depth-ordered scan of the tile counts, which also takes the capacity check
// (GS_ERR_CAPACITY, with K) before anything is emitted.  No kernel waits on
// another CTA.

// Ranking of an LSD pass's digits within a warp: one match instruction (1),
// or one ballot per digit bit (0).  A tuning knob.
#ifndef GS_LSD_MATCH
#define GS_LSD_MATCH 0
#endif
// Resident scatter CTAs per SM the register allocation targets (a tuning
// knob).
#ifndef GS_LSD_MINB
#define GS_LSD_MINB 2
#endif
// Rows of the digit-count matrix a warp of a locally scanned pass reads per
// round (a tuning knob).
#ifndef GS_LSD_ROWS
#define GS_LSD_ROWS 4
#endif
constexpr int kLsdThreads = 512;
constexpr int kLsdWarps = kLsdThreads / 32;

// The elements [lo, hi) of this CTA when `count` elements are split among
// the grid's CTAs in contiguous chunks.
__device__ __forceinline__ void lsd_chunk(uint64_t count, uint32_t &lo, uint32_t &hi) {
    const uint64_t chunk = (count + gridDim.x - 1) / gridDim.x;
    lo = (uint32_t)min((uint64_t)blockIdx.x * chunk, count);
    hi = (uint32_t)min((uint64_t)lo + chunk, count);
}

// The Gaussians' sort keys: the float bits of the depth (positive, so their
// order is the depth order) for Gaussians that touch a tile, all ones for
// the others; values: the ids.
__global__ void __launch_bounds__(256)
k_depth_init(int n, const int4 *__restrict__ rect, const float4 *__restrict__ xyod, int tiles_x, int tiles_y,
             uint32_t *__restrict__ keys, uint32_t *__restrict__ vals, const int32_t *__restrict__ status) {
    if (*(volatile const int32_t *)status != 0) return;
    const int g = blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= n) return;
    int x0, y0, w;
    const uint32_t c = rect_tiles(rect[g], tiles_x, tiles_y, x0, y0, w);
    keys[g] = c ? __float_as_uint(xyod[g].w) : 0xFFFFFFFFu;
    vals[g] = (uint32_t)g;
}

// Exclusive scan of 256 values in shared memory by the first 256 threads
// (all threads of the block meet the barriers).
__device__ __forceinline__ void scan256(uint32_t *v, uint32_t *s_w) {
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    uint32_t x = 0, y = 0;
    if (t < kRadix) {
        x = v[t];
        y = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t z = __shfl_up_sync(0xffffffffu, y, o);
            if (lane >= o) y += z;
        }
        if (lane == 31) s_w[w] = y;
    }
    __syncthreads();
    if (t < kRadix) {
        uint32_t base = 0;
        for (int k = 0; k < w; k++) base += s_w[k];
        v[t] = base + y - x;
    }
    __syncthreads();
}

// An LSD pass takes its elements in tiles of kScatterTile; CTA b of every
// kernel of the pass owns tile b.  H[d][b] (digit-major, T tiles per row)
// counts digit d in tile b; its exclusive scan in that order is the output
// position of tile b's first element of digit d.
constexpr int kScatterThreads = 512;
constexpr int kScatterWarps = kScatterThreads / 32;
constexpr int kScatterItems = 8;
constexpr int kScatterTile = kScatterThreads * kScatterItems;  // 4096
// dynamic shared memory of k_lsd_scatter: the tile's keys and values, and
// the per-warp digit counters
constexpr size_t kScatterSmem = (2 * (size_t)kScatterTile + (size_t)kScatterWarps * kRadix) * sizeof(uint32_t);
constexpr int kHistThreads = 256, kHistItems = kScatterTile / kHistThreads;
constexpr int kHistWarps = kHistThreads / 32;

// Digit counts of this CTA's tile into column blockIdx.x of H.  The element
// count is *count_dev when given (K), else count_host; tiles past it count
// nothing (their column is zero).  A thread's keys are loaded together, then
// counted.
__global__ void __launch_bounds__(kHistThreads)
k_lsd_hist(const uint32_t *__restrict__ keys, const uint64_t *__restrict__ count_dev, uint32_t count_host,
           int shift, int bits, uint32_t *__restrict__ H, const int32_t *__restrict__ status) {
    __shared__ uint32_t s_h[kHistWarps][kRadix];
    if (*(volatile const int32_t *)status != 0) return;
    const int warp = threadIdx.x >> 5;
    const uint32_t mask = (1u << bits) - 1u, ndig = 1u << bits;
    for (int i = threadIdx.x; i < kHistWarps * kRadix; i += kHistThreads) (&s_h[0][0])[i] = 0;
    const uint64_t count = count_dev ? *count_dev : count_host;
    const uint64_t t0 = (uint64_t)blockIdx.x * kScatterTile;
    const uint32_t m = t0 < count ? (uint32_t)min((uint64_t)kScatterTile, count - t0) : 0u;
    uint32_t kk[kHistItems];
#pragma unroll
    for (int k = 0; k < kHistItems; k++) {
        const uint32_t i = (uint32_t)(k * kHistThreads) + threadIdx.x;
        kk[k] = i < m ? keys[t0 + i] : 0u;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kHistItems; k++)
        if ((uint32_t)(k * kHistThreads) + threadIdx.x < m) atomicAdd(&s_h[warp][(kk[k] >> shift) & mask], 1u);
    __syncthreads();
    for (uint32_t d = threadIdx.x; d < ndig; d += kHistThreads) {
        uint32_t t = 0;
#pragma unroll
        for (int w = 0; w < kHistWarps; w++) t += s_h[w][d];
        H[(size_t)d * gridDim.x + blockIdx.x] = t;
    }
}

// Exclusive scan of H[0, m) in place, in blocks of kScanBlock: each CTA scans
// its block and writes the block's total to S (k_scan_blocks); each CTA then
// adds the totals of the blocks before it (k_scan_add).
constexpr int kScanThreads = 1024, kScanItems = 4, kScanBlock = kScanThreads * kScanItems;

__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t *s_w, uint32_t *total) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    uint32_t y = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t z = __shfl_up_sync(0xffffffffu, y, o);
        if (lane >= o) y += z;
    }
    if (lane == 31) s_w[w] = y;
    __syncthreads();
    if (w == 0) {
        const uint32_t x = lane < (int)(blockDim.x >> 5) ? s_w[lane] : 0u;
        uint32_t z = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t q = __shfl_up_sync(0xffffffffu, z, o);
            if (lane >= o) z += q;
        }
        s_w[lane] = z - x;  // exclusive warp bases
        if (lane == 31) s_w[32] = z;
    }
    __syncthreads();
    const uint32_t r = s_w[w] + y - v;
    *total = s_w[32];
    __syncthreads();
    return r;
}

__global__ void __launch_bounds__(kScanThreads)
k_scan_blocks(uint32_t *__restrict__ H, uint32_t m, uint32_t *__restrict__ S, const int32_t *__restrict__ status) {
    __shared__ uint32_t s_w[33];
    if (*(volatile const int32_t *)status != 0) return;
    const uint32_t b0 = blockIdx.x * kScanBlock + threadIdx.x * kScanItems;
    uint32_t v[kScanItems], sum = 0;
#pragma unroll
    for (int k = 0; k < kScanItems; k++) {
        v[k] = b0 + k < m ? H[b0 + k] : 0u;
        sum += v[k];
    }
    uint32_t total;
    uint32_t off = block_exclusive_scan(sum, s_w, &total);
#pragma unroll
    for (int k = 0; k < kScanItems; k++) {
        if (b0 + k < m) H[b0 + k] = off;
        off += v[k];
    }
    if (threadIdx.x == 0) S[blockIdx.x] = total;
}

__global__ void __launch_bounds__(kScanThreads)
k_scan_add(uint32_t *__restrict__ H, uint32_t m, const uint32_t *__restrict__ S, const int32_t *__restrict__ status) {
    __shared__ uint32_t s_w[33];
    if (*(volatile const int32_t *)status != 0) return;
    uint32_t pre = 0;
    for (uint32_t b = threadIdx.x; b < blockIdx.x; b += kScanThreads) pre += S[b];
    uint32_t total;
    block_exclusive_scan(pre, s_w, &total);  // only the block total is used
    const uint32_t b0 = blockIdx.x * kScanBlock + threadIdx.x * kScanItems;
#pragma unroll
    for (int k = 0; k < kScanItems; k++)
        if (b0 + k < m) H[b0 + k] += total;
}

// Stable scatter of one LSD pass, CTA b taking tile b: warp w holds elements
// w * 256 + 32 k + lane (k = 0 .. 7), so (w, k, lane) is the input order.
// Each warp ranks its elements within their digit in that order (one ballot
// per digit bit per 32 elements, per-warp counters in shared memory); a scan
// over the warps and over the digits places each element in the tile sorted
// by digit, in shared memory; the tile then goes out digit run by digit run,
// each run contiguous at the scanned H[d][b], so the writes are coalesced.
// With kLocal, H holds the tiles' digit counts unscanned (passes of at most
// kLocalScanTiles tiles): each CTA sums its digit's counts over the tiles
// before it and over all tiles, and scans the digit totals itself, in place
// of the two scan kernels.
constexpr int kLocalScanTiles = 256;
template <bool kLocal>
__global__ void __launch_bounds__(kScatterThreads, GS_LSD_MINB)
k_lsd_scatter(const uint32_t *__restrict__ keys_in, const uint32_t *__restrict__ vals_in,
              const uint64_t *__restrict__ count_dev, uint32_t count_host, int shift, int bits,
              const uint32_t *__restrict__ H, uint32_t *__restrict__ keys_out, uint32_t *__restrict__ vals_out,
              int32_t *__restrict__ status) {
    __shared__ uint32_t s_gbase[kRadix], s_start[kRadix], s_w[kScatterWarps];
    extern __shared__ uint32_t s_dyn[];
    uint32_t *s_key = s_dyn, *s_val = s_dyn + kScatterTile;
    uint32_t(*s_cnt)[kRadix] = reinterpret_cast<uint32_t(*)[kRadix]>(s_dyn + 2 * kScatterTile);
    if (*(volatile const int32_t *)status != 0) return;
    const uint64_t count = count_dev ? *count_dev : count_host;
    const uint64_t t0 = (uint64_t)blockIdx.x * kScatterTile;
    if (t0 >= count) return;  // uniform over the CTA
    const uint32_t m = (uint32_t)min((uint64_t)kScatterTile, count - t0);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t mask = (1u << bits) - 1u, ndig = 1u << bits, lt = lanemask_lt();
    uint32_t key[kScatterItems], val[kScatterItems], rank[kScatterItems];
#pragma unroll
    for (int k = 0; k < kScatterItems; k++) {
        const uint32_t i = (uint32_t)(warp * 32 * kScatterItems + 32 * k + lane);
        key[k] = i < m ? keys_in[t0 + i] : 0u;
        val[k] = i < m ? vals_in[t0 + i] : 0u;
    }
    for (int i = tid; i < kScatterWarps * kRadix; i += kScatterThreads) (&s_cnt[0][0])[i] = 0;
    if (kLocal) {
        // Each digit's count before this tile, and its total (in s_start for
        // now).  Warp w takes its digits GS_LSD_ROWS at a time; its lanes
        // read those rows' counts (tiles lane, lane + 32, ...) with every
        // load issued before the first is used, then sum over the warp.
        constexpr int kRowLoads = kLocalScanTiles / 32, kRowsAtOnce = GS_LSD_ROWS;
        static_assert(kRadix % (kScatterWarps * kRowsAtOnce) == 0, "every digit's row read once");
        const uint32_t T = gridDim.x;
        for (uint32_t d0 = (uint32_t)warp * kRowsAtOnce; d0 < kRadix; d0 += kScatterWarps * kRowsAtOnce) {
            uint32_t c[kRowsAtOnce][kRowLoads];
#pragma unroll
            for (int r = 0; r < kRowsAtOnce; r++)
#pragma unroll
                for (int j = 0; j < kRowLoads; j++) {
                    const uint32_t b = (uint32_t)(32 * j + lane);
                    c[r][j] = d0 + r < ndig && b < T ? H[(size_t)(d0 + r) * T + b] : 0u;
                }
#pragma unroll
            for (int r = 0; r < kRowsAtOnce; r++) {
                uint32_t before = 0, total = 0;
#pragma unroll
                for (int j = 0; j < kRowLoads; j++) {
                    total += c[r][j];
                    before += (uint32_t)(32 * j + lane) < blockIdx.x ? c[r][j] : 0u;
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    total += __shfl_xor_sync(0xffffffffu, total, o);
                    before += __shfl_xor_sync(0xffffffffu, before, o);
                }
                if (lane == 0) {
                    s_gbase[d0 + r] = before;
                    s_start[d0 + r] = total;
                }
            }
        }
        __syncthreads();
        scan256(s_start, s_w);  // each digit's first position in the output
        if (tid < kRadix) s_gbase[tid] += s_start[tid];
    } else if ((uint32_t)tid < ndig) {
        s_gbase[tid] = H[(size_t)tid * gridDim.x + blockIdx.x];
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kScatterItems; k++) {
        const uint32_t i = (uint32_t)(warp * 32 * kScatterItems + 32 * k + lane);
        const uint32_t d = i < m ? (key[k] >> shift) & mask : (uint32_t)kRadix;
#if GS_LSD_MATCH
        const uint32_t peers = __match_any_sync(0xffffffffu, d);
#else
        const uint32_t peers = digit_peers(d, bits);
#endif
        rank[k] = d < kRadix ? s_cnt[warp][d] + __popc(peers & lt) : 0u;
        __syncwarp();
        if (d < kRadix && lane == __ffs(peers) - 1) s_cnt[warp][d] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();
    if (tid < kRadix) {  // exclusive over the warps, per digit; digit totals of the tile
        uint32_t tot = 0;
#pragma unroll
        for (int w = 0; w < kScatterWarps; w++) {
            const uint32_t c = s_cnt[w][tid];
            s_cnt[w][tid] = tot;
            tot += c;
        }
        s_start[tid] = tot;
    }
    __syncthreads();
    scan256(s_start, s_w);  // digit starts within the tile
#pragma unroll
    for (int k = 0; k < kScatterItems; k++) {
        const uint32_t i = (uint32_t)(warp * 32 * kScatterItems + 32 * k + lane);
        if (i < m) {
            const uint32_t d = (key[k] >> shift) & mask;
            const uint32_t pos = s_start[d] + s_cnt[warp][d] + rank[k];
            s_key[pos] = key[k];
            s_val[pos] = val[k];
        }
    }
    __syncthreads();
    for (uint32_t i = tid; i < m; i += kScatterThreads) {
        const uint32_t kk = s_key[i], d = (kk >> shift) & mask;
        const uint32_t pos = s_gbase[d] + (i - s_start[d]);
        if (!in_bounds(pos, count, status)) continue;
        keys_out[pos] = kk;
        vals_out[pos] = s_val[i];
    }
}

// Per-CTA sums of the tile counts of the Gaussians in depth order (rank r:
// Gaussian order[r]), over contiguous chunks of ranks.
__device__ __forceinline__ uint32_t ranked_count(const int4 *__restrict__ rect, const uint32_t *__restrict__ order,
                                                 uint32_t r, int tiles_x, int tiles_y) {
    int x0, y0, w;
    return rect_tiles(rect[order[r]], tiles_x, tiles_y, x0, y0, w);
}

__device__ __forceinline__ uint64_t block_sum_512_u64(uint64_t v, uint64_t *s_w) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) s_w[w] = v;
    __syncthreads();
    uint64_t t = 0;
#pragma unroll
    for (int k = 0; k < kLsdWarps; k++) t += s_w[k];
    __syncthreads();
    return t;
}

__global__ void __launch_bounds__(kLsdThreads)
k_rank_sums(int n, const int4 *__restrict__ rect, const uint32_t *__restrict__ order, int tiles_x, int tiles_y,
            uint64_t *__restrict__ S, const int32_t *__restrict__ status) {
    __shared__ uint64_t s_w[kLsdWarps];
    if (*(volatile const int32_t *)status != 0) return;
    uint32_t lo, hi;
    lsd_chunk((uint64_t)n, lo, hi);
    uint64_t sum = 0;
    for (uint32_t r = lo + threadIdx.x; r < hi; r += kLsdThreads) sum += ranked_count(rect, order, r, tiles_x, tiles_y);
    sum = block_sum_512_u64(sum, s_w);
    if (threadIdx.x == 0) S[blockIdx.x] = sum;
}

// offsets[r] = pairs of the Gaussians ranked before r (exclusive scan).  The
// last CTA also records K and the capacity check (GS_ERR_CAPACITY: the
// kernels after it then write nothing).
__global__ void __launch_bounds__(kLsdThreads)
k_rank_offsets(int n, const int4 *__restrict__ rect, const uint32_t *__restrict__ order, int tiles_x, int tiles_y,
               const uint64_t *__restrict__ S, uint32_t *__restrict__ offsets, uint64_t *__restrict__ n_pairs,
               uint64_t max_pairs, int32_t *__restrict__ status) {
    __shared__ uint32_t s_w[kLsdWarps];
    __shared__ uint64_t s_w64[kLsdWarps];
    if (*(volatile const int32_t *)status != 0) return;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint64_t before = 0;
    for (int c = tid; c < (int)blockIdx.x; c += kLsdThreads) before += S[c];
    before = block_sum_512_u64(before, s_w64);
    if (blockIdx.x == gridDim.x - 1 && tid == 0) {
        const uint64_t K = before + S[blockIdx.x];
        *n_pairs = K;
        if (K > max_pairs) set_status(status, GS_ERR_CAPACITY);
    }
    if (before + S[blockIdx.x] > max_pairs) return;  // the capacity error: offsets are not needed
    uint32_t base = (uint32_t)before;
    uint32_t lo, hi;
    lsd_chunk((uint64_t)n, lo, hi);
    for (uint32_t c0 = lo; c0 < hi; c0 += kLsdThreads) {
        const uint32_t r = c0 + tid;
        const uint32_t v = r < hi ? ranked_count(rect, order, r, tiles_x, tiles_y) : 0u;
        uint32_t y = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t z = __shfl_up_sync(0xffffffffu, y, o);
            if (lane >= o) y += z;
        }
        if (lane == 31) s_w[warp] = y;
        __syncthreads();
        uint32_t wbase = 0, total = 0;
#pragma unroll
        for (int k = 0; k < kLsdWarps; k++) {
            const uint32_t x = s_w[k];
            wbase += k < warp ? x : 0u;
            total += x;
        }
        if (r < hi) offsets[r] = base + wbase + y - v;
        base += total;
        __syncthreads();
    }
}

// Each tile's [start, end) in the sorted pair list (ranges zeroed by the
// caller, so empty tiles stay [0, 0)), then each tile's total.  Thread j
// compares the four tile ids 4 j .. 4 j + 3 (one 16-byte load) and the next
// one: a change between positions p - 1 and p ends one tile's range and
// starts the next's at p.
__device__ __forceinline__ void tile_boundary(uint32_t a, uint32_t b, uint32_t p, uint32_t *__restrict__ ranges,
                                              uint32_t tiles, int32_t *__restrict__ status) {
    if (a == b) return;
    if (in_bounds(a, tiles, status)) ranges[2 * (size_t)a + 1] = p;
    if (in_bounds(b, tiles, status)) ranges[2 * (size_t)b] = p;
}

__global__ void __launch_bounds__(256)
k_tile_bounds(const uint32_t *__restrict__ pair_tile, const uint64_t *__restrict__ n_pairs,
              uint32_t *__restrict__ ranges, int32_t *__restrict__ status, uint32_t tiles) {
    if (*(volatile const int32_t *)status != 0) return;
    const uint32_t K = (uint32_t)*n_pairs;  // at most max_pairs < 2^30 here
    if (K == 0) return;
    const uint32_t groups = (K + 3) / 4;
    for (uint32_t j = blockIdx.x * blockDim.x + threadIdx.x; j < groups; j += gridDim.x * blockDim.x) {
        const uint32_t i0 = 4 * j;
        uint32_t t[5];
        if (i0 + 4 <= K) {
            const uint4 v = reinterpret_cast<const uint4 *>(pair_tile)[j];
            t[0] = v.x; t[1] = v.y; t[2] = v.z; t[3] = v.w;
        } else {
#pragma unroll
            for (int k = 0; k < 4; k++) t[k] = i0 + k < K ? pair_tile[i0 + k] : 0u;
        }
        t[4] = i0 + 4 < K ? pair_tile[i0 + 4] : 0u;
        if (j == 0 && in_bounds(t[0], tiles, status)) ranges[2 * (size_t)t[0]] = 0;
#pragma unroll
        for (int k = 0; k < 4; k++) {
            const uint32_t p = i0 + k + 1;  // boundary between positions p - 1 and p
            if (p > K) break;
            if (p == K) {
                if (in_bounds(t[k], tiles, status)) ranges[2 * (size_t)t[k] + 1] = K;
            } else {
                tile_boundary(t[k], t[k + 1], p, ranges, tiles, status);
            }
        }
    }
}

__global__ void __launch_bounds__(256)
k_tile_totals(const uint32_t *__restrict__ ranges, int tiles, uint32_t *__restrict__ totals) {
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t < tiles) totals[t] = ranges[2 * (size_t)t + 1] - ranges[2 * (size_t)t];
}

// Each Gaussian (rank r, id order[r]) writes the tile id and its id for
// every tile of its rectangle, row by row, at offsets[r]: rectangles of at
// most 16 tiles by their own lane, larger ones by the whole warp.
__global__ void __launch_bounds__(256)
k_emit_ranked(int n, const int4 *__restrict__ rect, const uint32_t *__restrict__ order,
              const uint32_t *__restrict__ offsets, int tiles_x, int tiles_y, uint32_t *__restrict__ tile_out,
              uint32_t *__restrict__ gid_out, int32_t *__restrict__ status, uint64_t max_pairs) {
    if (*(volatile const int32_t *)status != 0) return;
    const int lane = threadIdx.x & 31;
    const int stride = gridDim.x * blockDim.x;
    for (int r0 = blockIdx.x * blockDim.x + (threadIdx.x & ~31); r0 < n; r0 += stride) {
        const int r = r0 + lane;
        uint32_t g = 0, c = 0, off = 0;
        int x0 = 0, y0 = 0, w = 1;
        if (r < n) {
            g = order[r];
            c = rect_tiles(rect[g], tiles_x, tiles_y, x0, y0, w);
            if (c) off = offsets[r];
        }
        if (c <= kLaneTiles)
            rect_walk<1>(0u, c, x0, y0, (uint32_t)w, tiles_x, [&](uint32_t k, int t) {
                if (!in_bounds((uint64_t)off + k, max_pairs, status)) return;
                tile_out[off + k] = (uint32_t)t;
                gid_out[off + k] = g;
            });
        uint32_t big = __ballot_sync(0xffffffffu, c > kLaneTiles);
        while (big) {
            const int src = __ffs(big) - 1;
            big &= big - 1;
            const uint32_t gb = __shfl_sync(0xffffffffu, g, src), cb = __shfl_sync(0xffffffffu, c, src);
            const uint32_t ob = __shfl_sync(0xffffffffu, off, src);
            const int xb = __shfl_sync(0xffffffffu, x0, src), yb = __shfl_sync(0xffffffffu, y0, src);
            const uint32_t wb = (uint32_t)__shfl_sync(0xffffffffu, w, src);
            rect_walk<32>((uint32_t)lane, cb, xb, yb, wb, tiles_x, [&](uint32_t k, int t) {
                if (!in_bounds((uint64_t)ob + k, max_pairs, status)) return;
                tile_out[ob + k] = (uint32_t)t;
                gid_out[ob + k] = gb;
            });
        }
    }
}

// Per-device launch set-up of the binning kernels, done once per device with
// that device current: its SM count, and the dynamic shared memory the count,
// emit and wide sort kernels may use beyond the default 48 KB (a function
// attribute is a property of the device it was set on).
constexpr int kMaxDevices = 128;
struct DeviceSetup {
    int sms = 0;
    cudaError_t err = cudaSuccess;
};
DeviceSetup g_setup[kMaxDevices];
std::mutex g_setup_mutex;

// Every instantiation of k_lsd_scatter takes kScatterSmem of dynamic shared
// memory.
cudaError_t scatter_smem_attributes() {
    const void *kernels[] = {(const void *)k_lsd_scatter<true>, (const void *)k_lsd_scatter<false>};
    for (const void *k : kernels) {
        const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kScatterSmem);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t device_setup(int *sms) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    DeviceSetup &d = g_setup[dev];
    if (d.sms == 0) {
        int n = 0;
        if ((e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        const int cnt_bytes = (int)(kSmemTiles * sizeof(uint32_t));
        if ((e = cudaFuncSetAttribute(k_bin_count, cudaFuncAttributeMaxDynamicSharedMemorySize, cnt_bytes)) !=
                cudaSuccess ||
            (e = cudaFuncSetAttribute(k_bin_emit, cudaFuncAttributeMaxDynamicSharedMemorySize, cnt_bytes)) !=
                cudaSuccess ||
            (e = cudaFuncSetAttribute(k_tile_sort<kMidWarps, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)(2 * kTileSortMid * sizeof(uint64_t)))) != cudaSuccess ||
            (e = scatter_smem_attributes()) != cudaSuccess)
            return e;
        d.sms = n > 0 ? n : 148;
    }
    *sms = d.sms;
    return cudaSuccess;
}

}  // namespace

// The global path after the tile scan (see the kernels above).  ctas: CTAs
// of the LSD, rank and emit kernels.
// Entries of the count-matrix space one LSD pass over at most `cap`
// elements uses: the digit counts of its tiles and the scan's block totals.
int64_t lsd_space(int64_t cap) {
    const int64_t m = (int64_t)kRadix * ((cap + kScatterTile - 1) / kScatterTile);
    return m + (m + kScanBlock - 1) / kScanBlock;
}

// One stable LSD pass over the digit (key >> shift) & (2^bits - 1) of at
// most `cap` elements (*count_dev of them when given, else count_host):
// per-tile digit counts, their exclusive scan, the scatter.
// Returns the kernels it launched.
int lsd_pass(const uint32_t *ki, const uint32_t *vi, uint32_t *ko, uint32_t *vo, const uint64_t *count_dev,
             uint32_t count_host, int64_t cap, int shift, int bits, uint32_t *H, int32_t *status, cudaStream_t s) {
    const int tiles = (int)std::max<int64_t>(1, (cap + kScatterTile - 1) / kScatterTile);
    const uint32_t m = (uint32_t)((1u << bits) * (uint32_t)tiles);
    const int blocks = (int)((m + kScanBlock - 1) / kScanBlock);
    uint32_t *S = H + m;
    k_lsd_hist<<<tiles, kHistThreads, 0, s>>>(ki, count_dev, count_host, shift, bits, H, status);
    const bool local = tiles <= kLocalScanTiles;
    if (!local) {
        k_scan_blocks<<<blocks, kScanThreads, 0, s>>>(H, m, S, status);
        k_scan_add<<<blocks, kScanThreads, 0, s>>>(H, m, S, status);
    }
    (local ? k_lsd_scatter<true> : k_lsd_scatter<false>)<<<tiles, kScatterThreads, kScatterSmem, s>>>(
        ki, vi, count_dev, count_host, shift, bits, H, ko, vo, status);
    return local ? 2 : 4;
}

// The global path after the tile scan (see the kernels above).  ctas: CTAs
// of the rank and emit kernels.
cudaError_t launch_bin_global(const CamConst &c, int64_t n, const gs_projected &proj, const gs_bins &bins,
                              const BinsLayout &L, int ctas, int sms, cudaStream_t s) {
    char *base = static_cast<char *>(bins.scratch);
    auto U32 = [&](size_t off) { return reinterpret_cast<uint32_t *>(base + off); };
    int32_t *status = reinterpret_cast<int32_t *>(base + L.status);
    uint64_t *n_pairs = reinterpret_cast<uint64_t *>(base + L.n_pairs);
    uint32_t *H = U32(L.bin_hist);
    uint32_t *ranges = U32(L.ranges), *totals = U32(L.tile_total), *order = U32(L.tile_order);
    const int tiles_c = c.tiles_x * c.tiles_y;
    // no count phase on this path: ranges and totals start empty
    cudaError_t e = cudaMemsetAsync(totals, 0, (size_t)tiles_c * sizeof(uint32_t), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(ranges, 0, (size_t)tiles_c * 2 * sizeof(uint32_t), s);
    if (e != cudaSuccess) return e;
    if (n == 0) {  // K = 0: every range empty, every tile in the order
        k_tile_scan<<<1, kScanTilesThreads, 0, s>>>(tiles_c, totals, (uint64_t)bins.max_pairs, ranges, order,
                                                    n_pairs, status);
        return cudaGetLastError();
    }
    const size_t pb = align_up((size_t)bins.max_pairs * sizeof(uint32_t), 256);
    uint32_t *KA = U32(L.keys), *VA = U32(L.keys + pb);  // the key array's two halves
    uint32_t *KB = U32(L.long_keys), *VB = U32(L.long_ids);
    const int4 *rect = reinterpret_cast<const int4 *>(proj.rect);
    const float4 *xyod = reinterpret_cast<const float4 *>(proj.xy_opacity_depth);
    const int tiles = tiles_c;
    const uint32_t nn = (uint32_t)n;
    // 4. the Gaussians by depth: four stable 8-bit passes, A -> B -> A -> B -> A
    prof_before("depth_sort", s);
    k_depth_init<<<(unsigned)((n + 255) / 256), 256, 0, s>>>((int)n, rect, xyod, c.tiles_x, c.tiles_y, KA, VA,
                                                               status);
    int launched = 1;
    for (int p = 0; p < 4; p++) {
        uint32_t *ki = p & 1 ? KB : KA, *vi = p & 1 ? VB : VA, *ko = p & 1 ? KA : KB, *vo = p & 1 ? VA : VB;
        launched += lsd_pass(ki, vi, ko, vo, nullptr, nn, n, 8 * p, 8, H, status, s);
    }
    prof_after(s, launched);
    // 5. each Gaussian's first pair position in depth order (into KA), then
    // the pairs in (depth, id) order into (KB, VB)
    prof_before("emit", s);
    uint64_t *S = reinterpret_cast<uint64_t *>(H);
    k_rank_sums<<<ctas, kLsdThreads, 0, s>>>((int)n, rect, VA, c.tiles_x, c.tiles_y, S, status);
    k_rank_offsets<<<ctas, kLsdThreads, 0, s>>>((int)n, rect, VA, c.tiles_x, c.tiles_y, S, KA, n_pairs,
                                                (uint64_t)bins.max_pairs, status);
    const int emit_blocks = (int)std::min<int64_t>((n + 255) / 256, (int64_t)8 * sms);
    k_emit_ranked<<<emit_blocks, 256, 0, s>>>((int)n, rect, VA, KA, c.tiles_x, c.tiles_y, KB, VB, status,
                                              (uint64_t)bins.max_pairs);
    prof_after(s, 3);
    // 6. stable passes over the tile id, its bits split evenly into digits of
    // at most 8 bits: B -> A -> B ..., the last into pair_tile / pair_gid
    int tile_bits = 1;
    while (tile_bits < 31 && ((uint32_t)(tiles - 1) >> tile_bits)) tile_bits++;
    const int passes = (tile_bits + 7) / 8, digit = (tile_bits + passes - 1) / passes;
    prof_before("tile_sort", s);
    launched = 0;
    for (int p = 0; p < passes; p++) {
        const bool last = p == passes - 1;
        const int bits = std::min(digit, tile_bits - digit * p);
        uint32_t *ki = p & 1 ? KA : KB, *vi = p & 1 ? VA : VB;
        uint32_t *ko = last ? bins.pair_tile : (p & 1 ? KB : KA), *vo = last ? bins.pair_gid : (p & 1 ? VB : VA);
        launched += lsd_pass(ki, vi, ko, vo, n_pairs, 0u, bins.max_pairs, digit * p, bits, H, status, s);
    }
    prof_after(s, launched);
    // 7. each tile's range off the sorted list, its total, then the tile
    // scan as on the per-tile path (ranges again, K kept, the tile order)
    prof_before("tile_scan", s);
    const int bound_blocks = (int)std::min<int64_t>((bins.max_pairs / 4 + 255) / 256, (int64_t)32 * sms);
    k_tile_bounds<<<std::max(1, bound_blocks), 256, 0, s>>>(bins.pair_tile, n_pairs, ranges, status, (uint32_t)tiles);
    k_tile_totals<<<(tiles + 255) / 256, 256, 0, s>>>(ranges, tiles, totals);
    k_tile_scan<<<1, kScanTilesThreads, 0, s>>>(tiles, totals, (uint64_t)bins.max_pairs, ranges, order, n_pairs,
                                                status);
    prof_after(s, 3);
    return cudaGetLastError();
}

cudaError_t launch_bin_and_sort(const CamConst &c, int64_t n, const gs_projected &proj,
                                const gs_bins &bins, const BinsLayout &L, cudaStream_t s) {
    char *base = static_cast<char *>(bins.scratch);
    auto U32 = [&](size_t off) { return reinterpret_cast<uint32_t *>(base + off); };
    int32_t *status = reinterpret_cast<int32_t *>(base + L.status);
    uint64_t *n_pairs = reinterpret_cast<uint64_t *>(base + L.n_pairs);
    uint32_t *ranges = U32(L.ranges);
    uint32_t *totals = U32(L.tile_total);
    uint32_t *order = U32(L.tile_order);
    uint32_t *H = U32(L.bin_hist);
    uint64_t *keys = reinterpret_cast<uint64_t *>(base + L.keys);
    const int4 *rect = reinterpret_cast<const int4 *>(proj.rect);
    const int tiles = c.tiles_x * c.tiles_y;
    int sms = 0;
    cudaError_t e = device_setup(&sms);
    if (e != cudaSuccess) return e;
    // CTAs sharing the Gaussians: two per SM, within the count matrix's size
    int64_t ctas64 = std::min<int64_t>((int64_t)2 * sms, (int64_t)kBinCTAsMax);
    ctas64 = std::min<int64_t>(ctas64, kBinHistCap / tiles);
    const int ctas = (int)std::max<int64_t>(1, ctas64);
    const size_t cnt_smem = tiles <= kSmemTiles ? (size_t)tiles * sizeof(uint32_t) : 0;
    e = cudaMemsetAsync(base, 0, L.zero_bytes, s);
    if (e != cudaSuccess) return e;
    // the strategy (gs.h GS_BIN_*); the global path's LSD passes keep their
    // per-tile digit counts in the count matrix's space
    const int64_t hist_cap = std::min<int64_t>((int64_t)kBinCTAsMax * bins.max_tiles, kBinHistCap);
    // the rank kernels keep one u64 sum per CTA in the same space
    const int lsd_ctas = (int)std::max<int64_t>(1, std::min<int64_t>((int64_t)2 * sms, hist_cap / 2));
    bool global = bins.strategy == GS_BIN_GLOBAL;
    if (bins.strategy == GS_BIN_AUTO)
        global = bins.max_pairs >= (int64_t)1024 * tiles;
    global = global && n <= bins.max_pairs && lsd_space(bins.max_pairs) <= hist_cap;
    if (global) return launch_bin_global(c, n, proj, bins, L, lsd_ctas, sms, s);
    // 1. per-CTA tile counts, 2. offsets down each tile's column
    prof_before("bin_count", s);
    k_bin_count<<<ctas, kBinThreads, cnt_smem, s>>>((int)n, rect, c.tiles_x, c.tiles_y, H, status);
    k_bin_colscan<<<(tiles + 31) / 32, 256, 0, s>>>(tiles, ctas, H, totals);
    prof_after(s, 2);
    // 3. ranges, K, capacity check, tile order
    prof_before("tile_scan", s);
    k_tile_scan<<<1, kScanTilesThreads, 0, s>>>(tiles, totals, (uint64_t)bins.max_pairs, ranges, order,
                                                n_pairs, status);
    prof_after(s);
    if (n == 0) return cudaGetLastError();  // K = 0, all ranges empty
    // 4. emit the sort keys
    prof_before("emit", s);
    k_bin_emit<<<ctas, kBinThreads, cnt_smem, s>>>((int)n, rect, reinterpret_cast<const float4 *>(proj.xy_opacity_depth),
                                                   c.tiles_x, c.tiles_y, ranges, H, keys, status,
                                                   (uint64_t)bins.max_pairs);
    prof_after(s);
    // 5. sort each tile's list, by size class
    prof_before("tile_sort", s);
    const Bounds bd = bounds_of(bins, n, tiles);
    k_tile_sort<kShortWarps, false><<<tiles, kShortWarps * 32, 2 * kTileSortShort * sizeof(uint64_t), s>>>(
        ranges, order, tiles, keys, bins.pair_gid, bins.pair_tile, 256u, 0, nullptr, nullptr, bd);
    k_tile_sort<kMidWarps, true><<<std::min(tiles, sms), kMidWarps * 32, 2 * kTileSortMid * sizeof(uint64_t), s>>>(
        ranges, order, tiles, keys, bins.pair_gid, bins.pair_tile, kTileSortShort, 1, U32(L.long_keys),
        U32(L.long_ids), bd);
    prof_after(s, 2);
    return cudaGetLastError();
}

}  // namespace gs
