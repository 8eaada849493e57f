// gs_sort.cu -- tile binning: depth sort, count scan, pair emit, pair sort,
// per-tile ranges.
//
// Source: "SplatRs: The Week the Gap Closed", "Throughput: the tile
// rasterizer" (project, count, emit, sort, range, blend) and "Gaussian
// splatting in PyTorch" s5 (one global depth sort replaces per-tile sorts).
//
// The pages key each (tile, Gaussian) pair by (tile << 32 | depth bits) and
// radix-sort the pairs on that key.  Here the depth half of the key is sorted
// once per Gaussian instead of once per pair: Gaussians are first sorted by
// depth (31 used bits of the positive float), their pairs are emitted in that
// order, and a stable sort on the tile bits alone finishes the job.  The pair
// order is identical (ties in depth by Gaussian id), while each pair passes
// through ceil(tile_bits / 8) sort passes of 8 bytes instead of
// ceil(43..45 / 8) passes of 12 bytes.
//
// Both sorts are LSD radix sorts built from one "onesweep" pass kernel:
// a block ranks its 4096 keys with warp ballots and popc, publishes its digit
// counts, and resolves its global offsets by a decoupled look-back over the
// preceding partitions (bounded: a poll loop that runs out sets
// GS_ERR_DEVICE_TIMEOUT and the kernel still finishes).  Partitions are taken
// in ticket order so every block waits only on blocks already running.
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

// Exclusive block-wide scan of one value per thread (blockDim = 256).
__device__ __forceinline__ uint32_t block_exclusive_scan_256(uint32_t v, uint32_t *s_warp,
                                                             uint32_t *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    uint32_t wpre = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < 8; w++) {
        uint32_t t = s_warp[w];
        if (w < warp) wpre += t;
        tot += t;
    }
    __syncthreads();
    *total = tot;
    return wpre + x - v;
}

// Decoupled look-back for one digit: the sum of the digit's counts over
// partitions [0, q0], read from the partitions' published words back to the
// nearest inclusive one.  32 words are requested at a time, so a chain of
// aggregates costs one L2 round trip per 32 partitions.  A word that stays
// unpublished for kSpinLimit polls records GS_ERR_DEVICE_TIMEOUT and counts
// as zero, so the kernel always finishes.
__device__ __forceinline__ uint32_t lookback_digit(const uint32_t *lookback, int d, int64_t q0,
                                                   int32_t *status) {
    constexpr int kWindow = 32;
    uint32_t excl = 0;
    uint32_t spins = 0;
    for (int64_t q = q0; q >= 0; q -= kWindow) {
        uint32_t w[kWindow];
#pragma unroll
        for (int k = 0; k < kWindow; k++)
            w[k] = (q - k >= 0) ? ld_relaxed(lookback + (size_t)(q - k) * kRadix + d) : kFlagInclusive;
#pragma unroll
        for (int k = 0; k < kWindow; k++) {
            while ((w[k] & ~kValueMask) == 0u) {
                if (++spins > kSpinLimit) {
                    set_status(status, GS_ERR_DEVICE_TIMEOUT);
                    return excl;
                }
                w[k] = ld_relaxed(lookback + (size_t)(q - k) * kRadix + d);
            }
            excl += w[k] & kValueMask;
            if ((w[k] & ~kValueMask) == kFlagInclusive) return excl;
        }
    }
    return excl;
}

// Decoupled look-back over 64-bit partition words, by one full warp: lane l
// reads partition q0 - l, so each L2 round trip covers 32 partitions.
// Returns the inclusive prefix of partitions [0, q0] (to every lane).
__device__ __forceinline__ uint64_t lookback_warp64(const uint64_t *lookback, int64_t q0,
                                                    int32_t *status) {
    const int lane = threadIdx.x & 31;
    uint64_t prefix = 0;
    uint32_t spins = 0;
    for (int64_t base = q0; base >= 0; base -= 32) {
        const int64_t q = base - lane;
        uint64_t w = q >= 0 ? ld_relaxed64(lookback + q) : kFlag64Inclusive;
        bool timed_out = false;
        while (__any_sync(0xffffffffu, (w & ~kValue64Mask) == 0ull)) {
            if (++spins > kSpinLimit) {
                timed_out = true;
                break;
            }
            if ((w & ~kValue64Mask) == 0ull) w = ld_relaxed64(lookback + q);
        }
        if (timed_out) {
            if (lane == 0) set_status(status, GS_ERR_DEVICE_TIMEOUT);
            if ((w & ~kValue64Mask) == 0ull) w = kFlag64Inclusive;
        }
        const uint32_t incl = __ballot_sync(0xffffffffu, (w & ~kValue64Mask) == kFlag64Inclusive);
        const int first = incl ? __ffs(incl) - 1 : 31;
        uint64_t v = lane <= first ? (w & kValue64Mask) : 0ull;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        prefix += v;
        if (incl) break;
    }
    return prefix;
}

// Depth keys of the drawable Gaussians and the four digit histograms of the
// depth sort.
__global__ void __launch_bounds__(256)
k_depth_keys(int n, const float4 *__restrict__ xyod, const int4 *__restrict__ rect, int tiles_x,
             int tiles_y, uint32_t *__restrict__ keys, uint32_t *__restrict__ hist) {
    __shared__ uint32_t s_h[kMaxDepthPasses * kRadix];
    for (int i = threadIdx.x; i < kMaxDepthPasses * kRadix; i += blockDim.x) s_h[i] = 0;
    __syncthreads();
    for (int g = blockIdx.x * blockDim.x + threadIdx.x; g < n; g += gridDim.x * blockDim.x) {
        int x0, y0, w;
        const uint32_t c = rect_tiles(rect[g], tiles_x, tiles_y, x0, y0, w);
        const uint32_t key = c > 0 ? __float_as_uint(xyod[g].w) : kInvalidDepthKey;
        keys[g] = key;
#pragma unroll
        for (int k = 0; k < kMaxDepthPasses; k++) atomicAdd(&s_h[k * kRadix + ((key >> (8 * k)) & 0xFF)], 1u);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < kMaxDepthPasses * kRadix; i += blockDim.x)
        if (s_h[i]) atomicAdd(&hist[i], s_h[i]);
}

// One LSD radix pass over bits [shift, shift + bits) of 32-bit keys with
// 32-bit values.  n = min(*n_dev, n_cap) when n_dev is given, else n_host.
// With iota_vals the values are the input indices (first pass of a sort).
// When check_status is set the pass does nothing if *status is non-zero.
__global__ void __launch_bounds__(kSortThreads)
k_onesweep(const uint32_t *__restrict__ keys_in, const uint32_t *__restrict__ vals_in,
           uint32_t *__restrict__ keys_out, uint32_t *__restrict__ vals_out,
           const uint64_t *__restrict__ n_dev, uint32_t n_host, uint32_t n_cap, int shift, int bits,
           const uint32_t *__restrict__ hist, uint32_t *__restrict__ lookback,
           uint32_t *__restrict__ ticket, int32_t *__restrict__ status, int iota_vals,
           int check_status) {
    __shared__ uint32_t s_warp_hist[kSortThreads / 32][kRadix];
    __shared__ uint32_t s_digit_start[kRadix];
    __shared__ uint32_t s_global_base[kRadix];
    __shared__ uint32_t s_hist_excl[kRadix];
    __shared__ uint32_t s_keys[kSortPart];
    __shared__ uint32_t s_vals[kSortPart];
    __shared__ uint32_t s_scan[8];
    __shared__ uint32_t s_part;
    __shared__ int s_skip;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) s_skip = check_status ? (*(volatile int32_t *)status != 0) : 0;
    __syncthreads();
    if (s_skip) return;
    uint32_t n = n_host;
    if (n_dev) {
        const uint64_t nd = *n_dev;
        n = nd < (uint64_t)n_cap ? (uint32_t)nd : n_cap;
    }
    const uint32_t mask = (1u << bits) - 1u;
    const int radix = 1 << bits;

    // Exclusive scan of the global digit histogram: where each digit starts.
    {
        uint32_t tot;
        const uint32_t h = tid < radix ? hist[tid] : 0u;
        s_hist_excl[tid] = block_exclusive_scan_256(h, s_scan, &tot);
    }

    for (;;) {
        if (tid == 0) s_part = atomicAdd(ticket, 1u);
        __syncthreads();
        const uint32_t p = s_part;
        if ((uint64_t)p * kSortPart >= n) break;
        for (int i = tid; i < (kSortThreads / 32) * kRadix; i += kSortThreads)
            (&s_warp_hist[0][0])[i] = 0;
        __syncthreads();

        // Load: warp w owns keys [w*32*ITEMS, (w+1)*32*ITEMS) of the partition,
        // item i of lane l at offset i*32 + l: coalesced, and index order is
        // (warp, item, lane), which the ranking below preserves (stable).
        const uint32_t base = p * kSortPart + warp * (32 * kSortItems);
        uint32_t key[kSortItems], val[kSortItems], dig[kSortItems], rank[kSortItems];
        if (base + 32 * kSortItems <= n) {
            // a full slice: every load is issued before any is used (a
            // per-item guard and value select keep them from overlapping)
#pragma unroll
            for (int i = 0; i < kSortItems; i++) key[i] = __ldcg(keys_in + base + i * 32 + lane);
            if (iota_vals) {
#pragma unroll
                for (int i = 0; i < kSortItems; i++) val[i] = base + i * 32 + lane;
            } else {
#pragma unroll
                for (int i = 0; i < kSortItems; i++) val[i] = __ldcg(vals_in + base + i * 32 + lane);
            }
#pragma unroll
            for (int i = 0; i < kSortItems; i++) dig[i] = (key[i] >> shift) & mask;
        } else {
#pragma unroll
            for (int i = 0; i < kSortItems; i++) {
                const uint32_t idx = base + i * 32 + lane;
                if (idx < n) {
                    key[i] = keys_in[idx];
                    val[i] = iota_vals ? idx : vals_in[idx];
                    dig[i] = (key[i] >> shift) & mask;
                } else {
                    key[i] = 0; val[i] = 0;
                    dig[i] = kRadix;  // sentinel: not counted
                }
            }
        }
        // Warp-level ranking of each item among equal digits: the peer masks
        // first (independent ballots), then the per-digit counters in order.
        uint32_t peer[kSortItems];
#pragma unroll
        for (int i = 0; i < kSortItems; i++) peer[i] = digit_peers(dig[i], bits);
#pragma unroll
        for (int i = 0; i < kSortItems; i++) {
            const uint32_t d = dig[i];
            const uint32_t peers = peer[i];
            const int leader = __ffs(peers) - 1;
            uint32_t b = 0;
            if (d < kRadix) b = s_warp_hist[warp][d];
            __syncwarp();
            if (d < kRadix && lane == leader) s_warp_hist[warp][d] = b + __popc(peers);
            __syncwarp();
            rank[i] = b + __popc(peers & lanemask_lt());
        }
        __syncthreads();

        // Per digit (thread = digit): warp offsets, the block's count, and
        // where the digit's run starts in the partition's local order.
        uint32_t block_count = 0;
        {
            const int d = tid;
#pragma unroll
            for (int w = 0; w < kSortThreads / 32; w++) {
                const uint32_t c = s_warp_hist[w][d];
                s_warp_hist[w][d] = block_count;
                block_count += c;
            }
            uint32_t tot;
            s_digit_start[d] = block_exclusive_scan_256(d < radix ? block_count : 0u, s_scan, &tot);
        }
        __syncthreads();
        // Local reorder through shared memory first, so the look-back below
        // runs with the keys out of registers.
#pragma unroll
        for (int i = 0; i < kSortItems; i++) {
            const uint32_t d = dig[i];
            if (d < kRadix) {
                const uint32_t loc = s_digit_start[d] + s_warp_hist[warp][d] + rank[i];
                s_keys[loc] = key[i];
                s_vals[loc] = val[i];
            }
        }
        // Publish this partition's count for the digit, then look back.
        {
            const int d = tid;
            uint32_t *lb = lookback + (size_t)p * kRadix + d;
            uint32_t excl = 0;
            if (d < radix) {
                if (p == 0) {
                    st_relaxed(lb, kFlagInclusive | block_count);
                } else {
                    st_relaxed(lb, kFlagAggregate | block_count);
                    excl = lookback_digit(lookback, d, (int64_t)p - 1, status);
                    st_relaxed(lb, kFlagInclusive | ((excl + block_count) & kValueMask));
                }
            }
            s_global_base[d] = s_hist_excl[d] + excl;
        }
        uint32_t valid_count;
        {
            const uint64_t rem = (uint64_t)n - (uint64_t)p * kSortPart;
            valid_count = rem < (uint64_t)kSortPart ? (uint32_t)rem : (uint32_t)kSortPart;
        }
        __syncthreads();
        for (uint32_t j = tid; j < valid_count; j += kSortThreads) {
            const uint32_t k = s_keys[j];
            const uint32_t d = (k >> shift) & mask;
            const uint32_t pos = s_global_base[d] + (j - s_digit_start[d]);
            if (pos < n) {
                keys_out[pos] = k;
                vals_out[pos] = s_vals[j];
            }
        }
        __syncthreads();
    }
}

// Exclusive block-wide scan of one 64-bit value per thread (blockDim = 256).
__device__ __forceinline__ uint64_t block_exclusive_scan64_256(uint64_t v, uint64_t *s_warp,
                                                               uint64_t *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint64_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint64_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    uint64_t wpre = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < 8; w++) {
        const uint64_t t = s_warp[w];
        if (w < warp) wpre += t;
        tot += t;
    }
    __syncthreads();
    *total = tot;
    return wpre + x - v;
}

// Scan of the tile counts in depth order ("count" of the tile rasterizer).
// One block per 2048 Gaussians of the depth order; the block's offset comes
// from a decoupled look-back over 64-bit inclusive prefixes.  For each depth
// position i it writes the inclusive pair offset incl[i], the Gaussian's
// packed first tile (x0 | y0 << 16) and its rectangle width, next to the
// Gaussian id the depth sort left in sorted_gid: the emit reads these four
// contiguous arrays.  The last block stores K; K > max_pairs records
// GS_ERR_CAPACITY.
__global__ void __launch_bounds__(kScanThreads)
k_scan(int n, const uint32_t *__restrict__ sorted_gid, const int4 *__restrict__ rect, int tiles_x,
       int tiles_y, uint32_t *__restrict__ incl, uint32_t *__restrict__ rpack,
       uint32_t *__restrict__ width, uint64_t max_pairs, uint64_t *__restrict__ lookback,
       uint32_t *__restrict__ ticket, uint64_t *__restrict__ n_pairs, int32_t *__restrict__ status) {
    __shared__ uint64_t s_scan[8];
    __shared__ uint32_t s_part;
    __shared__ unsigned long long s_prefix;
    const int tid = threadIdx.x;
    if (tid == 0) s_part = atomicAdd(ticket, 1u);
    __syncthreads();
    const uint32_t p = s_part;
    const int64_t base = (int64_t)p * kScanPart;

    uint32_t c[kScanItems];
    uint64_t tsum = 0;
#pragma unroll
    for (int i = 0; i < kScanItems; i++) {
        const int64_t idx = base + tid * kScanItems + i;
        c[i] = 0;
        if (idx < n) {
            int x0, y0, w;
            c[i] = rect_tiles(rect[sorted_gid[idx]], tiles_x, tiles_y, x0, y0, w);
            rpack[idx] = (uint32_t)x0 | ((uint32_t)y0 << 16);
            width[idx] = (uint32_t)w;
        }
        tsum += c[i];
    }
    uint64_t block_total;
    const uint64_t toff = block_exclusive_scan64_256(tsum, s_scan, &block_total);
    if (tid < 32) {  // warp 0 publishes and looks back
        uint64_t *lb = lookback + p;
        uint64_t prefix = 0;
        if (p == 0) {
            if (tid == 0) st_relaxed64(lb, kFlag64Inclusive | (block_total & kValue64Mask));
        } else {
            if (tid == 0) st_relaxed64(lb, kFlag64Aggregate | (block_total & kValue64Mask));
            prefix = lookback_warp64(lookback, (int64_t)p - 1, status);
            if (tid == 0) st_relaxed64(lb, kFlag64Inclusive | ((prefix + block_total) & kValue64Mask));
        }
        if (tid == 0) {
            s_prefix = prefix;
            if (base + kScanPart >= n) {
                const uint64_t K = prefix + block_total;
                *n_pairs = K;
                if (K > max_pairs) set_status(status, GS_ERR_CAPACITY);
            }
        }
    }
    __syncthreads();
    uint64_t run = s_prefix + toff;
#pragma unroll
    for (int i = 0; i < kScanItems; i++) {
        const int64_t idx = base + tid * kScanItems + i;
        run += c[i];
        if (idx < n) incl[idx] = (uint32_t)run;  // meaningful while K <= max_pairs < 2^30
    }
}

// First index i in [lo, hi] with a[i] > t, for a non-decreasing array with
// a[hi] > t, by one full warp: each round probes 32 evenly spaced entries,
// so a search over N entries costs about log32(N) L2 round trips.
__device__ __forceinline__ uint32_t warp_upper_bound(const uint32_t *a, uint32_t lo, uint32_t hi,
                                                     uint32_t t) {
    const int lane = threadIdx.x & 31;
    while (hi - lo + 1 > 32) {
        const uint32_t stride = (hi - lo + 32) / 32;
        const uint32_t x = min(lo + lane * stride, hi);
        const uint32_t m = __ballot_sync(0xffffffffu, a[x] > t);
        if (m == 0) {
            lo = min(lo + 31 * stride, hi) + 1;
        } else {
            const int f = __ffs(m) - 1;
            const uint32_t xf = min(lo + f * stride, hi);
            lo = f == 0 ? lo : min(lo + (f - 1) * stride, hi) + 1;
            hi = xf;
        }
    }
    const uint32_t x = min(lo + lane, hi);
    const uint32_t m = __ballot_sync(0xffffffffu, a[x] > t);
    return lo + (__ffs(m) - 1);
}

// Pair emit ("emit" of the tile rasterizer), balanced by pairs: block b writes
// pairs [2048 b, 2048 b + 2048).  Warps 0 and 1 find the depth positions of
// the Gaussians holding its first and last pair; the block stages that span
// (at most 2048 Gaussians, since every drawable Gaussian has at least one
// pair and the undrawable ones sort last) in shared memory, and each thread
// finds its pair's Gaussian there by binary search.  A Gaussian's tiles are
// emitted row by row; the digit histograms of the tile sort are gathered on
// the way.  Nothing is emitted after a recorded error.
__global__ void __launch_bounds__(kEmitThreads)
k_emit(int n, const uint32_t *__restrict__ incl, const uint32_t *__restrict__ sorted_gid,
       const uint32_t *__restrict__ rpack, const uint32_t *__restrict__ width, int tiles_x,
       const uint64_t *__restrict__ n_pairs, const int32_t *__restrict__ status,
       uint32_t *__restrict__ ptile, uint32_t *__restrict__ pgid, uint32_t *__restrict__ tile_hist,
       int tile_passes, int tile_bpp) {
    __shared__ uint32_t s_incl[kEmitPairs];
    __shared__ uint32_t s_gid[kEmitPairs];
    __shared__ uint32_t s_rp[kEmitPairs];
    __shared__ uint32_t s_w[kEmitPairs];
    __shared__ uint32_t s_hist[kMaxTilePasses * kRadix];
    __shared__ uint32_t s_span[3];  // g0, g1, pairs before g0
    if (*(volatile const int32_t *)status != 0 || n == 0) return;
    const uint64_t K = *n_pairs;
    const int tid = threadIdx.x, warp = tid >> 5;
    for (int i = tid; i < kMaxTilePasses * kRadix; i += kEmitThreads) s_hist[i] = 0;
    const uint32_t dmask = (1u << tile_bpp) - 1u;
    for (uint64_t b = blockIdx.x; b * kEmitPairs < K; b += gridDim.x) {
        const uint32_t p0 = (uint32_t)(b * kEmitPairs);
        const uint64_t pe = (uint64_t)p0 + kEmitPairs;
        const uint32_t p1 = (uint32_t)(K < pe ? K : pe);  // exclusive
        __syncthreads();
        if (warp == 0) {
            const uint32_t g0 = warp_upper_bound(incl, 0, (uint32_t)n - 1, p0);
            if (tid == 0) {
                s_span[0] = g0;
                s_span[2] = g0 == 0 ? 0u : incl[g0 - 1];
            }
        } else if (warp == 1) {
            const uint32_t g1 = warp_upper_bound(incl, 0, (uint32_t)n - 1, p1 - 1);
            if ((tid & 31) == 0) s_span[1] = g1;
        }
        __syncthreads();
        const uint32_t g0 = s_span[0], g1 = s_span[1], before = s_span[2];
        const uint32_t span = g1 - g0 + 1;
        for (uint32_t k = tid; k < span && k < (uint32_t)kEmitPairs; k += kEmitThreads) {
            s_incl[k] = incl[g0 + k];
            s_gid[k] = sorted_gid[g0 + k];
            s_rp[k] = rpack[g0 + k];
            s_w[k] = width[g0 + k];
        }
        __syncthreads();
        const int last = (int)min(span, (uint32_t)kEmitPairs) - 1;
        for (uint32_t j = p0 + tid; j < p1; j += kEmitThreads) {
            int lo = 0, hi = last;
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (s_incl[mid] > j) hi = mid; else lo = mid + 1;
            }
            const uint32_t li = j - (lo == 0 ? before : s_incl[lo - 1]);
            const uint32_t w = s_w[lo], rp = s_rp[lo];
            const uint32_t row = li / w;
            const uint32_t tile = ((rp >> 16) + row) * (uint32_t)tiles_x + (rp & 0xFFFFu) + (li - row * w);
            ptile[j] = tile;
            pgid[j] = s_gid[lo];
            for (int k = 0; k < tile_passes; k++)
                atomicAdd(&s_hist[k * kRadix + ((tile >> (k * tile_bpp)) & dmask)], 1u);
        }
    }
    __syncthreads();
    for (int i = tid; i < tile_passes * kRadix; i += kEmitThreads)
        if (s_hist[i]) atomicAdd(&tile_hist[i], s_hist[i]);
}

// [start, end) of each tile in the sorted pair list.  Ranges were zeroed
// beforehand, so empty tiles stay [0, 0); on a recorded error all stay empty.
__global__ void __launch_bounds__(256)
k_ranges(const uint32_t *__restrict__ ptile, const uint64_t *__restrict__ n_pairs,
         uint32_t *__restrict__ ranges, const int32_t *__restrict__ status) {
    if (*(volatile const int32_t *)status != 0) return;
    const uint64_t K = *n_pairs;
    for (uint64_t j = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; j < K;
         j += (uint64_t)gridDim.x * blockDim.x) {
        const uint32_t t = ptile[j];
        if (j == 0 || ptile[j - 1] != t) ranges[2 * (size_t)t] = (uint32_t)j;
        if (j == K - 1 || ptile[j + 1] != t) ranges[2 * (size_t)t + 1] = (uint32_t)(j + 1);
    }
}

// Order in which the blend kernels take the tiles: longest list first, so
// that the heaviest tiles do not start last and leave SMs idle at the end
// (a counting sort on list length in steps of 4 entries, one CTA; the order
// within a bucket is arbitrary).
constexpr int kOrderBuckets = 1024;
__global__ void __launch_bounds__(kOrderBuckets)
k_tile_order(const uint32_t *__restrict__ ranges, int tiles, uint32_t *__restrict__ order) {
    __shared__ uint32_t s_off[kOrderBuckets];
    __shared__ uint32_t s_warp[kOrderBuckets / 32];
    const int t = threadIdx.x;
    auto bucket = [&](int i) {
        const uint32_t len = ranges[2 * (size_t)i + 1] - ranges[2 * (size_t)i];
        return kOrderBuckets - 1 - (int)min(len >> 2, (uint32_t)(kOrderBuckets - 1));
    };
    s_off[t] = 0;
    __syncthreads();
    for (int i = t; i < tiles; i += kOrderBuckets) atomicAdd(&s_off[bucket(i)], 1u);
    __syncthreads();
    // exclusive scan of the bucket counts
    const uint32_t v = s_off[t];
    uint32_t x = v;
    const int lane = t & 31, w = t >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[w] = x;
    __syncthreads();
    if (w == 0) {
        uint32_t z = s_warp[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, z, o);
            if (lane >= o) z += y;
        }
        s_warp[lane] = z;
    }
    __syncthreads();
    s_off[t] = x - v + (w > 0 ? s_warp[w - 1] : 0u);
    __syncthreads();
    for (int i = t; i < tiles; i += kOrderBuckets) order[atomicAdd(&s_off[bucket(i)], 1u)] = (uint32_t)i;
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

#ifndef GS_BIN_LOCAL
#define GS_BIN_LOCAL 1
#endif

constexpr int kBinThreads = 512;
// The count matrix holds at most kBinHistCap entries: min(SMs, kBinCTAsMax,
// kBinHistCap / tiles) CTAs share the Gaussians.
constexpr int kBinCTAsMax = 320;
constexpr int64_t kBinHistCap = 1 << 22;
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
            if (c <= kLaneTiles) {
                for (uint32_t k = 0; k < c; k++) {
                    const uint32_t dy = k / (uint32_t)w;
                    f(g, (y0 + (int)dy) * tiles_x + x0 + (int)(k - dy * (uint32_t)w));
                }
            }
            uint32_t big = __ballot_sync(0xffffffffu, c > kLaneTiles);
            while (big) {
                const int src = __ffs(big) - 1;
                big &= big - 1;
                const int gb = __shfl_sync(0xffffffffu, g, src);
                const uint32_t cb = __shfl_sync(0xffffffffu, c, src);
                const int xb = __shfl_sync(0xffffffffu, x0, src), yb = __shfl_sync(0xffffffffu, y0, src);
                const uint32_t wb = (uint32_t)__shfl_sync(0xffffffffu, w, src);
                for (uint32_t k = lane; k < cb; k += 32) {
                    const uint32_t dy = k / wb;
                    f(gb, (yb + (int)dy) * tiles_x + xb + (int)(k - dy * wb));
                }
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
k_bin_count(int n, const int4 *__restrict__ rect, int tiles_x, int tiles_y, uint32_t *__restrict__ H) {
    extern __shared__ uint32_t s_cnt[];
    const int tiles = tiles_x * tiles_y;
    uint32_t *row = H + (size_t)blockIdx.x * tiles;
    const bool smem = tiles <= kSmemTiles;
    uint32_t *cnt = smem ? s_cnt : row;
    for (int t = threadIdx.x; t < tiles; t += kBinThreads) cnt[t] = 0;
    __syncthreads();
    int g_begin, g_end;
    cta_range(n, g_begin, g_end);
    for_each_pair(g_begin, g_end, rect, tiles_x, tiles_y, [&](int, int t) { atomicAdd(&cnt[t], 1u); });
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
// order (longest list first, by a counting sort on length in steps of 4).
constexpr int kScanTilesThreads = 1024;
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
            *n_pairs = z;
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
        const uint32_t len = ranges[2 * (size_t)i + 1] - ranges[2 * (size_t)i];
        return kScanTilesThreads - 1 - (int)min(len >> 2, (uint32_t)(kScanTilesThreads - 1));
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
           const int32_t *__restrict__ status) {
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
    for_each_pair(g_begin, g_end, rect, tiles_x, tiles_y,
                  [&](int g, int t) { keys[atomicAdd(&cur[t], 1u)] = pair_key(xyod, (uint32_t)g); });
}

__device__ __forceinline__ uint32_t order_bucket(uint32_t len) {
    return min(len >> 2, (uint32_t)(kScanTilesThreads - 1));
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

// Tile lists of at most 256 entries: one warp each, in registers (CTA b,
// warp w take the (4 b + w)-th tile of the order).
__global__ void __launch_bounds__(128)
k_tile_sort_warp(const uint32_t *__restrict__ ranges, const uint32_t *__restrict__ order, int tiles,
                 const uint64_t *__restrict__ keys, uint32_t *__restrict__ pair_gid,
                 uint32_t *__restrict__ pair_tile) {
    const int lane = threadIdx.x & 31;
    const int b = blockIdx.x * 4 + (threadIdx.x >> 5);
    if (b >= tiles) return;
    const uint32_t tile = order[b];
    const uint32_t start = ranges[2 * (size_t)tile], end = ranges[2 * (size_t)tile + 1];
    const uint32_t L = end - start;
    if (L == 0 || L > 256) return;
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

// Tile lists in (lo, hi], hi = 256 kWarps: sorted by one CTA each.  Warp w
// sorts keys [256 w, 256 w + 256) in registers; the runs are then merged
// pairwise in shared memory (each key's output position is its index plus
// its rank in the other run).  With `persistent` a small grid walks the tile
// order (longest first) and stops at the first tile whose length bucket
// lies below lo's; otherwise CTA b takes the b-th tile of the order.
template <int kWarps>
__global__ void __launch_bounds__(kWarps * 32)
k_tile_sort(const uint32_t *__restrict__ ranges, const uint32_t *__restrict__ order, int tiles,
            const uint64_t *__restrict__ keys, uint32_t *__restrict__ pair_gid,
            uint32_t *__restrict__ pair_tile, uint32_t lo, int persistent) {
    constexpr int kThreads = kWarps * 32;
    constexpr uint32_t kHi = 256u * kWarps;
    extern __shared__ uint64_t s_buf[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int step = persistent ? (int)gridDim.x : tiles;
    for (int b = blockIdx.x; b < tiles; b += step) {
        const uint32_t tile = order[b];
        const uint32_t start = ranges[2 * (size_t)tile], end = ranges[2 * (size_t)tile + 1];
        const uint32_t L = end - start;
        if (persistent && order_bucket(L) < order_bucket(lo)) break;
        if (L <= lo || L > kHi) continue;
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

// Tiles longer than the shared-memory sort holds: one CTA per tile runs an
// LSD radix sort of the tile's keys in global memory (8-bit digits: four
// passes over the id, then four over the depth bits; each pass stable, in
// chunks of 256 ranked with warp ballots), ping-ponging between (ka, va) and
// (kb, vb) at the same offsets as the tile's range.
__global__ void __launch_bounds__(256)
k_tile_sort_long(const uint32_t *__restrict__ ranges, const uint32_t *__restrict__ order, int tiles,
                 const uint64_t *__restrict__ keys, uint32_t *__restrict__ pair_gid,
                 uint32_t *__restrict__ pair_tile, uint32_t lo, uint32_t *__restrict__ ka,
                 uint32_t *__restrict__ va, uint32_t *__restrict__ kb, uint32_t *__restrict__ vb) {
    __shared__ uint32_t s_base[kRadix];
    __shared__ uint32_t s_wc[8][kRadix];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int b = blockIdx.x; b < tiles; b += gridDim.x) {
        const uint32_t tile = order[b];
        const uint32_t start = ranges[2 * (size_t)tile], end = ranges[2 * (size_t)tile + 1];
        if (order_bucket(end - start) < order_bucket(lo)) break;
        if (end - start <= lo) continue;
        for (uint32_t i = start + tid; i < end; i += 256) {
            const uint64_t key = keys[i];
            ka[i] = (uint32_t)(key >> 32);
            va[i] = (uint32_t)key;
        }
        __syncthreads();
        uint32_t *sk = ka, *sv = va, *dk = kb, *dv = vb;
        for (int pass = 0; pass < 8; pass++) {
            const bool on_id = pass < 4;
            const int shift = 8 * (pass & 3);
            s_base[tid] = 0;
            __syncthreads();
            for (uint32_t i = start + tid; i < end; i += 256)
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
            for (uint32_t c0 = start; c0 < end; c0 += 256) {
                const uint32_t i = c0 + tid;
                const bool in = i < end;
                const uint32_t key = in ? sk[i] : 0u, val = in ? sv[i] : 0u;
                const uint32_t d = in ? ((on_id ? val : key) >> shift) & 0xFFu : (uint32_t)kRadix;
                for (int k = tid; k < 8 * kRadix; k += 256) (&s_wc[0][0])[k] = 0;
                __syncthreads();
                const uint32_t peers = digit_peers(d, 8);
                if (in && lane == __ffs(peers) - 1) s_wc[warp][d] = __popc(peers);
                __syncthreads();
                uint32_t acc = 0;  // per digit (thread = digit): exclusive over warps
                for (int ww = 0; ww < 8; ww++) {
                    const uint32_t c = s_wc[ww][tid];
                    s_wc[ww][tid] = acc;
                    acc += c;
                }
                __syncthreads();
                if (in) {
                    const uint32_t pos = s_base[d] + s_wc[warp][d] + __popc(peers & lanemask_lt());
                    dk[pos] = key;
                    dv[pos] = val;
                }
                __syncthreads();
                s_base[tid] += acc;
                __syncthreads();
            }
            uint32_t *t0 = sk, *t1 = sv;
            sk = dk; sv = dv; dk = t0; dv = t1;
            __syncthreads();
        }
        for (uint32_t i = start + tid; i < end; i += 256) {
            pair_gid[i] = sv[i];
            pair_tile[i] = tile;
        }
        __syncthreads();
    }
}

int num_sms() {
    static int sms = 0;
    if (sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms <= 0) sms = 148;
    }
    return sms;
}

}  // namespace

cudaError_t launch_bin_and_sort(const CamConst &c, int64_t n, const gs_projected &proj,
                                const gs_bins &bins, const BinsLayout &L, cudaStream_t s) {
    char *base = static_cast<char *>(bins.scratch);
    auto U32 = [&](size_t off) { return reinterpret_cast<uint32_t *>(base + off); };
    int32_t *status = reinterpret_cast<int32_t *>(base + L.status);
    uint64_t *n_pairs = reinterpret_cast<uint64_t *>(base + L.n_pairs);
    uint32_t *tickets = U32(L.tickets);
    uint32_t *depth_hist = U32(L.depth_hist);
    uint32_t *tile_hist = U32(L.tile_hist);
    uint32_t *ranges = U32(L.ranges);
    const int tiles = c.tiles_x * c.tiles_y;

    auto tile_order = [&]() {
        prof_before("tile_order", s);
        k_tile_order<<<1, kOrderBuckets, 0, s>>>(ranges, tiles, U32(L.tile_order));
        prof_after(s);
        return cudaGetLastError();
    };
    cudaError_t e = cudaMemsetAsync(base, 0, L.zero_bytes, s);
    if (e != cudaSuccess) return e;
#if GS_BIN_LOCAL
    {
        const int sms = num_sms();
        uint32_t *H = U32(L.bin_hist);
        uint32_t *totals = U32(L.tile_count);
        const int4 *rect = reinterpret_cast<const int4 *>(proj.rect);
        const float4 *xyod = reinterpret_cast<const float4 *>(proj.xy_opacity_depth);
        uint32_t *order = U32(L.tile_order);
        // the emitted sort keys, u64[max_pairs], over the (ptile_a, pgid_a) scratch
        uint64_t *keys = reinterpret_cast<uint64_t *>(base + L.ptile_a);
        int64_t ctas64 = std::min<int64_t>((int64_t)2 * sms, (int64_t)kBinCTAsMax);
        ctas64 = std::min<int64_t>(ctas64, kBinHistCap / tiles);
        const int ctas = (int)std::max<int64_t>(1, ctas64);
        const size_t cnt_smem = tiles <= kSmemTiles ? (size_t)tiles * sizeof(uint32_t) : 0;
        static bool attr = [] {
            cudaFuncSetAttribute(k_bin_count, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(kSmemTiles * sizeof(uint32_t)));
            cudaFuncSetAttribute(k_bin_emit, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(kSmemTiles * sizeof(uint32_t)));
            cudaFuncSetAttribute(k_tile_sort<kMidWarps>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(2 * kTileSortMid * sizeof(uint64_t)));
            return true;
        }();
        (void)attr;
        prof_before("bin_count", s);
        k_bin_count<<<ctas, kBinThreads, cnt_smem, s>>>((int)n, rect, c.tiles_x, c.tiles_y, H);
        k_bin_colscan<<<(tiles + 31) / 32, 256, 0, s>>>(tiles, ctas, H, totals);
        prof_after(s);
        prof_before("tile_scan", s);
        k_tile_scan<<<1, kScanTilesThreads, 0, s>>>(tiles, totals, (uint64_t)bins.max_pairs, ranges, order,
                                                    n_pairs, status);
        prof_after(s);
        if (n > 0) {
            prof_before("emit", s);
            k_bin_emit<<<ctas, kBinThreads, cnt_smem, s>>>((int)n, rect, xyod, c.tiles_x, c.tiles_y, ranges, H,
                                                           keys, status);
            prof_after(s);
            prof_before("tile_sort", s);
            k_tile_sort_warp<<<(tiles + 3) / 4, 128, 0, s>>>(ranges, order, tiles, keys, bins.pair_gid,
                                                              bins.pair_tile);
            k_tile_sort<kShortWarps><<<tiles, kShortWarps * 32, 2 * kTileSortShort * sizeof(uint64_t), s>>>(
                ranges, order, tiles, keys, bins.pair_gid, bins.pair_tile, 256u, 0);
            k_tile_sort<kMidWarps><<<std::min(tiles, sms), kMidWarps * 32, 2 * kTileSortMid * sizeof(uint64_t),
                                     s>>>(ranges, order, tiles, keys, bins.pair_gid, bins.pair_tile,
                                          kTileSortShort, 1);
            k_tile_sort_long<<<std::min(tiles, sms), 256, 0, s>>>(
                ranges, order, tiles, keys, bins.pair_gid, bins.pair_tile, kTileSortMid, U32(L.ptile_b),
                U32(L.pgid_b), bins.pair_tile, bins.pair_gid);
            prof_after(s);
        }
        return cudaGetLastError();
    }
#endif
    if (n == 0) return tile_order();  // K = 0, all ranges empty

    const int sms = num_sms();
    const uint32_t nn = (uint32_t)n;
    // 1. depth keys + histograms
    {
        const int blocks = (int)std::min<int64_t>((n + 255) / 256, (int64_t)sms * 4);
        prof_before("depth_keys", s);
        k_depth_keys<<<blocks, 256, 0, s>>>((int)n, reinterpret_cast<const float4 *>(proj.xy_opacity_depth),
                                             reinterpret_cast<const int4 *>(proj.rect), c.tiles_x, c.tiles_y,
                                             U32(L.keys_a), depth_hist);
        prof_after(s);
    }
    // 2. depth sort: 31 bits in four passes, A -> B -> A -> B -> A
    {
        const int shifts[4] = {0, 8, 16, 24}, bits[4] = {8, 8, 8, 7};
        uint32_t *ka = U32(L.keys_a), *va = U32(L.vals_a), *kb = U32(L.keys_b), *vb = U32(L.vals_b);
        const int64_t parts = (n + kSortPart - 1) / kSortPart;
        const int blocks = (int)std::min<int64_t>(parts, (int64_t)sms * 4);
        for (int pass = 0; pass < 4; pass++) {
            const bool even = (pass % 2) == 0;
            prof_before("depth_sort", s);
            k_onesweep<<<blocks, kSortThreads, 0, s>>>(
                even ? ka : kb, even ? va : vb, even ? kb : ka, even ? vb : va, nullptr, nn, nn,
                shifts[pass], bits[pass], depth_hist + pass * kRadix,
                U32(L.depth_lb) + (size_t)pass * L.depth_parts * kRadix, tickets + pass, status,
                pass == 0 ? 1 : 0, 0);
            prof_after(s);
        }
    }
    // 3. scan of the counts in depth order, then the pair emit.  The scan's
    //    per-Gaussian records reuse the depth sort's spare buffers: keys_b
    //    (inclusive offsets), vals_b (packed first tile), keys_a (widths);
    //    the sorted ids stay in vals_a.
    int tile_bits = 0;
    while ((1 << tile_bits) < tiles) tile_bits++;
    const int tile_passes = (tile_bits + kRadixBits - 1) / kRadixBits;
    const int tile_bpp = tile_passes ? (tile_bits + tile_passes - 1) / tile_passes : 1;
    uint32_t *ta = U32(L.ptile_a), *ga = U32(L.pgid_a), *tb = U32(L.ptile_b), *gb = U32(L.pgid_b);
    uint32_t *to = bins.pair_tile, *go = bins.pair_gid;
    {
        const int blocks = (int)((n + kScanPart - 1) / kScanPart);
        prof_before("scan", s);
        k_scan<<<blocks, kScanThreads, 0, s>>>((int)n, U32(L.vals_a), reinterpret_cast<const int4 *>(proj.rect),
                                              c.tiles_x, c.tiles_y, U32(L.keys_b), U32(L.vals_b),
                                              U32(L.keys_a), (uint64_t)bins.max_pairs,
                                              reinterpret_cast<uint64_t *>(base + L.scan_lb), tickets + 4,
                                              n_pairs, status);
        prof_after(s);
    }
    {
        const int64_t chunks = (bins.max_pairs + kEmitPairs - 1) / kEmitPairs;
        const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>(chunks, (int64_t)sms * 4));
        uint32_t *et = tile_passes == 0 ? to : ta, *eg = tile_passes == 0 ? go : ga;
        prof_before("emit", s);
        k_emit<<<blocks, kEmitThreads, 0, s>>>((int)n, U32(L.keys_b), U32(L.vals_a), U32(L.vals_b),
                                               U32(L.keys_a), c.tiles_x, n_pairs, status, et, eg, tile_hist,
                                               tile_passes, tile_bpp);
        prof_after(s);
    }
    // 4. stable pair sort on the tile bits
    {
        const int64_t parts = (bins.max_pairs + kSortPart - 1) / kSortPart;
        const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>(parts, (int64_t)sms * 4));
        uint32_t *st = ta, *sg = ga;
        for (int pass = 0; pass < tile_passes; pass++) {
            uint32_t *dt, *dg;
            if (pass == tile_passes - 1) { dt = to; dg = go; }
            else if (st == ta) { dt = tb; dg = gb; }
            else { dt = ta; dg = ga; }
            const int sh = pass * tile_bpp;
            const int nb = std::min(tile_bpp, tile_bits - sh);
            prof_before("tile_sort", s);
            k_onesweep<<<blocks, kSortThreads, 0, s>>>(
                st, sg, dt, dg, n_pairs, 0u, (uint32_t)bins.max_pairs, sh, nb, tile_hist + pass * kRadix,
                U32(L.tile_lb) + (size_t)pass * L.tile_parts * kRadix, tickets + 5 + pass, status, 0, 1);
            prof_after(s);
            st = dt; sg = dg;
        }
    }
    // 5. ranges
    {
        const int blocks = sms * 4;
        prof_before("ranges", s);
        k_ranges<<<blocks, 256, 0, s>>>(bins.pair_tile, n_pairs, ranges, status);
        prof_after(s);
    }
    // 6. the blend kernels' tile order
    return tile_order();
}

}  // namespace gs
