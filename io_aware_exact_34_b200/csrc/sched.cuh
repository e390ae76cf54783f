// sched.cuh -- band-mask arithmetic shared by the host scheduler and the kernels.
//
// The sliding-window FlashAttention prefill page (m.xxqk.cn/news/265020)
// skips a KV block when it lies wholly outside the band of every row of the
// Q block (§5.1), breaks once blocks start right of the band (§5.3), and in
// its kernel sketch computes the visited KV block range of a Q block in closed
// form, start_kv = max(0, q_blk - window_blocks), end_kv = min(n, q_blk +
// window_blocks) (§7.3).  Here the range is computed exactly from the first
// and last valid rows of the Q tile, so it holds every tile with an allowed
// pair and no other tile.  Partially covered tiles get the element mask of
// §5.2; fully covered tiles take no mask at all.
#pragma once

#include <stdint.h>

#ifndef FATTN_HD
#define FATTN_HD __host__ __device__ __forceinline__
#endif

namespace fattn {

// The mask of window_size = (window_left, window_right) (§7.1) with causal,
// in a form the kernels evaluate cheaply.  Negative bounds are unbounded.
struct Band {
    long long Lq, Lk;
    long long shift;   // Lk - Lq: query i sits at key position i + shift
    long long left;    // window_left, < 0 = unbounded
    long long right;   // effective right bound: 0 if causal, else window_right
};

FATTN_HD Band make_band(long long Lq, long long Lk, int causal, int window_left, int window_right) {
    Band b;
    b.Lq = Lq;
    b.Lk = Lk;
    b.shift = Lk - Lq;
    b.left = window_left < 0 ? -1 : window_left;
    if (causal)
        b.right = 0;
    else
        b.right = window_right < 0 ? -1 : window_right;
    return b;
}

// A relative index clamped into [-2^30, 2^30]: far enough outside any tile to
// compare correctly against tile columns, and safe to offset by a tile width.
FATTN_HD int clamp_int(long long x) {
    return (int)(x < -(1LL << 30) ? -(1LL << 30) : (x > (1LL << 30) ? (1LL << 30) : x));
}

// Visited KV tiles [*lo, *hi) (tiles of bk keys) for the valid query rows
// [q_first, q_last] of a Q tile.  Empty range: *lo == *hi.
FATTN_HD void kv_tile_range(const Band& b, long long q_first, long long q_last, int bk,
                            int* lo, int* hi) {
    long long jmin = 0, jmax = b.Lk - 1;
    if (b.left >= 0) {
        long long t = q_first + b.shift - b.left;
        jmin = t > jmin ? t : jmin;
    }
    if (b.right >= 0) {
        long long t = q_last + b.shift + b.right;
        jmax = t < jmax ? t : jmax;
    }
    if (q_last < q_first || jmax < jmin) {
        *lo = 0;
        *hi = 0;
        return;
    }
    *lo = (int)(jmin / bk);
    *hi = (int)(jmax / bk) + 1;
}

// The transposed range, for the backward pass that walks Q tiles per KV tile:
// Q tiles [*lo, *hi) (tiles of bq rows) that hold an allowed pair with the
// keys [k_first, k_last] (k_last <= Lk - 1).  Key k is allowed for query i
// iff k - shift - right <= i <= k - shift + left (each side only when
// bounded), so the queries of the key tile form the interval
// [k_first - shift - right, k_last - shift + left] clipped to [0, Lq - 1], and
// every query in it has an allowed key in the tile.  Empty: *lo == *hi.
FATTN_HD void q_tile_range(const Band& b, long long k_first, long long k_last, int bq, int* lo, int* hi) {
    long long imin = 0, imax = b.Lq - 1;
    if (b.right >= 0) {
        long long t = k_first - b.shift - b.right;
        imin = t > imin ? t : imin;
    }
    if (b.left >= 0) {
        long long t = k_last - b.shift + b.left;
        imax = t < imax ? t : imax;
    }
    if (k_last < k_first || imax < imin) {
        *lo = 0;
        *hi = 0;
        return;
    }
    *lo = (int)(imin / bq);
    *hi = (int)(imax / bq) + 1;
}

// True when every (query, key) pair of rows [q_first, q_last] x keys
// [k0, k0 + bk) is allowed, i.e. the tile needs no element mask.
FATTN_HD bool tile_is_full(const Band& b, long long q_first, long long q_last, long long k0, int bk) {
    const long long k_last = k0 + bk - 1;
    if (k_last > b.Lk - 1) return false;
    if (b.right >= 0 && k_last > q_first + b.shift + b.right) return false;
    if (b.left >= 0 && k0 < q_last + b.shift - b.left) return false;
    return true;
}

// Allowed key columns of query row i inside the tile starting at key k0:
// columns c with lo_col <= c <= hi_col (relative to k0).
FATTN_HD void row_col_bounds(const Band& b, long long i, long long k0, int* lo_col, int* hi_col) {
    const long long pos = i + b.shift;
    long long hi = b.Lk - 1;
    if (b.right >= 0 && pos + b.right < hi) hi = pos + b.right;
    long long lo = (b.left >= 0) ? pos - b.left : 0;
    if (lo < 0) lo = 0;
    long long h = hi - k0, l = lo - k0;
    // clamp into int range around the tile
    if (h > (1 << 30)) h = (1 << 30);
    if (h < -(1 << 30)) h = -(1 << 30);
    if (l > (1 << 30)) l = (1 << 30);
    if (l < -(1 << 30)) l = -(1 << 30);
    *lo_col = (int)l;
    *hi_col = (int)h;
}

}  // namespace fattn
