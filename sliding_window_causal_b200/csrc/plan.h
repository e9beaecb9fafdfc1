// plan.h: work decomposition shared by the host planner exports and the kernels.
//
// Prefill: query tiles of BM rows meet key tiles of BN keys. Only tiles that meet the
// band are visited; tiles wholly inside it skip the mask ("NNX Sliding-Window
// Attention", A local mask is not a sparse implementation: only the allowed windows
// need computing). Decode: a stream at position pos holds its in-window positions in
// ring slots 0 .. min(pos+1, W)-1 (slot = position mod W).
#pragma once
#include <stdint.h>

#if defined(__CUDACC__)
#define SWA_HD __host__ __device__ __forceinline__
#else
#define SWA_HD inline
#endif

namespace swa {

// First and last key tile visited by query tile qt.
SWA_HD void kv_tile_range(int64_t T, int64_t W, int64_t bm, int64_t bn, int64_t qt,
                          int64_t* kt_first, int64_t* kt_last) {
    int64_t i0 = qt * bm;
    int64_t i1 = i0 + bm - 1;
    int64_t lo = i0 - W + 1;
    if (lo < 0) lo = 0;
    int64_t hi = i1 < T - 1 ? i1 : T - 1;
    *kt_first = lo / bn;
    *kt_last = hi / bn;
}

// 0 = not visited, 1 = edge (masked), 2 = full (every pair in the band, keys < T).
// Rows of the last query tile at or past T are padding; counting them can only make
// a tile edge rather than full, never the other way.
SWA_HD int tile_class(int64_t T, int64_t W, int64_t bm, int64_t bn, int64_t qt, int64_t kt) {
    int64_t f, l;
    kv_tile_range(T, W, bm, bn, qt, &f, &l);
    if (kt < f || kt > l) return 0;
    int64_t i0 = qt * bm, i1 = i0 + bm - 1;
    int64_t j0 = kt * bn, j1 = j0 + bn - 1;
    bool full = (j1 <= i0) && (i1 - j0 < W) && (j1 < T);
    return full ? 2 : 1;
}

// Work items of the tensor-core prefill: pairs of query tiles (2p, 2p+1) of one (b,h),
// n_pairs = ceil(n_qt / 2) per head, BH * n_pairs items in all. Item u is (bh, pair):
//  - first the "full" pairs, both of whose tiles exist and every row of which sees a
//    whole window (256p >= W - 1, so they all do the same work), head after head with
//    the pairs of a head in order: the CTAs working at the same time then share the
//    key and value tiles of a few heads, which stay in L2;
//  - then the lighter pairs (rows near the start of a head, and a last pair that has
//    only one tile), heaviest first and head-minor, so that the persistent CTAs, which
//    take items in a snake order, finish together.
// W is the window clamped to T. Returns false if u is out of range. I is the integer type
// (int in the kernels, whose item counts fit 32 bits; int64_t on the host).
template <typename I>
SWA_HD bool prefill_item(I u, I BH, I n_qt, I W, I* bh, I* pair) {
    const I n_pairs = (n_qt + 1) / 2;
    if (u < 0 || BH < 1 || n_qt < 1 || u >= BH * n_pairs) return false;
    const I full_end = n_qt / 2;  // pairs with both tiles
    I pf0 = (W - 1 + 255) / 256;  // first pair whose rows all see W keys
    if (pf0 > full_end) pf0 = full_end;
    const I nf = full_end - pf0;
    if (u < BH * nf) {
        *bh = u / nf;
        *pair = pf0 + u % nf;
        return true;
    }
    const I v = u - BH * nf, idx = v / BH;
    *bh = v % BH;
    if (!(n_qt & 1)) {
        *pair = pf0 - 1 - idx;  // pairs pf0-1 .. 0: their work falls with the pair index
        return true;
    }
    // The last pair holds a single tile; it goes where its work falls among the others:
    // after the pairs p* .. pf0-1 that do at least as much (binary search: the work of
    // pair p, in 128-key tiles, is non-decreasing in p below pf0).
    auto tiles = [&](I qt) {  // key tiles visited by query tile qt
        const I lo = qt * 128 - W + 1;
        return qt - (lo > 0 ? lo / 128 : 0) + 1;
    };
    const I wh = tiles(n_qt - 1);
    I lo = 0, hi = pf0;  // smallest p in [0, pf0) with work(p) >= wh, or pf0
    while (lo < hi) {
        const I mid = (lo + hi) / 2;
        if (tiles(2 * mid) + tiles(2 * mid + 1) >= wh) hi = mid;
        else lo = mid + 1;
    }
    const I at = pf0 - lo;  // place of the single-tile pair in the list
    if (idx < at) *pair = pf0 - 1 - idx;
    else if (idx == at) *pair = n_pairs - 1;
    else *pair = pf0 - idx;
    return true;
}

// CTAs of the tensor-core backward: one per (bh, resident 128-row tile), BH * n_t in all;
// the resident tile is a key tile (kv) or a query tile. With a = ceil((W - 1) / 128), key
// tile kt streams the min(n_t - kt, a + 1) query tiles that meet its band (falling with
// kt) and query tile qt the min(qt, a) + 1 key tiles of its band (rising with qt), so the
// tiles that stream a + 1 tiles (full) are the first n_t - a key tiles or the last
// n_t - a query tiles. CTA u is:
//  - first the full tiles, head after head, those of a head in order: the CTAs at work
//    at one time stream the tiles of a few heads, which stay in L2;
//  - then the others heaviest first, head-minor, so that the last CTAs to start are the
//    lightest and the SMs finish together.
// W is the window clamped to T. Returns false if u is out of range.
template <typename I>
SWA_HD bool bwd_cta_tile(I u, I BH, I n_t, I W, bool kv, I* bh, I* xt) {
    if (u < 0 || BH < 1 || n_t < 1 || W < 1 || u >= BH * n_t) return false;
    const I a = (W + 126) / 128;
    const I np = a < n_t ? a : n_t;  // tiles that stream fewer than a + 1 tiles
    const I nf = n_t - np;
    if (u < BH * nf) {
        *bh = u / nf;
        const I r = u % nf;
        *xt = kv ? r : np + r;
        return true;
    }
    const I v = u - BH * nf, r = v / BH;  // r = 0: the heaviest of the others
    *bh = v % BH;
    *xt = kv ? nf + r : np - 1 - r;
    return true;
}

SWA_HD int64_t decode_valid_slots(int64_t pos, int64_t W) {
    return pos + 1 < W ? pos + 1 : W;
}

}  // namespace swa
