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

SWA_HD int64_t decode_valid_slots(int64_t pos, int64_t W) {
    return pos + 1 < W ? pos + 1 : W;
}

}  // namespace swa
