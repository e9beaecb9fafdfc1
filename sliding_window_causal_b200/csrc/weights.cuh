// weights.cuh: the softmax weights of every query's band, for inspection.
//
// "Mistral Architecture > Implementation: Sliding Window Attention" (Step 2) hands back the
// attention weight matrix beside the output. Only the band of that matrix can be nonzero,
// so this kernel writes the band alone: row i of (b,h) holds Wo = min(W, T) weights, and
// column c belongs to key j = i - Wo + 1 + c (the last column is the query itself). Columns
// with j < 0 hold 0. The weights are the softmax of the scaled scores over the band
// ("27. Sliding-Window Attention", Step-by-Step Approach steps 1-4), computed in fp32 from
// fp32 or bf16 inputs, with the row maximum subtracted (stable softmax, Step 2 of the
// Mistral page).
//
// One warp per row, two passes over the row's band: the first scores 32 keys at a time
// into the output row and keeps the running maximum and sum; the second rewrites each
// score as its weight. Every lane rereads only what it wrote itself.
#pragma once
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "prefill_simt.cuh"

namespace swa {

constexpr int kWeightWarps = 4;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// Dynamic shared memory: per warp q[D] floats. qs, ks: (b, h, t) element strides.
template <typename TIn>
__global__ void __launch_bounds__(kWeightWarps * 32)
    band_weights_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k, float* __restrict__ wout,
                        int64_t qsb, int64_t qsh, int64_t qst, int64_t ksb, int64_t ksh, int64_t kst,
                        int64_t nrows, int H, int T, int D, int Wo, float scale) {
    extern __shared__ float wsm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * kWeightWarps + warp;
    if (r >= nrows) return;
    float* sq = wsm + warp * D;
    const int64_t bh = r / T;
    const int i = (int)(r - bh * T);
    const int64_t b = bh / H, h = bh - b * H;
    const TIn* qr = q + b * qsb + h * qsh + (int64_t)i * qst;
    const TIn* kh = k + b * ksb + h * ksh;
    for (int d = lane; d < D; d += 32) sq[d] = to_f32(qr[d]);
    __syncwarp();
    float* wrow = wout + r * Wo;
    const int c_first = Wo - 1 - i > 0 ? Wo - 1 - i : 0;  // first column with j >= 0
    float m = -INFINITY, l = 0.f;
    for (int c0 = 0; c0 < Wo; c0 += 32) {
        const int c = c0 + lane;
        float s = -INFINITY;
        if (c < Wo && c >= c_first) {
            const TIn* kj = kh + (int64_t)(i - Wo + 1 + c) * kst;
            float dot = 0.f;
            for (int d = 0; d < D; ++d) dot = fmaf(sq[d], to_f32(kj[d]), dot);
            s = dot * scale;
        }
        if (c < Wo) wrow[c] = s;
        const float bm = warp_max(s);
        if (bm == -INFINITY) continue;  // no key of this batch is in the band
        const float m_new = fmaxf(m, bm);
        const float p = s == -INFINITY ? 0.f : expf(s - m_new);
        l = l * expf(m - m_new) + warp_sum(p);
        m = m_new;
    }
    const float inv_l = 1.f / l;  // l >= 1: the row maximum contributes exp(0)
    for (int c = lane; c < Wo; c += 32) {
        const float s = wrow[c];
        wrow[c] = s == -INFINITY ? 0.f : expf(s - m) * inv_l;
    }
}

}  // namespace swa
