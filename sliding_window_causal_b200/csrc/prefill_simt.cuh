// prefill_simt.cuh: fp32 sliding-window causal attention on the CUDA cores.
//
// fp32 inputs and outputs are served in fp32 arithmetic end to end (TF32 tensor cores
// would round the operands to 10 mantissa bits). One warp owns one query row i and
// walks its band max(0, i-W+1) .. i in batches of 32 keys: each lane scores one key
// (scaled dot product, "27. Sliding-Window Attention", Step-by-Step Approach step 1),
// the warp folds the batch into a running max and sum (stable softmax with the max
// subtracted, "Mistral Architecture > Implementation: Sliding Window Attention",
// Step 2, in its online form), and the lanes accumulate weights x v over the head
// dimension. Keys outside the band are never read. Any head dimension 1..4096.
#pragma once
#include <math.h>

namespace swa {

constexpr int kSimtWarps = 4;

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Dynamic shared memory: per warp q[D], acc[D], p[32] floats.
__global__ void __launch_bounds__(kSimtWarps * 32)
    prefill_simt_kernel(const float* __restrict__ q, const float* __restrict__ k,
                        const float* __restrict__ v, float* __restrict__ out, int64_t nrows, int T,
                        int D, int W, float scale) {
    extern __shared__ float sm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * kSimtWarps + warp;
    if (r >= nrows) return;
    float* sq = sm + warp * (2 * D + 32);
    float* sacc = sq + D;
    float* sp = sacc + D;
    const int64_t bh = r / T;
    const int i = (int)(r - bh * T);
    const float* qr = q + r * D;
    const float* kh = k + bh * (int64_t)T * D;
    const float* vh = v + bh * (int64_t)T * D;
    for (int d = lane; d < D; d += 32) {
        sq[d] = qr[d];
        sacc[d] = 0.f;
    }
    __syncwarp();
    const int lo = i - W + 1 > 0 ? i - W + 1 : 0;
    float m = -INFINITY, l = 0.f;
    for (int j0 = lo; j0 <= i; j0 += 32) {
        const int j = j0 + lane;
        const bool valid = j <= i;
        float s = -INFINITY;
        if (valid) {
            const float* kj = kh + (int64_t)j * D;
            float dot = 0.f;
            for (int d = 0; d < D; ++d) dot = fmaf(sq[d], kj[d], dot);
            s = dot * scale;
        }
        const float m_new = fmaxf(m, warp_max(s));  // finite: key j0 is in the band
        const float alpha = expf(m - m_new);
        const float p = valid ? expf(s - m_new) : 0.f;
        l = l * alpha + warp_sum(p);
        sp[lane] = p;
        __syncwarp();
        const int cnt = (i - j0 + 1) < 32 ? (i - j0 + 1) : 32;
        for (int d = lane; d < D; d += 32) {
            float a = sacc[d] * alpha;
            for (int t = 0; t < cnt; ++t) a = fmaf(sp[t], vh[(int64_t)(j0 + t) * D + d], a);
            sacc[d] = a;
        }
        __syncwarp();
        m = m_new;
    }
    float* orow = out + r * D;
    for (int d = lane; d < D; d += 32) orow[d] = sacc[d] / l;
}

}  // namespace swa
