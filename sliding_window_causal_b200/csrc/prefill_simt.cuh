// prefill_simt.cuh: fp32 sliding-window causal attention on the CUDA cores.
//
// fp32 inputs and outputs are served in fp32 arithmetic end to end (TF32 tensor cores
// would round the operands to 10 mantissa bits). One warp owns one query row i and
// walks its band max(0, i-W+1) .. i in batches of 32 keys: each lane scores one key
// (scaled dot product, "27. Sliding-Window Attention", Step-by-Step Approach step 1),
// the warp folds the batch into a running max and sum (stable softmax with the max
// subtracted, "Mistral Architecture > Implementation: Sliding Window Attention",
// Step 2, in its online form), and the lanes accumulate weights x v over the head
// dimension. Keys outside the band are never read. Any head dimension 1..4096, and any
// (b, h, t) element strides (the head dimension is contiguous).
#pragma once
#include <math.h>
#include <stdint.h>

namespace swa {

// Element strides (b, h, t) of q, k, v and out; the head-dimension stride is 1.
struct Strides {
    int64_t q[3], k[3], v[3], o[3];
};

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
                        const float* __restrict__ v, float* __restrict__ out, Strides st,
                        float* __restrict__ lse, int64_t nrows, int H, int T, int D, int W, float scale) {
    extern __shared__ float sm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * kSimtWarps + warp;
    if (r >= nrows) return;
    float* sq = sm + warp * (2 * D + 32);
    float* sacc = sq + D;
    float* sp = sacc + D;
    const int64_t bh = r / T;
    const int i = (int)(r - bh * T);
    const int64_t b = bh / H, h = bh - b * H;
    const float* qr = q + b * st.q[0] + h * st.q[1] + (int64_t)i * st.q[2];
    const float* kh = k + b * st.k[0] + h * st.k[1];
    const float* vh = v + b * st.v[0] + h * st.v[1];
    const int64_t kt = st.k[2], vt = st.v[2];
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
            const float* kj = kh + (int64_t)j * kt;
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
            for (int t = 0; t < cnt; ++t) a = fmaf(sp[t], vh[(int64_t)(j0 + t) * vt + d], a);
            sacc[d] = a;
        }
        __syncwarp();
        m = m_new;
    }
    float* orow = out + b * st.o[0] + h * st.o[1] + (int64_t)i * st.o[2];
    for (int d = lane; d < D; d += 32) orow[d] = sacc[d] / l;
    if (lse != nullptr && lane == 0) lse[r] = m + logf(l);  // natural log-sum-exp
}

}  // namespace swa
