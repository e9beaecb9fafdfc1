// prefill_narrow.cuh: bf16 sliding-window causal attention for bands of at most
// kNarrowMaxW keys, on the CUDA cores.
//
// With W keys per row the work is 4·T·W·D FLOPs against about 8·T·D bytes of q, k, v and
// out, so for small W the prefill is bound by HBM. The tensor-core kernel would spend such
// a band filling and draining its pipeline (TMA ring, a 128-key score tile of which W
// columns count, the TMEM round trip of S and P). Here one warp takes four consecutive
// rows, eight lanes per row, each lane a slice of D/8 head-dimension elements read as
// 16-byte vectors:
//   1. the row's W scores, scaled dot products q_i . k_j with j = i, i-1, .., i-W+1
//      (j >= 0) ("27. Sliding-Window Attention", Step-by-Step Approach step 1), each
//      summed over the row's eight lanes;
//   2. softmax over those W scores with their maximum subtracted ("Mistral Architecture >
//      Implementation: Sliding Window Attention", step 2), in fp32;
//   3. the weighted sum of the W value rows in fp32 (step 3), divided by the weight sum
//      and rounded to bf16 once.
// A key/value row is used by the W query rows after it, which run in the same or the next
// warps of the CTA, so it is read from HBM about once. Any (b, h, t) element strides; the
// head dimension is contiguous.
#pragma once
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "prefill_simt.cuh"  // Strides
#include "ptx.cuh"

namespace swa {

// Bands of at most this many keys take this kernel. Measured on B2 H16 T8192 D128: 50.5 us
// at W = 1 (5.3 TB/s) against 80.1 us for the tensor-core kernel, 89.1 against 103.6 at
// W = 6, and even at W = 8 (106.3 against 103.1).
constexpr int kNarrowMaxW = 7;
constexpr int kNarrowWarps = 8;
constexpr int kNarrowRows = 4 * kNarrowWarps;  // rows per CTA

// n elements of bf16 (n a multiple of 8, 16-byte aligned) to fp32
template <int N>
__device__ __forceinline__ void narrow_load(const __nv_bfloat16* p, float (&f)[N]) {
    static_assert(N % 8 == 0, "16-byte vectors");
#pragma unroll
    for (int x = 0; x < N / 8; ++x) {
        const uint4 u = *reinterpret_cast<const uint4*>(p + 8 * x);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int y = 0; y < 4; ++y) {
            f[8 * x + 2 * y] = ptx::bf16lo_f32(w[y]);
            f[8 * x + 2 * y + 1] = ptx::bf16hi_f32(w[y]);
        }
    }
}

// One CTA per (b, h, 32-row block); grid = B*H*n_rb. scale_log2 = scale * log2(e).
template <int D>
__global__ void __launch_bounds__(kNarrowWarps * 32)
    prefill_narrow_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                          const __nv_bfloat16* __restrict__ v, __nv_bfloat16* __restrict__ out, Strides st,
                          float* __restrict__ lse, int H, int T, int W, float scale_log2, int n_rb) {
    static_assert(D == 64 || D == 128, "head dim 64 or 128");
    constexpr int E = D / 8;  // elements per lane
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane & 7;
    const int64_t bh = blockIdx.x / n_rb;
    const int rb = (int)(blockIdx.x - bh * n_rb);
    const int i = rb * kNarrowRows + warp * 4 + (lane >> 3);  // this lane's row
    const bool live = i < T;
    const int64_t b = bh / H, h = bh - b * H;
    const int e0 = sub * E;
    const __nv_bfloat16* kh = k + b * st.k[0] + h * st.k[1] + e0;
    const __nv_bfloat16* vh = v + b * st.v[0] + h * st.v[1] + e0;

    float qf[E];
    if (live) {
        narrow_load<E>(q + b * st.q[0] + h * st.q[1] + (int64_t)i * st.q[2] + e0, qf);
#pragma unroll
        for (int e = 0; e < E; ++e) qf[e] *= scale_log2;
    }
    // scores in log2 units; key i - t for t < W (t = 0 is the diagonal, always in the band)
    float s[kNarrowMaxW];
#pragma unroll
    for (int t = 0; t < kNarrowMaxW; ++t) {
        if (t < W) {  // uniform across the warp: the shuffles below see every lane
            const int j = i - t;
            const bool ok = live && j >= 0;
            float dot = 0.f;
            if (ok) {
                float kf[E];
                narrow_load<E>(kh + (int64_t)j * st.k[2], kf);
#pragma unroll
                for (int e = 0; e < E; ++e) dot = fmaf(qf[e], kf[e], dot);
            }
            dot += __shfl_xor_sync(0xffffffffu, dot, 1);
            dot += __shfl_xor_sync(0xffffffffu, dot, 2);
            dot += __shfl_xor_sync(0xffffffffu, dot, 4);
            s[t] = ok ? dot : -INFINITY;
        }
    }
    if (!live) return;
    float m = s[0];
#pragma unroll
    for (int t = 1; t < kNarrowMaxW; ++t)
        if (t < W) m = fmaxf(m, s[t]);
    float l = 0.f, acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
#pragma unroll
    for (int t = 0; t < kNarrowMaxW; ++t) {
        const int j = i - t;
        if (t < W && j >= 0) {
            const float p = ptx::ex2(s[t] - m);
            l += p;
            float vf[E];
            narrow_load<E>(vh + (int64_t)j * st.v[2], vf);
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] = fmaf(p, vf[e], acc[e]);
        }
    }
    const float inv = 1.f / l;  // l >= 1: the maximum's own weight is 1
    __nv_bfloat16* orow = out + b * st.o[0] + h * st.o[1] + (int64_t)i * st.o[2] + e0;
#pragma unroll
    for (int x = 0; x < E / 8; ++x) {
        uint4 u;
        u.x = ptx::pack_bf16x2(acc[8 * x + 0] * inv, acc[8 * x + 1] * inv);
        u.y = ptx::pack_bf16x2(acc[8 * x + 2] * inv, acc[8 * x + 3] * inv);
        u.z = ptx::pack_bf16x2(acc[8 * x + 4] * inv, acc[8 * x + 5] * inv);
        u.w = ptx::pack_bf16x2(acc[8 * x + 6] * inv, acc[8 * x + 7] * inv);
        *reinterpret_cast<uint4*>(orow + 8 * x) = u;
    }
    // natural log-sum-exp of the scaled scores: (m + log2 l) ln 2
    if (lse != nullptr && sub == 0) lse[bh * T + i] = (m + log2f(l)) * 0.6931471805599453f;
}

}  // namespace swa
