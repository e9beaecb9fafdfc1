// backward.cuh: gradients of the sliding-window prefill with respect to q, k and v, on the
// CUDA cores in fp32 arithmetic (fp32 or bf16 operands).
//
// With c the score scale, p_ij the forward weights of row i and dout the output gradient
// ("NNX Sliding-Window Attention", Mask before softmax: the gradients are well defined for
// finite allowed scores; they follow from the chain rule through the forward):
//   dv_j = sum_i p_ij dout_i            dp_ij = dout_i . v_j
//   ds_ij = p_ij (dp_ij - delta_i)       delta_i = sum_j p_ij dp_ij
//   dq_i = c sum_j ds_ij k_j             dk_j = c sum_i ds_ij q_i
// over the band pairs only (0 <= i - j < W). Two kernels, neither with atomics, so every
// sum has one fixed order and the results are deterministic:
//   bwd_rows_kernel  one warp per query row i: the row's max and sum (lse_i), delta_i and
//                    dq_i, walking the band 32 keys at a time (lanes = keys).
//   bwd_cols_kernel  one warp per key row j: dk_j and dv_j, walking the queries that see j
//                    (i = j .. j+W-1) 32 at a time (lanes = queries), with lse_i and
//                    delta_i from the first kernel.
#pragma once
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "prefill_simt.cuh"
#include "weights.cuh"

namespace swa {

constexpr int kBwdWarps = 4;

__device__ __forceinline__ void store_val(float* p, float x) { *p = x; }
__device__ __forceinline__ void store_val(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// Dynamic shared memory per warp: q_i[D], dout_i[D], dq[D], p[32], ds[32] floats.
// stats: [rows][2] = (lse_i, delta_i), fp32. Contiguous [B,H,T,D] operands.
template <typename TIn>
__global__ void __launch_bounds__(kBwdWarps * 32)
    bwd_rows_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k, const TIn* __restrict__ v,
                    const TIn* __restrict__ dout, TIn* __restrict__ dq, float* __restrict__ stats, int64_t nrows,
                    int T, int D, int W, float c) {
    extern __shared__ float bsm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * kBwdWarps + warp;
    if (r >= nrows) return;
    float* sq = bsm + warp * (3 * D + 64);
    float* sdo = sq + D;
    float* sdq = sdo + D;
    float* sp = sdq + D;
    float* sds = sp + 32;
    const int64_t bh = r / T;
    const int i = (int)(r - bh * T);
    const TIn* kh = k + bh * (int64_t)T * D;
    const TIn* vh = v + bh * (int64_t)T * D;
    for (int d = lane; d < D; d += 32) {
        sq[d] = to_f32(q[r * D + d]);
        sdo[d] = to_f32(dout[r * D + d]);
        sdq[d] = 0.f;
    }
    __syncwarp();
    const int lo = i - W + 1 > 0 ? i - W + 1 : 0;
    // pass 1: row maximum and sum of the scaled scores (online)
    float m = -INFINITY, l = 0.f;
    for (int j0 = lo; j0 <= i; j0 += 32) {
        const int j = j0 + lane;
        float s = -INFINITY;
        if (j <= i) {
            float dot = 0.f;
            for (int d = 0; d < D; ++d) dot = fmaf(sq[d], to_f32(kh[(int64_t)j * D + d]), dot);
            s = dot * c;
        }
        const float m_new = fmaxf(m, warp_max(s));  // finite: key j0 is in the band
        l = l * expf(m - m_new) + warp_sum(j <= i ? expf(s - m_new) : 0.f);
        m = m_new;
    }
    const float lse = m + logf(l);
    // pass 2: delta = sum_j p_j dp_j
    float delta = 0.f;
    for (int j0 = lo; j0 <= i; j0 += 32) {
        const int j = j0 + lane;
        float pdp = 0.f;
        if (j <= i) {
            float dot = 0.f, dp = 0.f;
            for (int d = 0; d < D; ++d) {
                dot = fmaf(sq[d], to_f32(kh[(int64_t)j * D + d]), dot);
                dp = fmaf(sdo[d], to_f32(vh[(int64_t)j * D + d]), dp);
            }
            pdp = expf(dot * c - lse) * dp;
        }
        delta += warp_sum(pdp);
    }
    // pass 3: dq = c sum_j ds_j k_j
    for (int j0 = lo; j0 <= i; j0 += 32) {
        const int j = j0 + lane;
        float ds = 0.f;
        if (j <= i) {
            float dot = 0.f, dp = 0.f;
            for (int d = 0; d < D; ++d) {
                dot = fmaf(sq[d], to_f32(kh[(int64_t)j * D + d]), dot);
                dp = fmaf(sdo[d], to_f32(vh[(int64_t)j * D + d]), dp);
            }
            ds = expf(dot * c - lse) * (dp - delta);
        }
        sds[lane] = ds;
        __syncwarp();
        const int cnt = (i - j0 + 1) < 32 ? (i - j0 + 1) : 32;
        for (int d = lane; d < D; d += 32) {
            float a = sdq[d];
            for (int t = 0; t < cnt; ++t) a = fmaf(sds[t], to_f32(kh[(int64_t)(j0 + t) * D + d]), a);
            sdq[d] = a;
        }
        __syncwarp();
    }
    for (int d = lane; d < D; d += 32) store_val(dq + r * D + d, sdq[d] * c);
    if (lane == 0) {
        stats[2 * r] = lse;
        stats[2 * r + 1] = delta;
    }
}

// Dynamic shared memory per warp: k_j[D], v_j[D], dk[D], dv[D], p[32], ds[32] floats.
template <typename TIn>
__global__ void __launch_bounds__(kBwdWarps * 32)
    bwd_cols_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k, const TIn* __restrict__ v,
                    const TIn* __restrict__ dout, const float* __restrict__ stats, TIn* __restrict__ dk,
                    TIn* __restrict__ dv, int64_t nrows, int T, int D, int W, float c) {
    extern __shared__ float bsm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * kBwdWarps + warp;
    if (r >= nrows) return;
    float* sk = bsm + warp * (4 * D + 64);
    float* sv = sk + D;
    float* sdk = sv + D;
    float* sdv = sdk + D;
    float* sp = sdv + D;
    float* sds = sp + 32;
    const int64_t bh = r / T;
    const int j = (int)(r - bh * T);
    const TIn* qh = q + bh * (int64_t)T * D;
    const TIn* doh = dout + bh * (int64_t)T * D;
    const float* st = stats + 2 * bh * (int64_t)T;
    for (int d = lane; d < D; d += 32) {
        sk[d] = to_f32(k[r * D + d]);
        sv[d] = to_f32(v[r * D + d]);
        sdk[d] = 0.f;
        sdv[d] = 0.f;
    }
    __syncwarp();
    const int hi = j + W - 1 < T - 1 ? j + W - 1 : T - 1;  // the last query that sees key j
    for (int i0 = j; i0 <= hi; i0 += 32) {
        const int i = i0 + lane;
        float p = 0.f, ds = 0.f;
        if (i <= hi) {
            float dot = 0.f, dp = 0.f;
            for (int d = 0; d < D; ++d) {
                dot = fmaf(to_f32(qh[(int64_t)i * D + d]), sk[d], dot);
                dp = fmaf(to_f32(doh[(int64_t)i * D + d]), sv[d], dp);
            }
            p = expf(dot * c - st[2 * i]);
            ds = p * (dp - st[2 * i + 1]);
        }
        sp[lane] = p;
        sds[lane] = ds;
        __syncwarp();
        const int cnt = (hi - i0 + 1) < 32 ? (hi - i0 + 1) : 32;
        for (int d = lane; d < D; d += 32) {
            float a = sdv[d], b = sdk[d];
            for (int t = 0; t < cnt; ++t) {
                const int64_t row = (int64_t)(i0 + t) * D + d;
                a = fmaf(sp[t], to_f32(doh[row]), a);
                b = fmaf(sds[t], to_f32(qh[row]), b);
            }
            sdv[d] = a;
            sdk[d] = b;
        }
        __syncwarp();
    }
    for (int d = lane; d < D; d += 32) {
        store_val(dk + r * D + d, sdk[d] * c);
        store_val(dv + r * D + d, sdv[d]);
    }
}

}  // namespace swa
