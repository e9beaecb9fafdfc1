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
//   bwd_rows_kernel  a CTA takes kBwdRows consecutive query rows of one (b,h), one warp per
//                    row. It walks the union of their bands 32 keys at a time: the CTA
//                    stages the 32 key rows (and value rows) in shared memory with
//                    coalesced loads, and each lane scores one key from there. Three
//                    walks: the row statistics (lse_i), delta_i, and dq_i.
//   bwd_cols_kernel  a CTA takes kBwdRows consecutive key rows, one warp per key; it walks
//                    the queries that see them (i = j .. j+W-1) 32 at a time, staging q
//                    and dout rows, with lse_i and delta_i from the first kernel: dk_j, dv_j.
// Shared-memory rows are padded by one float so that 32 lanes reading 32 different rows
// hit 32 different banks. Head dimension D <= kBwdMaxD.
#pragma once
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "prefill_simt.cuh"
#include "weights.cuh"

namespace swa {

constexpr int kBwdRows = 8;      // rows (warps) per CTA
constexpr int kBwdMaxD = 512;

__device__ __forceinline__ void store_val(float* p, float x) { *p = x; }
__device__ __forceinline__ void store_val(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// Shared memory (floats): two staged blocks of 32 rows x (D+1), then per warp two rows of
// D and two vectors of 32.
__host__ __device__ constexpr size_t bwd_smem_floats(int D) { return 2 * 32 * (size_t)(D + 1) + kBwdRows * (2 * (size_t)D + 64); }

// Stage rows r0 .. r0+n-1 (n <= 32) of a [T, D] head into sh (stride D+1), zero-filling
// the rest of the 32-row block. All threads of the CTA take part.
template <typename TIn>
__device__ __forceinline__ void bwd_stage(float* sh, const TIn* __restrict__ head, int r0, int n, int D) {
    for (int x = threadIdx.x; x < 32 * D; x += kBwdRows * 32) {
        const int rr = x / D, d = x - rr * D;
        sh[rr * (D + 1) + d] = rr < n ? to_f32(head[(int64_t)(r0 + rr) * D + d]) : 0.f;
    }
}

template <typename TIn>
__global__ void __launch_bounds__(kBwdRows * 32)
    bwd_rows_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k, const TIn* __restrict__ v,
                    const TIn* __restrict__ dout, TIn* __restrict__ dq, float* __restrict__ stats, int T, int D,
                    int W, float c) {
    extern __shared__ float bsm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int blocks_per_head = (T + kBwdRows - 1) / kBwdRows;
    const int64_t bh = blockIdx.x / blocks_per_head;
    const int i0 = (int)(blockIdx.x - bh * blocks_per_head) * kBwdRows;
    const int i = i0 + warp;  // this warp's query row (may be past T: then it only helps stage)
    const bool live = i < T;
    const int last = min(T - 1, i0 + kBwdRows - 1);
    float* sk = bsm;
    float* sv = sk + 32 * (D + 1);
    float* sq = sv + 32 * (D + 1) + warp * (2 * D + 64);
    float* sdo = sq + D;
    float* sds = sdo + D;
    const TIn* kh = k + bh * (int64_t)T * D;
    const TIn* vh = v + bh * (int64_t)T * D;
    const int64_t r = bh * (int64_t)T + i;
    if (live)
        for (int d = lane; d < D; d += 32) {
            sq[d] = to_f32(q[r * D + d]);
            sdo[d] = to_f32(dout[r * D + d]);
        }
    const int lo = live ? max(0, i - W + 1) : 0;
    const int blo = max(0, i0 - W + 1);  // first key any row of the CTA needs
    // walk 1: row maximum and sum (online)
    float m = -INFINITY, l = 0.f;
    for (int j0 = blo; j0 <= last; j0 += 32) {
        __syncthreads();
        bwd_stage(sk, kh, j0, min(32, last - j0 + 1), D);
        __syncthreads();
        const int j = j0 + lane;
        const bool in = live && j >= lo && j <= i;
        float s = -INFINITY;
        if (in) {
            float dot = 0.f;
            const float* kr = sk + lane * (D + 1);
            for (int d = 0; d < D; ++d) dot = fmaf(sq[d], kr[d], dot);
            s = dot * c;
        }
        const float bm = warp_max(s);
        if (bm != -INFINITY) {
            const float m_new = fmaxf(m, bm);
            l = l * expf(m - m_new) + warp_sum(in ? expf(s - m_new) : 0.f);
            m = m_new;
        }
    }
    const float lse = m + logf(l);
    // walk 2: delta = sum_j p_j dp_j
    float delta = 0.f;
    for (int j0 = blo; j0 <= last; j0 += 32) {
        __syncthreads();
        const int n = min(32, last - j0 + 1);
        bwd_stage(sk, kh, j0, n, D);
        bwd_stage(sv, vh, j0, n, D);
        __syncthreads();
        const int j = j0 + lane;
        float pdp = 0.f;
        if (live && j >= lo && j <= i) {
            float dot = 0.f, dp = 0.f;
            const float* kr = sk + lane * (D + 1);
            const float* vr = sv + lane * (D + 1);
            for (int d = 0; d < D; ++d) {
                dot = fmaf(sq[d], kr[d], dot);
                dp = fmaf(sdo[d], vr[d], dp);
            }
            pdp = expf(dot * c - lse) * dp;
        }
        delta += warp_sum(pdp);
    }
    // walk 3: dq = c sum_j ds_j k_j; lanes then own columns d = lane, lane+32, ...
    constexpr int kMaxPerLane = kBwdMaxD / 32;
    float acc[kMaxPerLane];
#pragma unroll
    for (int x = 0; x < kMaxPerLane; ++x) acc[x] = 0.f;
    for (int j0 = blo; j0 <= last; j0 += 32) {
        __syncthreads();
        const int n = min(32, last - j0 + 1);
        bwd_stage(sk, kh, j0, n, D);
        bwd_stage(sv, vh, j0, n, D);
        __syncthreads();
        const int j = j0 + lane;
        float ds = 0.f;
        if (live && j >= lo && j <= i) {
            float dot = 0.f, dp = 0.f;
            const float* kr = sk + lane * (D + 1);
            const float* vr = sv + lane * (D + 1);
            for (int d = 0; d < D; ++d) {
                dot = fmaf(sq[d], kr[d], dot);
                dp = fmaf(sdo[d], vr[d], dp);
            }
            ds = expf(dot * c - lse) * (dp - delta);
        }
        sds[lane] = ds;
        __syncwarp();
#pragma unroll
        for (int x = 0; x < kMaxPerLane; ++x) {
            const int d = lane + 32 * x;
            if (d < D) {
                float a = acc[x];
                for (int t = 0; t < n; ++t) a = fmaf(sds[t], sk[t * (D + 1) + d], a);
                acc[x] = a;
            }
        }
        __syncwarp();
    }
    if (live) {
#pragma unroll
        for (int x = 0; x < kMaxPerLane; ++x) {
            const int d = lane + 32 * x;
            if (d < D) store_val(dq + r * D + d, acc[x] * c);
        }
        if (lane == 0) {
            stats[2 * r] = lse;
            stats[2 * r + 1] = delta;
        }
    }
}

template <typename TIn>
__global__ void __launch_bounds__(kBwdRows * 32)
    bwd_cols_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k, const TIn* __restrict__ v,
                    const TIn* __restrict__ dout, const float* __restrict__ stats, TIn* __restrict__ dk,
                    TIn* __restrict__ dv, int T, int D, int W, float c) {
    extern __shared__ float bsm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int blocks_per_head = (T + kBwdRows - 1) / kBwdRows;
    const int64_t bh = blockIdx.x / blocks_per_head;
    const int j0b = (int)(blockIdx.x - bh * blocks_per_head) * kBwdRows;
    const int j = j0b + warp;  // this warp's key row
    const bool live = j < T;
    const int jl = min(T - 1, j0b + kBwdRows - 1);
    const int qhi = min(T - 1, jl + W - 1);  // last query any key of the CTA is seen by
    float* sq = bsm;
    float* sdo = sq + 32 * (D + 1);
    float* sk = sdo + 32 * (D + 1) + warp * (2 * D + 64);
    float* sv = sk + D;
    float* sp = sv + D;
    float* sds = sp + 32;
    const TIn* qh = q + bh * (int64_t)T * D;
    const TIn* doh = dout + bh * (int64_t)T * D;
    const float* st = stats + 2 * bh * (int64_t)T;
    const int64_t r = bh * (int64_t)T + j;
    if (live)
        for (int d = lane; d < D; d += 32) {
            sk[d] = to_f32(k[r * D + d]);
            sv[d] = to_f32(v[r * D + d]);
        }
    const int hi = live ? min(T - 1, j + W - 1) : -1;  // last query that sees key j
    constexpr int kMaxPerLane = kBwdMaxD / 32;
    float ak[kMaxPerLane], av[kMaxPerLane];
#pragma unroll
    for (int x = 0; x < kMaxPerLane; ++x) ak[x] = av[x] = 0.f;
    for (int i0 = j0b; i0 <= qhi; i0 += 32) {
        __syncthreads();
        const int n = min(32, qhi - i0 + 1);
        bwd_stage(sq, qh, i0, n, D);
        bwd_stage(sdo, doh, i0, n, D);
        __syncthreads();
        const int i = i0 + lane;
        float p = 0.f, ds = 0.f;
        if (live && i >= j && i <= hi) {
            float dot = 0.f, dp = 0.f;
            const float* qr = sq + lane * (D + 1);
            const float* dr = sdo + lane * (D + 1);
            for (int d = 0; d < D; ++d) {
                dot = fmaf(qr[d], sk[d], dot);
                dp = fmaf(dr[d], sv[d], dp);
            }
            p = expf(dot * c - st[2 * i]);
            ds = p * (dp - st[2 * i + 1]);
        }
        sp[lane] = p;
        sds[lane] = ds;
        __syncwarp();
#pragma unroll
        for (int x = 0; x < kMaxPerLane; ++x) {
            const int d = lane + 32 * x;
            if (d < D) {
                float a = av[x], b = ak[x];
                for (int t = 0; t < n; ++t) {
                    a = fmaf(sp[t], sdo[t * (D + 1) + d], a);
                    b = fmaf(sds[t], sq[t * (D + 1) + d], b);
                }
                av[x] = a;
                ak[x] = b;
            }
        }
        __syncwarp();
    }
    if (live) {
#pragma unroll
        for (int x = 0; x < kMaxPerLane; ++x) {
            const int d = lane + 32 * x;
            if (d < D) {
                store_val(dk + r * D + d, ak[x] * c);
                store_val(dv + r * D + d, av[x]);
            }
        }
    }
}

}  // namespace swa
