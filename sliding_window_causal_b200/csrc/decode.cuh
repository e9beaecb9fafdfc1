// decode.cuh: one query per stream against a W-slot rolling KV buffer, bf16, D = 64/128.
//
// The buffer of stream b keeps position p in slot p mod W; at position P the query sees
// positions max(0, P-W+1) .. P, which sit in slots 0 .. n-1 with n = min(P+1, W)
// ("25. Sliding-Window Causal Attention for Streaming Inference", Problem: a KV cache
// bounded to the window). The softmax does not depend on the order of the keys, so the
// slots are visited in slot order. Slots n .. W-1 are never read.
//
// Grid (B*H, S): CTA (bh, s) streams slots [s*chunk, min((s+1)*chunk, n)) of K and V
// with 16-byte non-coherent loads (D/8 lanes per slot, several slots in flight per lane),
// scores in fp32 with q pre-scaled by log2(e)/sqrt(D), and keeps an online softmax state
// (max m, sum l, unnormalised acc[D]) per warp. The four warps merge in shared memory.
// With S > 1 each CTA writes (m, l, acc) to the workspace, and the last CTA of a stream
// to finish (atomic ticket) merges the S states in split order, which makes the result
// independent of the order in which CTAs finish:
//   m* = max_s m_s,  out = sum_s 2^(m_s - m*) acc_s / sum_s 2^(m_s - m*) l_s.
// That CTA also resets the stream's ticket counter to zero for the next call.
#pragma once
#include <cuda_bf16.h>
#include <math.h>

#include "ptx.cuh"

namespace swa {

constexpr int kDecodeWarps = 4;
constexpr int kDecodeUnroll = 4;
constexpr int kStatusInvalid = 1;  // SWA_ERR_INVALID_ARG

template <int D>
struct DecodeCfg {
    static_assert(D == 64 || D == 128, "head dim 64 or 128");
    static constexpr int kLanesPerRow = D / 8;
    static constexpr int kRowsPerStep = 32 / kLanesPerRow;
    static constexpr int kRowsPerBatch = kDecodeWarps * kRowsPerStep * kDecodeUnroll;
};

__device__ __forceinline__ uint4 ld_stream_16(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
    f[0] = __uint_as_float(u.x << 16); f[1] = __uint_as_float(u.x & 0xFFFF0000u);
    f[2] = __uint_as_float(u.y << 16); f[3] = __uint_as_float(u.y & 0xFFFF0000u);
    f[4] = __uint_as_float(u.z << 16); f[5] = __uint_as_float(u.z & 0xFFFF0000u);
    f[6] = __uint_as_float(u.w << 16); f[7] = __uint_as_float(u.w & 0xFFFF0000u);
}

template <int D>
__global__ void __launch_bounds__(kDecodeWarps * 32)
    decode_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kring,
                  const __nv_bfloat16* __restrict__ vring, const int64_t* __restrict__ pos,
                  __nv_bfloat16* __restrict__ out, int H, int W, int chunk, int S, float scale_log2,
                  float* __restrict__ part, int* __restrict__ counters, int* status) {
    using C = DecodeCfg<D>;
    constexpr int LPR = C::kLanesPerRow, RPS = C::kRowsPerStep, U = kDecodeUnroll;
    __shared__ float sm_m[kDecodeWarps], sm_l[kDecodeWarps];
    __shared__ float sm_acc[kDecodeWarps][D];
    __shared__ int sm_last;

    const int bh = blockIdx.x;
    const int s = blockIdx.y;
    const int b = bh / H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane / LPR;   // which slot of a load step this lane serves
    const int cl = lane % LPR;  // which 8 columns of the head dimension

    const int64_t P = pos[b];
    const bool bad = P < 0;
    if (bad && s == 0 && tid == 0) atomicCAS(status, 0, kStatusInvalid);
    const int n = bad ? 0 : (int)(P + 1 < (int64_t)W ? P + 1 : (int64_t)W);
    const int r0 = s * chunk;
    const int r1 = r0 + chunk < n ? r0 + chunk : n;

    float qf[8];
    {
        const uint4 qu = *reinterpret_cast<const uint4*>(q + (int64_t)bh * D + cl * 8);
        bf16x8_to_f32(qu, qf);
#pragma unroll
        for (int e = 0; e < 8; ++e) qf[e] *= scale_log2;
    }
    const __nv_bfloat16* kb = kring + (int64_t)bh * W * D + cl * 8;
    const __nv_bfloat16* vb = vring + (int64_t)bh * W * D + cl * 8;

    float m = -INFINITY, l = 0.f;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;

    for (int base = r0 + warp * RPS * U; base < r1; base += C::kRowsPerBatch) {
        uint4 kr[U], vr[U];
        bool valid[U];
#pragma unroll
        for (int t = 0; t < U; ++t) {
            const int row = base + t * RPS + g;
            valid[t] = row < r1;
            if (valid[t]) {
                kr[t] = ld_stream_16(kb + (int64_t)row * D);
                vr[t] = ld_stream_16(vb + (int64_t)row * D);
            } else {
                kr[t] = make_uint4(0, 0, 0, 0);
                vr[t] = make_uint4(0, 0, 0, 0);
            }
        }
        float sc[U];
#pragma unroll
        for (int t = 0; t < U; ++t) {
            float kf[8];
            bf16x8_to_f32(kr[t], kf);
            float dot = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) dot = fmaf(qf[e], kf[e], dot);
            sc[t] = dot;
        }
#pragma unroll
        for (int o = LPR / 2; o > 0; o >>= 1) {
#pragma unroll
            for (int t = 0; t < U; ++t) sc[t] += __shfl_xor_sync(0xffffffffu, sc[t], o);
        }
        float mb = -INFINITY;
#pragma unroll
        for (int t = 0; t < U; ++t) {
            if (!valid[t]) sc[t] = -INFINITY;
            mb = fmaxf(mb, sc[t]);
        }
#pragma unroll
        for (int o = LPR; o < 32; o <<= 1) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, o));
        // mb is finite: slot `base` (t = 0, g = 0) is in range
        const float m_new = fmaxf(m, mb);
        const float alpha = ptx::ex2(m - m_new);
        l *= alpha;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] *= alpha;
#pragma unroll
        for (int t = 0; t < U; ++t) {
            const float p = ptx::ex2(sc[t] - m_new);
            float vf[8];
            bf16x8_to_f32(vr[t], vf);
            l += p;
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = fmaf(p, vf[e], acc[e]);
        }
        m = m_new;
    }
    // merge the slot groups of this warp (same m, so plain sums)
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1) {
        l += __shfl_xor_sync(0xffffffffu, l, o);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
    }
    if (g == 0) {
#pragma unroll
        for (int e = 0; e < 8; ++e) sm_acc[warp][cl * 8 + e] = acc[e];
    }
    if (lane == 0) {
        sm_m[warp] = m;
        sm_l[warp] = l;
    }
    __syncthreads();

    // merge the warps: thread c owns column c
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecodeWarps; ++w) M = fmaxf(M, sm_m[w]);
    float L = 0.f, A = 0.f;
    if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < kDecodeWarps; ++w) {
            const float f = ptx::ex2(sm_m[w] - M);
            L = fmaf(sm_l[w], f, L);
            if (tid < D) A = fmaf(sm_acc[w][tid], f, A);
        }
    }
    __nv_bfloat16* orow = out + (int64_t)bh * D;
    if (S == 1) {
        if (tid < D) orow[tid] = __float2bfloat16_rn(L > 0.f ? A / L : 0.f);
        return;
    }
    float* mine = part + ((int64_t)bh * S + s) * (D + 2);
    if (tid < D) mine[2 + tid] = A;
    if (tid == 0) {
        mine[0] = M;
        mine[1] = L;
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const int ticket = atomicAdd(counters + bh, 1);
        sm_last = (ticket == S - 1);
    }
    __syncthreads();
    if (!sm_last) return;
    __threadfence();
    const float* all = part + (int64_t)bh * S * (D + 2);
    float Ms = -INFINITY;
    for (int t = 0; t < S; ++t) Ms = fmaxf(Ms, __ldcg(all + (int64_t)t * (D + 2)));
    float Ls = 0.f, As = 0.f;
    if (Ms != -INFINITY) {
        for (int t = 0; t < S; ++t) {
            const float* pt = all + (int64_t)t * (D + 2);
            const float f = ptx::ex2(__ldcg(pt) - Ms);
            Ls = fmaf(__ldcg(pt + 1), f, Ls);
            if (tid < D) As = fmaf(__ldcg(pt + 2 + tid), f, As);
        }
    }
    if (tid < D) orow[tid] = __float2bfloat16_rn(Ls > 0.f ? As / Ls : 0.f);
    if (tid == 0) counters[bh] = 0;
}

}  // namespace swa
