// backward_tc.cuh: gradients of the bf16 sliding-window prefill on the sm_100a tensor
// cores (D = 64 or 128).
//
// The gradients ("NNX Sliding-Window Attention", Mask before softmax: well defined for
// finite allowed scores), with s_ij = q_i . k_j, c the scale, P_ij = exp(c s_ij - lse_i)
// the forward weights and delta_i = dout_i . out_i:
//   dV = P^T dO,   dS = P o (dO V^T - delta),   dK = c dS^T Q,   dQ = c dS K
// over the band pairs only. Three kernels, no atomics (deterministic):
//   bwd_stats_kernel  delta_i from dout and out, and lse_i (from the forward) in log2
//                     units, into a [B*H, Tpad] layout padded to whole 128-row tiles
//                     (padding rows get lse = +inf, delta = 0, so they weigh nothing).
//   bwd_tc_kernel<D, true>: one CTA per (b, h, 128-key tile): K and V stay in shared memory;
//                     for every query tile that meets the band, TMA brings Q, dO and the
//                     tile's (lse, delta); S^T = K Q^T and dP^T = V dO^T go to TMEM; eight
//                     warps (two threads per key row, 64 columns each) turn them into bf16 P^T and
//                     dS^T over the dP^T columns; then dV += P^T dO and dK += dS^T Q
//                     accumulate in TMEM (TS form: A from TMEM, B from shared memory). The
//                     next tile's S^T is computed while the element-wise warps work: they
//                     read their scores into registers first and release the S columns. They
//                     then take the tile's columns in two halves of 64; the gradient products
//                     of a half, and the next tile's dP^T for that half, run on the tensor
//                     cores while the warps work on the other half.
//   bwd_tc_kernel<D, false>: one CTA per (b, h, 128-query tile): Q and dO stay; for every key
//                     tile of the band S = Q K^T and dP = dO V^T, then dS (bf16, in TMEM)
//                     and dQ += dS K.
// Work per band pair: seven 128x128xD products (the score and dP products are formed in
// both kernels, so that neither needs atomics), against five in the useful-FLOP count.
// Every mbarrier wait is bounded as in the forward kernels.
#pragma once
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "plan.h"
#include "prefill_pp.cuh"
#include "ptx.cuh"
#include "umma.h"

namespace swa {

// mbar_wait for a whole warp: true only if every lane's wait completed, so that the warp
// stays converged (its elected-lane MMAs need the full warp).
__device__ __forceinline__ bool bwd_wait_warp(uint64_t* bar, uint32_t parity, uint64_t limit_ns, volatile int* abort) {
    return __all_sync(0xffffffffu, ptx::mbar_wait(bar, parity, limit_ns, abort));
}

constexpr int kBwdTcThreads = 320;  // warp 0 producer, warp 1 MMA, warps 2..9 element-wise
constexpr int kBwdTcEw = 256;       // element-wise threads: two warps per row quarter

template <int D, bool KV>
struct BwdTcCfg {
    static_assert(D == 64 || D == 128, "head dim 64 or 128");
    static constexpr int kBoxBytes = 128 * 128;
    static constexpr int kTileBytes = 128 * D * 2;
    // the key-tile kernel keeps K and V in shared memory; the query-tile kernel keeps Q and
    // dO in TMEM and gives their room to the ring of streamed tiles (Q/dO or K/V)
    static constexpr int kStages = KV ? (D == 128 ? 4 : 8) : (D == 128 ? 6 : 10);
    static constexpr int kFixOff = 0;
    static constexpr int kRingOff = KV ? 2 * kTileBytes : 0;
    static constexpr int kStatStages = 2;
    static constexpr int kStatBytes = 2 * 128 * 4;    // nlse2[128], delta[128]
    static constexpr int kStatOff = kRingOff + kStages * kTileBytes;
    static constexpr int kBarOff = kStatOff + kStatStages * kStatBytes;
    // fix_full, ring_full[S], ring_empty[S], stat_full[2], stat_empty[2], s_full, s_read,
    // dp_full[2], p_full[2], o_final, drain
    static constexpr int kNumBars = 1 + 2 * kStages + 4 + 8;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kSmemBytes = kMiscOff + 16 + 1024;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColS = 0, kColDP = 128, kColA = 256, kColB = 384;
    // the query-tile kernel's resident Q and dO rows (A operands of S and dP)
    static constexpr uint32_t kColQ = 384, kColDO = 448;
};

// delta_i = sum_d dout_i[d] out_i[d] (fp32) and nlse2_i = -lse_i * log2(e), one warp per row
// (negated, so that the exponent s*c2 - lse*log2(e) is one fused multiply-add, s*c2 + nlse2).
__global__ void __launch_bounds__(256)
    bwd_stats_kernel(const __nv_bfloat16* __restrict__ dout, const __nv_bfloat16* __restrict__ out,
                     const float* __restrict__ lse, float* __restrict__ nlse2, float* __restrict__ delta,
                     int64_t BH, int T, int Tpad, int D) {
    const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= BH * Tpad) return;
    const int64_t bh = r / Tpad;
    const int i = (int)(r - bh * Tpad);
    if (i >= T) {
        if (lane == 0) {
            nlse2[r] = -INFINITY;  // padding rows: P = 0
            delta[r] = 0.f;
        }
        return;
    }
    const int64_t src = (bh * T + i) * D;
    float acc = 0.f;
    // D/32 consecutive elements a lane (D is 64 or 128, rows 16-byte aligned): one 4- or
    // 8-byte load of each tensor, so a warp reads each row in one coalesced pass
    if (D == 128) {
        const uint2 a = *reinterpret_cast<const uint2*>(dout + src + 4 * lane);
        const uint2 o = *reinterpret_cast<const uint2*>(out + src + 4 * lane);
        acc = ptx::bf16lo_f32(a.x) * ptx::bf16lo_f32(o.x);
        acc = fmaf(ptx::bf16hi_f32(a.x), ptx::bf16hi_f32(o.x), acc);
        acc = fmaf(ptx::bf16lo_f32(a.y), ptx::bf16lo_f32(o.y), acc);
        acc = fmaf(ptx::bf16hi_f32(a.y), ptx::bf16hi_f32(o.y), acc);
    } else {
        const uint32_t a = *reinterpret_cast<const uint32_t*>(dout + src + 2 * lane);
        const uint32_t o = *reinterpret_cast<const uint32_t*>(out + src + 2 * lane);
        acc = ptx::bf16lo_f32(a) * ptx::bf16lo_f32(o);
        acc = fmaf(ptx::bf16hi_f32(a), ptx::bf16hi_f32(o), acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
        delta[r] = acc;
        nlse2[r] = lse[bh * T + i] * -1.4426950408889634f;
    }
}

// One chunk of 32 columns of one TMEM row, already in registers: scores s (fp32, raw q.k)
// and dp, to bf16 P and dS = P (dp - delta), with P = exp2(s*c2 + nlse2) where the column
// is valid, else 0 (nlse2 = -lse in log2 units). COLSTATS: each column has its own nlse2
// and delta (32 values each at col_nlse, col_delta in shared memory, 16-byte aligned);
// else the row's row_nlse, row_delta apply to every column. On EDGE tiles only columns
// cmin..cmax are valid (band membership of one row is an interval of columns); other tiles
// are valid throughout. dS goes to columns dpcol .. dpcol+15 and, when STORE_P, P to
// dpcol+16 .. dpcol+31 (both over dp values already read), leaving the S columns free for
// the next tile's scores. Pairs of columns go through the packed f32x2 arithmetic.
template <bool STORE_P, bool EDGE, bool COLSTATS>
__device__ __forceinline__ void bwd_chunk(const uint32_t (&s)[32], const uint32_t (&dp)[32], uint32_t dpcol,
                                          float c2, const float* col_nlse, const float* col_delta,
                                          float row_nlse, float row_delta, int cmin, int cmax) {
    uint32_t ph[16], dh[16];
    const ptx::f32x2 cc = {c2, c2};
#pragma unroll
    for (int t2 = 0; t2 < 16; t2 += 2) {
        float4 nl4, dl4;
        if (COLSTATS) {
            nl4 = *reinterpret_cast<const float4*>(col_nlse + 2 * t2);
            dl4 = *reinterpret_cast<const float4*>(col_delta + 2 * t2);
        } else {
            nl4 = make_float4(row_nlse, row_nlse, row_nlse, row_nlse);
            dl4 = make_float4(row_delta, row_delta, row_delta, row_delta);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int t = t2 + u;
            const ptx::f32x2 nl = u ? ptx::f32x2{nl4.z, nl4.w} : ptx::f32x2{nl4.x, nl4.y};
            const ptx::f32x2 dl = u ? ptx::f32x2{dl4.z, dl4.w} : ptx::f32x2{dl4.x, dl4.y};
            const ptx::f32x2 z = ptx::fma2({__uint_as_float(s[2 * t]), __uint_as_float(s[2 * t + 1])}, cc, nl);
            ptx::f32x2 p = {ptx::ex2(z.x), ptx::ex2(z.y)};
            if (EDGE) {
                if (!(2 * t >= cmin && 2 * t <= cmax)) p.x = 0.f;
                if (!(2 * t + 1 >= cmin && 2 * t + 1 <= cmax)) p.y = 0.f;
            }
            const ptx::f32x2 ds =
                ptx::mul2(p, ptx::sub2({__uint_as_float(dp[2 * t]), __uint_as_float(dp[2 * t + 1])}, dl));
            ph[t] = ptx::pack_bf16x2(p.x, p.y);
            dh[t] = ptx::pack_bf16x2(ds.x, ds.y);
        }
    }
    ptx::tmem_st16(dpcol, dh);
    if (STORE_P) ptx::tmem_st16(dpcol + 16, ph);
}

// Store one 128-column TMEM accumulator row (D fp32 values from column col) times a, as
// bf16, to dst (a row of D elements), 16 bytes at a time.
template <int D>
__device__ __forceinline__ void bwd_store_row(uint32_t col, float a, __nv_bfloat16* dst, bool live) {
#pragma unroll 1
    for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        ptx::tmem_ld32(col + cc * 32, o);
        ptx::tmem_ld_wait();
        ptx::reg_fence(o);
        if (live) {
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                uint4 val;
                val.x = ptx::pack_bf16x2(__uint_as_float(o[8 * t + 0]) * a, __uint_as_float(o[8 * t + 1]) * a);
                val.y = ptx::pack_bf16x2(__uint_as_float(o[8 * t + 2]) * a, __uint_as_float(o[8 * t + 3]) * a);
                val.z = ptx::pack_bf16x2(__uint_as_float(o[8 * t + 4]) * a, __uint_as_float(o[8 * t + 5]) * a);
                val.w = ptx::pack_bf16x2(__uint_as_float(o[8 * t + 6]) * a, __uint_as_float(o[8 * t + 7]) * a);
                *reinterpret_cast<uint4*>(dst + cc * 32 + t * 8) = val;
            }
        }
    }
}

// KV = true: bwd_kv_kernel (resident K, V in shared memory; streamed Q, dO; dK, dV out).
// KV = false: bwd_q_kernel (resident Q, dO in TMEM, read from rq, rdo; streamed K, V; dQ out).
// Maps are 4-D {D, T, H, B} of contiguous [B,H,T,D] tensors. nlse2/delta: [B*H, Tpad].
template <int D, bool KV>
__global__ void __launch_bounds__(kBwdTcThreads, 1)
    bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const __nv_bfloat16* __restrict__ rq, const __nv_bfloat16* __restrict__ rdo,
                  const float* __restrict__ nlse2, const float* __restrict__ delta, __nv_bfloat16* __restrict__ g1,
                  __nv_bfloat16* __restrict__ g2, int H, int T, int Tpad, int W, int n_t, float c, float c2,
                  uint64_t wait_limit_ns, int* status) {
    using Cf = BwdTcCfg<D, KV>;
    constexpr int NS = Cf::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cf::kBarOff);
    uint64_t* fix_full = bars;
    uint64_t* ring_full = bars + 1;  // [NS]
    uint64_t* ring_empty = ring_full + NS;
    uint64_t* stat_full = ring_empty + NS;  // [2]
    uint64_t* stat_empty = stat_full + 2;   // [2]
    uint64_t* s_full = stat_empty + 2;
    uint64_t* s_read = s_full + 1;   // the element-wise warps have read a tile's S
    uint64_t* dp_full = s_read + 1;  // [2]: dP of one half of the tile's columns
    uint64_t* p_full = dp_full + 2;  // [2]: P and dS of one half of the tile's columns
    uint64_t* o_final = p_full + 2;
    uint64_t* drain = o_final + 1;
    const float* st_smem = reinterpret_cast<const float*>(smem + Cf::kStatOff);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cf::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cf::kMiscOff + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int bh, xt;  // the resident tile: key tile (KV) or query tile
    bwd_cta_tile<int>((int)blockIdx.x, (int)gridDim.x / n_t, n_t, W, KV, &bh, &xt);
    // The query-tile kernel follows this one as a programmatic dependent launch: it reads
    // nothing this kernel writes, so its CTAs may take the SMs this grid's last CTAs leave.
    if (KV) ptx::launch_dependents();
    const int b = bh / H, h = bh - b * H;
    // the streamed tiles that meet the band: query tiles xt .. (KV), or key tiles (Q)
    int lo, hi;
    if (KV) {
        lo = xt;
        hi = min(n_t - 1, (128 * xt + 127 + W - 1) / 128);
    } else {
        int64_t f, l;
        kv_tile_range(T, W, 128, 128, xt, &f, &l);
        lo = (int)f;
        hi = (int)l;
    }
    auto cls = [&](int yt) { return KV ? tile_class(T, W, 128, 128, yt, xt) : tile_class(T, W, 128, 128, xt, yt); };

    if (threadIdx.x == 0) {
        ptx::mbar_init(fix_full, KV ? 1 : kBwdTcEw);
        for (int s = 0; s < NS; ++s) {
            ptx::mbar_init(ring_full + s, 1);
            ptx::mbar_init(ring_empty + s, 1);
        }
        for (int x = 0; x < 2; ++x) {
            ptx::mbar_init(stat_full + x, 1);
            ptx::mbar_init(stat_empty + x, kBwdTcEw);
        }
        ptx::mbar_init(s_full, 1);
        ptx::mbar_init(s_read, kBwdTcEw);
        for (int x = 0; x < 2; ++x) {
            ptx::mbar_init(dp_full + x, 1);
            ptx::mbar_init(p_full + x, kBwdTcEw);
        }
        ptx::mbar_init(o_final, 1);
        ptx::mbar_init(drain, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tmap(&tm_q);
        ptx::prefetch_tmap(&tm_k);
        ptx::prefetch_tmap(&tm_v);
        ptx::prefetch_tmap(&tm_do);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, Cf::kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    uint32_t loads = 0, stat_loads = 0;
    bool fix_issued = false;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------------------- producer
            bool ok = true;
            const CUtensorMap* fa = KV ? &tm_k : &tm_q;   // resident operands
            const CUtensorMap* fb = KV ? &tm_v : &tm_do;
            const CUtensorMap* sa = KV ? &tm_q : &tm_k;   // streamed operands
            const CUtensorMap* sb = KV ? &tm_do : &tm_v;
            if (KV) {
                ptx::mbar_arrive_expect_tx(fix_full, 2 * Cf::kTileBytes);
                for (int x = 0; x < 2; ++x)
                    for (int cc = 0; cc < D / 64; ++cc)
                        ptx::tma_load_4d(smem + Cf::kFixOff + x * Cf::kTileBytes + cc * Cf::kBoxBytes, x ? fb : fa,
                                         fix_full, cc * 64, 128 * xt, h, b);
                fix_issued = true;
            }
            for (int yt = lo; yt <= hi && ok; ++yt) {
                if (cls(yt) == 0) continue;
                for (int x = 0; x < 2 && ok; ++x) {
                    const uint32_t st = loads % NS;
                    if (loads >= (uint32_t)NS)
                        ok = ptx::mbar_wait(ring_empty + st, ((loads / NS) - 1) & 1, wait_limit_ns, abort_flag);
                    if (!ok) break;
                    uint8_t* dst = smem + Cf::kRingOff + st * Cf::kTileBytes;
                    ptx::mbar_arrive_expect_tx(ring_full + st, Cf::kTileBytes);
                    for (int cc = 0; cc < D / 64; ++cc)
                        ptx::tma_load_4d(dst + cc * Cf::kBoxBytes, x ? sb : sa, ring_full + st, cc * 64, 128 * yt, h, b);
                    ++loads;
                }
                if (KV && ok) {
                    // the query tile's nlse2 and delta (512 bytes each, contiguous in [B*H, Tpad])
                    const uint32_t ss = stat_loads % 2;
                    if (stat_loads >= 2)
                        ok = ptx::mbar_wait(stat_empty + ss, ((stat_loads / 2) - 1) & 1, wait_limit_ns, abort_flag);
                    if (!ok) break;
                    uint8_t* dst = smem + Cf::kStatOff + ss * Cf::kStatBytes;
                    ptx::mbar_arrive_expect_tx(stat_full + ss, Cf::kStatBytes);
                    const int64_t off = (int64_t)bh * Tpad + 128 * yt;
                    ptx::bulk_load(dst, nlse2 + off, 512, stat_full + ss);
                    ptx::bulk_load(dst + 512, delta + off, 512, stat_full + ss);
                    ++stat_loads;
                }
            }
            if (!ok) {
                atomicCAS(status, 0, 5);
                *abort_flag = 1;
            }
        }
    } else if (warp == 1) {
        {
            // ---------------------------------------------------------------- MMA issuer
            // (the whole warp runs this loop; its waits are warp-uniform, one lane issues).
            // A tile's 128 streamed columns are handled in two halves of 64: the element-wise
            // warps turn half h of dP into P and dS, the gradient products of that half follow
            // at once, and so does the next tile's dP for the same half (over the P and dS
            // those products have just read), while the warps work on the other half.
            const uint32_t idesc_s = umma::idesc_bf16_f32(128, 128, 0);
            const uint32_t idesc_dp = umma::idesc_bf16_f32(128, 64, 0);
            const uint32_t idesc_o = umma::idesc_bf16_f32(128, D, 1);
            const uint64_t desc_hi = umma::smem_desc(0, 0, 1024) & 0xFFFFFFFF00000000ull;
            const uint32_t lo_k = (uint32_t)umma::smem_desc(0, 16, 1024);
            const uint32_t lo_mn = (uint32_t)umma::smem_desc(0, Cf::kBoxBytes, 1024);
            const uint32_t fa_lo = ptx::smem_u32(smem + Cf::kFixOff) >> 4;
            const uint32_t fb_lo = ptx::smem_u32(smem + Cf::kFixOff + Cf::kTileBytes) >> 4;
            const uint32_t ring_lo = ptx::smem_u32(smem + Cf::kRingOff) >> 4;
            constexpr uint32_t kStageLo = Cf::kTileBytes >> 4;
            bool ok = bwd_wait_warp(fix_full, 0, wait_limit_ns, abort_flag);
            auto next_visited = [&](int y) {  // the first visited tile after y (> hi if none)
                for (++y; y <= hi && cls(y) == 0; ++y) {
                }
                return y;
            };
            auto wait_stage = [&](uint32_t idx) {
                return bwd_wait_warp(ring_full + idx % NS, (idx / NS) & 1, wait_limit_ns, abort_flag);
            };
            // KV: S^T = K Q^T, dP^T = V dO^T.   Q: S = Q K^T, dP = dO V^T.
            // Tile j's streamed operands sit in stages L % NS (a: Q or K) and (L+1) % NS (b: dO or V).
            auto issue_s = [&](uint32_t Lj) {
                const uint32_t a_lo = ring_lo + (Lj % NS) * kStageLo;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * Cf::kBoxBytes + (kk & 3) * 32) >> 4;
                    if (KV)
                        ptx::mma_ss_one(tmem + Cf::kColS, desc_hi | ((fa_lo + off) | lo_k),
                                        desc_hi | ((a_lo + off) | lo_k), idesc_s, kk > 0 ? 1u : 0u);
                    else
                        ptx::mma_ts_one(tmem + Cf::kColS, tmem + Cf::kColQ + 8 * kk, desc_hi | ((a_lo + off) | lo_k),
                                        idesc_s, kk > 0 ? 1u : 0u);
                }
                ptx::tc_commit_one(s_full);
            };
            // dP of the streamed rows 64 hf .. 64 hf + 63 into TMEM columns 64 hf .. of the dP buffer
            auto issue_dp = [&](uint32_t Lj, uint32_t hf) {
                const uint32_t b_lo = ring_lo + ((Lj + 1) % NS) * kStageLo + hf * (64 * 128 >> 4);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * Cf::kBoxBytes + (kk & 3) * 32) >> 4;
                    if (KV)
                        ptx::mma_ss_one(tmem + Cf::kColDP + 64 * hf, desc_hi | ((fb_lo + off) | lo_k),
                                        desc_hi | ((b_lo + off) | lo_k), idesc_dp, kk > 0 ? 1u : 0u);
                    else
                        ptx::mma_ts_one(tmem + Cf::kColDP + 64 * hf, tmem + Cf::kColDO + 8 * kk,
                                        desc_hi | ((b_lo + off) | lo_k), idesc_dp, kk > 0 ? 1u : 0u);
                }
                ptx::tc_commit_one(dp_full + hf);
            };
            uint32_t L = 0;
            int j = 0;  // visited tiles
            int yt = next_visited(lo - 1);
            if (ok) ok = wait_stage(0) && wait_stage(1);
            if (ok) {
                ptx::tc_fence_after();
                issue_s(0);
                issue_dp(0, 0);
                issue_dp(0, 1);
            }
            while (ok) {
                const int ynext = next_visited(yt);
                // the next tile's scores as soon as this tile's S is in registers
                ok = bwd_wait_warp(s_read, j & 1, wait_limit_ns, abort_flag);
                if (ok && ynext <= hi) {
                    ok = wait_stage(L + 2);
                    if (ok) {
                        ptx::tc_fence_after();
                        issue_s(L + 2);
                    }
                }
                const uint32_t sta = L % NS, stb = (L + 1) % NS;
                const uint32_t a_lo = ring_lo + sta * kStageLo, b_lo = ring_lo + stb * kStageLo;
                for (uint32_t hf = 0; hf < 2 && ok; ++hf) {
                    ok = bwd_wait_warp(p_full + hf, j & 1, wait_limit_ns, abort_flag);
                    if (!ok) break;
                    ptx::tc_fence_after();
                    if (KV) {
                        // dV += P^T dO (A = P^T, the +16 half of each dP chunk; B = dO);
                        // dK += dS^T Q (A = dS^T, the first half; B = Q)
#pragma unroll
                        for (int k4 = 0; k4 < 4; ++k4) {
                            const int kk = 4 * hf + k4;
                            ptx::mma_ts_one(tmem + Cf::kColA, tmem + Cf::kColDP + pp_pcol(kk) + 16,
                                        desc_hi | ((b_lo + kk * (2048 >> 4)) | lo_mn), idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
                        }
#pragma unroll
                        for (int k4 = 0; k4 < 4; ++k4) {
                            const int kk = 4 * hf + k4;
                            ptx::mma_ts_one(tmem + Cf::kColB, tmem + Cf::kColDP + pp_pcol(kk),
                                        desc_hi | ((a_lo + kk * (2048 >> 4)) | lo_mn), idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
                        }
                    } else {
                        // dQ += dS K (A = dS in the dP columns, B = K)
#pragma unroll
                        for (int k4 = 0; k4 < 4; ++k4) {
                            const int kk = 4 * hf + k4;
                            ptx::mma_ts_one(tmem + Cf::kColA, tmem + Cf::kColDP + pp_pcol(kk),
                                        desc_hi | ((a_lo + kk * (2048 >> 4)) | lo_mn), idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
                        }
                    }
                    if (hf == 1) {
                        ptx::tc_commit_one(ring_empty + sta);
                        ptx::tc_commit_one(ring_empty + stb);
                    }
                    // the next tile's dP for this half, after the products above read its P and dS
                    if (ynext <= hi) {
                        ok = wait_stage(L + 3);
                        if (!ok) break;
                        ptx::tc_fence_after();
                        issue_dp(L + 2, hf);
                    }
                }
                if (!ok || ynext > hi) break;
                L += 2;
                ++j;
                yt = ynext;
            }
            if (ok) ptx::tc_commit_one(o_final);
            if (!ok && lane == 0) {
                atomicCAS(status, 0, 5);
                *abort_flag = 1;
            }
        }
    } else {
        // -------------------------------------------------------------------- element-wise
        // warps 2..9: warp w serves TMEM lanes 32*(w%4).. and column chunks half, 2+half
        const int quarter = warp & 3;
        const int half = (warp - 2) >> 2;
        const int r = quarter * 32 + lane;  // the TMEM lane = this thread's resident row
        const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
        const int xr = 128 * xt + r;         // key index (KV) or query index (Q)
        float my_nlse2 = 0.f, my_delta = 0.f;
        if (!KV) {
            my_nlse2 = nlse2[(int64_t)bh * Tpad + xr];  // -inf on padding rows: P = 0
            my_delta = delta[(int64_t)bh * Tpad + xr];
            // this thread's half of its rows of q and dout (zero past T) into TMEM, where
            // column c holds elements 2c and 2c+1: the A operands of S and dP
            constexpr int HE = D / 2;
            const bool live = xr < T;
            const int64_t src = ((int64_t)bh * T + (live ? xr : 0)) * D + HE * half;
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const uint4* p4 = reinterpret_cast<const uint4*>((x ? rdo : rq) + src);
                uint32_t w[HE / 2];
#pragma unroll
                for (int t = 0; t < HE / 8; ++t) {
                    const uint4 u = live ? p4[t] : make_uint4(0u, 0u, 0u, 0u);
                    w[4 * t] = u.x;
                    w[4 * t + 1] = u.y;
                    w[4 * t + 2] = u.z;
                    w[4 * t + 3] = u.w;
                }
                const uint32_t col = tl + (x ? Cf::kColDO : Cf::kColQ) + (HE / 2) * half;
                if constexpr (D == 128) ptx::tmem_st32(col, w);
                else ptx::tmem_st16(col, w);
            }
            ptx::tmem_st_wait();
            ptx::tc_fence_before();
            ptx::mbar_arrive(fix_full);
        }
        bool ok = true;
        int j = 0;
        for (int yt = lo; yt <= hi && ok; ++yt) {
            const int k = cls(yt);
            if (k == 0) continue;
            bool w = ptx::mbar_wait(s_full, j & 1, wait_limit_ns, abort_flag);
            const float* sts = st_smem + (j & 1) * 256;
            if (KV && w) w = ptx::mbar_wait(stat_full + (j & 1), (j >> 1) & 1, wait_limit_ns, abort_flag);
            if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
            ptx::tc_fence_after();
            const bool edge = k != 2;
            // valid columns of this row in the tile, as an interval of tile columns
            int clo, chi;
            if (KV) {  // row = key xr, columns = queries: xr <= i <= min(xr + W - 1, T - 1)
                clo = xr - 128 * yt;
                chi = (xr < T ? min(xr + W - 1, T - 1) : -1) - 128 * yt;
            } else {   // row = query xr, columns = keys: max(0, xr - W + 1) <= j <= min(xr, T - 1)
                clo = max(0, xr - W + 1) - 128 * yt;
                chi = (xr < T ? xr : -1) - 128 * yt;
                if (xr >= T) clo = chi + 1;
            }
            if (KV && xr >= T) clo = chi + 1;
            // the scores first, so that the S columns can take the next tile's scores; this
            // warp's chunks are half (columns 0..63) and 2 + half (columns 64..127)
            uint32_t sv[2][32];
#pragma unroll
            for (int x = 0; x < 2; ++x) ptx::tmem_ld32(tl + Cf::kColS + 32 * (2 * x + half), sv[x]);
            ptx::tmem_ld_wait();
#pragma unroll
            for (int x = 0; x < 2; ++x) ptx::reg_fence(sv[x]);
            ptx::tc_fence_before();
            ptx::mbar_arrive(s_read);
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const int cc = 2 * x + half;
                if (!__all_sync(0xffffffffu, ptx::mbar_wait(dp_full + x, j & 1, wait_limit_ns, abort_flag))) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t dc = tl + Cf::kColDP + 32 * cc;
                uint32_t dpv[32];
                ptx::tmem_ld32(dc, dpv);
                ptx::tmem_ld_wait();
                ptx::reg_fence(dpv);
                const int cmin = clo - 32 * cc, cmax = chi - 32 * cc;
                if (KV) {
                    const float* sl = sts + 32 * cc;  // the columns' nlse2, then (at +128) their delta
                    if (edge) bwd_chunk<true, true, true>(sv[x], dpv, dc, c2, sl, sl + 128, 0.f, 0.f, cmin, cmax);
                    else bwd_chunk<true, false, true>(sv[x], dpv, dc, c2, sl, sl + 128, 0.f, 0.f, cmin, cmax);
                } else {
                    if (edge) bwd_chunk<false, true, false>(sv[x], dpv, dc, c2, nullptr, nullptr, my_nlse2, my_delta, cmin, cmax);
                    else bwd_chunk<false, false, false>(sv[x], dpv, dc, c2, nullptr, nullptr, my_nlse2, my_delta, cmin, cmax);
                }
                ptx::tmem_st_wait();
                ptx::tc_fence_before();
                ptx::mbar_arrive(p_full + x);
            }
            if (!ok) break;
            if (KV) ptx::mbar_arrive(stat_empty + (j & 1));
            ++j;
        }
        if (ok) {
            const bool w = ptx::mbar_wait(o_final, 0, wait_limit_ns, abort_flag);
            if (!__all_sync(0xffffffffu, w)) ok = false;
        }
        if (ok) {
            ptx::tc_fence_after();
            const bool live = xr < T;
            const int64_t row = ((int64_t)bh * T + xr) * D;
            // each of the two warps of a quarter stores half of the D columns
            const int dh = (D / 2) * half;
            if (KV) {
                bwd_store_row<D / 2>(tl + Cf::kColB + dh, c, g1 + row + dh, live);    // dK = c dS^T Q
                bwd_store_row<D / 2>(tl + Cf::kColA + dh, 1.f, g2 + row + dh, live);  // dV = P^T dO
            } else {
                bwd_store_row<D / 2>(tl + Cf::kColA + dh, c, g1 + row + dh, live);    // dQ = c dS K
            }
        } else {
            atomicCAS(status, 0, 5);
            *abort_flag = 1;
        }
    }

    // -------------------------------------------------------------------- teardown
    ptx::tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        if (warp == 0 && lane == 0) {
            if (fix_issued) ptx::mbar_wait(fix_full, 0, kPPDrainLimitNs, nullptr);
            for (uint32_t st = 0; st < (uint32_t)NS && st < loads; ++st) {
                const uint32_t t = st + ((loads - 1 - st) / NS) * NS;
                ptx::mbar_wait(ring_full + st, (t / NS) & 1, kPPDrainLimitNs, nullptr);
            }
            for (uint32_t ss = 0; ss < 2 && ss < stat_loads; ++ss) {
                const uint32_t t = ss + ((stat_loads - 1 - ss) / 2) * 2;
                ptx::mbar_wait(stat_full + ss, (t / 2) & 1, kPPDrainLimitNs, nullptr);
            }
        }
        if (warp == 1) {
            ptx::tc_commit_one(drain);
            ptx::mbar_wait(drain, 0, kPPDrainLimitNs, nullptr);
        }
        __syncthreads();
    }
    if (warp == 1) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, Cf::kTmemCols);
    }
    // The query-tile grid ends only after the key-tile grid it may overlap, so that the
    // stream's next work sees dK and dV as well as dQ.
    if (!KV) ptx::grid_dependency_wait();
}

}  // namespace swa
