// prefill_tc.cuh: bf16 sliding-window causal attention prefill on the sm_100a tensor cores.
//
// One CTA computes one 128-row query tile of one (b,h). It visits only the 128-key
// tiles that meet the band (tile plan in plan.h) and masks only the edge tiles, as an
// implementation doing O(T * min(W,T) * D) work must ("NNX Sliding-Window Attention",
// A local mask is not a sparse implementation).
//
// Roles (192 threads):
//   warp 0, lane 0   TMA producer: Q once, then K_j and V_j through NS-stage rings.
//   warp 1           allocates 512 TMEM columns; lane 0 issues the tcgen05 MMAs:
//                      S_j = Q K_j^T     -> TMEM S[j%2] (fp32, 128 x 128)
//                      O  += P_j V_j     -> TMEM O (fp32, 128 x D), P_j read from TMEM
//   warps 2..5       softmax: warp w reads TMEM lanes 32*(w%4).. (one query row per
//                    thread), masks edge tiles by selecting -inf, keeps the running
//                    max m and sum l of the online softmax, writes P_j = exp2(s*c - m)
//                    as bf16 over the first 64 columns of S[j%2], rescales O when the
//                    max grows past a threshold, and finally writes O/l through smem
//                    with a TMA store.
// Stable softmax with the row max subtracted: "Mistral Architecture > Implementation:
// Sliding Window Attention", Step 2. The online form (running max, rescaling earlier
// partial sums) gives the same value by the shift invariance of softmax.
//
// Every mbarrier wait is bounded by wait_limit_ns. On a timeout the role records
// SWA_ERR_TIMEOUT in *status, raises the CTA's abort flag (other roles then stop
// waiting), and the CTA drains its in-flight TMA loads and MMAs, frees its TMEM and
// returns.
#pragma once
#include <cuda_bf16.h>
#include <math.h>

#include "plan.h"
#include "ptx.cuh"
#include "umma.h"

namespace swa {

constexpr int kTileM = 128;  // query rows per tile
constexpr int kTileN = 128;  // keys per tile
constexpr float kRescaleThreshold = 8.0f;  // lazy O rescale: max may grow by 2^8 first
// Query tiles whose rows see few keys (the first tile of every head, or any tile when
// W <= kPreciseWindow) carry P as a bf16 pair hi + lo (two P.V MMAs). There a couple of
// weights decide each output, |out| can reach 2 and more, and the 2^-9 relative rounding
// of a single bf16 P would use up most of the error budget left by the output rounding.
constexpr int kPreciseWindow = 32;
constexpr uint64_t kDrainLimitNs = 200000000ull;
constexpr int kStatusTimeout = 5;  // SWA_ERR_TIMEOUT

template <int D, int NS>
struct TcCfg {
    static_assert(D == 64 || D == 128, "head dim 64 or 128");
    static constexpr int kBoxBytes = 128 * 128;           // 128 rows x 64 bf16
    static constexpr int kTileBytes = kTileM * D * 2;     // one 128-row tile
    static constexpr int kQOff = 0;
    static constexpr int kKOff = kQOff + kTileBytes;
    static constexpr int kVOff = kKOff + NS * kTileBytes;
    static constexpr int kBarOff = kVOff + NS * kTileBytes;
    // q_full, k_full[NS], k_empty[NS], v_full[NS], v_empty[NS], s_full[2], p_full[2],
    // o_done, o_final, drain
    static constexpr int kNumBars = 1 + 4 * NS + 2 + 2 + 3;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kSmemBytes = kMiscOff + 16 + 1024;  // + alignment slack
    static constexpr uint32_t kTmemCols = 512;
    __device__ static constexpr uint32_t colS(int b) { return b ? 128u : 0u; }  // S/P buffers
    static constexpr uint32_t kColO = 256;
    static constexpr int kThreads = 192;
};

__device__ __forceinline__ void record_status(int* status, int code) {
    atomicCAS(status, 0, code);
}

// P = exp2(s*c - m) for one 128-key row held by this thread, written to TMEM at column
// col as bf16 pairs (rounded toward zero by a byte permute). PRECISE also writes the
// remainder p - bf16(p), again as bf16, 64 columns further on. Returns the sum of the
// weights exactly as written (so that O is normalised by the weights the MMAs used).
template <bool PRECISE>
__device__ __forceinline__ float write_p(const float (&sv)[128], float scale_log2, float m_use,
                                         uint32_t col) {
    float ls0 = 0.f, ls1 = 0.f;
    if (!PRECISE) {
        uint32_t p[2][32];
#pragma unroll
        for (int c = 0; c < 64; ++c) {
            const float e0 = ptx::ex2(fmaf(sv[2 * c], scale_log2, -m_use));
            const float e1 = ptx::ex2(fmaf(sv[2 * c + 1], scale_log2, -m_use));
            p[c >> 5][c & 31] = ptx::pack_bf16x2_trunc(e0, e1);
            ls0 += ptx::trunc_bf16(e0);
            ls1 += ptx::trunc_bf16(e1);
        }
        __syncwarp();
        ptx::tmem_st32(col, p[0]);
        ptx::tmem_st32(col + 32, p[1]);
    } else {
        __syncwarp();
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
            uint32_t ph[16], pl[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const int cp = q4 * 16 + c;
                const float e0 = ptx::ex2(fmaf(sv[2 * cp], scale_log2, -m_use));
                const float e1 = ptx::ex2(fmaf(sv[2 * cp + 1], scale_log2, -m_use));
                const float h0 = ptx::trunc_bf16(e0), h1 = ptx::trunc_bf16(e1);
                const float r0 = e0 - h0, r1 = e1 - h1;  // exact in fp32
                ph[c] = ptx::pack_bf16x2_trunc(e0, e1);
                pl[c] = ptx::pack_bf16x2_trunc(r0, r1);
                ls0 += h0 + ptx::trunc_bf16(r0);
                ls1 += h1 + ptx::trunc_bf16(r1);
            }
            ptx::tmem_st16(col + q4 * 16, ph);
            ptx::tmem_st16(col + 64 + q4 * 16, pl);
        }
    }
    return ls0 + ls1;
}

template <int D, int NS>
__global__ void __launch_bounds__(192, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                      int BH, int T, int W, int n_qt, float scale_log2, uint64_t wait_limit_ns,
                      int* status) {
    using C = TcCfg<D, NS>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem + C::kQOff;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    uint64_t* q_full = bars;
    uint64_t* k_full = bars + 1;
    uint64_t* k_empty = k_full + NS;
    uint64_t* v_full = k_empty + NS;
    uint64_t* v_empty = v_full + NS;
    uint64_t* s_full = v_empty + NS;
    uint64_t* p_full = s_full + 2;
    uint64_t* o_done = p_full + 2;
    uint64_t* o_final = o_done + 1;
    uint64_t* drain = o_final + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // Heavy query tiles (full windows) first, so that the light ones fill the tail.
    const int u = blockIdx.x;
    const int qt = n_qt - 1 - u / BH;
    const int bh = u % BH;
    int64_t ktf64, ktl64;
    kv_tile_range(T, W, kTileM, kTileN, qt, &ktf64, &ktl64);
    const int kt_first = (int)ktf64;
    const int n_tiles = (int)(ktl64 - ktf64 + 1);
    const bool precise = (qt == 0) || (W <= kPreciseWindow);

    if (threadIdx.x == 0) {
        ptx::mbar_init(q_full, 1);
        for (int s = 0; s < NS; ++s) {
            ptx::mbar_init(k_full + s, 1);
            ptx::mbar_init(k_empty + s, 1);
            ptx::mbar_init(v_full + s, 1);
            ptx::mbar_init(v_empty + s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(s_full + b, 1);
            ptx::mbar_init(p_full + b, 128);
        }
        ptx::mbar_init(o_done, 1);
        ptx::mbar_init(o_final, 1);
        ptx::mbar_init(drain, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tmap(&tm_q);
        ptx::prefetch_tmap(&tm_k);
        ptx::prefetch_tmap(&tm_v);
        ptx::prefetch_tmap(&tm_o);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, C::kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    int k_issued = 0, v_issued = 0;  // producer bookkeeping for the drain

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            bool ok = true;
            ptx::mbar_arrive_expect_tx(q_full, C::kTileBytes);
            for (int c = 0; c < D / 64; ++c)
                ptx::tma_load_3d(sQ + c * C::kBoxBytes, &tm_q, q_full, c * 64, qt * kTileM, bh);
            for (int j = 0; j <= n_tiles && ok; ++j) {
                if (j < n_tiles) {
                    const int st = j % NS;
                    if (j >= NS) ok = ptx::mbar_wait(k_empty + st, ((j / NS) - 1) & 1, wait_limit_ns, abort_flag);
                    if (!ok) break;
                    uint8_t* dst = smem + C::kKOff + st * C::kTileBytes;
                    ptx::mbar_arrive_expect_tx(k_full + st, C::kTileBytes);
                    for (int c = 0; c < D / 64; ++c)
                        ptx::tma_load_3d(dst + c * C::kBoxBytes, &tm_k, k_full + st, c * 64,
                                         (kt_first + j) * kTileN, bh);
                    ++k_issued;
                }
                if (j >= 1) {
                    const int jv = j - 1, st = jv % NS;
                    if (jv >= NS) ok = ptx::mbar_wait(v_empty + st, ((jv / NS) - 1) & 1, wait_limit_ns, abort_flag);
                    if (!ok) break;
                    uint8_t* dst = smem + C::kVOff + st * C::kTileBytes;
                    ptx::mbar_arrive_expect_tx(v_full + st, C::kTileBytes);
                    for (int c = 0; c < D / 64; ++c)
                        ptx::tma_load_3d(dst + c * C::kBoxBytes, &tm_v, v_full + st, c * 64,
                                         (kt_first + jv) * kTileN, bh);
                    ++v_issued;
                }
            }
            if (!ok) {
                record_status(status, kStatusTimeout);
                *abort_flag = 1;
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            const uint32_t idesc_s = umma::idesc_bf16_f32(kTileM, kTileN, 0);
            const uint32_t idesc_o = umma::idesc_bf16_f32(kTileM, D, 1);
            const uint32_t q_addr = ptx::smem_u32(sQ);
            bool ok = ptx::mbar_wait(q_full, 0, wait_limit_ns, abort_flag);
            for (int j = 0; j <= n_tiles && ok; ++j) {
                if (j < n_tiles) {
                    const int st = j % NS, b = j & 1;
                    ok = ptx::mbar_wait(k_full + st, (j / NS) & 1, wait_limit_ns, abort_flag);
                    if (!ok) break;
                    ptx::tc_fence_after();
                    const uint32_t k_addr = ptx::smem_u32(smem + C::kKOff + st * C::kTileBytes);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * C::kBoxBytes + (kk & 3) * 32;
                        ptx::mma_ss(tmem + C::colS(b), umma::smem_desc(q_addr + off, 16, 1024),
                                    umma::smem_desc(k_addr + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
                    }
                    ptx::tc_commit(s_full + b);
                    ptx::tc_commit(k_empty + st);
                }
                if (j >= 1) {
                    const int jp = j - 1, bp = jp & 1, st = jp % NS;
                    ok = ptx::mbar_wait(p_full + bp, (jp >> 1) & 1, wait_limit_ns, abort_flag);
                    if (!ok) break;
                    ok = ptx::mbar_wait(v_full + st, (jp / NS) & 1, wait_limit_ns, abort_flag);
                    if (!ok) break;
                    ptx::tc_fence_after();
                    const uint32_t v_addr = ptx::smem_u32(smem + C::kVOff + st * C::kTileBytes);
#pragma unroll
                    for (int kk = 0; kk < kTileN / 16; ++kk) {
                        ptx::mma_ts(tmem + C::kColO, tmem + C::colS(bp) + kk * 8,
                                    umma::smem_desc(v_addr + kk * 2048, C::kBoxBytes, 1024), idesc_o,
                                    (jp > 0 || kk > 0) ? 1u : 0u);
                    }
                    if (precise) {  // low halves of P, stored 64 columns further on
#pragma unroll
                        for (int kk = 0; kk < kTileN / 16; ++kk)
                            ptx::mma_ts(tmem + C::kColO, tmem + C::colS(bp) + 64 + kk * 8,
                                        umma::smem_desc(v_addr + kk * 2048, C::kBoxBytes, 1024),
                                        idesc_o, 1u);
                    }
                    ptx::tc_commit(v_empty + st);
                    ptx::tc_commit(o_done);
                    if (jp == n_tiles - 1) ptx::tc_commit(o_final);
                }
            }
            if (!ok) {
                record_status(status, kStatusTimeout);
                *abort_flag = 1;
            }
        }
    } else {
        // ---------------------------------------------------- softmax / epilogue
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;  // row of the tile this thread owns
        const int i = qt * kTileM + r;      // query position (>= T: padding row)
        const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
        int lo = i - W + 1;
        if (lo < 0) lo = 0;
        const int hi = i < T - 1 ? i : T - 1;
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < n_tiles; ++j) {
            const int b = j & 1;
            bool w = ptx::mbar_wait(s_full + b, (j >> 1) & 1, wait_limit_ns, abort_flag);
            if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
            ptx::tc_fence_after();
            uint32_t sr[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) ptx::tmem_ld32(tl + C::colS(b) + c * 32, sr[c]);
            ptx::tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 4; ++c) ptx::reg_fence(sr[c]);
            float sv[128];
#pragma unroll
            for (int c = 0; c < 128; ++c) sv[c] = __uint_as_float(sr[c >> 5][c & 31]);

            const int kt = kt_first + j;
            if (tile_class(T, W, kTileM, kTileN, qt, kt) != 2) {
                const int cmin = lo - kt * kTileN, cmax = hi - kt * kTileN;
#pragma unroll
                for (int c = 0; c < 128; ++c) sv[c] = (c >= cmin && c <= cmax) ? sv[c] : -INFINITY;
            }
            float mx[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) mx[t] = sv[t];
#pragma unroll
            for (int c = 8; c < 128; ++c) mx[c & 7] = fmaxf(mx[c & 7], sv[c]);
            const float mtile = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                      fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
            const float m_cand = mtile * scale_log2;
            bool need = false;
            float alpha = 1.f;
            if (m_cand > m_ref) {
                if (m_ref == -INFINITY) {
                    m_ref = m_cand;  // first in-band keys of this row: O row and l are 0
                } else if (m_cand > m_ref + kRescaleThreshold) {
                    need = true;
                    alpha = ptx::ex2(m_ref - m_cand);
                }
            }
            if (__any_sync(0xffffffffu, need)) {
                // O must hold P_{j-1} V_{j-1} and nothing later: wait for that MMA.
                w = ptx::mbar_wait(o_done, (j - 1) & 1, wait_limit_ns, abort_flag);
                if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
                ptx::tc_fence_after();
#pragma unroll 1
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t o[32];
                    ptx::tmem_ld32(tl + C::kColO + cc * 32, o);
                    ptx::tmem_ld_wait();
                    ptx::reg_fence(o);
#pragma unroll
                    for (int t = 0; t < 32; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * alpha);
                    ptx::tmem_st32(tl + C::kColO + cc * 32, o);
                }
                ptx::tmem_st_wait();
                if (need) {
                    l *= alpha;
                    m_ref = m_cand;
                }
            }
            const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
            l += precise ? write_p<true>(sv, scale_log2, m_use, tl + C::colS(b))
                         : write_p<false>(sv, scale_log2, m_use, tl + C::colS(b));
            ptx::tmem_st_wait();
            ptx::tc_fence_before();
            ptx::mbar_arrive(p_full + b);
        }
        if (ok) {
            bool w = ptx::mbar_wait(o_final, 0, wait_limit_ns, abort_flag);
            ok = __all_sync(0xffffffffu, w);
        }
        if (ok) {
            ptx::tc_fence_after();
            const float inv_l = l > 0.f ? 1.f / l : 0.f;
            // O/l as bf16 into the Q buffer (free: every MMA that read it is done), in
            // the 128-byte-swizzled layout the output tensor map expects.
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t o[32];
                ptx::tmem_ld32(tl + C::kColO + cc * 32, o);
                ptx::tmem_ld_wait();
                ptx::reg_fence(o);
                const int box = cc >> 1;
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    uint4 val;
                    val.x = ptx::pack_bf16x2(__uint_as_float(o[8 * t + 0]) * inv_l, __uint_as_float(o[8 * t + 1]) * inv_l);
                    val.y = ptx::pack_bf16x2(__uint_as_float(o[8 * t + 2]) * inv_l, __uint_as_float(o[8 * t + 3]) * inv_l);
                    val.z = ptx::pack_bf16x2(__uint_as_float(o[8 * t + 4]) * inv_l, __uint_as_float(o[8 * t + 5]) * inv_l);
                    val.w = ptx::pack_bf16x2(__uint_as_float(o[8 * t + 6]) * inv_l, __uint_as_float(o[8 * t + 7]) * inv_l);
                    const int chunk = (cc & 1) * 4 + t;
                    const int phys = chunk ^ (r & 7);
                    *reinterpret_cast<uint4*>(sQ + box * C::kBoxBytes + r * 128 + phys * 16) = val;
                }
            }
            ptx::fence_async_smem();
        }
        if (!ok) {
            record_status(status, kStatusTimeout);
            *abort_flag = 1;
        }
        // every softmax warp passes this barrier exactly once, on every path
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (threadIdx.x == 64 && !*abort_flag) {
            for (int c = 0; c < D / 64; ++c)
                ptx::tma_store_3d(&tm_o, sQ + c * C::kBoxBytes, c * 64, qt * kTileM, bh);
            ptx::bulk_commit();
            ptx::bulk_wait0();
        }
    }

    // ---------------------------------------------------------------- teardown
    ptx::tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        if (warp == 0 && lane == 0) {
            // let every TMA load this CTA issued land before its smem goes away
            ptx::mbar_wait(q_full, 0, kDrainLimitNs, nullptr);
            for (int st = 0; st < NS; ++st) {
                if (st < k_issued) {
                    const int t = st + ((k_issued - 1 - st) / NS) * NS;
                    ptx::mbar_wait(k_full + st, (t / NS) & 1, kDrainLimitNs, nullptr);
                }
                if (st < v_issued) {
                    const int t = st + ((v_issued - 1 - st) / NS) * NS;
                    ptx::mbar_wait(v_full + st, (t / NS) & 1, kDrainLimitNs, nullptr);
                }
            }
        }
        if (warp == 1 && lane == 0) {
            ptx::tc_commit(drain);  // completes when every MMA issued so far is done
            ptx::mbar_wait(drain, 0, kDrainLimitNs, nullptr);
        }
        __syncthreads();
    }
    if (warp == 1) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace swa
