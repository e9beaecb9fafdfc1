// chunk.cuh: chunked streaming prefill over the rolling KV buffer, and the ring append.
//
// A stream that has seen positions 0 .. pos-1 keeps the last min(pos, W) of them in a
// W-slot ring, position p in slot p mod W ("25. Sliding-Window Causal Attention for
// Streaming Inference", Problem: a KV cache bounded by the window; "Sliding Window
// Attention", Advantages: a cache of size W). A chunk of C new tokens takes positions
// pos .. pos+C-1. Query row i of the chunk (position P = pos + i) attends to positions
// max(0, P-W+1) .. P: the older ones from the ring, the chunk's own from the chunk. Among
// the chunk's own keys this is exactly the prefill band over chunk indices (0 <= i-j < W).
//
// chunk_kernel<D>: one CTA per (b, h, 128-row query tile of the chunk), 256 threads:
//   warp 0, lane 0   TMA producer: the Q tile, then K and V of every visited key tile
//                    through an NSTAGE ring: first the ring's slot tiles (128 slots each),
//                    then the chunk's key tiles.
//   warp 1           allocates TMEM; the warp runs the MMA loop and an elected lane issues
//                    the tcgen05 MMAs. S is double buffered,
//                    S_j = Q K_j^T -> TMEM columns [128 + 128(j&1), +128), and the
//                    order S_0, S_1, PV_0, S_2, PV_1, ... computes S_{j+1} while the softmax
//                    works on S_j, so the softmax never waits for its own P.V product.
//                    O += P_j V_j accumulates in TMEM columns [0, D).
//   warps 4..7       online softmax, one query row per thread (pp_tile of the prefill):
//                    a ring tile masks each slot by the position it holds, a chunk tile by
//                    the prefill band. Because PV_{j-1} may still run while S_j is read,
//                    a row that must rescale O first waits for PV_{j-1} (rare: only when
//                    the row maximum grows past the lazy-rescale threshold).
// The ring slot s holds position p(s) = pos - r + s - (s >= r ? W : 0) with r = pos mod W
// (the slot the chunk's first token will take); slots with p(s) < 0 hold nothing yet.
//
// ring_append_kernel: writes the chunk's k and v rows into slots (pos + c) mod W, only the
// last min(C, W) of them (the earlier ones would be overwritten within the same chunk), so
// every slot is written at most once per call. Launched after chunk_kernel on the same
// stream, it cannot overwrite anything the attention still reads.
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "plan.h"
#include "prefill_pp.cuh"
#include "ptx.cuh"
#include "umma.h"

namespace swa {

constexpr int kChunkThreads = 256;

template <int D>
struct ChunkCfg {
    static_assert(D == 64 || D == 128, "head dim 64 or 128");
    static constexpr int kBoxBytes = 128 * 128;         // 128 rows x 64 bf16
    static constexpr int kTileBytes = 128 * D * 2;      // one 128-row tile of Q, K or V
    static constexpr int kStages = D == 128 ? 6 : 12;   // unified K/V ring
    static constexpr int kQOff = 0;
    static constexpr int kRingOff = kTileBytes;
    static constexpr int kBarOff = kRingOff + kStages * kTileBytes;
    // q_full, ring_full[S], ring_empty[S], s_full[2], p_full[2], pv_done, o_final, drain
    static constexpr int kNumBars = 1 + 2 * kStages + 7;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kSmemBytes = kMiscOff + 16 + 1024;  // + alignment slack
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColO = 0;
    __device__ static constexpr uint32_t colS(int x) { return 128u + 128u * x; }
};

// What every role of a CTA derives from (b, h, qt) and the stream position.
struct ChunkItem {
    int bh, b, h, qt;
    int64_t pos0;     // stream position of chunk row 0
    int r;            // pos0 mod W
    int64_t lo_r;     // lowest position the tile's first row needs: max(0, P0 - W + 1)
    int64_t lb_last;  // lowest position the tile's last real row needs
    int n_st;         // slot tiles of the ring
    int kf, kl;       // chunk key tiles of the tile
    bool precise;
};

__device__ __forceinline__ ChunkItem chunk_item(int u, int n_qt, int H, int C, int W, int64_t pos0) {
    ChunkItem it;
    it.bh = u / n_qt;
    it.qt = u - it.bh * n_qt;
    it.b = it.bh / H;
    it.h = it.bh - it.b * H;
    it.pos0 = pos0;
    it.r = (int)(pos0 % W);
    const int64_t P0 = pos0 + 128 * (int64_t)it.qt;
    const int last = min(C, 128 * it.qt + 128) - 1;
    it.lo_r = P0 - W + 1 > 0 ? P0 - W + 1 : 0;
    it.lb_last = pos0 + last - W + 1 > 0 ? pos0 + last - W + 1 : 0;
    it.n_st = (W + 127) / 128;
    int64_t f, l;
    kv_tile_range(C, W, 128, 128, it.qt, &f, &l);
    it.kf = (int)f;
    it.kl = (int)l;
    it.precise = P0 < 128 || W <= kPPPreciseWindow;
    return it;
}

// Position held by ring slot s.
__device__ __forceinline__ int64_t chunk_slot_pos(const ChunkItem& it, int W, int s) {
    return it.pos0 - it.r + s - (s >= it.r ? W : 0);
}

// How the query tile treats ring slot tile t: 0 not visited, 1 edge, 2 full (every slot
// of the tile exists and is in every real row's band).
__device__ __forceinline__ int chunk_ring_class(const ChunkItem& it, int W, int t) {
    if (it.lo_r > it.pos0 - 1) return 0;  // the tile's band holds no position before the chunk
    const int s0 = 128 * t, s1 = min(W, s0 + 128) - 1;
    int64_t pmin, pmax;
    if (it.r > s0 && it.r <= s1) {  // the tile holds both the newest and the oldest slot
        pmin = it.pos0 - W;
        pmax = it.pos0 - 1;
    } else {
        pmin = chunk_slot_pos(it, W, s0);
        pmax = chunk_slot_pos(it, W, s1);
    }
    if (pmax < it.lo_r) return 0;
    return (s1 - s0 == 127 && pmin >= it.lb_last) ? 2 : 1;
}

__device__ __forceinline__ int clamp_col(int64_t x) { return (int)(x < -1 ? -1 : (x > 128 ? 128 : x)); }

template <int D>
__global__ void __launch_bounds__(kChunkThreads, 1)
    chunk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kc,
                 const __grid_constant__ CUtensorMap tm_vc, const __grid_constant__ CUtensorMap tm_kr,
                 const __grid_constant__ CUtensorMap tm_vr, const int64_t* __restrict__ pos,
                 __nv_bfloat16* __restrict__ out, int H, int C, int W, int n_qt, float scale_log2,
                 uint64_t wait_limit_ns, int* status) {
    using Cfg = ChunkCfg<D>;
    constexpr int NS = Cfg::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOff);
    uint64_t* q_full = bars;
    uint64_t* ring_full = bars + 1;  // [NS]
    uint64_t* ring_empty = ring_full + NS;
    uint64_t* s_full = ring_empty + NS;  // [2]
    uint64_t* p_full = s_full + 2;       // [2]
    uint64_t* pv_done = p_full + 2;
    uint64_t* o_final = pv_done + 1;
    uint64_t* drain = o_final + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kMiscOff + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u = blockIdx.x;
    const int b_of_u = (u / n_qt) / H;
    const int64_t pos0 = pos[b_of_u];
    if (pos0 < 0) {
        // Invalid position: this tile's rows are written as zeros and the status records it.
        if (threadIdx.x == 0) atomicCAS(status, 0, 1);
        const int bh = u / n_qt, qt = u - bh * n_qt;
        const int rows = min(C, 128 * qt + 128) - 128 * qt;
        uint4* o = reinterpret_cast<uint4*>(out + ((int64_t)bh * C + 128 * qt) * D);
        for (int x = threadIdx.x; x < rows * D / 8; x += kChunkThreads) o[x] = make_uint4(0, 0, 0, 0);
        return;
    }
    const ChunkItem it = chunk_item(u, n_qt, H, C, W, pos0);

    if (threadIdx.x == 0) {
        ptx::mbar_init(q_full, 1);
        for (int s = 0; s < NS; ++s) {
            ptx::mbar_init(ring_full + s, 1);
            ptx::mbar_init(ring_empty + s, 1);
        }
        for (int x = 0; x < 2; ++x) {
            ptx::mbar_init(s_full + x, 1);
            ptx::mbar_init(p_full + x, 128);
        }
        ptx::mbar_init(pv_done, 1);
        ptx::mbar_init(o_final, 1);
        ptx::mbar_init(drain, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tmap(&tm_q);
        ptx::prefetch_tmap(&tm_kc);
        ptx::prefetch_tmap(&tm_vc);
        ptx::prefetch_tmap(&tm_kr);
        ptx::prefetch_tmap(&tm_vr);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, Cfg::kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    uint32_t loads = 0;  // producer: K/V tiles issued
    bool q_issued = false;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------------------- producer
            bool ok = true;
            ptx::mbar_arrive_expect_tx(q_full, Cfg::kTileBytes);
            for (int c = 0; c < D / 64; ++c)
                ptx::tma_load_4d(smem + Cfg::kQOff + c * Cfg::kBoxBytes, &tm_q, q_full, c * 64, 128 * it.qt,
                                 it.h, it.b);
            q_issued = true;
            auto load = [&](const CUtensorMap* m, int row) {
                const uint32_t st = loads % NS;
                if (loads >= (uint32_t)NS)
                    ok = ptx::mbar_wait(ring_empty + st, ((loads / NS) - 1) & 1, wait_limit_ns, abort_flag);
                if (!ok) return;
                uint8_t* dst = smem + Cfg::kRingOff + st * Cfg::kTileBytes;
                ptx::mbar_arrive_expect_tx(ring_full + st, Cfg::kTileBytes);
                for (int c = 0; c < D / 64; ++c)
                    ptx::tma_load_4d(dst + c * Cfg::kBoxBytes, m, ring_full + st, c * 64, row, it.h, it.b);
                ++loads;
            };
            for (int t = 0; t < it.n_st && ok; ++t) {
                if (chunk_ring_class(it, W, t) == 0) continue;
                load(&tm_kr, 128 * t);
                if (ok) load(&tm_vr, 128 * t);
            }
            for (int kt = it.kf; kt <= it.kl && ok; ++kt) {
                load(&tm_kc, 128 * kt);
                if (ok) load(&tm_vc, 128 * kt);
            }
            if (!ok) {
                atomicCAS(status, 0, 5);
                *abort_flag = 1;
            }
        }
    } else if (warp == 1) {
        {
            // ---------------------------------------------------------------- MMA issuer
            // (the whole warp runs this loop; its waits are warp-uniform, one lane issues)
            const uint32_t idesc_s = umma::idesc_bf16_f32(128, 128, 0);
            const uint32_t idesc_o = umma::idesc_bf16_f32(128, D, 1);
            const uint64_t desc_hi = umma::smem_desc(0, 0, 1024) & 0xFFFFFFFF00000000ull;
            const uint32_t lo_k = (uint32_t)umma::smem_desc(0, 16, 1024);
            const uint32_t lo_v = (uint32_t)umma::smem_desc(0, Cfg::kBoxBytes, 1024);
            const uint32_t q_lo = (ptx::smem_u32(smem + Cfg::kQOff) >> 4) | lo_k;
            const uint32_t ring_lo = ptx::smem_u32(smem + Cfg::kRingOff) >> 4;
            constexpr uint32_t kStageLo = Cfg::kTileBytes >> 4;
            int n = 0;
            for (int t = 0; t < it.n_st; ++t) n += chunk_ring_class(it, W, t) != 0;
            n += it.kl - it.kf + 1;
            bool ok = pp_wait_warp(q_full, 0, wait_limit_ns, abort_flag);
            auto issue_s = [&](int j) {
                const uint32_t L = 2u * j, st = L % NS;
                ok = pp_wait_warp(ring_full + st, (L / NS) & 1, wait_limit_ns, abort_flag);
                if (!ok) return;
                ptx::tc_fence_after();
                const uint32_t k_lo = (ring_lo + st * kStageLo) | lo_k;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * Cfg::kBoxBytes + (kk & 3) * 32) >> 4;
                    ptx::mma_ss_one(tmem + Cfg::colS(j & 1), desc_hi | (q_lo + off), desc_hi | (k_lo + off), idesc_s,
                                kk > 0 ? 1u : 0u);
                }
                ptx::tc_commit_one(s_full + (j & 1));
                ptx::tc_commit_one(ring_empty + st);  // K_j read
            };
            auto issue_pv = [&](int j) {
                ok = pp_wait_warp(p_full + (j & 1), (j >> 1) & 1, wait_limit_ns, abort_flag);
                const uint32_t L = 2u * j + 1, st = L % NS;
                if (ok) ok = pp_wait_warp(ring_full + st, (L / NS) & 1, wait_limit_ns, abort_flag);
                if (!ok) return;
                ptx::tc_fence_after();
                const uint32_t v_lo = (ring_lo + st * kStageLo) | lo_v;
                const uint32_t scol = tmem + Cfg::colS(j & 1);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    ptx::mma_ts_one(tmem + Cfg::kColO, scol + pp_pcol(kk), desc_hi | (v_lo + kk * (2048 >> 4)), idesc_o,
                                (j > 0 || kk > 0) ? 1u : 0u);
                if (it.precise) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        ptx::mma_ts_one(tmem + Cfg::kColO, scol + pp_pcol(kk) + 16, desc_hi | (v_lo + kk * (2048 >> 4)),
                                    idesc_o, 1u);
                }
                ptx::tc_commit_one(pv_done);
                ptx::tc_commit_one(ring_empty + st);  // V_j read
                if (j == n - 1) ptx::tc_commit_one(o_final);
            };
            if (ok) issue_s(0);
            for (int j = 0; j < n && ok; ++j) {
                if (j + 1 < n) issue_s(j + 1);
                if (ok) issue_pv(j);
            }
            if (!ok && lane == 0) {
                atomicCAS(status, 0, 5);
                *abort_flag = 1;
            }
        }
    } else if (warp >= 4) {
        // -------------------------------------------------------------------- softmax
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const int i = 128 * it.qt + row;             // chunk row
        const int64_t Pi = it.pos0 + i;               // stream position
        const int64_t lb = Pi - W + 1 > 0 ? Pi - W + 1 : 0;
        const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
        float m_ref = -INFINITY, l = 0.f;
        int j = 0;
        bool ok = true;
        auto before = [&] {
            if (j > 0) {
                // PV_{j-1} may still be accumulating into O
                const bool w = ptx::mbar_wait(pv_done, (j - 1) & 1, wait_limit_ns, abort_flag);
                if (!__all_sync(0xffffffffu, w)) ok = false;
            }
        };
        auto next_s = [&]() -> bool {
            const bool w = ptx::mbar_wait(s_full + (j & 1), (j >> 1) & 1, wait_limit_ns, abort_flag);
            if (!__all_sync(0xffffffffu, w)) return false;
            ptx::tc_fence_after();
            return true;
        };
        auto done_p = [&] {
            ptx::tmem_st_wait();
            ptx::tc_fence_before();
            ptx::mbar_arrive(p_full + (j & 1));
            ++j;
        };
        for (int t = 0; t < it.n_st && ok; ++t) {
            const int cls = chunk_ring_class(it, W, t);
            if (cls == 0) continue;
            if (!next_s()) { ok = false; break; }
            const uint32_t scol = tl + Cfg::colS(j & 1), ocol = tl + Cfg::kColO;
            if (cls == 2) {
                if (it.precise) pp_tile<D, 0, true>(scol, ocol, scale_log2, m_ref, l, 0, 127, 0, -1, before);
                else pp_tile<D, 0, false>(scol, ocol, scale_log2, m_ref, l, 0, 127, 0, -1, before);
            } else {
                // valid slots: [lb - pos0 + r, r - 1] (newest positions) and
                // [max(r, lb - pos0 + r + W), W - 1] (older ones), as tile columns
                const int s0 = 128 * t;
                const int64_t a0 = lb - it.pos0 + it.r, a1 = it.r - 1;
                int64_t b0 = lb - it.pos0 + it.r + W;
                if (b0 < it.r) b0 = it.r;
                const int64_t b1 = W - 1;
                const int c0 = clamp_col(a0 - s0), c1 = clamp_col(a1 - s0);
                const int c2 = clamp_col(b0 - s0), c3 = clamp_col(b1 - s0);
                if (it.precise) pp_tile<D, 2, true>(scol, ocol, scale_log2, m_ref, l, c0, c1, c2, c3, before);
                else pp_tile<D, 2, false>(scol, ocol, scale_log2, m_ref, l, c0, c1, c2, c3, before);
            }
            done_p();
        }
        int lo = i - W + 1;
        if (lo < 0) lo = 0;
        const int hi = i < C - 1 ? i : C - 1;
        for (int kt = it.kf; kt <= it.kl && ok; ++kt) {
            if (!next_s()) { ok = false; break; }
            const uint32_t scol = tl + Cfg::colS(j & 1), ocol = tl + Cfg::kColO;
            const bool edge = tile_class(C, W, 128, 128, it.qt, kt) != 2;
            const int cmin = lo - kt * 128, cmax = hi - kt * 128;
            if (edge) {
                if (it.precise) pp_tile<D, 1, true>(scol, ocol, scale_log2, m_ref, l, cmin, cmax, 0, -1, before);
                else pp_tile<D, 1, false>(scol, ocol, scale_log2, m_ref, l, cmin, cmax, 0, -1, before);
            } else {
                if (it.precise) pp_tile<D, 0, true>(scol, ocol, scale_log2, m_ref, l, cmin, cmax, 0, -1, before);
                else pp_tile<D, 0, false>(scol, ocol, scale_log2, m_ref, l, cmin, cmax, 0, -1, before);
            }
            done_p();
        }
        if (ok) {
            // ------------------------------------------------------------ epilogue
            const bool w = ptx::mbar_wait(o_final, 0, wait_limit_ns, abort_flag);
            if (!__all_sync(0xffffffffu, w)) ok = false;
        }
        if (ok) {
            ptx::tc_fence_after();
            const float inv_l = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16* orow = out + ((int64_t)it.bh * C + i) * D;
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t o[32];
                ptx::tmem_ld32(tl + Cfg::kColO + cc * 32, o);
                ptx::tmem_ld_wait();
                ptx::reg_fence(o);
                if (i < C) {
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        uint4 val;
                        val.x = ptx::pack_bf16x2(__uint_as_float(o[8 * t + 0]) * inv_l, __uint_as_float(o[8 * t + 1]) * inv_l);
                        val.y = ptx::pack_bf16x2(__uint_as_float(o[8 * t + 2]) * inv_l, __uint_as_float(o[8 * t + 3]) * inv_l);
                        val.z = ptx::pack_bf16x2(__uint_as_float(o[8 * t + 4]) * inv_l, __uint_as_float(o[8 * t + 5]) * inv_l);
                        val.w = ptx::pack_bf16x2(__uint_as_float(o[8 * t + 6]) * inv_l, __uint_as_float(o[8 * t + 7]) * inv_l);
                        *reinterpret_cast<uint4*>(orow + cc * 32 + t * 8) = val;
                    }
                }
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
            // let every TMA load this CTA issued land before its shared memory goes away
            if (q_issued) ptx::mbar_wait(q_full, 0, kPPDrainLimitNs, nullptr);
            for (uint32_t st = 0; st < (uint32_t)NS && st < loads; ++st) {
                const uint32_t t = st + ((loads - 1 - st) / NS) * NS;
                ptx::mbar_wait(ring_full + st, (t / NS) & 1, kPPDrainLimitNs, nullptr);
            }
        }
        if (warp == 1) {
            ptx::tc_commit_one(drain);  // completes when every MMA issued so far is done
            ptx::mbar_wait(drain, 0, kPPDrainLimitNs, nullptr);
        }
        __syncthreads();
    }
    if (warp == 1) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, Cfg::kTmemCols);
    }
}

// Ring append: 16-byte vectors, one thread per vector, grid-stride. Rows c < c_first of
// the chunk are skipped (c_first = max(0, C - W)).
__global__ void __launch_bounds__(256)
    ring_append_kernel(const uint4* __restrict__ kc, const uint4* __restrict__ vc, uint4* __restrict__ kr,
                       uint4* __restrict__ vr, const int64_t* __restrict__ pos, int H, int C, int W,
                       int vpr, int c_first, int64_t n_vec, int* status) {
    const int rows = C - c_first;
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < n_vec;
         x += (int64_t)gridDim.x * blockDim.x) {
        const int e = (int)(x % vpr);
        const int64_t rr = x / vpr;
        const int c = c_first + (int)(rr % rows);
        const int64_t bh = rr / rows;
        const int64_t p0 = pos[bh / H];
        if (p0 < 0) {
            atomicCAS(status, 0, 1);
            continue;
        }
        const int64_t slot = (p0 + c) % W;
        const int64_t src = (bh * C + c) * vpr + e, dst = (bh * W + slot) * vpr + e;
        kr[dst] = kc[src];
        vr[dst] = vc[src];
    }
}

}  // namespace swa
