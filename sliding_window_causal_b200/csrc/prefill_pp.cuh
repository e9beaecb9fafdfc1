// prefill_pp.cuh: persistent, ping-pong bf16 sliding-window causal attention prefill on
// the sm_100a tensor cores.
//
// Work items are pairs of consecutive 128-row query tiles (A = 2p, B = 2p+1) of one (b,h).
// Both tiles meet nearly the same 128-key tiles of the band, so every K and V tile is
// loaded once for the pair. Only the key tiles that meet a tile's band are computed for
// it, and only edge tiles are masked ("NNX Sliding-Window Attention", A local mask is not
// a sparse implementation: only the allowed windows need computing).
//
// Q, K and V are read through 4-D tensor maps {D, T, H, B}, so any (b, h, t) element
// strides the TMA unit accepts work: contiguous [B,H,T,D], or the [B,T,H,D] layout of
// "Mistral Architecture > Implementation: Sliding Window Attention" (Step 2). The output is
// written with its own (b, h, t) strides.
//
// The grid holds at most one CTA per SM; CTA g takes items g, then 2G-1-g, then 2G+g, ...
// (a snake over the list of prefill_item in plan.h: first the equal-work pairs head after
// head, so that the CTAs at work share a few heads' key and value tiles in L2, then the
// lighter pairs heaviest first), which balances the load without any device-side queue.
//
// Roles (384 threads = 3 warpgroups, one CTA per SM):
//   warp 0, lane 0     TMA producer: Q_A, Q_B per item, then K_kt and V_kt through one
//                      NSTAGE-deep ring of 128-row tiles.
//   warp 1 (and 3)     warp 1 allocates the 512 TMEM columns. With one issuer (TWO = false)
//                      the whole of warp 1 runs the MMA loop and an elected lane issues every
//                      tcgen05 MMA in the order PV_A(kt-1), S_A(kt), PV_B(kt-1), S_B(kt); with
//                      two (TWO = true, for short bands), warp 1 issues tile A's products and
//                      warp 3 tile B's, each in the order S_x(kt), PV_x(kt), S_x(kt+1), ...
//                      Either way the tensor
//                      core works on one tile's products while the other tile's softmax runs:
//                        S_X = Q_X K^T   -> TMEM columns [128X, 128X+128)   (fp32)
//                        O_X += P_X V    -> TMEM columns [256+128X, +D)     (fp32)
//   warp 2             recomputes, in fp32 on the CUDA cores, the rows the softmax warps
//                      found sharp (pp_fix_row), taking them from a queue in shared memory.
//   warps 4..7 (A), 8..11 (B)   softmax of one query tile each, one row per thread (warp w
//                      reads TMEM lanes 32*(w%4)..): running max and sum of the online
//                      softmax ("Mistral Architecture > Implementation: Sliding Window
//                      Attention", Step 2, stable softmax), -inf select on edge tiles, P
//                      written over the S columns as bf16, lazy rescale of O, and finally
//                      O/l rounded to bf16 and stored to global memory.
// Because the MMAs of one thread complete in issue order, S_X(kt) completing implies that
// PV_X(kt-1) is complete: the softmax may rescale O_X right after it sees S_X(kt).
//
// Every mbarrier wait is bounded by wait_limit_ns. A role that runs past it records
// SWA_ERR_TIMEOUT, raises the CTA's abort flag (the other roles then stop waiting), and
// the CTA lets its in-flight TMA loads and MMAs finish, frees its TMEM and returns.
#pragma once
#include <cuda_bf16.h>
#include <math.h>

#include <type_traits>

#include "plan.h"
#include "ptx.cuh"
#include "umma.h"

namespace swa {

constexpr int kPPThreads = 384;
// Register split (setmaxnreg): the CTA is launched with kPPLaunchRegs per thread
// (384 x 168 = 64512); the producer/MMA warpgroup gives registers back down to
// kPPRoleRegs and the two softmax warpgroups take them up to kPPSoftmaxRegs:
// 128 x 104 + 256 x 200 = 64512. The host refuses to launch if the compiled kernel does
// not use exactly kPPLaunchRegs (an increase the pool cannot cover would never return).
constexpr int kPPLaunchRegs = 168;
constexpr int kPPRoleRegs = 104;
constexpr int kPPSoftmaxRegs = 200;
static_assert(128 * kPPRoleRegs + 256 * kPPSoftmaxRegs <= kPPThreads * kPPLaunchRegs, "register split");
constexpr float kPPRescaleThreshold = 8.0f;  // lazy O rescale: the max may grow by 2^8 first
// Query tiles whose rows see few keys (the first tile of every head, or any tile when
// W <= kPPPreciseWindow) carry P as two bf16 parts hi + lo with a second P.V MMA: there a
// couple of weights decide each output and |out| can exceed 2, so a single bf16 P would
// use up the error budget left by the output's own bf16 rounding. With single-bf16 P, such
// rows are found sharp at the epilogue and recomputed one by one on the CUDA cores; for
// bands of up to 144 keys and N(0,1) scores so many rows are sharp that the one
// recomputing warp sets the pace (B2 H16 T8192 D128: 389 us at W = 48 and 231 at W = 64,
// against 105 and 104 with hi + lo P; 138 against 104 at W = 129, whose bands still span
// two key tiles), while from 152 keys on hi + lo P costs more than it saves (W = 152: 134.5
// against 125.6 us; W = 256: 128 against 115).
constexpr int kPPPreciseWindow = 144;
constexpr uint64_t kPPDrainLimitNs = 200000000ull;
// Bands of at most this many keys use two MMA issuers (one per query tile), longer ones one.
constexpr int kPPTwoIssuerWindow = 1024;
// P of a tile is handed to the MMA issuer in this many parts (1, 2 or 4), so that the
// first keys' P.V products run while the softmax still works on the last keys.
constexpr int kPPParts = 2;
static_assert(kPPParts == 1 || kPPParts == 2 || kPPParts == 4, "parts of a tile's P");
// A row whose largest weight from a single-bf16-P tile ends up above kPPSharpShare of the
// row's total weight, and one of whose outputs reaches kPPSharpOut in magnitude, is
// recomputed in fp32 on the CUDA cores (pp_fix_row): such a key's bf16 rounding reaches
// the output almost undamped, on top of the output's own bf16 rounding (2^-8 relative).
constexpr float kPPSharpShare = 0.25f;
constexpr float kPPSharpOut = 1.0f;
// ADAPT (a kernel template argument): a softmax warp writes hi + lo parts of P on any tile
// where one of its rows meets a key that could end up above a quarter of the row's weight,
// and the MMA issuer adds the second P.V product for those warps' rows, so that no row
// becomes sharp. On N(0,1) inputs this costs about an eighth of the throughput; on inputs
// whose rows are dominated by a few keys it saves recomputing nearly every row. Without
// ADAPT, once one CTA has recomputed kPPAdaptAfter sharp rows the kernel sets *auto_flag
// (when given: a word of host memory mapped for the device), which the host reads to run
// later launches with ADAPT.
constexpr int kPPAdaptAfter = 8;

// Sharp rows go through a queue in shared memory to warp 2 (otherwise idle), which
// recomputes them while the softmax warps carry on; a full queue makes a softmax thread
// wait for a free slot.
constexpr int kPPFixSlots = 64;

// Raw operand pointers and their (b, h, t) element strides, for the fp32 recomputation
// of sharp rows (the tensor-core path reads q, k, v through tensor maps).
struct PPRaw {
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    const __nv_bfloat16* v;
    int64_t sq[3], sk[3], sv[3];
};

// TWO (two MMA issuers, short bands): two sets of Q_A, Q_B buffers, so that the producer
// loads the next item's Q while the current item still uses its own, and a shallower ring.
// An item of a short band streams few key tiles, so its start (Q and the first key tile
// arriving) weighs more than the ring depth within it.
template <int D, bool TWO = false>
struct PPCfg {
    static_assert(D == 64 || D == 128, "head dim 64 or 128");
    static constexpr int kBoxBytes = 128 * 128;        // 128 rows x 64 bf16
    static constexpr int kTileBytes = 128 * D * 2;     // one 128-row tile of Q, K or V
    static constexpr int kQSets = TWO ? 2 : 1;         // sets of Q_A, Q_B
    static constexpr int kStages = D == 128 ? (TWO ? 3 : 5) : (TWO ? 10 : 12);  // unified K/V ring
    static constexpr int kQOff = 0;                    // Q set s, tile x at (2s + x) tiles
    static constexpr int kRingOff = 2 * kQSets * kTileBytes;
    static constexpr int kBarOff = kRingOff + kStages * kTileBytes;
    // q_full[2][2], q_empty[2][2] (set, tile), ring_full[S], ring_empty[2][S], s_full[2],
    // p_full[2][4], o_final[2], o_free[2], drain[2]
    static constexpr int kNumBars = 8 + 3 * kStages + 16;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;  // tmem slot, abort flag, 4 queue counters
    static constexpr int kLoOff = (kMiscOff + 24 + 15) & ~15;  // low-part flags [2 tiles][2 parities][4 warps]
    static constexpr int kFixOff = kLoOff + 64;                 // queue of sharp rows: kPPFixSlots x 16 B
    static constexpr int kSmemBytes = kFixOff + kPPFixSlots * 16 + 1024;  // + alignment slack
    static constexpr uint32_t kTmemCols = 512;
    __device__ static constexpr uint32_t colS(int x) { return 128u * x; }
    __device__ static constexpr uint32_t colO(int x) { return 256u + 128u * x; }
};

// The r-th item of CTA g among n items on G CTAs (snake order), or -1.
__device__ __forceinline__ int pp_item(int r, int g, int G, int n) {
    const int u = r * G + ((r & 1) ? (G - 1 - g) : g);
    return u < n ? u : -1;
}

struct PPItem {
    int b, h, qt[2], f[2], l[2], k0, k1;
    bool hasB;
};

// single: each item is one query tile (used when a problem has fewer pairs of query tiles
// than the grid has SMs, so that more CTAs work); item u is tile u % n_qt of (b, h) u / n_qt.
__device__ __forceinline__ PPItem pp_decode(int u, int BH, int H, int n_qt, int T, int W, bool single) {
    PPItem it;
    int bh, p;
    if (single) {
        bh = u / n_qt;
        it.qt[0] = u - bh * n_qt;
        it.qt[1] = it.qt[0] + 1;
        it.hasB = false;
    } else {
        prefill_item<int>(u, BH, n_qt, W, &bh, &p);  // u is in range: pp_item checked it
        it.qt[0] = 2 * p;
        it.qt[1] = 2 * p + 1;
        it.hasB = it.qt[1] < n_qt;
    }
    it.b = bh / H;
    it.h = bh - it.b * H;
    int64_t f, l;
    kv_tile_range(T, W, 128, 128, it.qt[0], &f, &l);
    it.f[0] = (int)f;
    it.l[0] = (int)l;
    it.f[1] = it.l[1] = -1;
    if (it.hasB) {
        kv_tile_range(T, W, 128, 128, it.qt[1], &f, &l);
        it.f[1] = (int)f;
        it.l[1] = (int)l;
    }
    it.k0 = it.f[0];
    it.k1 = it.hasB ? it.l[1] : it.l[0];
    return it;
}

// mbar_wait for a whole warp: true only if every lane's wait completed, so that the warp
// stays converged (its elected-lane MMAs need the full warp).
__device__ __forceinline__ bool pp_wait_warp(uint64_t* bar, uint32_t parity, uint64_t limit_ns, volatile int* abort) {
    return __all_sync(0xffffffffu, ptx::mbar_wait(bar, parity, limit_ns, abort));
}

__device__ __forceinline__ bool pp_precise(int qt, int W) { return qt == 0 || W <= kPPPreciseWindow; }

// Which warps of tile x's softmax wrote low parts of P for the side-x tile number t (the
// flags of its parity; read after the tile's first part was handed over): dis[w] disables
// the 32 TMEM lanes of warp w in the second P.V product when it did not. Returns whether
// any did.
__device__ __forceinline__ bool pp_lo_lanes(volatile const uint32_t* lo_flag, int x, uint32_t t, uint32_t (&dis)[4]) {
    uint32_t w[4];  // one 16-byte load (the four flags of a tile are 16-byte aligned)
    asm volatile("ld.volatile.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                 : "r"(ptx::smem_u32(const_cast<const uint32_t*>(lo_flag + 4 * (2 * x + (t & 1))))));
#pragma unroll
    for (int j = 0; j < 4; ++j) dis[j] = w[j] != 0u ? 0u : 0xFFFFFFFFu;
    return (w[0] | w[1] | w[2] | w[3]) != 0u;
}

// Column of TMEM (relative to the S buffer) that holds P for keys 16kk..16kk+15: keys
// 32c..32c+31 are packed into columns 32c..32c+15 (and, for precise tiles, the low parts
// into 32c+16..32c+31), so that P only ever overwrites S values already read.
__device__ __forceinline__ uint32_t pp_pcol(int kk) { return 32u * (kk >> 1) + 8u * (kk & 1); }

// 2^-k for an integer k in [0, 126], exactly.
__device__ __forceinline__ float pp_pow2_neg(int k) { return __uint_as_float((uint32_t)(127 - k) << 23); }

// Multiply this thread's O row (D fp32 columns at TMEM column ocol) by a, and the bf16 P
// already written for the first `chunks` 32-key chunks of the S buffer at scol (and
// their low parts when PRECISE) by the same a. Warp-collective; a = 1 leaves a row as is.
// With a a power of two the products are exact (barring underflow to zero).
template <int D, bool PRECISE>
__device__ __forceinline__ void pp_rescale(uint32_t ocol, uint32_t scol, int chunks, float a) {
    ptx::tmem_st_wait();  // the P chunks read back below were written by this thread
#pragma unroll 1
    for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        ptx::tmem_ld32(ocol + cc * 32, o);
        ptx::tmem_ld_wait();
        ptx::reg_fence(o);
#pragma unroll
        for (int t = 0; t < 32; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * a);
        ptx::tmem_st32(ocol + cc * 32, o);
    }
#pragma unroll 1
    for (int c = 0; c < chunks; ++c) {
#pragma unroll
        for (int part = 0; part < (PRECISE ? 2 : 1); ++part) {
            uint32_t p[16];
            ptx::tmem_ld16(scol + 32 * c + 16 * part, p);
            ptx::tmem_ld_wait();
            ptx::reg_fence(p);
#pragma unroll
            for (int t = 0; t < 16; ++t)
                p[t] = ptx::pack_bf16x2(ptx::bf16lo_f32(p[t]) * a, ptx::bf16hi_f32(p[t]) * a);
            ptx::tmem_st16(scol + 32 * c + 16 * part, p);
        }
    }
    ptx::tmem_st_wait();
}

// P = exp2(s*c - mu) for the thread's 128 scores v (c = scale_log2), written over S as bf16
// in columns 32c..32c+15 of each 32-column chunk; LO = 1 also writes the low parts
// P - bf16(P), rounded to bf16, in columns 32c+16..32c+31, LO = 0 nothing. after_part(s) runs once part s's stores are issued and the next chunk's
// arithmetic is done. Returns the sum of the weights as written (hi + lo).
template <int LO, typename AfterPart>
__device__ __forceinline__ float pp_exps(uint32_t scol, const uint32_t (&v)[4][32], float scale_log2, float mu,
                                         AfterPart after_part) {
    const ptx::f32x2 sc = {scale_log2, scale_log2}, nm = {-mu, -mu};
    ptx::f32x2 acc[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint32_t ph[16], pl[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) {
            const ptx::f32x2 s2 = {__uint_as_float(v[c][2 * t]), __uint_as_float(v[c][2 * t + 1])};
            const ptx::f32x2 z = ptx::fma2(s2, sc, nm);
            const float e0 = ptx::ex2(z.x), e1 = ptx::ex2(z.y);
            ph[t] = ptx::pack_bf16x2(e0, e1);
            if (LO == 1) {
                const ptx::f32x2 w = {ptx::bf16lo_f32(ph[t]), ptx::bf16hi_f32(ph[t])};
                pl[t] = ptx::pack_bf16x2(e0 - w.x, e1 - w.y);
                acc[(t + 2) & 3] = ptx::add2(acc[(t + 2) & 3], {ptx::bf16lo_f32(pl[t]), ptx::bf16hi_f32(pl[t])});
                acc[t & 3] = ptx::add2(acc[t & 3], w);
            } else {
                acc[t & 3] = ptx::add_bf16x2_f32(ph[t], acc[t & 3]);
            }
        }
        // the previous part's stores have had this chunk's arithmetic to land
        if (c > 0 && c % (4 / kPPParts) == 0) after_part(c / (4 / kPPParts) - 1);
        ptx::tmem_st16(scol + 32 * c, ph);
        if (LO == 1) ptx::tmem_st16(scol + 32 * c + 16, pl);
    }
    after_part(kPPParts - 1);
    return ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) + ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
}

struct PPNoPublish {
    __device__ void operator()(bool) const {}
};

// One tile of one row: the thread's 128 scores are read from TMEM in one round trip,
// masked on edge tiles, reduced to the row maximum (log2 units), and P = exp2(s*c - m)
// is written back over the S columns as bf16 pairs (round to nearest): keys 32c..32c+31
// into columns 32c..32c+15 and, for PRECISE tiles, the remainders p - bf16(p) (again
// bf16) into columns 32c+16..32c+31.
// m is the row's reference maximum (-inf until the row meets its first in-band key). A
// row that sees its first keys takes the tile maximum; a row whose maximum exceeds m by
// more than the rescale threshold moves m up by the integer k = ceil(excess) and scales
// O and l by 2^-k (exact; zero when k > 126, where they are negligible). The row sum adds
// the weights exactly as written, so O is normalised by the weights the MMAs multiply by.
// MASK: 0 every key of the tile is in the row's band; 1 only columns cmin..cmax are; 2
// columns cmin..cmax and cmin2..cmax2 are. before_rescale() runs (warp-uniformly) before O
// is rescaled, for callers whose last P.V product may still be in flight. after_part(s)
// runs (warp-uniformly) once the stores of part s of P (keys 128s/kPPParts ..) have been
// issued and the next chunk's arithmetic is done, so that the caller can hand that part
// to the MMA issuer while the rest of the tile is computed. ADAPT (with PRECISE false): the
// warp chooses hi + lo parts for this tile when one of its rows meets a key that could end
// up above a quarter of the row's weight, or always when force is set; publish(bool) tells
// the caller which.
// Returns the row's largest scaled score in the tile (log2 units; -inf if none is in band,
// or if the tile's weights were written in two parts).
struct PPNoPart {
    __device__ void operator()(int) const {}
};

template <int D, int MASK, bool PRECISE, bool ADAPT = false, typename BeforeRescale, typename AfterPart = PPNoPart,
          typename Publish = PPNoPublish>
__device__ __forceinline__ float pp_tile(uint32_t scol, uint32_t ocol, float scale_log2, float& m,
                                        float& l, int cmin, int cmax, int cmin2, int cmax2,
                                        BeforeRescale before_rescale, AfterPart after_part = AfterPart(),
                                        Publish publish = Publish(), bool force = false) {
    uint32_t v[4][32];
#pragma unroll
    for (int c = 0; c < 4; ++c) ptx::tmem_ld32(scol + 32 * c, v[c]);
    ptx::tmem_ld_wait();
#pragma unroll
    for (int c = 0; c < 4; ++c) ptx::reg_fence(v[c]);
    if (MASK == 1) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int t = 0; t < 32; ++t) {
                const int k = 32 * c + t;
                if (!(k >= cmin && k <= cmax)) v[c][t] = __float_as_uint(-INFINITY);
            }
    } else if (MASK == 2) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int t = 0; t < 32; ++t) {
                const int k = 32 * c + t;
                if (!((k >= cmin && k <= cmax) || (k >= cmin2 && k <= cmax2)))
                    v[c][t] = __float_as_uint(-INFINITY);
            }
    }
    // eight independent max chains, so that the row maximum is not one long dependent chain
    float q[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) q[j] = -INFINITY;
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int t = 0; t < 32; t += 16) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
                q[j] = ptx::max3(q[j], __uint_as_float(v[c][t + 2 * j]), __uint_as_float(v[c][t + 2 * j + 1]));
        }
    const float tm = ptx::max3(ptx::max3(q[0], q[1], q[2]), ptx::max3(q[3], q[4], q[5]), fmaxf(q[6], q[7])) * scale_log2;
    const bool need = m != -INFINITY && tm > m + kPPRescaleThreshold;
    if (__any_sync(0xffffffffu, need)) {
        // k = ceil(excess) in full, so that no weight of this tile exceeds 2^0 (a capped k
        // would leave exp2 of the rest to overflow); beyond 2^-126 the old O and l are below
        // fp32's normal range relative to the new maximum and are dropped (f = 0)
        const int k = need ? (int)fminf(ceilf(tm - m), 1048576.0f) : 0;
        const float f = k > 126 ? 0.f : pp_pow2_neg(k);
        before_rescale();
        __syncwarp();
        pp_rescale<D, PRECISE>(ocol, scol, 0, f);
        l *= f;
        m += (float)k;
    }
    if (m == -INFINITY) m = tm;  // first in-band keys of the row (or still none)
    const float mu = m == -INFINITY ? 0.f : m;
    if (ADAPT) {
        // A key of this tile can end up above a quarter of its row's weight (the test for a
        // sharp row) only if its weight exceeds a third of the weight met before the tile:
        // w > (l + w)/4 needs 3w > l, and later tiles only add weight. Such a row, or any in
        // the warp, takes P as hi + lo parts; the warp tells the MMA issuer (publish) before
        // it hands the first part over, and the issuer's second P.V product leaves the
        // rows of the other warps unchanged.
        const bool flag = force || (tm != -INFINITY && 3.f * ptx::ex2(tm - mu) > l);
        const bool any = __any_sync(0xffffffffu, flag);
        publish(any);
        if (any) {
            l += pp_exps<1>(scol, v, scale_log2, mu, after_part);
            return -INFINITY;  // every weight of the tile is carried in two parts
        }
        l += pp_exps<0>(scol, v, scale_log2, mu, after_part);
        return tm;
    }
    l += pp_exps<PRECISE ? 1 : 0>(scol, v, scale_log2, mu, after_part);
    return tm;
}

__device__ __forceinline__ float pp_bf16_lo(uint32_t p) { return __uint_as_float(p << 16); }
__device__ __forceinline__ float pp_bf16_hi(uint32_t p) { return __uint_as_float(p & 0xFFFF0000u); }

// Row i of head (b, h), recomputed by the whole warp in fp32 on the CUDA cores. The band
// is taken 32 keys at a time: lane t scores key j0+t (fp32 FMA over d, ascending), the
// chunk's maximum moves the running maximum, and each lane accumulates its D/32 output
// columns over the chunk's keys in order. Loads are issued in batches ahead of their use
// (128 bytes of a lane's key row; half a chunk of value columns at a time). The weights are
// exact fp32 exponentials: no key's weight carries a bf16 rounding. Writes the bf16
// output row and, when lse_out is not null, the natural log-sum-exp. Warp-collective; the
// row has at least one key. Runs on the sharp-row worker warp, within that warpgroup's
// register share.
template <int D>
__device__ __forceinline__ void pp_fix_row(const PPRaw& raw, int b, int h, int i, int W, float scale_log2,
                                        __nv_bfloat16* orow, float* lse_out, int lane) {
    constexpr int DPL = D / 32;  // output columns per lane: 4 (8 bytes) or 2 (4 bytes)
    constexpr int NQ = D / 8;    // 16-byte pieces of a row
    using VT = typename std::conditional<DPL == 4, uint2, uint32_t>::type;
    const __nv_bfloat16* qrow = raw.q + b * raw.sq[0] + h * raw.sq[1] + (int64_t)i * raw.sq[2];
    const __nv_bfloat16* kbase = raw.k + b * raw.sk[0] + h * raw.sk[1];
    const __nv_bfloat16* vbase = raw.v + b * raw.sv[0] + h * raw.sv[1] + lane * DPL;
    const int lo = i - W + 1 > 0 ? i - W + 1 : 0;
    float m = -INFINITY, lsum = 0.f, o[DPL];
#pragma unroll
    for (int c = 0; c < DPL; ++c) o[c] = 0.f;
    for (int j0 = lo; j0 <= i; j0 += 32) {
        const int j = j0 + lane;
        const bool mine = j <= i;
        const __nv_bfloat16* krow = kbase + (int64_t)(mine ? j : i) * raw.sk[2];
        VT vv[16];
        auto load_v = [&](int t0) {
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                const int jt = j0 + t0 + t <= i ? j0 + t0 + t : i;  // rows past i are never read
                vv[t] = *reinterpret_cast<const VT*>(vbase + (int64_t)jt * raw.sv[2]);
            }
        };
        load_v(0);
        float acc = 0.f;
#pragma unroll
        for (int c0 = 0; c0 < NQ; c0 += 8) {  // the key row in pieces of 128 bytes
            uint4 kv[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) kv[c] = *reinterpret_cast<const uint4*>(krow + 8 * (c0 + c));
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 qc = *reinterpret_cast<const uint4*>(qrow + 8 * (c0 + c));  // the same for every lane
                const uint32_t qw[4] = {qc.x, qc.y, qc.z, qc.w};
                const uint32_t kw[4] = {kv[c].x, kv[c].y, kv[c].z, kv[c].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    acc = fmaf(pp_bf16_lo(qw[e]), pp_bf16_lo(kw[e]), acc);
                    acc = fmaf(pp_bf16_hi(qw[e]), pp_bf16_hi(kw[e]), acc);
                }
            }
        }
        const float s = mine ? acc * scale_log2 : -INFINITY;
        float cm = s;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, off));
        if (cm > m) {  // warp-uniform: the chunk raises the running maximum
            const float a = exp2f(m - cm);  // 0 on the first chunk
            lsum *= a;
#pragma unroll
            for (int c = 0; c < DPL; ++c) o[c] *= a;
            m = cm;
        }
        const float p = mine ? exp2f(s - m) : 0.f;
        lsum += p;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            if (half == 1) load_v(16);
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                const float pt = __shfl_sync(0xffffffffu, p, 16 * half + t);  // 0 for keys past i
                if constexpr (DPL == 4) {
                    o[0] = fmaf(pt, pp_bf16_lo(vv[t].x), o[0]);
                    o[1] = fmaf(pt, pp_bf16_hi(vv[t].x), o[1]);
                    o[2] = fmaf(pt, pp_bf16_lo(vv[t].y), o[2]);
                    o[3] = fmaf(pt, pp_bf16_hi(vv[t].y), o[3]);
                } else {
                    o[0] = fmaf(pt, pp_bf16_lo(vv[t]), o[0]);
                    o[1] = fmaf(pt, pp_bf16_hi(vv[t]), o[1]);
                }
            }
        }
    }
    float l = lsum;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
    const float inv = 1.f / l;
    if constexpr (DPL == 4) {
        uint2 w;
        w.x = ptx::pack_bf16x2(o[0] * inv, o[1] * inv);
        w.y = ptx::pack_bf16x2(o[2] * inv, o[3] * inv);
        *reinterpret_cast<uint2*>(orow + lane * DPL) = w;
    } else {
        *reinterpret_cast<uint32_t*>(orow + lane * DPL) = ptx::pack_bf16x2(o[0] * inv, o[1] * inv);
    }
    if (lse_out != nullptr && lane == 0) *lse_out = (m + log2f(l)) * 0.6931471805599453f;
}

// Push row i of head (b, h) to the sharp-row queue: take the next push number s, wait
// (bounded) until the worker has finished push s - kPPFixSlots, whose slot this is, write
// the row, then its sequence word s + 1. Returns false on abort or time-out.
__device__ __forceinline__ bool pp_push_sharp(uint32_t* fix_head, const uint32_t* fix_tail, uint4* fix_slot, int b,
                                              int h, int i, uint64_t limit_ns, volatile int* abort) {
    const uint32_t sl = atomicAdd(fix_head, 1u);
    volatile uint4* e = fix_slot + (sl % kPPFixSlots);
    const uint64_t t0 = ptx::globaltimer_ns();
    while (*reinterpret_cast<const volatile uint32_t*>(fix_tail) + kPPFixSlots <= sl) {
        if (*abort || ptx::globaltimer_ns() - t0 > limit_ns) return false;
        __nanosleep(256);
    }
    e->x = (uint32_t)b;
    e->y = (uint32_t)h;
    e->z = (uint32_t)i;
    __threadfence_block();
    e->w = sl + 1;
    return true;
}

// LSE: also write the natural log-sum-exp of each row (a separate instantiation, so that
// the plain prefill keeps its register allocation). ADAPT: hi + lo P chosen per warp and
// tile (above); likewise its own instantiation, so that the kernel without it is not slowed.
template <int D, bool LSE = false, bool TWO = false, bool ADAPT = false>
__global__ void __launch_bounds__(kPPThreads, 1)
    prefill_pp_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, __nv_bfloat16* __restrict__ out,
                      int64_t osb, int64_t osh, int64_t ost, float* __restrict__ lse, int BH, int H,
                      int T, int W, int n_qt, float scale_log2, uint64_t wait_limit_ns,
                      int* status, const __grid_constant__ PPRaw raw, int* auto_flag) {
    using C = PPCfg<D, TWO>;
    constexpr int NS = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    uint64_t* q_full = bars;            // [2][2]: Q set s, tile x at 2s + x
    uint64_t* q_empty = bars + 4;       // [2][2]
    uint64_t* ring_full = bars + 8;     // [NS]
    uint64_t* ring_empty = ring_full + NS;  // [2][NS]: tile x's issuer is done with the stage
    uint64_t* s_full = ring_empty + 2 * NS;  // [2]
    uint64_t* p_full = s_full + 2;       // [2][4]: P of tile x, part s, is in TMEM
    uint64_t* o_final = p_full + 8;      // [2]
    uint64_t* o_free = o_final + 2;      // [2]
    uint64_t* drain = o_free + 2;  // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);
    // queue of sharp rows: fix_head counts the rows pushed, fix_tail the rows the worker has
    // finished, fix_done the softmax warps that finished, fix_beat their items (progress);
    // push number s sits in slot s % kPPFixSlots as (b, h, i, s + 1)
    uint32_t* fix_head = reinterpret_cast<uint32_t*>(smem + C::kMiscOff + 8);
    uint32_t* fix_done = reinterpret_cast<uint32_t*>(smem + C::kMiscOff + 12);
    uint32_t* fix_beat = reinterpret_cast<uint32_t*>(smem + C::kMiscOff + 16);
    uint32_t* fix_tail = reinterpret_cast<uint32_t*>(smem + C::kMiscOff + 20);
    uint4* fix_slot = reinterpret_cast<uint4*>(smem + C::kFixOff);
    // lo_flag[4 * (2x + parity) + w]: warp w of tile x's softmax wrote low parts of P for the
    // x-tile of that parity (counted in tiles of side x); read by the MMA issuer once the
    // tile's first part is handed over
    volatile uint32_t* lo_flag = reinterpret_cast<volatile uint32_t*>(smem + C::kLoOff);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x, g = blockIdx.x;
    // pairs of query tiles as items, or single tiles when there are fewer pairs than CTAs
    // (the host then sizes the grid by the single tiles)
    const int n_pairs = ((n_qt + 1) >> 1) * BH;
    const bool single = G > n_pairs;
    const int n_items = single ? n_qt * BH : n_pairs;

    if (threadIdx.x == 0) {
        for (int x = 0; x < 4; ++x) {
            ptx::mbar_init(q_full + x, 1);
            ptx::mbar_init(q_empty + x, 1);
        }
        for (int x = 0; x < 2; ++x) {
            ptx::mbar_init(s_full + x, 1);
            for (int c = 0; c < 4; ++c) ptx::mbar_init(p_full + 4 * x + c, 4);  // one arrival per warp
            ptx::mbar_init(o_final + x, 1);
            ptx::mbar_init(o_free + x, 128);
        }
        for (int s = 0; s < NS; ++s) {
            ptx::mbar_init(ring_full + s, 1);
            ptx::mbar_init(ring_empty + s, 1);
            ptx::mbar_init(ring_empty + NS + s, 1);
        }
        ptx::mbar_init(drain, 1);
        ptx::mbar_init(drain + 1, 1);
        *abort_flag = 0;
        *fix_head = 0;
        *fix_done = 0;
        *fix_beat = 0;
        *fix_tail = 0;
        for (int q = 0; q < kPPFixSlots; ++q) fix_slot[q] = make_uint4(0, 0, 0, 0);
        for (int q = 0; q < 16; ++q) lo_flag[q] = 0u;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tmap(&tm_q);
        ptx::prefetch_tmap(&tm_k);
        ptx::prefetch_tmap(&tm_v);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, C::kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    constexpr bool adapt = ADAPT;

    uint32_t loads = 0;  // producer: K/V tiles issued so far
    int nq[2] = {0, 0};  // producer: Q tiles issued per side

    if (warp < 4) {
      ptx::regs_dec<kPPRoleRegs>();
      if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------------------ producer
            bool ok = true;
            for (int r = 0; ok; ++r) {
                const int u = pp_item(r, g, G, n_items);
                if (u < 0) break;
                const PPItem it = pp_decode(u, BH, H, n_qt, T, W, single);
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    if (!ok || (x == 1 && !it.hasB)) break;
                    // the n-th Q tile of side x goes to set n % kQSets, once that set's previous
                    // tile (n - kQSets) is no longer read
                    const int n = nq[x], qb = 2 * (n % C::kQSets) + x;
                    if (n >= C::kQSets)
                        ok = ptx::mbar_wait(q_empty + qb, ((n / C::kQSets) - 1) & 1, wait_limit_ns, abort_flag);
                    if (!ok) break;
                    uint8_t* dst = smem + C::kQOff + qb * C::kTileBytes;
                    ptx::mbar_arrive_expect_tx(q_full + qb, C::kTileBytes);
                    for (int c = 0; c < D / 64; ++c)
                        ptx::tma_load_4d(dst + c * C::kBoxBytes, &tm_q, q_full + qb, c * 64, it.qt[x] * 128, it.h, it.b);
                    ++nq[x];
                }
                for (int kt = it.k0; kt <= it.k1 && ok; ++kt) {
                    for (int kv = 0; kv < 2; ++kv) {
                        const uint32_t st = loads % NS;
                        if (loads >= (uint32_t)NS)
                            ok = ptx::mbar_wait(ring_empty + st, ((loads / NS) - 1) & 1, wait_limit_ns, abort_flag) &&
                                 (!TWO ||
                                  ptx::mbar_wait(ring_empty + NS + st, ((loads / NS) - 1) & 1, wait_limit_ns, abort_flag));
                        if (!ok) break;
                        uint8_t* dst = smem + C::kRingOff + st * C::kTileBytes;
                        ptx::mbar_arrive_expect_tx(ring_full + st, C::kTileBytes);
                        for (int c = 0; c < D / 64; ++c)
                            ptx::tma_load_4d(dst + c * C::kBoxBytes, kv ? &tm_v : &tm_k, ring_full + st, c * 64,
                                             kt * 128, it.h, it.b);
                        ++loads;
                    }
                }
            }
            if (!ok) {
                atomicCAS(status, 0, 5);
                *abort_flag = 1;
            }
        }
    } else if (!TWO && warp == 1) {
        {
            // ------------------------------------------------------------ MMA issuer (one warp)
            // (the whole warp runs this loop; its waits are warp-uniform, one lane issues)
            // Descriptors: the high word (SBO = 1024, sm_100 version, 128-byte swizzle) is
            // the same for every operand; the low word is start >> 4 plus the leading byte
            // offset field, so each MMA needs one add (shared memory is far below 256 KiB, so
            // start >> 4 + offset never carries out of its 14-bit field).
            const uint32_t idesc_s = umma::idesc_bf16_f32(128, 128, 0);
            const uint32_t idesc_o = umma::idesc_bf16_f32(128, D, 1);
            const uint64_t desc_hi = umma::smem_desc(0, 0, 1024) & 0xFFFFFFFF00000000ull;
            const uint32_t lo_k = (uint32_t)umma::smem_desc(0, 16, 1024);              // K-major LBO field
            const uint32_t lo_v = (uint32_t)umma::smem_desc(0, C::kBoxBytes, 1024);   // MN-major LBO field
            const uint32_t q_base = ptx::smem_u32(smem + C::kQOff) >> 4;
            const uint32_t ring_lo = ptx::smem_u32(smem + C::kRingOff) >> 4;
            constexpr uint32_t kStageLo = C::kTileBytes >> 4;
            uint32_t L = 0;               // K/V tiles consumed so far (same count as the producer)
            int ni[2] = {0, 0};           // items seen per side
            uint32_t ns[2] = {0, 0};      // S tiles issued per side
            bool ok = true;
            for (int r = 0; ok; ++r) {
                const int u = pp_item(r, g, G, n_items);
                if (u < 0) break;
                const PPItem it = pp_decode(u, BH, H, n_qt, T, W, single);
                const int nx = it.hasB ? 2 : 1;
                const bool prec[2] = {pp_precise(it.qt[0], W), pp_precise(it.qt[1], W)};
                // this item's Q_x: the ni[x]-th of side x, in set ni[x] % kQSets
                const int qb[2] = {2 * (ni[0] % C::kQSets), 2 * (ni[1] % C::kQSets) + 1};
                const uint32_t q_lo[2] = {(q_base + qb[0] * (C::kTileBytes >> 4)) | lo_k,
                                          (q_base + qb[1] * (C::kTileBytes >> 4)) | lo_k};
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    if (x < nx && ok) ok = pp_wait_warp(q_full + qb[x], (ni[x] / C::kQSets) & 1, wait_limit_ns, abort_flag);
                }
                if (!ok) break;
                int pend[2] = {-1, -1};
                bool first_pv[2] = {true, true};
                const uint32_t Lbase = L;
                for (int kt = it.k0; kt <= it.k1 + 1 && ok; ++kt) {
                    const uint32_t j = (uint32_t)(kt - it.k0);
                    const uint32_t Lk = Lbase + 2 * j, Lv = Lk - 1;
                    const uint32_t stk = Lk % NS, stv = Lv % NS;
                    if (kt <= it.k1) ok = pp_wait_warp(ring_full + stk, (Lk / NS) & 1, wait_limit_ns, abort_flag);
                    if (ok && kt > it.k0) ok = pp_wait_warp(ring_full + stv, (Lv / NS) & 1, wait_limit_ns, abort_flag);
                    if (!ok) break;
                    const uint32_t k_lo = (ring_lo + stk * kStageLo) | lo_k;
                    const uint32_t v_lo = (ring_lo + stv * kStageLo) | lo_v;
#pragma unroll
                    for (int x = 0; x < 2; ++x) {
                        if (x >= nx || !ok) break;
                        if (pend[x] >= 0) {
                            // PV_x(kt-1) part by part as the softmax hands P_x(kt-1) over; O_x
                            // must be free if it starts the item
                            if (first_pv[x] && ni[x] > 0)
                                ok = pp_wait_warp(o_free + x, (ni[x] - 1) & 1, wait_limit_ns, abort_flag);
                            // low parts: every lane on tiles that always carry them, else the lanes
                            // of the softmax warps that wrote them for this tile
                            bool lo_parts = prec[x];
                            uint32_t dis[4] = {0u, 0u, 0u, 0u};
#pragma unroll
                            for (int part = 0; part < kPPParts && ok; ++part) {
                                ok = pp_wait_warp(p_full + 4 * x + part, (ns[x] - 1) & 1, wait_limit_ns, abort_flag);
                                if (!ok) break;
                                ptx::tc_fence_after();
                                constexpr int kPer = 8 / kPPParts;  // 16-key MMA steps per part
#pragma unroll
                                for (int kk = part * kPer; kk < (part + 1) * kPer; ++kk)
                                    ptx::mma_ts_one(tmem + C::colO(x), tmem + C::colS(x) + pp_pcol(kk),
                                                    desc_hi | (v_lo + kk * (2048 >> 4)), idesc_o,
                                                    (!first_pv[x] || kk > 0) ? 1u : 0u);
                                // the warps' choices, read while the tensor pipe takes the part's
                                // products; every warp's rows: the unmasked form
                                if (part == 0 && adapt && !prec[x]) lo_parts = pp_lo_lanes(lo_flag, x, ns[x] - 1, dis);
                                if (lo_parts && adapt && (dis[0] | dis[1] | dis[2] | dis[3]) != 0u) {
#pragma unroll
                                    for (int kk = part * kPer; kk < (part + 1) * kPer; ++kk)
                                        ptx::mma_ts_one_masked(tmem + C::colO(x), tmem + C::colS(x) + pp_pcol(kk) + 16,
                                                               desc_hi | (v_lo + kk * (2048 >> 4)), idesc_o, 1u, dis);
                                } else if (lo_parts) {
#pragma unroll
                                    for (int kk = part * kPer; kk < (part + 1) * kPer; ++kk)
                                        ptx::mma_ts_one(tmem + C::colO(x), tmem + C::colS(x) + pp_pcol(kk) + 16,
                                                        desc_hi | (v_lo + kk * (2048 >> 4)), idesc_o, 1u);
                                }
                            }
                            if (!ok) break;
                            first_pv[x] = false;
                            if (pend[x] == it.l[x]) ptx::tc_commit_one(o_final + x);
                            pend[x] = -1;
                        } else {
                            ptx::tc_fence_after();
                        }
                        if (kt <= it.k1 && kt >= it.f[x] && kt <= it.l[x]) {
                            // S_x(kt) = Q_x K(kt)^T
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk) {
                                const uint32_t off = ((kk >> 2) * C::kBoxBytes + (kk & 3) * 32) >> 4;
                                ptx::mma_ss_one(tmem + C::colS(x), desc_hi | (q_lo[x] + off), desc_hi | (k_lo + off),
                                            idesc_s, kk > 0 ? 1u : 0u);
                            }
                            ptx::tc_commit_one(s_full + x);
                            ++ns[x];
                            if (kt == it.l[x]) ptx::tc_commit_one(q_empty + qb[x]);
                            pend[x] = kt;
                        }
                    }
                    if (!ok) break;
                    if (kt <= it.k1) ptx::tc_commit_one(ring_empty + stk);  // K(kt) read by its S MMAs
                    if (kt > it.k0) ptx::tc_commit_one(ring_empty + stv);   // V(kt-1) read by its PV MMAs
                }
                L = Lbase + 2u * (uint32_t)(it.k1 - it.k0 + 1);
                ++ni[0];
                if (it.hasB) ++ni[1];
            }
            if (!ok && lane == 0) {
                atomicCAS(status, 0, 5);
                *abort_flag = 1;
            }
        }
    } else if (TWO && (warp == 1 || warp == 3)) {
        {
            // ------------------------------------------------------------ MMA issuers (two warps)
            // Warp 1 issues tile A's products, warp 3 tile B's, each as a whole warp
            // (warp-uniform waits, one elected lane issues): S_x(f), PV_x(f), S_x(f+1), ...
            // Two issuers keep one tile's wait for its P from holding up the other tile's
            // products. Each issuer releases every ring stage of the item, used or not, on its
            // own ring_empty barrier (after the products that read it, or once the stage is
            // filled if it does not use it), so the producer waits for both.
            // Descriptors: the high word (SBO = 1024, sm_100 version, 128-byte swizzle) is
            // the same for every operand; the low word is start >> 4 plus the leading byte
            // offset field, so each MMA needs one add (shared memory is far below 256 KiB, so
            // start >> 4 + offset never carries out of its 14-bit field).
            const int x = warp == 1 ? 0 : 1;
            const uint32_t idesc_s = umma::idesc_bf16_f32(128, 128, 0);
            const uint32_t idesc_o = umma::idesc_bf16_f32(128, D, 1);
            const uint64_t desc_hi = umma::smem_desc(0, 0, 1024) & 0xFFFFFFFF00000000ull;
            const uint32_t lo_k = (uint32_t)umma::smem_desc(0, 16, 1024);              // K-major LBO field
            const uint32_t lo_v = (uint32_t)umma::smem_desc(0, C::kBoxBytes, 1024);   // MN-major LBO field
            const uint32_t ring_lo = ptx::smem_u32(smem + C::kRingOff) >> 4;
            constexpr uint32_t kStageLo = C::kTileBytes >> 4;
            uint64_t* my_empty = ring_empty + x * NS;
            const auto release = [&](uint32_t st, bool used) {
                if (used) ptx::tc_commit_one(my_empty + st);  // once the products that read it are done
                else if (lane == 0) ptx::mbar_arrive(my_empty + st);
            };
            uint32_t L = 0;   // K/V tiles consumed so far (same count as the producer)
            int ni = 0;       // items of this tile seen
            uint32_t ns = 0;  // S tiles issued
            bool ok = true;
            for (int r = 0; ok; ++r) {
                const int u = pp_item(r, g, G, n_items);
                if (u < 0) break;
                const PPItem it = pp_decode(u, BH, H, n_qt, T, W, single);
                const bool mine = x == 0 || it.hasB;
                const int f = it.f[x], l = it.l[x];
                const bool prec = pp_precise(it.qt[x], W);
                // this item's Q_x: the ni-th of side x, in set ni % kQSets
                const int qb = 2 * (ni % C::kQSets) + x;
                const uint32_t q_lo = (ptx::smem_u32(smem + C::kQOff + qb * C::kTileBytes) >> 4) | lo_k;
                if (mine) ok = pp_wait_warp(q_full + qb, (ni / C::kQSets) & 1, wait_limit_ns, abort_flag);
                if (!ok) break;
                int pend = -1;
                bool first_pv = true;
                const uint32_t Lbase = L;
                for (int kt = it.k0; kt <= it.k1 + 1 && ok; ++kt) {
                    const uint32_t j = (uint32_t)(kt - it.k0);
                    const uint32_t Lk = Lbase + 2 * j, Lv = Lk - 1;
                    if (kt > it.k0) {
                        // PV_x(kt-1) (before S_x(kt), which overwrites P_x(kt-1)); V(kt-1) released
                        const uint32_t stv = Lv % NS;
                        ok = pp_wait_warp(ring_full + stv, (Lv / NS) & 1, wait_limit_ns, abort_flag);
                        if (ok && pend >= 0) {
                            // part by part as the softmax hands P_x(kt-1) over; O_x must be
                            // free if it starts the item
                            if (first_pv && ni > 0)
                                ok = pp_wait_warp(o_free + x, (ni - 1) & 1, wait_limit_ns, abort_flag);
                            const uint32_t v_lo = (ring_lo + stv * kStageLo) | lo_v;
                            // low parts: every lane on tiles that always carry them, else the lanes
                            // of the softmax warps that wrote them for this tile
                            bool lo_parts = prec;
                            uint32_t dis[4] = {0u, 0u, 0u, 0u};
#pragma unroll
                            for (int part = 0; part < kPPParts && ok; ++part) {
                                ok = pp_wait_warp(p_full + 4 * x + part, (ns - 1) & 1, wait_limit_ns, abort_flag);
                                if (!ok) break;
                                ptx::tc_fence_after();
                                constexpr int kPer = 8 / kPPParts;  // 16-key MMA steps per part
#pragma unroll
                                for (int kk = part * kPer; kk < (part + 1) * kPer; ++kk)
                                    ptx::mma_ts_one(tmem + C::colO(x), tmem + C::colS(x) + pp_pcol(kk),
                                                    desc_hi | (v_lo + kk * (2048 >> 4)), idesc_o,
                                                    (!first_pv || kk > 0) ? 1u : 0u);
                                // the warps' choices, read while the tensor pipe takes the part's
                                // products; every warp's rows: the unmasked form
                                if (part == 0 && adapt && !prec) lo_parts = pp_lo_lanes(lo_flag, x, ns - 1, dis);
                                if (lo_parts && adapt && (dis[0] | dis[1] | dis[2] | dis[3]) != 0u) {
#pragma unroll
                                    for (int kk = part * kPer; kk < (part + 1) * kPer; ++kk)
                                        ptx::mma_ts_one_masked(tmem + C::colO(x), tmem + C::colS(x) + pp_pcol(kk) + 16,
                                                               desc_hi | (v_lo + kk * (2048 >> 4)), idesc_o, 1u, dis);
                                } else if (lo_parts) {
#pragma unroll
                                    for (int kk = part * kPer; kk < (part + 1) * kPer; ++kk)
                                        ptx::mma_ts_one(tmem + C::colO(x), tmem + C::colS(x) + pp_pcol(kk) + 16,
                                                        desc_hi | (v_lo + kk * (2048 >> 4)), idesc_o, 1u);
                                }
                            }
                            if (!ok) break;
                            first_pv = false;
                            if (pend == l) ptx::tc_commit_one(o_final + x);
                        }
                        if (!ok) break;
                        release(stv, pend >= 0);
                        pend = -1;
                    }
                    if (kt <= it.k1) {
                        // S_x(kt) = Q_x K(kt)^T; K(kt) released
                        const uint32_t stk = Lk % NS;
                        ok = pp_wait_warp(ring_full + stk, (Lk / NS) & 1, wait_limit_ns, abort_flag);
                        if (!ok) break;
                        const bool use = mine && kt >= f && kt <= l;
                        if (use) {
                            ptx::tc_fence_after();
                            const uint32_t k_lo = (ring_lo + stk * kStageLo) | lo_k;
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk) {
                                const uint32_t off = ((kk >> 2) * C::kBoxBytes + (kk & 3) * 32) >> 4;
                                ptx::mma_ss_one(tmem + C::colS(x), desc_hi | (q_lo + off), desc_hi | (k_lo + off),
                                                idesc_s, kk > 0 ? 1u : 0u);
                            }
                            ptx::tc_commit_one(s_full + x);
                            ++ns;
                            if (kt == l) ptx::tc_commit_one(q_empty + qb);
                            pend = kt;
                        }
                        release(stk, use);
                    }
                }
                L = Lbase + 2u * (uint32_t)(it.k1 - it.k0 + 1);
                if (mine) ++ni;
            }
            if (!ok && lane == 0) {
                atomicCAS(status, 0, 5);
                *abort_flag = 1;
            }
        }
      } else if (warp == 2) {
        // ------------------------------------------------------------ sharp-row worker
        // Slots are taken in push order. The loop ends once every softmax warp has
        // finished and no push is left, or on abort, or when the softmax warps have made
        // no progress (no item finished, nothing pushed) for the wait limit.
        uint64_t t0 = ptx::globaltimer_ns();
        uint32_t seen = 0;
        for (uint32_t sl = 0;; ++sl) {
            volatile uint4* e = fix_slot + (sl % kPPFixSlots);
            bool have = false;
            while (true) {
                const uint32_t now = *reinterpret_cast<volatile uint32_t*>(fix_beat) +
                                     *reinterpret_cast<volatile uint32_t*>(fix_head);
                if (now != seen) {
                    seen = now;
                    t0 = ptx::globaltimer_ns();
                }
                if (e->w == sl + 1) {
                    have = true;
                    break;
                }
                if (*reinterpret_cast<volatile uint32_t*>(fix_done) == 8u &&
                    *reinterpret_cast<volatile uint32_t*>(fix_head) <= sl)
                    break;  // all softmax warps are done and nothing more was pushed
                if (*abort_flag) break;
                if (ptx::globaltimer_ns() - t0 > wait_limit_ns) {
                    atomicCAS(status, 0, 5);
                    *abort_flag = 1;
                    break;
                }
                __nanosleep(256);
            }
            if (!__all_sync(0xffffffffu, have)) break;
            __threadfence_block();
            const uint4 ent = *const_cast<const uint4*>(reinterpret_cast<volatile uint4*>(e));
            const int fb = (int)ent.x, fh = (int)ent.y, fi = (int)ent.z;
            pp_fix_row<D>(raw, fb, fh, fi, W, scale_log2, out + fb * osb + fh * osh + (int64_t)fi * ost,
                          LSE ? lse + ((int64_t)fb * H + fh) * T + fi : nullptr, lane);
            // inputs that make this many rows sharp in one CTA run adaptive from the next launch
            if (!ADAPT && auto_flag != nullptr && sl + 1 == (uint32_t)kPPAdaptAfter && lane == 0) {
                *reinterpret_cast<volatile int*>(auto_flag) = 1;
                __threadfence_system();
            }
            __syncwarp();
            if (lane == 0) *reinterpret_cast<volatile uint32_t*>(fix_tail) = sl + 1;  // slot free again
        }
      }
    } else {
        ptx::regs_inc<kPPSoftmaxRegs>();
        // ---------------------------------------------------------------- softmax A / B
        const int x = (warp - 4) >> 2;   // 0: tile A, 1: tile B
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
        uint32_t ns = 0;   // S tiles seen
        int ni = 0;        // items seen
        bool ok = true;
        for (int rr = 0; ok; ++rr) {
            const int u = pp_item(rr, g, G, n_items);
            if (u < 0) break;
            const PPItem it = pp_decode(u, BH, H, n_qt, T, W, single);
            if (x == 1 && !it.hasB) continue;
            const int qt = x ? it.qt[1] : it.qt[0];
            const int fx = x ? it.f[1] : it.f[0];
            const int lx = x ? it.l[1] : it.l[0];
            const bool precise = pp_precise(qt, W);
            const int i = qt * 128 + r;
            int lo = i - W + 1;
            if (lo < 0) lo = 0;
            const int hi = i < T - 1 ? i : T - 1;
            float m_ref = -INFINITY, l = 0.f;
            float t_np = -INFINITY;  // largest scaled score met in a single-bf16-P tile
            for (int kt = fx; kt <= lx; ++kt) {
                bool w = ptx::mbar_wait(s_full + x, ns & 1, wait_limit_ns, abort_flag);
                ++ns;
                if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
                ptx::tc_fence_after();
                const bool edge = tile_class(T, W, 128, 128, qt, kt) != 2;
                const int cmin = lo - kt * 128, cmax = hi - kt * 128;
                const uint32_t scol = tl + C::colS(x), ocol = tl + C::colO(x);
                // S_x(kt) complete implies PV_x(kt-1) complete: nothing to wait for
                const auto none = [] {};
                // part s of P is in TMEM: the warp's stores have completed
                const auto hand = [&](int part) {
                    ptx::tmem_st_wait();
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(p_full + 4 * x + part);
                };
                // whether this warp wrote low parts of P, for the MMA issuer (before part 0's
                // arrival, which releases it)
                const auto publish = [&](bool lo_parts) {
                    if (lane == 0) lo_flag[4 * (2 * x + ((ns - 1) & 1)) + (warp & 3)] = lo_parts ? 1u : 0u;
                };
                if (adapt) {
                    // (tiles that always carry low parts take the same code with force set)
                    if (edge)
                        t_np = fmaxf(t_np, pp_tile<D, 1, false, true>(scol, ocol, scale_log2, m_ref, l, cmin, cmax, 0,
                                                                      -1, none, hand, publish, precise));
                    else
                        t_np = fmaxf(t_np, pp_tile<D, 0, false, true>(scol, ocol, scale_log2, m_ref, l, cmin, cmax, 0,
                                                                      -1, none, hand, publish, precise));
                } else if (edge) {
                    if (precise) pp_tile<D, 1, true>(scol, ocol, scale_log2, m_ref, l, cmin, cmax, 0, -1, none, hand);
                    else t_np = fmaxf(t_np, pp_tile<D, 1, false>(scol, ocol, scale_log2, m_ref, l, cmin, cmax, 0, -1, none, hand));
                } else {
                    if (precise) pp_tile<D, 0, true>(scol, ocol, scale_log2, m_ref, l, cmin, cmax, 0, -1, none, hand);
                    else t_np = fmaxf(t_np, pp_tile<D, 0, false>(scol, ocol, scale_log2, m_ref, l, cmin, cmax, 0, -1, none, hand));
                }
            }
            if (!ok) break;
            // ------------------------------------------------------------ epilogue
            bool w = ptx::mbar_wait(o_final + x, ni & 1, wait_limit_ns, abort_flag);
            ++ni;
            if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
            ptx::tc_fence_after();
            const float inv_l = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16* orow = out + it.b * osb + it.h * osh + (int64_t)i * ost;
            const auto store_chunk = [&](int cc, const uint32_t (&o)[32]) {
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    uint4 val;
                    val.x = ptx::pack_bf16x2(__uint_as_float(o[8 * t + 0]) * inv_l, __uint_as_float(o[8 * t + 1]) * inv_l);
                    val.y = ptx::pack_bf16x2(__uint_as_float(o[8 * t + 2]) * inv_l, __uint_as_float(o[8 * t + 3]) * inv_l);
                    val.z = ptx::pack_bf16x2(__uint_as_float(o[8 * t + 4]) * inv_l, __uint_as_float(o[8 * t + 5]) * inv_l);
                    val.w = ptx::pack_bf16x2(__uint_as_float(o[8 * t + 6]) * inv_l, __uint_as_float(o[8 * t + 7]) * inv_l);
                    *reinterpret_cast<uint4*>(orow + cc * 32 + t * 8) = val;
                }
            };
            // A row is sharp when one key of a single-bf16-P tile holds more than
            // kPPSharpShare of its weight (t_np and m_ref are both log2 units; l is in the
            // frame of m_ref) and some output reaches kPPSharpOut in magnitude, where the
            // output's own bf16 spacing leaves little of the error budget to the weights. A
            // sharp row is recomputed by the worker instead of stored from O.
            const bool dominated = i < T && t_np != -INFINITY && ptx::ex2(t_np - m_ref) > kPPSharpShare * l;
            bool sharp = false;
            if (__any_sync(0xffffffffu, dominated)) {
                // rare: the whole row of O first, to see its largest output
                uint32_t o[D / 32][32];
#pragma unroll
                for (int cc = 0; cc < D / 32; ++cc) ptx::tmem_ld32(tl + C::colO(x) + cc * 32, o[cc]);
                ptx::tmem_ld_wait();
                float big = 0.f;
#pragma unroll
                for (int cc = 0; cc < D / 32; ++cc) {
                    ptx::reg_fence(o[cc]);
#pragma unroll
                    for (int t = 0; t < 32; ++t) big = fmaxf(big, fabsf(__uint_as_float(o[cc][t])));
                }
                sharp = dominated && big * inv_l >= kPPSharpOut;
                if (i < T && !sharp) {
#pragma unroll
                    for (int cc = 0; cc < D / 32; ++cc) store_chunk(cc, o[cc]);
                }
            } else {
#pragma unroll 1
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t o[32];
                    ptx::tmem_ld32(tl + C::colO(x) + cc * 32, o);
                    ptx::tmem_ld_wait();
                    ptx::reg_fence(o);
                    if (i < T) store_chunk(cc, o);
                }
            }
            // natural log-sum-exp of the row's scaled scores: (m + log2 l) ln 2
            if (LSE && i < T && !sharp)
                lse[((int64_t)it.b * H + it.h) * T + i] = (m_ref + log2f(l)) * 0.6931471805599453f;
            ptx::tc_fence_before();
            ptx::mbar_arrive(o_free + x);  // O_x may be overwritten by the next item
            if (sharp && !pp_push_sharp(fix_head, fix_tail, fix_slot, it.b, it.h, i, wait_limit_ns, abort_flag)) {
                atomicCAS(status, 0, 5);
                *abort_flag = 1;
            }
            if (lane == 0) atomicAdd(fix_beat, 1u);  // progress, for the worker's time limit
        }
        __syncwarp();
        __threadfence_block();  // this warp's pushes are visible before it counts as done
        if (lane == 0) atomicAdd(fix_done, 1u);
        if (!ok) {
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
            // (the last Q tile of each set: the latest use of that set's barrier)
#pragma unroll
            for (int x = 0; x < 2; ++x)
                for (int n = nq[x] - 1; n >= 0 && n >= nq[x] - C::kQSets; --n)
                    ptx::mbar_wait(q_full + 2 * (n % C::kQSets) + x, (n / C::kQSets) & 1, kPPDrainLimitNs, nullptr);
            for (uint32_t st = 0; st < (uint32_t)NS && st < loads; ++st) {
                const uint32_t t = st + ((loads - 1 - st) / NS) * NS;
                ptx::mbar_wait(ring_full + st, (t / NS) & 1, kPPDrainLimitNs, nullptr);
            }
        }
        if (warp == 1 || (TWO && warp == 3)) {
            const int x = warp == 1 ? 0 : 1;
            ptx::tc_commit_one(drain + x);  // completes when every MMA this warp issued is done
            ptx::mbar_wait(drain + x, 0, kPPDrainLimitNs, nullptr);
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
