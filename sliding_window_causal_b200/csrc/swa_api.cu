// swa_api.cu: the C ABI declared in include/swa.h. Validates arguments, encodes the TMA
// tensor maps, picks a kernel by dtype and head dimension, and launches it on the
// caller's stream. No torch types cross this boundary.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <type_traits>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <map>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "swa.h"
#include "api_internal.h"
#include "backward.cuh"
#include "backward_tc.cuh"
#include "chunk.cuh"
#include "decode.cuh"
#include "plan.h"
#include "prefill_narrow.cuh"
#include "prefill_simt.cuh"
#include "prefill_pp.cuh"
#include "weights.cuh"

// Per-device status word: kernels record the first error here (atomicCAS from 0).
__device__ int g_swa_status = 0;

namespace {

thread_local std::string t_error;

int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    t_error = buf;
    return code;
}
int success() {
    t_error.clear();
    return SWA_OK;
}
int cuda_fail(cudaError_t e, const char* what) {
    return fail(SWA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;
std::atomic<uint64_t> g_wait_limit{0};
std::atomic<int> g_prefill_mode{SWA_PREFILL_AUTO};

uint64_t env_wait_limit() {
    static uint64_t v = [] {
        const char* s = getenv("SWA_WAIT_LIMIT_NS");
        if (s && *s) {
            unsigned long long x = strtoull(s, nullptr, 10);
            if (x > 0) return (uint64_t)x;
        }
        return kDefaultWaitLimitNs;
    }();
    return v;
}
uint64_t wait_limit() {
    uint64_t v = g_wait_limit.load();
    return v ? v : env_wait_limit();
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// ------------------------------------------------------------------ per-device state
std::mutex g_mu;

struct DeviceState {
    bool attrs_set = false;
    int* status = nullptr;  // device address of g_swa_status
    int num_sms = 0;
    bool pp_regs_ok = false;  // the persistent prefill kernels use exactly kPPLaunchRegs
    // SWA_PREFILL_AUTO's switch: a word of pinned host memory that the prefill kernel without
    // adaptive P sets (through its device mapping) when its inputs make many rows sharp
    volatile int* auto_host = nullptr;
    int* auto_dev = nullptr;
};
std::map<int, DeviceState> g_dev;

// The sixteen tensor-core prefill kernels (D 64/128, with and without the log-sum-exp, one or
// two MMA issuers, with and without adaptive P): set the shared-memory size, and check that
// each was compiled with the kPPLaunchRegs registers per thread that its register split
// assumes.
template <int D, bool LSE, bool TWO, bool ADAPT>
cudaError_t set_pp_attrs_one(bool* regs_ok) {
    cudaError_t e = cudaFuncSetAttribute(swa::prefill_pp_kernel<D, LSE, TWO, ADAPT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, swa::PPCfg<D, TWO>::kSmemBytes);
    cudaFuncAttributes a;
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&a, swa::prefill_pp_kernel<D, LSE, TWO, ADAPT>);
    if (e == cudaSuccess && a.numRegs != swa::kPPLaunchRegs) *regs_ok = false;
    return e;
}
template <int D, bool LSE, bool TWO>
cudaError_t set_pp_attrs(bool* regs_ok) {
    cudaError_t e = set_pp_attrs_one<D, LSE, TWO, false>(regs_ok);
    return e == cudaSuccess ? set_pp_attrs_one<D, LSE, TWO, true>(regs_ok) : e;
}

template <int D>
cudaError_t set_bwd_tc_attrs() {
    cudaError_t e = cudaFuncSetAttribute(swa::bwd_tc_kernel<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         swa::BwdTcCfg<D, true>::kSmemBytes);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(swa::bwd_tc_kernel<D, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 swa::BwdTcCfg<D, false>::kSmemBytes);
    return e;
}

template <typename TIn>
cudaError_t set_bwd_attrs() {
    const int bytes = (int)(swa::bwd_smem_floats(swa::kBwdMaxD) * 4);
    cudaError_t e = cudaFuncSetAttribute(swa::bwd_rows_kernel<TIn>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(swa::bwd_cols_kernel<TIn>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    return e;
}

int device_state(DeviceState** out) {
    int dev;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceState& st = g_dev[dev];
    if (!st.status) {
        e = cudaGetSymbolAddress(reinterpret_cast<void**>(&st.status), g_swa_status);
        if (e != cudaSuccess) {
            st.status = nullptr;
            return cuda_fail(e, "cudaGetSymbolAddress(status)");
        }
    }
    if (!st.auto_dev) {
        int* h = nullptr;
        e = cudaHostAlloc(reinterpret_cast<void**>(&h), sizeof(int), cudaHostAllocMapped);
        if (e != cudaSuccess) return cuda_fail(e, "cudaHostAlloc(prefill mode word)");
        *h = 0;
        e = cudaHostGetDevicePointer(reinterpret_cast<void**>(&st.auto_dev), h, 0);
        if (e != cudaSuccess) {
            cudaFreeHost(h);
            st.auto_dev = nullptr;
            return cuda_fail(e, "cudaHostGetDevicePointer(prefill mode word)");
        }
        st.auto_host = h;
    }
    if (!st.attrs_set) {
        e = cudaSuccess;
        bool regs_ok = true;  // the register split inside the kernels assumes this launch allocation
        if (e == cudaSuccess) e = set_pp_attrs<128, false, false>(&regs_ok);
        if (e == cudaSuccess) e = set_pp_attrs<128, true, false>(&regs_ok);
        if (e == cudaSuccess) e = set_pp_attrs<128, false, true>(&regs_ok);
        if (e == cudaSuccess) e = set_pp_attrs<128, true, true>(&regs_ok);
        if (e == cudaSuccess) e = set_pp_attrs<64, false, false>(&regs_ok);
        if (e == cudaSuccess) e = set_pp_attrs<64, true, false>(&regs_ok);
        if (e == cudaSuccess) e = set_pp_attrs<64, false, true>(&regs_ok);
        if (e == cudaSuccess) e = set_pp_attrs<64, true, true>(&regs_ok);
        st.pp_regs_ok = e == cudaSuccess && regs_ok;
        if (e == cudaSuccess) e = set_bwd_tc_attrs<64>();
        if (e == cudaSuccess) e = set_bwd_tc_attrs<128>();
        if (e == cudaSuccess) e = set_bwd_attrs<float>();
        if (e == cudaSuccess) e = set_bwd_attrs<__nv_bfloat16>();
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(swa::chunk_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     swa::ChunkCfg<128>::kSmemBytes);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(swa::chunk_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     swa::ChunkCfg<64>::kSmemBytes);
        if (e == cudaSuccess)
            e = cudaDeviceGetAttribute(&st.num_sms, cudaDevAttrMultiProcessorCount, dev);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(swa::prefill_simt_kernel,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     swa::kSimtWarps * (2 * 4096 + 32) * 4);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(swa::band_weights_kernel<float>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     swa::kWeightWarps * 4096 * 4);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(swa::band_weights_kernel<__nv_bfloat16>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     swa::kWeightWarps * 4096 * 4);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        st.attrs_set = true;
    }
    *out = &st;
    return SWA_OK;
}

// ------------------------------------------------------------------ TMA tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return (EncodeTiledFn) nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// A bf16 [B, H, T, D] tensor with element strides st = (b, h, t) (D contiguous), viewed as
// the 4-D tensor {D, T, H, B}: boxes of 64 columns x 128 rows of one (b, h), 128-byte
// swizzle. Rows past T read as zeros.
int make_map(CUtensorMap* m, const void* ptr, int64_t B, int64_t H, int64_t T, int64_t D,
             const int64_t st[3]) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return fail(SWA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)T, (cuuint64_t)H, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)(st[2] * 2), (cuuint64_t)(st[1] * 2), (cuuint64_t)(st[0] * 2)};
    cuuint32_t box[4] = {64, 128, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(SWA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return SWA_OK;
}

// Element strides (b, h, t) of q, k, v and out. NULL means contiguous [B, H, T, D]. The
// stride of a dimension of size 1 is never used to address memory; it is replaced by the
// contiguous one so that every stride the TMA unit sees is valid.
int read_strides(const char* fn, const int64_t* in, int n, int64_t B, int64_t H, int64_t T,
                 int64_t D, int64_t out[][3]) {
    const int64_t dense[3] = {H * T * D, T * D, D};
    const int64_t size[3] = {B, H, T};
    for (int a = 0; a < n; ++a)
        for (int x = 0; x < 3; ++x) {
            int64_t v = in ? in[3 * a + x] : dense[x];
            if (v < 0 || v > (int64_t(1) << 38))
                return fail(SWA_ERR_INVALID_ARG, "%s: stride %lld of operand %d is negative or too large",
                            fn, (long long)v, a);
            if (size[x] == 1) v = dense[x];
            out[a][x] = v;
        }
    return SWA_OK;
}

// ------------------------------------------------------------------ decode workspace
// Per (device, stream): the split partial states (m, l, acc[D]) and, in a separate
// allocation, one ticket counter per stream. Every counter is zero between calls: the
// allocation is zeroed and the last CTA of each stream resets its counter.
struct Workspace {
    void* part = nullptr;
    size_t part_bytes = 0;
    int* counters = nullptr;
    size_t n_counters = 0;
};
std::map<std::pair<int, void*>, Workspace> g_ws;

int decode_workspace(void* stream, size_t part_need, size_t counters_need, float** part,
                     int** counters) {
    int dev;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    std::lock_guard<std::mutex> lk(g_mu);
    Workspace& w = g_ws[std::make_pair(dev, stream)];
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (w.part_bytes < part_need || w.n_counters < counters_need) {
        // the stream may still be using the old buffers
        e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    }
    if (w.part_bytes < part_need) {
        if (w.part) cudaFree(w.part);
        w.part = nullptr;
        w.part_bytes = 0;
        e = cudaMalloc(&w.part, part_need);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(decode partials)");
        w.part_bytes = part_need;
    }
    if (w.n_counters < counters_need) {
        if (w.counters) cudaFree(w.counters);
        w.counters = nullptr;
        w.n_counters = 0;
        e = cudaMalloc(&w.counters, counters_need * sizeof(int));
        if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(decode counters)");
        e = cudaMemsetAsync(w.counters, 0, counters_need * sizeof(int), s);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
        w.n_counters = counters_need;
    }
    *part = static_cast<float*>(w.part);
    *counters = w.counters;
    return SWA_OK;
}

// The splits are the grid's y dimension, whose limit is 65535 blocks. The library's own
// plan stays below 148 * 16; only a small SWA_DECODE_CHUNK over a long ring can exceed it.
constexpr int kMaxDecodeSplits = 65535;

void split_plan(int64_t B, int64_t H, int64_t D, int64_t W, int32_t* splits, int32_t* chunk) {
    const int64_t rows_per_batch = (D == 64) ? swa::DecodeCfg<64>::kRowsPerBatch
                                             : swa::DecodeCfg<128>::kRowsPerBatch;
    int64_t c = 0;
    if (const char* e = getenv("SWA_DECODE_CHUNK")) c = strtoll(e, nullptr, 10);
    if (c <= 0) {
        // Enough CTAs to keep ~16 resident per SM on 148 SMs, chunks of whole batches.
        const int64_t target = 148 * 16;
        int64_t S = (target + B * H - 1) / (B * H);
        if (S < 1) S = 1;
        c = (W + S - 1) / S;
    }
    c = ((c + rows_per_batch - 1) / rows_per_batch) * rows_per_batch;
    if (c > W) c = ((W + rows_per_batch - 1) / rows_per_batch) * rows_per_batch;
    *chunk = (int32_t)c;
    *splits = (int32_t)((W + c - 1) / c);
}

// Checks shared by the prefill entry points. OK means "go on" (B*H*T may still be 0).
int check_sizes(const char* fn, int64_t B, int64_t H, int64_t T, int64_t D, int64_t W, int dtype,
                double scale) {
    if (dtype != SWA_F32 && dtype != SWA_BF16)
        return fail(SWA_ERR_INVALID_ARG, "%s: dtype %d is neither SWA_F32 nor SWA_BF16", fn, dtype);
    if (W < 1) return fail(SWA_ERR_INVALID_ARG, "%s: window W=%lld must be >= 1", fn, (long long)W);
    if (B < 0 || H < 0 || T < 0)
        return fail(SWA_ERR_INVALID_ARG, "%s: negative size B=%lld H=%lld T=%lld", fn, (long long)B,
                    (long long)H, (long long)T);
    if (D < 1) return fail(SWA_ERR_INVALID_ARG, "%s: head dim D=%lld must be >= 1", fn, (long long)D);
    if (!std::isfinite(scale)) return fail(SWA_ERR_INVALID_ARG, "%s: scale must be finite", fn);
    if (B > INT32_MAX || H > INT32_MAX || T > INT32_MAX || (B > 0 && H > INT32_MAX / B) ||
        (T > 0 && B * H > INT64_MAX / T) || (B * H * T > 0 && B * H * T > INT64_MAX / D / 4))
        return fail(SWA_ERR_UNSUPPORTED, "%s: sizes too large", fn);
    return SWA_OK;
}

}  // namespace

namespace swa_internal {

int check_forward(const char* fn, const void* q, const void* k, const void* v, const void* out, int64_t B,
                  int64_t H, int64_t T, int64_t D, int64_t W, double scale, const int64_t* strides, int dtype,
                  int64_t st[4][3]) {
    if (int rc = check_sizes(fn, B, H, T, D, W, dtype, scale)) return rc;
    if (B == 0 || H == 0 || T == 0) return SWA_OK;
    if (!q || !k || !v || !out) return fail(SWA_ERR_INVALID_ARG, "%s: null pointer", fn);
    if (int rc = read_strides(fn, strides, 4, B, H, T, D, st)) return rc;
    if (dtype == SWA_BF16) {
        if (D != 64 && D != 128)
            return fail(SWA_ERR_UNSUPPORTED, "%s: bf16 needs D = 64 or 128 (got %lld)", fn, (long long)D);
        // The kernel takes the row maximum of the raw scores and scales it, which is the
        // maximum of the scaled scores only for a positive scale.
        if (!(scale > 0.0))
            return fail(SWA_ERR_UNSUPPORTED, "%s: the bf16 path needs scale > 0 (got %g)", fn, scale);
        if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
            return fail(SWA_ERR_MISALIGNED, "%s: bf16 tensors must be 16-byte aligned", fn);
        for (int a = 0; a < 4; ++a)
            for (int x = 0; x < 3; ++x)
                if (st[a][x] % 8 != 0)
                    return fail(SWA_ERR_MISALIGNED,
                                "%s: bf16 strides must be multiples of 8 elements (16 bytes); operand %d "
                                "has stride %lld",
                                fn, a, (long long)st[a][x]);
        if ((T + 127) / 128 * (B * H) > INT32_MAX) return fail(SWA_ERR_UNSUPPORTED, "%s: too many tiles", fn);
        if ((W < T ? W : T) <= swa::kNarrowMaxW && (T + swa::kNarrowRows - 1) / swa::kNarrowRows * (B * H) > INT32_MAX)
            return fail(SWA_ERR_UNSUPPORTED, "%s: too many row blocks", fn);
    } else {
        if (D > 4096) return fail(SWA_ERR_UNSUPPORTED, "%s: fp32 supports D <= 4096", fn);
        if (!aligned(q, 4) || !aligned(k, 4) || !aligned(v, 4) || !aligned(out, 4))
            return fail(SWA_ERR_MISALIGNED, "%s: fp32 tensors must be 4-byte aligned", fn);
        if ((B * H * T + swa::kSimtWarps - 1) / swa::kSimtWarps > INT32_MAX)
            return fail(SWA_ERR_UNSUPPORTED, "%s: too many rows", fn);
    }
    return SWA_OK;
}

}  // namespace swa_internal

namespace {

int forward_impl(const char* fn, const void* q, const void* k, const void* v, void* out, int64_t B,
                 int64_t H, int64_t T, int64_t D, int64_t W, double scale, const int64_t* strides,
                 int dtype, void* stream, float* lse = nullptr) {
    int64_t st[4][3];
    if (int rc = swa_internal::check_forward(fn, q, k, v, out, B, H, T, D, W, scale, strides, dtype, st))
        return rc;
    if (B == 0 || H == 0 || T == 0) return success();
    const int Wi = (int)(W < T ? W : T);  // W >= T is causal attention
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    DeviceState* ds;
    if (int rc = device_state(&ds)) return rc;

    if (dtype == SWA_BF16 && Wi <= swa::kNarrowMaxW) {
        // bands of a few keys: bound by HBM, served on the CUDA cores without the tensor-core
        // pipeline's fill and drain
        const int64_t BH = B * H;
        const int n_rb = (int)((T + swa::kNarrowRows - 1) / swa::kNarrowRows);
        swa::Strides sx;
        for (int x = 0; x < 3; ++x) {
            sx.q[x] = st[0][x];
            sx.k[x] = st[1][x];
            sx.v[x] = st[2][x];
            sx.o[x] = st[3][x];
        }
        const float scale_log2 = (float)(1.4426950408889634 * scale);
        const auto* qb = static_cast<const __nv_bfloat16*>(q);
        const auto* kb = static_cast<const __nv_bfloat16*>(k);
        const auto* vb = static_cast<const __nv_bfloat16*>(v);
        auto* ob = static_cast<__nv_bfloat16*>(out);
        const unsigned grid = (unsigned)(BH * n_rb);
        if (D == 128)
            swa::prefill_narrow_kernel<128><<<grid, swa::kNarrowWarps * 32, 0, s>>>(qb, kb, vb, ob, sx, lse, (int)H,
                                                                                 (int)T, Wi, scale_log2, n_rb);
        else
            swa::prefill_narrow_kernel<64><<<grid, swa::kNarrowWarps * 32, 0, s>>>(qb, kb, vb, ob, sx, lse, (int)H,
                                                                                (int)T, Wi, scale_log2, n_rb);
    } else if (dtype == SWA_BF16) {
        const int64_t BH = B * H;
        const int n_qt = (int)((T + 127) / 128);
        CUtensorMap mq, mk, mv;
        int rc;
        if ((rc = make_map(&mq, q, B, H, T, D, st[0])) || (rc = make_map(&mk, k, B, H, T, D, st[1])) ||
            (rc = make_map(&mv, v, B, H, T, D, st[2])))
            return rc;
        const float scale_log2 = (float)(1.4426950408889634 * scale);
        if (!ds->pp_regs_ok)
            return fail(SWA_ERR_UNSUPPORTED, "%s: prefill kernel was not compiled with %d registers per thread",
                        fn, swa::kPPLaunchRegs);
        // pairs of query tiles as work items; single tiles when there are fewer pairs than SMs
        // (the kernel tells the two apart by the grid size)
        const int64_t n_pairs = (int64_t)((n_qt + 1) / 2) * BH;
        const int64_t n_items = n_pairs < ds->num_sms ? (int64_t)n_qt * BH : n_pairs;
        const unsigned G = (unsigned)(n_items < ds->num_sms ? n_items : ds->num_sms);
        auto* ob = static_cast<__nv_bfloat16*>(out);
        swa::PPRaw raw;
        raw.q = static_cast<const __nv_bfloat16*>(q);
        raw.k = static_cast<const __nv_bfloat16*>(k);
        raw.v = static_cast<const __nv_bfloat16*>(v);
        for (int x = 0; x < 3; ++x) {
            raw.sq[x] = st[0][x];
            raw.sk[x] = st[1][x];
            raw.sv[x] = st[2][x];
        }
        // Bands of at most kPPTwoIssuerWindow keys are short: an item's pipeline fills and
        // drains every few tiles, and one MMA issuer per query tile keeps either tile from
        // waiting on the other's P. Longer bands keep the single issuer, whose ping-pong order
        // completes each tile's scores sooner.
        const bool two = Wi <= swa::kPPTwoIssuerWindow;
        // adaptive P when asked for, or when an earlier launch on this device in AUTO mode
        // met inputs that make many rows sharp (the kernel without it sets the word)
        const int mode = g_prefill_mode.load();
        const bool adapt = mode == SWA_PREFILL_ADAPTIVE || (mode == SWA_PREFILL_AUTO && *ds->auto_host != 0);
        int* auto_flag = mode == SWA_PREFILL_AUTO ? ds->auto_dev : nullptr;
        auto launch = [&](auto kern, int smem) {
            kern<<<G, swa::kPPThreads, smem, s>>>(mq, mk, mv, ob, st[3][0], st[3][1], st[3][2], lse, (int)BH, (int)H,
                                                 (int)T, Wi, n_qt, scale_log2, wait_limit(), ds->status, raw, auto_flag);
        };
        constexpr int S128 = swa::PPCfg<128, false>::kSmemBytes, S64 = swa::PPCfg<64, false>::kSmemBytes;
        constexpr int S128t = swa::PPCfg<128, true>::kSmemBytes, S64t = swa::PPCfg<64, true>::kSmemBytes;
        // one launch of the instantiation <D, lse, two, adapt>
        auto pick = [&](auto d_tag, int smem1, int smem2) {
            constexpr int DD = decltype(d_tag)::value;
            if (lse) {
                if (two) adapt ? launch(swa::prefill_pp_kernel<DD, true, true, true>, smem2) : launch(swa::prefill_pp_kernel<DD, true, true, false>, smem2);
                else adapt ? launch(swa::prefill_pp_kernel<DD, true, false, true>, smem1) : launch(swa::prefill_pp_kernel<DD, true, false, false>, smem1);
            } else {
                if (two) adapt ? launch(swa::prefill_pp_kernel<DD, false, true, true>, smem2) : launch(swa::prefill_pp_kernel<DD, false, true, false>, smem2);
                else adapt ? launch(swa::prefill_pp_kernel<DD, false, false, true>, smem1) : launch(swa::prefill_pp_kernel<DD, false, false, false>, smem1);
            }
        };
        if (D == 128) pick(std::integral_constant<int, 128>(), S128, S128t);
        else pick(std::integral_constant<int, 64>(), S64, S64t);
    } else {
        const int64_t nrows = B * H * T;
        const int64_t blocks = (nrows + swa::kSimtWarps - 1) / swa::kSimtWarps;
        const size_t smem = (size_t)swa::kSimtWarps * (2 * D + 32) * sizeof(float);
        swa::Strides sx;
        for (int x = 0; x < 3; ++x) {
            sx.q[x] = st[0][x];
            sx.k[x] = st[1][x];
            sx.v[x] = st[2][x];
            sx.o[x] = st[3][x];
        }
        swa::prefill_simt_kernel<<<(unsigned)blocks, swa::kSimtWarps * 32, smem, s>>>(
            static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
            static_cast<float*>(out), sx, lse, nrows, (int)H, (int)T, (int)D, Wi, (float)scale);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "swa_forward launch");
    return success();
}

// ------------------------------------------------------------------ host-buffer pipeline
// Per device: the three streams of swa_forward_host (host-to-device copies, attention,
// device-to-host copies) and a pool of events that order them. Created on first use and
// kept until exit. A call holds `mu` while it enqueues, so calls from several host
// threads take the streams one after another.
struct HostPipe {
    std::mutex mu;
    cudaStream_t in = nullptr, cmp = nullptr, out = nullptr;
    std::vector<cudaEvent_t> ev;
};
std::map<int, HostPipe> g_pipe;

HostPipe& host_pipe(int dev) {
    std::lock_guard<std::mutex> lk(g_mu);
    return g_pipe[dev];
}

// Streams and at least n_events events; the caller holds hp.mu.
int host_pipe_ready(HostPipe& hp, size_t n_events) {
    cudaError_t e = cudaSuccess;
    for (cudaStream_t* st : {&hp.in, &hp.cmp, &hp.out})
        if (!*st && e == cudaSuccess) e = cudaStreamCreateWithFlags(st, cudaStreamNonBlocking);
    while (e == cudaSuccess && hp.ev.size() < n_events) {
        cudaEvent_t x;
        e = cudaEventCreateWithFlags(&x, cudaEventDisableTiming);
        if (e == cudaSuccess) hp.ev.push_back(x);
    }
    if (e != cudaSuccess) return cuda_fail(e, "swa_forward_host: stream/event creation");
    return SWA_OK;
}

}  // namespace

// ==================================================================== C ABI
extern "C" {

const char* swa_last_error(void) { return t_error.c_str(); }

uint64_t swa_set_wait_limit_ns(uint64_t ns) {
    uint64_t prev = wait_limit();
    g_wait_limit.store(ns);
    return prev;
}

int swa_set_prefill_mode(int mode) {
    if (mode != SWA_PREFILL_AUTO && mode != SWA_PREFILL_ADAPTIVE && mode != SWA_PREFILL_FAST) {
        fail(SWA_ERR_INVALID_ARG, "swa_set_prefill_mode: mode %d", mode);
        return -1;
    }
    return g_prefill_mode.exchange(mode);
}

int swa_prefill_auto_state(int clear) {
    DeviceState* ds;
    if (device_state(&ds)) return -1;
    const int v = *ds->auto_host;
    if (clear) *ds->auto_host = 0;
    return v;
}

int swa_prefill_tile_class(int64_t T, int64_t W, int64_t bm, int64_t bn, int64_t qt, int64_t kt) {
    if (T < 1 || W < 1 || bm < 1 || bn < 1 || qt < 0 || kt < 0 || qt * bm >= T) return -1;
    return swa::tile_class(T, W, bm, bn, qt, kt);
}

int swa_prefill_work_item(int64_t u, int64_t B, int64_t H, int64_t T, int64_t W, int64_t* b, int64_t* h,
                          int64_t* pair) {
    if (B < 1 || H < 1 || T < 1 || W < 1 || !b || !h || !pair || B > INT32_MAX || H > INT32_MAX || T > INT32_MAX)
        return -1;
    int64_t bh;
    if (!swa::prefill_item<int64_t>(u, B * H, (T + 127) / 128, W < T ? W : T, &bh, pair)) return -1;
    *b = bh / H;
    *h = bh % H;
    return 0;
}

int swa_backward_cta_tile(int64_t u, int64_t B, int64_t H, int64_t T, int64_t W, int kv, int64_t* b, int64_t* h,
                          int64_t* tile) {
    if (B < 1 || H < 1 || T < 1 || W < 1 || !b || !h || !tile || B > INT32_MAX || H > INT32_MAX || T > INT32_MAX)
        return -1;
    int64_t bh;
    if (!swa::bwd_cta_tile<int64_t>(u, B * H, (T + 127) / 128, W < T ? W : T, kv != 0, &bh, tile)) return -1;
    *b = bh / H;
    *h = bh % H;
    return 0;
}

int64_t swa_decode_valid_slots(int64_t pos, int64_t W) {
    if (pos < 0 || W < 1) return -1;
    return swa::decode_valid_slots(pos, W);
}

int swa_decode_split_plan(int64_t B, int64_t H, int64_t D, int64_t W, int32_t* splits,
                          int32_t* chunk) {
    if (B < 1 || H < 1 || W < 1 || (D != 64 && D != 128) || !splits || !chunk)
        return fail(SWA_ERR_INVALID_ARG, "swa_decode_split_plan: bad arguments");
    split_plan(B, H, D, W, splits, chunk);
    return success();
}

int swa_forward(const void* q, const void* k, const void* v, void* out, int64_t B, int64_t H,
                int64_t T, int64_t D, int64_t W, int dtype, void* stream) {
    return forward_impl("swa_forward", q, k, v, out, B, H, T, D, W,
                        D >= 1 ? 1.0 / std::sqrt((double)D) : 0.0, nullptr, dtype, stream);
}

int swa_forward_host(const void* q, const void* k, const void* v, void* out, void* dq, void* dk, void* dv,
                     void* dout, int64_t B, int64_t H, int64_t T, int64_t D, int64_t W, int64_t heads_per_group,
                     int dtype, void* stream) {
    const char* fn = "swa_forward_host";
    const double scale = D >= 1 ? 1.0 / std::sqrt((double)D) : 0.0;
    int64_t st[4][3];
    if (int rc = swa_internal::check_forward(fn, dq, dk, dv, dout, B, H, T, D, W, scale, nullptr, dtype, st))
        return rc;
    if (B == 0 || H == 0 || T == 0) return success();
    if (!q || !k || !v || !out) return fail(SWA_ERR_INVALID_ARG, "%s: null host pointer", fn);
    if (heads_per_group < 0) return fail(SWA_ERR_INVALID_ARG, "%s: heads_per_group < 0", fn);
    const int64_t BH = B * H;
    int64_t hpg = heads_per_group > 0 ? heads_per_group : (BH + 7) / 8;  // about 8 groups
    if (hpg > BH) hpg = BH;
    const int64_t n_groups = (BH + hpg - 1) / hpg;
    const size_t head_bytes = (size_t)T * (size_t)D * (dtype == SWA_BF16 ? 2 : 4);
    int dev;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    HostPipe* hp = &host_pipe(dev);
    std::lock_guard<std::mutex> lk(hp->mu);
    if (int rc = host_pipe_ready(*hp, (size_t)(2 * n_groups + 2))) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaEvent_t* ev = hp->ev.data();  // [0] start, [1] done, then (copied in, computed) per group
    auto bytes_at = [&](const void* base, int64_t g0) {
        return static_cast<const char*>(base) + (size_t)g0 * head_bytes;
    };
    // everything already on the caller's stream (earlier users of the staging buffers) first
    if ((e = cudaEventRecord(ev[0], s)) != cudaSuccess || (e = cudaStreamWaitEvent(hp->in, ev[0], 0)) != cudaSuccess)
        return cuda_fail(e, "swa_forward_host: ordering after the caller's stream");
    for (int64_t g = 0; g < n_groups; ++g) {
        const int64_t g0 = g * hpg, nh = (g0 + hpg <= BH ? hpg : BH - g0);
        const size_t nb = (size_t)nh * head_bytes;
        cudaEvent_t e_in = ev[2 + 2 * g], e_cmp = ev[3 + 2 * g];
        // the (b, h) heads are independent problems: heads g0 .. g0+nh-1 of the contiguous
        // [B,H,T,D] tensors are one [1, nh, T, D] problem
        if ((e = cudaMemcpyAsync(const_cast<char*>(bytes_at(dq, g0)), bytes_at(q, g0), nb, cudaMemcpyHostToDevice, hp->in)) ||
            (e = cudaMemcpyAsync(const_cast<char*>(bytes_at(dk, g0)), bytes_at(k, g0), nb, cudaMemcpyHostToDevice, hp->in)) ||
            (e = cudaMemcpyAsync(const_cast<char*>(bytes_at(dv, g0)), bytes_at(v, g0), nb, cudaMemcpyHostToDevice, hp->in)) ||
            (e = cudaEventRecord(e_in, hp->in)) || (e = cudaStreamWaitEvent(hp->cmp, e_in, 0)))
            return cuda_fail(e, "swa_forward_host: host-to-device copies");
        if (int rc = forward_impl(fn, bytes_at(dq, g0), bytes_at(dk, g0), bytes_at(dv, g0),
                                  const_cast<char*>(bytes_at(dout, g0)), 1, nh, T, D, W, scale, nullptr, dtype,
                                  hp->cmp))
            return rc;
        if ((e = cudaEventRecord(e_cmp, hp->cmp)) || (e = cudaStreamWaitEvent(hp->out, e_cmp, 0)) ||
            (e = cudaMemcpyAsync(const_cast<char*>(bytes_at(out, g0)), bytes_at(dout, g0), nb, cudaMemcpyDeviceToHost,
                                 hp->out)))
            return cuda_fail(e, "swa_forward_host: device-to-host copy");
    }
    if ((e = cudaEventRecord(ev[1], hp->out)) != cudaSuccess || (e = cudaStreamWaitEvent(s, ev[1], 0)) != cudaSuccess)
        return cuda_fail(e, "swa_forward_host: ordering the caller's stream after the copies");
    return success();
}

int swa_forward_ex(const void* q, const void* k, const void* v, void* out, int64_t B, int64_t H,
                   int64_t T, int64_t D, int64_t W, double scale, const int64_t* strides, int dtype,
                   void* stream) {
    return forward_impl("swa_forward_ex", q, k, v, out, B, H, T, D, W, scale, strides, dtype, stream);
}

int swa_band_weights(const void* q, const void* k, float* weights, int64_t B, int64_t H, int64_t T,
                     int64_t D, int64_t W, double scale, const int64_t* strides, int dtype,
                     void* stream) {
    const char* fn = "swa_band_weights";
    if (int rc = check_sizes(fn, B, H, T, D, W, dtype, scale)) return rc;
    if (B == 0 || H == 0 || T == 0) return success();
    if (!q || !k || !weights) return fail(SWA_ERR_INVALID_ARG, "%s: null pointer", fn);
    const int64_t Wo = W < T ? W : T;
    if (D > 4096) return fail(SWA_ERR_UNSUPPORTED, "%s: D <= 4096", fn);
    if (B * H * T > INT64_MAX / Wo / 4) return fail(SWA_ERR_UNSUPPORTED, "%s: sizes too large", fn);
    const size_t esz = dtype == SWA_BF16 ? 2 : 4;
    if (!aligned(q, esz) || !aligned(k, esz) || !aligned(weights, 4))
        return fail(SWA_ERR_MISALIGNED, "%s: tensors must be aligned to their element size", fn);
    int64_t st[2][3] = {};
    if (int rc = read_strides(fn, strides, 2, B, H, T, D, st)) return rc;
    const int64_t nrows = B * H * T;
    const int64_t blocks = (nrows + swa::kWeightWarps - 1) / swa::kWeightWarps;
    if (blocks > INT32_MAX) return fail(SWA_ERR_UNSUPPORTED, "%s: too many rows", fn);
    DeviceState* ds;
    if (int rc = device_state(&ds)) return rc;
    const size_t smem = (size_t)swa::kWeightWarps * D * sizeof(float);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dtype == SWA_BF16)
        swa::band_weights_kernel<__nv_bfloat16><<<(unsigned)blocks, swa::kWeightWarps * 32, smem, s>>>(
            static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), weights,
            st[0][0], st[0][1], st[0][2], st[1][0], st[1][1], st[1][2], nrows, (int)H, (int)T, (int)D,
            (int)Wo, (float)scale);
    else
        swa::band_weights_kernel<float><<<(unsigned)blocks, swa::kWeightWarps * 32, smem, s>>>(
            static_cast<const float*>(q), static_cast<const float*>(k), weights, st[0][0], st[0][1],
            st[0][2], st[1][0], st[1][1], st[1][2], nrows, (int)H, (int)T, (int)D, (int)Wo, (float)scale);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "swa_band_weights launch");
    return success();
}

int swa_decode(const void* q, const void* kring, const void* vring, const int64_t* pos, void* out,
               int64_t B, int64_t H, int64_t D, int64_t W, void* stream) {
    if (W < 1) return fail(SWA_ERR_INVALID_ARG, "swa_decode: window W=%lld must be >= 1", (long long)W);
    if (B < 0 || H < 0)
        return fail(SWA_ERR_INVALID_ARG, "swa_decode: negative size B=%lld H=%lld", (long long)B, (long long)H);
    if (D < 1) return fail(SWA_ERR_INVALID_ARG, "swa_decode: head dim D=%lld must be >= 1", (long long)D);
    if (B == 0 || H == 0) return success();
    if (!q || !kring || !vring || !pos || !out) return fail(SWA_ERR_INVALID_ARG, "swa_decode: null pointer");
    if (D != 64 && D != 128)
        return fail(SWA_ERR_UNSUPPORTED, "swa_decode: D must be 64 or 128 (got %lld)", (long long)D);
    if (!aligned(q, 16) || !aligned(kring, 16) || !aligned(vring, 16) || !aligned(out, 16) ||
        !aligned(pos, 8))
        return fail(SWA_ERR_MISALIGNED, "swa_decode: tensors must be 16-byte aligned (pos 8-byte)");
    if (B * H > INT32_MAX || W > INT32_MAX / 2 || B * H > INT64_MAX / W / D)
        return fail(SWA_ERR_UNSUPPORTED, "swa_decode: sizes too large");
    int32_t S, chunk;
    split_plan(B, H, D, W, &S, &chunk);
    if (S > kMaxDecodeSplits)
        return fail(SWA_ERR_UNSUPPORTED, "swa_decode: %d splits exceed the grid limit of %d (a larger SWA_DECODE_CHUNK)",
                    (int)S, kMaxDecodeSplits);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    DeviceState* ds;
    if (int rc = device_state(&ds)) return rc;
    float* part = nullptr;
    int* counters = nullptr;
    if (S > 1) {
        const size_t part_bytes = (size_t)(B * H) * S * (D + 2) * sizeof(float);
        if (int rc = decode_workspace(stream, part_bytes, (size_t)(B * H), &part, &counters))
            return rc;
    }
    const float scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
    const dim3 grid((unsigned)(B * H), (unsigned)S);
    const auto* qb = static_cast<const __nv_bfloat16*>(q);
    const auto* kb = static_cast<const __nv_bfloat16*>(kring);
    const auto* vb = static_cast<const __nv_bfloat16*>(vring);
    auto* ob = static_cast<__nv_bfloat16*>(out);
    if (D == 128)
        swa::decode_kernel<128><<<grid, swa::kDecodeWarps * 32, 0, s>>>(
            qb, kb, vb, pos, ob, (int)H, (int)W, chunk, S, scale_log2, part, counters, ds->status);
    else
        swa::decode_kernel<64><<<grid, swa::kDecodeWarps * 32, 0, s>>>(
            qb, kb, vb, pos, ob, (int)H, (int)W, chunk, S, scale_log2, part, counters, ds->status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "swa_decode launch");
    return success();
}

}  // extern "C"

namespace {
// Checks shared by the streaming entry points (chunk attention and ring append).
int check_stream_args(const char* fn, int64_t B, int64_t H, int64_t C, int64_t D, int64_t W) {
    if (W < 1) return fail(SWA_ERR_INVALID_ARG, "%s: window W=%lld must be >= 1", fn, (long long)W);
    if (B < 0 || H < 0 || C < 0)
        return fail(SWA_ERR_INVALID_ARG, "%s: negative size B=%lld H=%lld C=%lld", fn, (long long)B,
                    (long long)H, (long long)C);
    if (D < 1) return fail(SWA_ERR_INVALID_ARG, "%s: head dim D=%lld must be >= 1", fn, (long long)D);
    if (B * H * C == 0) return SWA_OK;
    if (D != 64 && D != 128)
        return fail(SWA_ERR_UNSUPPORTED, "%s: D must be 64 or 128 (got %lld)", fn, (long long)D);
    if (B > INT32_MAX || H > INT32_MAX || B * H > INT32_MAX || C > INT32_MAX || W > INT32_MAX / 2 ||
        B * H > INT64_MAX / (W > C ? W : C) / D)
        return fail(SWA_ERR_UNSUPPORTED, "%s: sizes too large", fn);
    return SWA_OK;
}

int launch_append(const char* fn, const void* k, const void* v, void* kring, void* vring, const int64_t* pos,
                  int64_t B, int64_t H, int64_t C, int64_t D, int64_t W, cudaStream_t s, int* status) {
    const int64_t c_first = C > W ? C - W : 0;
    const int vpr = (int)(D / 8);
    const int64_t n_vec = B * H * (C - c_first) * vpr;
    int64_t blocks = (n_vec + 255) / 256;
    if (blocks > 148 * 32) blocks = 148 * 32;
    swa::ring_append_kernel<<<(unsigned)blocks, 256, 0, s>>>(
        static_cast<const uint4*>(k), static_cast<const uint4*>(v), static_cast<uint4*>(kring),
        static_cast<uint4*>(vring), pos, (int)H, (int)C, (int)W, vpr, (int)c_first, n_vec, status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, fn);
    return SWA_OK;
}
}  // namespace

extern "C" {

int swa_ring_append(const void* k, const void* v, void* kring, void* vring, const int64_t* pos, int64_t B,
                    int64_t H, int64_t C, int64_t D, int64_t W, void* stream) {
    const char* fn = "swa_ring_append";
    if (int rc = check_stream_args(fn, B, H, C, D, W)) return rc;
    if (B * H * C == 0) return success();
    if (!k || !v || !kring || !vring || !pos) return fail(SWA_ERR_INVALID_ARG, "%s: null pointer", fn);
    if (!aligned(k, 16) || !aligned(v, 16) || !aligned(kring, 16) || !aligned(vring, 16) || !aligned(pos, 8))
        return fail(SWA_ERR_MISALIGNED, "%s: tensors must be 16-byte aligned (pos 8-byte)", fn);
    DeviceState* ds;
    if (int rc = device_state(&ds)) return rc;
    if (int rc = launch_append(fn, k, v, kring, vring, pos, B, H, C, D, W, static_cast<cudaStream_t>(stream),
                               ds->status))
        return rc;
    return success();
}

int swa_chunk_forward(const void* q, const void* k, const void* v, void* kring, void* vring,
                      const int64_t* pos, void* out, int64_t B, int64_t H, int64_t C, int64_t D, int64_t W,
                      void* stream) {
    const char* fn = "swa_chunk_forward";
    if (int rc = check_stream_args(fn, B, H, C, D, W)) return rc;
    if (B * H * C == 0) return success();
    if (!q || !k || !v || !kring || !vring || !pos || !out)
        return fail(SWA_ERR_INVALID_ARG, "%s: null pointer", fn);
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(kring, 16) || !aligned(vring, 16) ||
        !aligned(out, 16) || !aligned(pos, 8))
        return fail(SWA_ERR_MISALIGNED, "%s: tensors must be 16-byte aligned (pos 8-byte)", fn);
    const int64_t n_qt = (C + 127) / 128;
    if (B * H * n_qt > INT32_MAX) return fail(SWA_ERR_UNSUPPORTED, "%s: too many tiles", fn);
    DeviceState* ds;
    if (int rc = device_state(&ds)) return rc;
    const int64_t cst[3] = {H * C * D, C * D, D}, rst[3] = {H * W * D, W * D, D};
    CUtensorMap mq, mk, mv, mkr, mvr;
    int rc;
    if ((rc = make_map(&mq, q, B, H, C, D, cst)) || (rc = make_map(&mk, k, B, H, C, D, cst)) ||
        (rc = make_map(&mv, v, B, H, C, D, cst)) || (rc = make_map(&mkr, kring, B, H, W, D, rst)) ||
        (rc = make_map(&mvr, vring, B, H, W, D, rst)))
        return rc;
    const float scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    auto* ob = static_cast<__nv_bfloat16*>(out);
    const unsigned grid = (unsigned)(B * H * n_qt);
    if (D == 128)
        swa::chunk_kernel<128><<<grid, swa::kChunkThreads, swa::ChunkCfg<128>::kSmemBytes, s>>>(
            mq, mk, mv, mkr, mvr, pos, ob, (int)H, (int)C, (int)W, (int)n_qt, scale_log2, wait_limit(), ds->status);
    else
        swa::chunk_kernel<64><<<grid, swa::kChunkThreads, swa::ChunkCfg<64>::kSmemBytes, s>>>(
            mq, mk, mv, mkr, mvr, pos, ob, (int)H, (int)C, (int)W, (int)n_qt, scale_log2, wait_limit(), ds->status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "swa_chunk_forward launch");
    // the ring takes the chunk only after every read of the attention above (same stream)
    if ((rc = launch_append(fn, k, v, kring, vring, pos, B, H, C, D, W, s, ds->status))) return rc;
    return success();
}

int64_t swa_backward_workspace_bytes(int64_t B, int64_t H, int64_t T) {
    if (B < 0 || H < 0 || T < 0) return -1;
    const int64_t Tpad = (T + 127) / 128 * 128;
    if (B > 0 && H > 0 && Tpad > 0 && (B * H > INT64_MAX / Tpad || B * H * Tpad > INT64_MAX / 8)) return -1;
    return B * H * Tpad * 8;
}

int swa_forward_lse(const void* q, const void* k, const void* v, void* out, float* lse, int64_t B, int64_t H,
                    int64_t T, int64_t D, int64_t W, double scale, int dtype, void* stream) {
    if (!lse && B > 0 && H > 0 && T > 0) return fail(SWA_ERR_INVALID_ARG, "swa_forward_lse: null lse");
    if (lse && !aligned(lse, 4)) return fail(SWA_ERR_MISALIGNED, "swa_forward_lse: lse must be 4-byte aligned");
    return forward_impl("swa_forward_lse", q, k, v, out, B, H, T, D, W, scale, nullptr, dtype, stream, lse);
}

int swa_backward(const void* q, const void* k, const void* v, const void* out, const void* dout,
                 const float* lse, void* dq, void* dk, void* dv, void* workspace, int64_t workspace_bytes,
                 int64_t B, int64_t H, int64_t T, int64_t D, int64_t W, double scale, int dtype, void* stream) {
    const char* fn = "swa_backward";
    if (int rc = check_sizes(fn, B, H, T, D, W, dtype, scale)) return rc;
    if (B == 0 || H == 0 || T == 0) return success();
    const bool tc = dtype == SWA_BF16 && (D == 64 || D == 128);
    if (!q || !k || !v || !dout || !dq || !dk || !dv || !workspace || (tc && (!out || !lse)))
        return fail(SWA_ERR_INVALID_ARG, "%s: null pointer", fn);
    if (workspace_bytes < swa_backward_workspace_bytes(B, H, T))
        return fail(SWA_ERR_INVALID_ARG, "%s: workspace of %lld bytes, %lld needed", fn, (long long)workspace_bytes,
                    (long long)swa_backward_workspace_bytes(B, H, T));
    if (tc) {
        const void* ptrs16[] = {q, k, v, out, dout, dq, dk, dv};
        for (const void* p : ptrs16)
            if (!aligned(p, 16)) return fail(SWA_ERR_MISALIGNED, "%s: bf16 tensors must be 16-byte aligned", fn);
        if (!aligned(workspace, 256) || !aligned(lse, 4))
            return fail(SWA_ERR_MISALIGNED, "%s: workspace must be 256-byte aligned, lse 4-byte", fn);
        if (!(scale > 0.0)) return fail(SWA_ERR_UNSUPPORTED, "%s: the bf16 path needs scale > 0", fn);
        const int64_t BH = B * H;
        const int n_t = (int)((T + 127) / 128);
        const int64_t Tpad = (int64_t)n_t * 128;
        // one CTA per (b, h, tile) in the products, one warp per padded row in the statistics
        if (BH * n_t > INT32_MAX || (BH * Tpad + 7) / 8 > INT32_MAX)
            return fail(SWA_ERR_UNSUPPORTED, "%s: too many tiles", fn);
        DeviceState* ds;
        if (int rc = device_state(&ds)) return rc;
        const int64_t cst[3] = {H * T * D, T * D, D};
        CUtensorMap mq, mk, mv, mdo;
        int rc;
        if ((rc = make_map(&mq, q, B, H, T, D, cst)) || (rc = make_map(&mk, k, B, H, T, D, cst)) ||
            (rc = make_map(&mv, v, B, H, T, D, cst)) || (rc = make_map(&mdo, dout, B, H, T, D, cst)))
            return rc;
        cudaStream_t s = static_cast<cudaStream_t>(stream);
        float* nlse2 = static_cast<float*>(workspace);
        float* delta = nlse2 + BH * Tpad;
        const int Wi = (int)(W < T ? W : T);
        swa::bwd_stats_kernel<<<(unsigned)((BH * Tpad + 7) / 8), 256, 0, s>>>(
            static_cast<const __nv_bfloat16*>(dout), static_cast<const __nv_bfloat16*>(out), lse, nlse2, delta, BH,
            (int)T, (int)Tpad, (int)D);
        const float c = (float)scale, c2 = (float)(1.4426950408889634 * scale);
        const unsigned grid = (unsigned)(BH * n_t);
        auto* gq = static_cast<__nv_bfloat16*>(dq);
        auto* gk = static_cast<__nv_bfloat16*>(dk);
        auto* gv = static_cast<__nv_bfloat16*>(dv);
        // The key-tile kernel, then the query-tile kernel as its programmatic dependent:
        // the two share no output, so the second may start on the SMs the first one's
        // last CTAs free (it waits for the first grid before it ends).
        const auto* rq = static_cast<const __nv_bfloat16*>(q);
        const auto* rdo = static_cast<const __nv_bfloat16*>(dout);
        const uint64_t lim = wait_limit();
        cudaLaunchAttribute pdl[1];
        pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        pdl[0].val.programmaticStreamSerializationAllowed = 1;
        cudaLaunchConfig_t qc = {};
        qc.gridDim = dim3(grid);
        qc.blockDim = dim3(swa::kBwdTcThreads);
        qc.stream = s;
        qc.attrs = pdl;
        qc.numAttrs = 1;
        cudaError_t e;
        if (D == 128) {
            swa::bwd_tc_kernel<128, true><<<grid, swa::kBwdTcThreads, swa::BwdTcCfg<128, true>::kSmemBytes, s>>>(
                mq, mk, mv, mdo, nullptr, nullptr, nlse2, delta, gk, gv, (int)H, (int)T, (int)Tpad, Wi, n_t, c, c2, lim,
                ds->status);
            qc.dynamicSmemBytes = swa::BwdTcCfg<128, false>::kSmemBytes;
            e = cudaLaunchKernelEx(&qc, swa::bwd_tc_kernel<128, false>, mq, mk, mv, mdo, rq, rdo, (const float*)nlse2,
                                   (const float*)delta, gq, (__nv_bfloat16*)nullptr, (int)H, (int)T, (int)Tpad, Wi, n_t,
                                   c, c2, lim, ds->status);
        } else {
            swa::bwd_tc_kernel<64, true><<<grid, swa::kBwdTcThreads, swa::BwdTcCfg<64, true>::kSmemBytes, s>>>(
                mq, mk, mv, mdo, nullptr, nullptr, nlse2, delta, gk, gv, (int)H, (int)T, (int)Tpad, Wi, n_t, c, c2, lim,
                ds->status);
            qc.dynamicSmemBytes = swa::BwdTcCfg<64, false>::kSmemBytes;
            e = cudaLaunchKernelEx(&qc, swa::bwd_tc_kernel<64, false>, mq, mk, mv, mdo, rq, rdo, (const float*)nlse2,
                                   (const float*)delta, gq, (__nv_bfloat16*)nullptr, (int)H, (int)T, (int)Tpad, Wi, n_t,
                                   c, c2, lim, ds->status);
        }
        if (e == cudaSuccess) e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "swa_backward launch");
        return success();
    }
    // CUDA-core path: the row statistics are recomputed from q and k
    if (D > swa::kBwdMaxD) return fail(SWA_ERR_UNSUPPORTED, "%s: D <= %d", fn, swa::kBwdMaxD);
    const size_t esz = dtype == SWA_BF16 ? 2 : 4;
    const void* ptrs[] = {q, k, v, dout, dq, dk, dv};
    for (const void* p : ptrs)
        if (!aligned(p, esz)) return fail(SWA_ERR_MISALIGNED, "%s: tensors must be aligned to their element size", fn);
    if (!aligned(workspace, 8)) return fail(SWA_ERR_MISALIGNED, "%s: workspace must be 8-byte aligned", fn);
    const int64_t blocks = B * H * ((T + swa::kBwdRows - 1) / swa::kBwdRows);
    if (blocks > INT32_MAX) return fail(SWA_ERR_UNSUPPORTED, "%s: too many rows", fn);
    DeviceState* ds;
    if (int rc = device_state(&ds)) return rc;
    const int Wi = (int)(W < T ? W : T);
    const size_t smem = swa::bwd_smem_floats((int)D) * 4;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    float* stats = static_cast<float*>(workspace);
    const float c = (float)scale;
    const unsigned grid = (unsigned)blocks, block = swa::kBwdRows * 32;
    if (dtype == SWA_BF16) {
        using T16 = __nv_bfloat16;
        swa::bwd_rows_kernel<T16><<<grid, block, smem, s>>>(
            static_cast<const T16*>(q), static_cast<const T16*>(k), static_cast<const T16*>(v),
            static_cast<const T16*>(dout), static_cast<T16*>(dq), stats, (int)T, (int)D, Wi, c);
        swa::bwd_cols_kernel<T16><<<grid, block, smem, s>>>(
            static_cast<const T16*>(q), static_cast<const T16*>(k), static_cast<const T16*>(v),
            static_cast<const T16*>(dout), stats, static_cast<T16*>(dk), static_cast<T16*>(dv), (int)T, (int)D, Wi, c);
    } else {
        swa::bwd_rows_kernel<float><<<grid, block, smem, s>>>(
            static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
            static_cast<const float*>(dout), static_cast<float*>(dq), stats, (int)T, (int)D, Wi, c);
        swa::bwd_cols_kernel<float><<<grid, block, smem, s>>>(
            static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
            static_cast<const float*>(dout), stats, static_cast<float*>(dk), static_cast<float*>(dv), (int)T, (int)D,
            Wi, c);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "swa_backward launch");
    return success();
}

int swa_device_status(void* stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "swa_device_status: cudaStreamSynchronize");
    int v = 0;
    e = cudaMemcpyFromSymbol(&v, g_swa_status, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "swa_device_status: read");
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_swa_status, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "swa_device_status: clear");
    if (v != SWA_OK) return fail(v, "a kernel recorded status %d", v);
    return success();
}

}  // extern "C"

// ------------------------------------------------------------------ timeout probe
namespace {
__global__ void timeout_probe_kernel(uint64_t limit_ns, int* status) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        swa::ptx::mbar_init(&bar, 1);
        abort_flag = 0;
        swa::ptx::fence_mbar_init();
    }
    __syncthreads();
    // Nothing ever arrives on bar: phase 0 never completes, so this wait runs out.
    if (threadIdx.x == 0 && !swa::ptx::mbar_wait(&bar, 0, limit_ns, &abort_flag))
        atomicCAS(status, 0, (int)SWA_ERR_TIMEOUT);
}
}  // namespace

extern "C" int swa_timeout_probe(void* stream) {
    DeviceState* ds;
    if (int rc = device_state(&ds)) return rc;
    timeout_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(wait_limit(), ds->status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "swa_timeout_probe launch");
    return success();
}

// ------------------------------------------------------------------ allocation-free decode
// Some callers cannot let a library call cudaMalloc: their device memory is owned end to
// end by another allocator (a framework's caching allocator, or a serving runtime that
// carves a fixed arena at start-up and treats any other allocation as a leak), or they
// run a latency-bound decode step that must not take cudaMalloc's implicit device-wide
// synchronisation. For them, swa_decode_noalloc keeps the split partial states and ticket
// counters in this fixed file-scope array instead of a cudaMalloc'd workspace. Every GPU
// that loads the library holds the array until the process exits.
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
constexpr size_t kNoAllocCounterAlign = 256;
static __device__ __align__(256) unsigned char g_decode_noalloc_scratch[kNoAllocScratchBytes];

std::map<int, void*> g_noalloc_scratch;  // device address of the array, per device

// Once per device, with that device current: the array's name is only a host-side
// stand-in in host code, so fetch the device address the kernels must be given.
int noalloc_scratch(void** out) {
    int dev;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    std::lock_guard<std::mutex> lk(g_mu);
    void*& ptr = g_noalloc_scratch[dev];
    if (!ptr) {
        e = cudaGetSymbolAddress(&ptr, g_decode_noalloc_scratch);
        if (e != cudaSuccess) {
            ptr = nullptr;
            return cuda_fail(e, "cudaGetSymbolAddress(decode scratch)");
        }
    }
    *out = ptr;
    return SWA_OK;
}
}  // namespace

extern "C" int swa_decode_noalloc(const void* q, const void* kring, const void* vring,
                                  const int64_t* pos, void* out, int64_t B, int64_t H, int64_t D,
                                  int64_t W, void* stream) {
    if (W < 1) return fail(SWA_ERR_INVALID_ARG, "swa_decode_noalloc: window W=%lld must be >= 1", (long long)W);
    if (B < 0 || H < 0)
        return fail(SWA_ERR_INVALID_ARG, "swa_decode_noalloc: negative size B=%lld H=%lld", (long long)B, (long long)H);
    if (D < 1) return fail(SWA_ERR_INVALID_ARG, "swa_decode_noalloc: head dim D=%lld must be >= 1", (long long)D);
    if (B == 0 || H == 0) return success();
    if (!q || !kring || !vring || !pos || !out)
        return fail(SWA_ERR_INVALID_ARG, "swa_decode_noalloc: null pointer");
    if (D != 64 && D != 128)
        return fail(SWA_ERR_UNSUPPORTED, "swa_decode_noalloc: D must be 64 or 128 (got %lld)", (long long)D);
    if (!aligned(q, 16) || !aligned(kring, 16) || !aligned(vring, 16) || !aligned(out, 16) ||
        !aligned(pos, 8))
        return fail(SWA_ERR_MISALIGNED, "swa_decode_noalloc: tensors must be 16-byte aligned (pos 8-byte)");
    if (B * H > INT32_MAX || W > INT32_MAX / 2 || B * H > INT64_MAX / W / D)
        return fail(SWA_ERR_UNSUPPORTED, "swa_decode_noalloc: sizes too large");
    int32_t S, chunk;
    split_plan(B, H, D, W, &S, &chunk);
    if (S > kMaxDecodeSplits)
        return fail(SWA_ERR_UNSUPPORTED,
                    "swa_decode_noalloc: %d splits exceed the grid limit of %d (a larger SWA_DECODE_CHUNK)", (int)S,
                    kMaxDecodeSplits);
    const size_t counter_bytes =
        ((size_t)(B * H) * sizeof(int) + kNoAllocCounterAlign - 1) / kNoAllocCounterAlign * kNoAllocCounterAlign;
    const size_t part_bytes = (size_t)(B * H) * S * (D + 2) * sizeof(float);
    if (S > 1 && counter_bytes + part_bytes > kNoAllocScratchBytes)
        return fail(SWA_ERR_UNSUPPORTED,
                    "swa_decode_noalloc: %lld streams x %d splits need %zu bytes of scratch; the fixed "
                    "array holds %zu (use swa_decode)",
                    (long long)(B * H), (int)S, counter_bytes + part_bytes, kNoAllocScratchBytes);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    DeviceState* ds;
    if (int rc = device_state(&ds)) return rc;
    float* part = nullptr;
    int* counters = nullptr;
    if (S > 1) {
        void* base;
        if (int rc = noalloc_scratch(&base)) return rc;
        counters = static_cast<int*>(base);
        part = reinterpret_cast<float*>(static_cast<unsigned char*>(base) + counter_bytes);
        // The array keeps the last call's contents and the ticket counters must start at
        // zero. Every decode kernel that runs to its end puts its counters back to zero, so
        // after ordered calls they already are; the clear guards against a launch that
        // never ran to its end (a kernel stopped by an error), at the cost of one memset
        // node of B*H*4 bytes per call.
        cudaError_t e = cudaMemsetAsync(counters, 0, (size_t)(B * H) * sizeof(int), s);
        if (e != cudaSuccess) return cuda_fail(e, "swa_decode_noalloc: clearing counters");
    }
    const float scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
    const dim3 grid((unsigned)(B * H), (unsigned)S);
    const auto* qb = static_cast<const __nv_bfloat16*>(q);
    const auto* kb = static_cast<const __nv_bfloat16*>(kring);
    const auto* vb = static_cast<const __nv_bfloat16*>(vring);
    auto* ob = static_cast<__nv_bfloat16*>(out);
    if (D == 128)
        swa::decode_kernel<128><<<grid, swa::kDecodeWarps * 32, 0, s>>>(
            qb, kb, vb, pos, ob, (int)H, (int)W, chunk, S, scale_log2, part, counters, ds->status);
    else
        swa::decode_kernel<64><<<grid, swa::kDecodeWarps * 32, 0, s>>>(
            qb, kb, vb, pos, ob, (int)H, (int)W, chunk, S, scale_log2, part, counters, ds->status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "swa_decode_noalloc launch");
    return success();
}

namespace swa_internal {
int set_error(int code, const char* msg) {
    t_error = msg;
    return code;
}
int clear_error() {
    t_error.clear();
    return SWA_OK;
}
}  // namespace swa_internal
