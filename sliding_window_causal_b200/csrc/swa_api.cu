// swa_api.cu: the C ABI declared in include/swa.h. Validates arguments, encodes the TMA
// tensor maps, picks a kernel by dtype and head dimension, and launches it on the
// caller's stream. No torch types cross this boundary.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <map>
#include <mutex>
#include <string>
#include <utility>

#include "swa.h"
#include "decode.cuh"
#include "plan.h"
#include "prefill_simt.cuh"
#include "prefill_pp.cuh"

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
};
std::map<int, DeviceState> g_dev;

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
    if (!st.attrs_set) {
        e = cudaSuccess;
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(swa::prefill_pp_kernel<128>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     swa::PPCfg<128>::kSmemBytes);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(swa::prefill_pp_kernel<64>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     swa::PPCfg<64>::kSmemBytes);
        if (e == cudaSuccess)
            e = cudaDeviceGetAttribute(&st.num_sms, cudaDevAttrMultiProcessorCount, dev);
        if (e == cudaSuccess) {
            // The register split inside the kernel assumes this launch allocation.
            cudaFuncAttributes a128, a64;
            e = cudaFuncGetAttributes(&a128, swa::prefill_pp_kernel<128>);
            if (e == cudaSuccess) e = cudaFuncGetAttributes(&a64, swa::prefill_pp_kernel<64>);
            st.pp_regs_ok = e == cudaSuccess && a128.numRegs == swa::kPPLaunchRegs &&
                            a64.numRegs == swa::kPPLaunchRegs;
        }
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(swa::prefill_simt_kernel,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     swa::kSimtWarps * (2 * 4096 + 32) * 4);
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

// [BH, T, D] bf16 viewed as a 3-D tensor (D fastest), boxes of 64 columns x 128 rows,
// 128-byte swizzle. Rows past T read as zeros; stores past T are dropped.
int make_map(CUtensorMap* m, const void* ptr, int64_t BH, int64_t T, int64_t D) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return fail(SWA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)T, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)(D * 2), (cuuint64_t)(T * D * 2)};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(SWA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
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

}  // namespace

// ==================================================================== C ABI
extern "C" {

const char* swa_last_error(void) { return t_error.c_str(); }

uint64_t swa_set_wait_limit_ns(uint64_t ns) {
    uint64_t prev = wait_limit();
    g_wait_limit.store(ns);
    return prev;
}

int swa_prefill_tile_class(int64_t T, int64_t W, int64_t bm, int64_t bn, int64_t qt, int64_t kt) {
    if (T < 1 || W < 1 || bm < 1 || bn < 1 || qt < 0 || kt < 0 || qt * bm >= T) return -1;
    return swa::tile_class(T, W, bm, bn, qt, kt);
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
    if (dtype != SWA_F32 && dtype != SWA_BF16)
        return fail(SWA_ERR_INVALID_ARG, "swa_forward: dtype %d is neither SWA_F32 nor SWA_BF16", dtype);
    if (W < 1) return fail(SWA_ERR_INVALID_ARG, "swa_forward: window W=%lld must be >= 1", (long long)W);
    if (B < 0 || H < 0 || T < 0)
        return fail(SWA_ERR_INVALID_ARG, "swa_forward: negative size B=%lld H=%lld T=%lld",
                    (long long)B, (long long)H, (long long)T);
    if (D < 1) return fail(SWA_ERR_INVALID_ARG, "swa_forward: head dim D=%lld must be >= 1", (long long)D);
    if (B == 0 || H == 0 || T == 0) return success();
    if (!q || !k || !v || !out) return fail(SWA_ERR_INVALID_ARG, "swa_forward: null pointer");
    if (B > INT32_MAX || H > INT32_MAX || B * H > INT32_MAX || T > INT32_MAX ||
        B * H > INT64_MAX / T || B * H * T > INT64_MAX / D / 4)
        return fail(SWA_ERR_UNSUPPORTED, "swa_forward: sizes too large");
    const int Wi = (int)(W < T ? W : T);  // W >= T is causal attention
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    DeviceState* ds;
    if (int rc = device_state(&ds)) return rc;

    if (dtype == SWA_BF16) {
        if (D != 64 && D != 128)
            return fail(SWA_ERR_UNSUPPORTED, "swa_forward: bf16 needs D = 64 or 128 (got %lld)", (long long)D);
        if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
            return fail(SWA_ERR_MISALIGNED, "swa_forward: bf16 tensors must be 16-byte aligned");
        const int64_t BH = B * H;
        const int n_qt = (int)((T + 127) / 128);
        if ((int64_t)n_qt * BH > INT32_MAX) return fail(SWA_ERR_UNSUPPORTED, "swa_forward: too many tiles");
        CUtensorMap mq, mk, mv;
        int rc;
        if ((rc = make_map(&mq, q, BH, T, D)) || (rc = make_map(&mk, k, BH, T, D)) ||
            (rc = make_map(&mv, v, BH, T, D)))
            return rc;
        const float scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
        if (!ds->pp_regs_ok)
            return fail(SWA_ERR_UNSUPPORTED,
                        "swa_forward: prefill kernel was not compiled with %d registers per thread",
                        swa::kPPLaunchRegs);
        const int64_t n_items = (int64_t)((n_qt + 1) / 2) * BH;
        const unsigned G = (unsigned)(n_items < ds->num_sms ? n_items : ds->num_sms);
        auto* ob = static_cast<__nv_bfloat16*>(out);
        if (D == 128)
            swa::prefill_pp_kernel<128><<<G, swa::kPPThreads, swa::PPCfg<128>::kSmemBytes, s>>>(
                mq, mk, mv, ob, (int)BH, (int)T, Wi, n_qt, scale_log2, wait_limit(), ds->status);
        else
            swa::prefill_pp_kernel<64><<<G, swa::kPPThreads, swa::PPCfg<64>::kSmemBytes, s>>>(
                mq, mk, mv, ob, (int)BH, (int)T, Wi, n_qt, scale_log2, wait_limit(), ds->status);
    } else {
        if (D > 4096) return fail(SWA_ERR_UNSUPPORTED, "swa_forward: fp32 supports D <= 4096");
        if (!aligned(q, 4) || !aligned(k, 4) || !aligned(v, 4) || !aligned(out, 4))
            return fail(SWA_ERR_MISALIGNED, "swa_forward: fp32 tensors must be 4-byte aligned");
        const int64_t nrows = B * H * T;
        const int64_t blocks = (nrows + swa::kSimtWarps - 1) / swa::kSimtWarps;
        if (blocks > INT32_MAX) return fail(SWA_ERR_UNSUPPORTED, "swa_forward: too many rows");
        const size_t smem = (size_t)swa::kSimtWarps * (2 * D + 32) * sizeof(float);
        const float scale = (float)(1.0 / std::sqrt((double)D));
        swa::prefill_simt_kernel<<<(unsigned)blocks, swa::kSimtWarps * 32, smem, s>>>(
            static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
            static_cast<float*>(out), nrows, (int)T, (int)D, Wi, scale);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "swa_forward launch");
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
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    DeviceState* ds;
    if (int rc = device_state(&ds)) return rc;
    int32_t S, chunk;
    split_plan(B, H, D, W, &S, &chunk);
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
        // the array keeps the last call's contents: the ticket counters must start at zero
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
