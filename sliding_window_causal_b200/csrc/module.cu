// module.cu: the sliding-window multi-head attention module of "NNX Sliding-Window
// Attention" (A complete example with moving averages) around the attention kernels.
//
//   q = x Wq + bq,  k = x Wk + bk,  v = x Wv + bv        (y = x @ kernel + bias, [d, d] kernels)
//   split q, k, v into H heads of Dh = d / H columns, sliding-window attention per head,
//   concatenate the heads, out = concat Wo + bo.
//
// The four projections are plain dense GEMMs and run in cuBLASLt (fp32 accumulation, the
// bias added in its epilogue). Their [B*T, d] outputs are already the [B, T, H, Dh] layout
// the attention reads through strides (swa_forward_ex), so nothing is transposed: the
// attention writes its heads straight into the [B*T, d] concatenation the last GEMM reads.
#include <cublasLt.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <map>
#include <mutex>
#include <tuple>

#include "api_internal.h"
#include "swa.h"

namespace {

constexpr size_t kLtWorkspaceBytes = size_t(32) << 20;

int fail(int code, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    return swa_internal::set_error(code, buf);
}

std::mutex g_mu;
std::map<int, cublasLtHandle_t> g_lt;  // one handle per device, kept until exit
// heuristic algorithm per (device, dtype, M, N, K, has_bias)
std::map<std::tuple<int, int, int64_t, int64_t, int64_t, bool>, cublasLtMatmulAlgo_t> g_algo;

int lt_handle(int dev, cublasLtHandle_t* out) {
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_lt.find(dev);
    if (it == g_lt.end()) {
        cublasLtHandle_t h;
        cublasStatus_t st = cublasLtCreate(&h);
        if (st != CUBLAS_STATUS_SUCCESS) return fail(SWA_ERR_CUDA, "cublasLtCreate failed (%d)", (int)st);
        it = g_lt.emplace(dev, h).first;
    }
    *out = it->second;
    return SWA_OK;
}

// Y[M, N] = X[M, K] @ Wt[K, N] (+ bias[N]), all row-major of one dtype. cuBLASLt is
// column-major, so it computes Y^T = Wt^T X^T with Wt and X read as they are.
int gemm(int dev, cublasLtHandle_t h, int dtype, const void* X, const void* Wt, const void* bias, void* Y,
         int64_t M, int64_t N, int64_t K, void* ws, cudaStream_t s) {
    const cudaDataType_t dt = dtype == SWA_BF16 ? CUDA_R_16BF : CUDA_R_32F;
    cublasLtMatmulDesc_t op = nullptr;
    cublasLtMatrixLayout_t la = nullptr, lb = nullptr, lc = nullptr;
    cublasLtMatmulPreference_t pref = nullptr;
    int rc = SWA_OK;
    cublasStatus_t st = cublasLtMatmulDescCreate(&op, CUBLAS_COMPUTE_32F, CUDA_R_32F);  // no TF32
    const cublasOperation_t no = CUBLAS_OP_N;
    if (st == CUBLAS_STATUS_SUCCESS)
        st = cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSA, &no, sizeof(no));
    if (st == CUBLAS_STATUS_SUCCESS)
        st = cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSB, &no, sizeof(no));
    if (st == CUBLAS_STATUS_SUCCESS && bias) {
        const cublasLtEpilogue_t epi = CUBLASLT_EPILOGUE_BIAS;
        st = cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_EPILOGUE, &epi, sizeof(epi));
        if (st == CUBLAS_STATUS_SUCCESS)
            st = cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_BIAS_POINTER, &bias, sizeof(bias));
        if (st == CUBLAS_STATUS_SUCCESS)
            st = cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_BIAS_DATA_TYPE, &dt, sizeof(dt));
    }
    if (st == CUBLAS_STATUS_SUCCESS) st = cublasLtMatrixLayoutCreate(&la, dt, N, K, N);
    if (st == CUBLAS_STATUS_SUCCESS) st = cublasLtMatrixLayoutCreate(&lb, dt, K, M, K);
    if (st == CUBLAS_STATUS_SUCCESS) st = cublasLtMatrixLayoutCreate(&lc, dt, N, M, N);
    cublasLtMatmulAlgo_t algo;
    if (st == CUBLAS_STATUS_SUCCESS) {
        const auto key = std::make_tuple(dev, dtype, M, N, K, bias != nullptr);
        std::unique_lock<std::mutex> lk(g_mu);
        auto it = g_algo.find(key);
        if (it != g_algo.end()) {
            algo = it->second;
        } else {
            lk.unlock();
            st = cublasLtMatmulPreferenceCreate(&pref);
            const uint64_t wsb = kLtWorkspaceBytes;
            if (st == CUBLAS_STATUS_SUCCESS)
                st = cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES, &wsb,
                                                          sizeof(wsb));
            cublasLtMatmulHeuristicResult_t res;
            int n = 0;
            if (st == CUBLAS_STATUS_SUCCESS)
                st = cublasLtMatmulAlgoGetHeuristic(h, op, la, lb, lc, lc, pref, 1, &res, &n);
            if (st == CUBLAS_STATUS_SUCCESS && n < 1) st = CUBLAS_STATUS_NOT_SUPPORTED;
            if (st == CUBLAS_STATUS_SUCCESS) {
                algo = res.algo;
                lk.lock();
                g_algo[key] = algo;
            }
        }
    }
    if (st == CUBLAS_STATUS_SUCCESS) {
        const float alpha = 1.f, beta = 0.f;
        st = cublasLtMatmul(h, op, &alpha, Wt, la, X, lb, &beta, Y, lc, Y, lc, &algo, ws, kLtWorkspaceBytes, s);
    }
    if (st != CUBLAS_STATUS_SUCCESS)
        rc = fail(SWA_ERR_CUDA, "swa_mha_forward: cuBLASLt GEMM [%lld x %lld x %lld] failed (%d)", (long long)M,
                  (long long)N, (long long)K, (int)st);
    if (pref) cublasLtMatmulPreferenceDestroy(pref);
    if (lc) cublasLtMatrixLayoutDestroy(lc);
    if (lb) cublasLtMatrixLayoutDestroy(lb);
    if (la) cublasLtMatrixLayoutDestroy(la);
    if (op) cublasLtMatmulDescDestroy(op);
    return rc;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

extern "C" {

int64_t swa_mha_workspace_bytes(int64_t B, int64_t T, int64_t d_model, int dtype) {
    if (B < 0 || T < 0 || d_model < 1 || (dtype != SWA_F32 && dtype != SWA_BF16)) return -1;
    if (B > 0 && T > 0 && B * T > INT64_MAX / d_model / 16) return -1;
    const size_t esz = dtype == SWA_BF16 ? 2 : 4;
    return (int64_t)(4 * round256((size_t)(B * T * d_model) * esz) + kLtWorkspaceBytes);
}

int swa_mha_forward(const void* x, const void* wq, const void* bq, const void* wk, const void* bk,
                    const void* wv, const void* bv, const void* wo, const void* bo, void* out, void* workspace,
                    int64_t workspace_bytes, int64_t B, int64_t T, int64_t d_model, int64_t H, int64_t W,
                    int dtype, void* stream) {
    const char* fn = "swa_mha_forward";
    if (dtype != SWA_F32 && dtype != SWA_BF16) return fail(SWA_ERR_INVALID_ARG, "%s: bad dtype %d", fn, dtype);
    if (W < 1) return fail(SWA_ERR_INVALID_ARG, "%s: window W=%lld must be >= 1", fn, (long long)W);
    if (B < 0 || T < 0 || d_model < 1 || H < 1 || d_model % H != 0)
        return fail(SWA_ERR_INVALID_ARG, "%s: bad sizes B=%lld T=%lld d_model=%lld H=%lld", fn, (long long)B,
                    (long long)T, (long long)d_model, (long long)H);
    if (B == 0 || T == 0) return swa_internal::clear_error();
    const int64_t need = swa_mha_workspace_bytes(B, T, d_model, dtype);
    if (need < 0 || B * T > INT32_MAX || d_model > INT32_MAX)
        return fail(SWA_ERR_UNSUPPORTED, "%s: sizes too large", fn);
    if (!x || !wq || !wk || !wv || !wo || !out || !workspace)
        return fail(SWA_ERR_INVALID_ARG, "%s: null pointer", fn);
    if (workspace_bytes < need)
        return fail(SWA_ERR_INVALID_ARG, "%s: workspace of %lld bytes, %lld needed", fn, (long long)workspace_bytes,
                    (long long)need);
    const int64_t Dh = d_model / H;
    if (dtype == SWA_BF16 && Dh != 64 && Dh != 128)
        return fail(SWA_ERR_UNSUPPORTED, "%s: bf16 needs a head width d_model/H of 64 or 128 (got %lld)", fn,
                    (long long)Dh);
    if (dtype == SWA_F32 && Dh > 4096) return fail(SWA_ERR_UNSUPPORTED, "%s: fp32 head width <= 4096", fn);
    const size_t esz = dtype == SWA_BF16 ? 2 : 4;
    const void* ptrs[] = {x, wq, wk, wv, wo, out, bq, bk, bv, bo};
    for (const void* p : ptrs)
        if (p && !aligned(p, 16)) return fail(SWA_ERR_MISALIGNED, "%s: tensors must be 16-byte aligned", fn);
    if (!aligned(workspace, 256)) return fail(SWA_ERR_MISALIGNED, "%s: workspace must be 256-byte aligned", fn);
    if (dtype == SWA_BF16 && d_model % 8 != 0)
        return fail(SWA_ERR_MISALIGNED, "%s: bf16 d_model must be a multiple of 8", fn);

    const int64_t M = B * T;
    const size_t part = round256((size_t)(M * d_model) * esz);
    char* base = static_cast<char*>(workspace);
    void *q = base, *k = base + part, *v = base + 2 * part, *attn = base + 3 * part, *lt_ws = base + 4 * part;
    // [B*T, d] is [B, T, H, Dh]: element strides b = T*d, h = Dh, t = d for every operand
    const int64_t st[12] = {T * d_model, Dh, d_model, T * d_model, Dh, d_model,
                            T * d_model, Dh, d_model, T * d_model, Dh, d_model};
    const double scale = 1.0 / std::sqrt((double)Dh);
    // the attention's own refusals come before the first GEMM is enqueued
    int64_t eff[4][3];
    if (int rc = swa_internal::check_forward(fn, q, k, v, attn, B, H, T, Dh, W, scale, st, dtype, eff)) return rc;

    int dev;
    cudaError_t ce = cudaGetDevice(&dev);
    if (ce != cudaSuccess) return fail(SWA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(ce));
    cublasLtHandle_t h;
    if (int rc = lt_handle(dev, &h)) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int rc;
    if ((rc = gemm(dev, h, dtype, x, wq, bq, q, M, d_model, d_model, lt_ws, s)) ||
        (rc = gemm(dev, h, dtype, x, wk, bk, k, M, d_model, d_model, lt_ws, s)) ||
        (rc = gemm(dev, h, dtype, x, wv, bv, v, M, d_model, d_model, lt_ws, s)))
        return rc;
    if ((rc = swa_forward_ex(q, k, v, attn, B, H, T, Dh, W, scale, st, dtype, stream))) return rc;
    if ((rc = gemm(dev, h, dtype, attn, wo, bo, out, M, d_model, d_model, lt_ws, s))) return rc;
    return swa_internal::clear_error();
}

}  // extern "C"
