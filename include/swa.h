/*
 * swa.h: C ABI of the B200 (sm_100a) sliding-window causal attention library.
 *
 * The operation. Query position i of a sequence attends only to key positions j
 * with 0 <= i - j < W, that is to the W most recent positions including itself:
 *
 *   out[b,h,i,:] = sum_{j in band(i)} softmax_j( q[b,h,i,:] . k[b,h,j,:] / sqrt(D) ) v[b,h,j,:]
 *   band(i)      = { j : max(0, i-W+1) <= j <= i }
 *
 * Sources: "27. Sliding-Window Attention" (Problem; Step-by-Step Approach steps 1-5:
 * scaled scores, a mask that keeps j <= i with i - j below the window, -inf outside it,
 * a softmax over the keys, then the weighted sum of v); "25. Sliding-Window Causal
 * Attention for Streaming Inference" (Step-by-Step Approach step 3: the oldest key kept
 * is strictly newer than i - W); "NNX Sliding-Window Attention" (opening
 * paragraph: keys max(0, i-W+1) .. i; W = 1 is self-attention only; W >= T is
 * ordinary causal attention). The one-key-wider interval [i-W, i] of "Sliding
 * Window Attention" (Mathematical Formulation and Attention Masking) is not
 * used; a caller who wants it passes W+1.
 *
 * Conventions for every call below:
 *  - Every tensor pointer is a DEVICE pointer to row-major contiguous memory (or to a
 *    strided view, where a call takes strides), owned by the caller. The library keeps
 *    no pointer after a call returns.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *    Calls enqueue work on it and return without waiting (asynchronous).
 *  - Calls return an swa_status code and never throw. All validation happens before
 *    any work is enqueued, so a non-OK return has enqueued nothing; the reason is in
 *    swa_last_error(). A failure detected inside a kernel (a pipeline wait that ran
 *    past its time limit, a negative decode position) is recorded in a per-device
 *    status word and reported by swa_device_status().
 *  - `out` must not alias q, k, v (or the rings); this is documented, not checked.
 *  - Results are deterministic: the same inputs and sizes give bitwise-identical
 *    outputs on every run (swa_mha_forward: its attention is; its projections are as
 *    reproducible as the GEMM algorithm cuBLASLt picks).
 */
#ifndef SWA_H
#define SWA_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { SWA_F32 = 0, SWA_BF16 = 1 } swa_dtype;

typedef enum {
    SWA_OK = 0,
    SWA_ERR_INVALID_ARG = 1, /* bad size, window, dtype or null pointer */
    SWA_ERR_UNSUPPORTED = 2, /* a valid request this build does not implement (e.g. bf16 D=96) */
    SWA_ERR_MISALIGNED = 3,  /* a pointer is not aligned as the kernel needs */
    SWA_ERR_CUDA = 4,        /* a CUDA runtime/driver call or a launch failed */
    SWA_ERR_TIMEOUT = 5      /* a kernel wait ran past its limit (reported by swa_device_status) */
} swa_status;

/*
 * swa_forward: prefill. out[B,H,T,D] = sliding-window causal attention of q, k, v.
 *
 *   q, k, v, out : [B, H, T, D] contiguous, all of `dtype`. Element (b,h,t,d) is at
 *                  ((b*H + h)*T + t)*D + d. (A (B,T,H,D) caller transposes first; a
 *                  3-D (B,T,D) input is H = 1.)
 *   W            : window, W >= 1. W >= T is ordinary causal attention; W = 1 returns v.
 *   dtype        : SWA_BF16 - bf16 in and out, fp32 accumulation, tensor cores
 *                  (tcgen05), D must be 64 or 128, pointers 16-byte aligned;
 *                  SWA_F32  - fp32 in and out, fp32 arithmetic on the CUDA cores
 *                  (no TF32), any 1 <= D <= 4096, pointers 4-byte aligned.
 *   scale        : 1/sqrt(D), fixed.
 * Errors: W < 1, a negative size, D < 1, a null pointer (unless B*H*T == 0) or a bad
 * dtype -> SWA_ERR_INVALID_ARG; B*H*T == 0 -> SWA_OK with nothing enqueued; an
 * unsupported D or sizes beyond 2^31-1 rows -> SWA_ERR_UNSUPPORTED; misaligned
 * pointers -> SWA_ERR_MISALIGNED; a failed launch -> SWA_ERR_CUDA.
 */
int swa_forward(const void* q, const void* k, const void* v, void* out,
                int64_t B, int64_t H, int64_t T, int64_t D, int64_t W,
                int dtype, void* stream);

/*
 * swa_forward_ex: swa_forward with a caller-chosen score scale and strided operands.
 *
 * "Mistral Architecture > Implementation: Sliding Window Attention" (Step 2) lays its
 * inputs out batch, position, head, feature ([B,T,H,D]) and lets the caller choose the
 * score scale, 1/sqrt(D) when none is given. This call covers both:
 *   scale   : scores are (q . k) * scale. swa_forward is scale = 1/sqrt(D). SWA_BF16 takes
 *             any scale > 0 (the tensor-core softmax scales the row maximum of the raw
 *             scores, which is the maximum of the scaled ones only for a positive scale);
 *             SWA_F32 takes any finite value, 0 giving equal weights over the band (a
 *             trailing moving average of v).
 *   strides : NULL for contiguous [B,H,T,D], or 12 element strides (not bytes), in the
 *             order q(b,h,t), k(b,h,t), v(b,h,t), out(b,h,t); the head dimension is always
 *             contiguous. Element (b,h,t,d) of q is at q + b*s[0] + h*s[1] + t*s[2] + d.
 *             The [B,T,H,D] layout of the page is (T*H*D, D, H*D) for every operand.
 *             The stride of a size-1 dimension is ignored. The rows of out must not overlap
 *             each other or the inputs; this is documented, not checked.
 * Everything else is as swa_forward. Extra errors: a non-finite scale, or a negative
 * stride or one above 2^38 -> SWA_ERR_INVALID_ARG; for SWA_BF16 a scale <= 0 ->
 * SWA_ERR_UNSUPPORTED, and a stride that is not a multiple of 8 elements (16 bytes) ->
 * SWA_ERR_MISALIGNED.
 */
int swa_forward_ex(const void* q, const void* k, const void* v, void* out,
                   int64_t B, int64_t H, int64_t T, int64_t D, int64_t W,
                   double scale, const int64_t* strides, int dtype, void* stream);

/*
 * swa_forward_host: swa_forward from and to HOST memory, the copies overlapped with the
 * attention and with each other.
 *
 *   q, k, v, out     : HOST [B,H,T,D] contiguous, of `dtype`. Page-locked (pinned) memory
 *                      lets the copies run asynchronously and overlap; pageable memory
 *                      works, but the copies then wait for each other.
 *   dq, dk, dv, dout : DEVICE staging tensors of the same shape, owned by the caller; on
 *                      return they hold the inputs and the output.
 *   heads_per_group  : the (b,h) heads are independent problems (each row's band lies in
 *                      its own head), so the B*H heads are processed in groups of this many
 *                      consecutive heads; 0 lets the library pick (about eight groups).
 * Group g's host-to-device copies, its attention (swa_forward on heads g) and its
 * device-to-host copy run on three library-owned streams, created once per device and
 * ordered by events, so the copies of one group overlap the attention of another and the
 * two copy directions overlap each other. The work starts after everything already
 * enqueued on `stream`, and `stream` waits for all of it: once the stream reaches this
 * point, out holds the result, bitwise equal to swa_forward on the device copies. The
 * copies are asynchronous: the host buffers must stay allocated and q, k, v unchanged
 * until then. Calls from several host threads enqueue one after another.
 * Errors: as swa_forward (on the device pointers), a null host pointer ->
 * SWA_ERR_INVALID_ARG, heads_per_group < 0 -> SWA_ERR_INVALID_ARG. A CUDA failure after
 * the first copy was enqueued returns SWA_ERR_CUDA with the earlier groups enqueued.
 */
int swa_forward_host(const void* q, const void* k, const void* v, void* out,
                     void* dq, void* dk, void* dv, void* dout,
                     int64_t B, int64_t H, int64_t T, int64_t D, int64_t W,
                     int64_t heads_per_group, int dtype, void* stream);

/*
 * swa_band_weights: the softmax weights of every query's band, for inspection.
 *
 * "Mistral Architecture > Implementation: Sliding Window Attention" (Step 2) returns the
 * attention weights beside the output. Outside the band they are zero, so only the band is
 * written: weights is [B, H, T, Wo] fp32 contiguous with Wo = min(W, T), and
 * weights[b,h,i,c] is the weight of key j = i - Wo + 1 + c (c = Wo-1 is the query itself),
 * or 0 where j < 0. Each row of weights sums to 1 (up to fp32 rounding). The weights are
 * computed in fp32 on the CUDA cores, from q and k of `dtype` (SWA_F32 or SWA_BF16).
 *   q, k    : [B,H,T,D] device tensors; strides NULL (contiguous) or 6 element strides
 *             q(b,h,t), k(b,h,t) as in swa_forward_ex. D <= 4096.
 *   scale   : as swa_forward_ex (pass 1/sqrt(D) for the scores of swa_forward).
 * This is a debugging aid: it writes B*H*T*Wo*4 bytes, so it is not on the prefill path.
 * Errors: as swa_forward_ex; pointers must be aligned to their element size.
 */
int swa_band_weights(const void* q, const void* k, float* weights,
                     int64_t B, int64_t H, int64_t T, int64_t D, int64_t W,
                     double scale, const int64_t* strides, int dtype, void* stream);

/*
 * swa_decode: one new query per stream against a W-slot rolling KV buffer.
 *
 * "25. Sliding-Window Causal Attention for Streaming Inference" (Problem) pairs the
 * window with a bounded KV cache that drops anything older than the window. Here the
 * cache of stream b holds position p in slot p mod W. pos[b] is the 0-based absolute
 * position of stream b's new query; the caller has already written that position's
 * k and v into slot pos[b] mod W. The query attends to positions
 * max(0, pos[b]-W+1) .. pos[b], which always occupy slots 0 .. min(pos[b]+1, W)-1.
 * Slots outside that range are never read.
 *
 *   q, out       : [B, H, D] bf16.
 *   kring, vring : [B, H, W, D] bf16; slot s of (b,h) starts at ((b*H + h)*W + s)*D.
 *   pos          : [B] int64, on the device, each >= 0.
 *   D            : 64 or 128. All pointers 16-byte aligned (pos 8-byte aligned).
 * The work is split along the ring into chunks whose partial softmax states are merged
 * in a fixed order (deterministic). The chunk length follows from the sizes (about 16
 * CTAs per SM in total); the SWA_DECODE_CHUNK environment variable overrides it (in
 * slots) for tuning. The partial states live in a workspace that the
 * library allocates with cudaMalloc on the first call for each (device, stream) and
 * keeps, growing it when a larger call needs more: make that first call before any
 * stream capture. Calls on one stream share its workspace; calls on different
 * streams do not.
 * Errors: as swa_forward, plus more than 65535 splits (possible only when SWA_DECODE_CHUNK
 * forces a small chunk over a long ring) -> SWA_ERR_UNSUPPORTED. A negative pos[b] is found
 * on the device: that stream's output is written as zeros and swa_device_status() reports
 * SWA_ERR_INVALID_ARG.
 */
int swa_decode(const void* q, const void* kring, const void* vring, const int64_t* pos,
               void* out, int64_t B, int64_t H, int64_t D, int64_t W, void* stream);

/*
 * swa_chunk_forward: chunked streaming prefill. C new tokens per stream attend to the
 * rolling buffer and to each other, then join the buffer.
 *
 * "25. Sliding-Window Causal Attention for Streaming Inference" (Problem) processes an
 * unbounded stream with a KV cache bounded by the window. Stream b has seen positions
 * 0 .. pos[b]-1, and its rings hold the last min(pos[b], W) of them, position p in slot
 * p mod W (the swa_decode layout). The chunk's tokens take positions pos[b] .. pos[b]+C-1.
 * Chunk row c (position P = pos[b] + c) attends to positions max(0, P-W+1) .. P: those
 * below pos[b] are read from the rings, the others from k and v. Then the chunk is
 * appended as swa_ring_append does, so after the call the rings hold positions up to
 * pos[b]+C-1, ready for the next chunk (pos[b] + C) or for swa_decode.
 *
 *   q, k, v, out : [B, H, C, D] bf16 contiguous, the chunk's queries, keys, values and
 *                  the output.
 *   kring, vring : [B, H, W, D] bf16 contiguous, read, then updated in place.
 *   pos          : [B] int64 on the device: tokens stream b had before the chunk (>= 0).
 *   D            : 64 or 128. All pointers 16-byte aligned (pos 8-byte).
 * The attention runs on the tensor cores (tcgen05, fp32 accumulation, one rounding of the
 * output to bf16); the append is a copy. Both are enqueued on `stream`, in that order.
 * Errors: as swa_decode; B*H*C == 0 -> SWA_OK with nothing enqueued. A negative pos[b]
 * is found on the device: that stream's output is written as zeros, its rings are left
 * as they were, and swa_device_status() reports SWA_ERR_INVALID_ARG. out must not alias
 * any input; k, v must not alias the rings.
 */
int swa_chunk_forward(const void* q, const void* k, const void* v, void* kring, void* vring,
                      const int64_t* pos, void* out, int64_t B, int64_t H, int64_t C,
                      int64_t D, int64_t W, void* stream);

/*
 * swa_ring_append: write C new tokens' keys and values into the rolling buffer.
 *
 * Position pos[b] + c of stream b goes to slot (pos[b] + c) mod W of kring and vring
 * ("25. Sliding-Window Causal Attention for Streaming Inference", Problem: the cache keeps
 * only the last W positions). When C > W only the last W tokens are written (the earlier
 * ones would be overwritten by the same call). Use it to seed the rings after a prefill
 * (pos = 0, C = T: the last min(T, W) positions land in their slots) or to add the token
 * a decode step will query (C = 1, pos = that token's position) before swa_decode.
 *   k, v         : [B, H, C, D] bf16 contiguous.  kring, vring : [B, H, W, D] bf16.
 *   pos          : [B] int64 on the device, each >= 0.  D : 64 or 128.
 * Errors: as swa_chunk_forward (a negative pos[b] leaves that stream's rings untouched and
 * is reported by swa_device_status()).
 */
int swa_ring_append(const void* k, const void* v, void* kring, void* vring, const int64_t* pos,
                    int64_t B, int64_t H, int64_t C, int64_t D, int64_t W, void* stream);

/*
 * swa_mha_forward: the sliding-window multi-head attention module of "NNX Sliding-Window
 * Attention" (A complete example with moving averages):
 *
 *   q = x Wq + bq, k = x Wk + bk, v = x Wv + bv   (y = x @ kernel + bias)
 *   head h of q, k, v is columns h*Dh .. h*Dh+Dh-1, Dh = d_model / H
 *   per head: sliding-window causal attention with window W and scale 1/sqrt(Dh)
 *   out = concat(heads) Wo + bo
 *
 *   x, out       : [B, T, d_model] contiguous, of `dtype`.
 *   wq, wk, wv, wo : [d_model, d_model] contiguous (input x output, the layout of the
 *                  page's Linear kernels), of `dtype`.
 *   bq, bk, bv, bo : [d_model] of `dtype`, or NULL for a zero bias.
 *   workspace    : caller-owned device buffer of workspace_bytes >= swa_mha_workspace_bytes
 *                  bytes, 256-byte aligned: q, k, v, the concatenated heads, and the GEMM
 *                  library's scratch. The library allocates no device memory here.
 *   dtype        : SWA_BF16 (Dh must be 64 or 128; projections in fp32 accumulation,
 *                  each of q, k, v and the heads rounded once to bf16) or SWA_F32 (any
 *                  Dh <= 4096; fp32 projections without TF32).
 * The projections are dense GEMMs run by cuBLASLt; the attention is swa_forward_ex reading
 * q, k, v in place as [B, T, H, Dh] (no transposes). All work is enqueued on `stream`.
 * Errors: as swa_forward_ex, plus d_model % H != 0 or a short workspace ->
 * SWA_ERR_INVALID_ARG, pointers not 16-byte aligned (workspace 256) -> SWA_ERR_MISALIGNED,
 * a GEMM library failure -> SWA_ERR_CUDA. B*T == 0 -> SWA_OK with nothing enqueued. Every
 * refusal, the attention's included, is decided before the first GEMM is enqueued; only
 * a CUDA or GEMM-library failure can come after earlier steps were enqueued, and out is
 * then undefined.
 */
int swa_mha_forward(const void* x, const void* wq, const void* bq, const void* wk, const void* bk,
                    const void* wv, const void* bv, const void* wo, const void* bo, void* out,
                    void* workspace, int64_t workspace_bytes, int64_t B, int64_t T,
                    int64_t d_model, int64_t H, int64_t W, int dtype, void* stream);

/* swa_mha_workspace_bytes: bytes of workspace swa_mha_forward needs for these sizes
 * (4 * B*T*d_model elements, each part rounded up to 256 bytes, plus 32 MiB of GEMM
 * scratch), or -1 for invalid sizes or dtype. */
int64_t swa_mha_workspace_bytes(int64_t B, int64_t T, int64_t d_model, int dtype);

/*
 * swa_forward_lse: swa_forward (contiguous operands, the given scale) that also writes the
 * natural log-sum-exp of every row's scaled scores, the statistic swa_backward needs:
 *   lse[b,h,i] = log( sum_{j in band(i)} exp(scale * q_i . k_j) )    [B, H, T] fp32.
 * Errors: as swa_forward_ex; a null lse (for a non-empty batch) -> SWA_ERR_INVALID_ARG,
 * an lse not 4-byte aligned -> SWA_ERR_MISALIGNED.
 */
int swa_forward_lse(const void* q, const void* k, const void* v, void* out, float* lse,
                    int64_t B, int64_t H, int64_t T, int64_t D, int64_t W, double scale,
                    int dtype, void* stream);

/*
 * swa_backward: gradients of the prefill with respect to q, k and v.
 *
 * "NNX Sliding-Window Attention" (Mask before softmax) notes that with the band masked to
 * -inf before the softmax the gradients stay well defined. With c = scale and p the
 * forward weights (only band pairs 0 <= i-j < W take part):
 *   dv_j = sum_i p_ij dout_i,  ds_ij = p_ij (dout_i . v_j - delta_i),
 *   delta_i = dout_i . out_i,  dq_i = c sum_j ds_ij k_j,  dk_j = c sum_i ds_ij q_i.
 *   q, k, v       : [B,H,T,D] contiguous inputs of `dtype`.
 *   out, lse      : the forward's output and log-sum-exp, from swa_forward_lse with the
 *                   same inputs and scale.
 *   dout          : [B,H,T,D] = dL/dout, of `dtype`.
 *   dq, dk, dv    : [B,H,T,D] contiguous outputs of `dtype` (overwritten).
 *   workspace     : caller-owned device buffer of workspace_bytes >=
 *                   swa_backward_workspace_bytes(B,H,T) bytes, 256-byte aligned.
 *   scale         : the forward's score scale (1/sqrt(D) for swa_forward), finite.
 *   dtype         : SWA_BF16 with D = 64 or 128 runs on the tensor cores (tcgen05):
 *                   P and dS are rounded to bf16 for the products, accumulation is fp32,
 *                   scale must be > 0. Other cases (SWA_F32, or bf16 with another D) run
 *                   in fp32 on the CUDA cores, D <= 512, recomputing the statistics
 *                   (out and lse are then not read and may be NULL).
 * There are no atomics: the results are deterministic. Errors (nothing is enqueued):
 *   invalid sizes, dtype or scale, a null pointer (out and lse included on the tensor-core
 *   path) or a workspace shorter than swa_backward_workspace_bytes -> SWA_ERR_INVALID_ARG;
 *   tensor-core path: tensors not 16-byte aligned, workspace not 256-byte aligned or lse
 *   not 4-byte aligned -> SWA_ERR_MISALIGNED, scale <= 0 -> SWA_ERR_UNSUPPORTED;
 *   CUDA-core path: D > 512 -> SWA_ERR_UNSUPPORTED, tensors not aligned to their element
 *   size or workspace not 8-byte aligned -> SWA_ERR_MISALIGNED.
 * B, H or T = 0 is a no-op that returns SWA_OK.
 */
int swa_backward(const void* q, const void* k, const void* v, const void* out,
                 const void* dout, const float* lse, void* dq, void* dk, void* dv,
                 void* workspace, int64_t workspace_bytes, int64_t B, int64_t H, int64_t T,
                 int64_t D, int64_t W, double scale, int dtype, void* stream);

/* swa_backward_workspace_bytes: 8*B*H*Tpad with Tpad = T rounded up to a multiple of 128,
 * or -1 for negative or overflowing sizes. */
int64_t swa_backward_workspace_bytes(int64_t B, int64_t H, int64_t T);

/*
 * swa_device_status: synchronize `stream`, then read and clear the current device's
 * status word. Returns SWA_OK, or the first error a kernel recorded since the last
 * call (SWA_ERR_TIMEOUT, SWA_ERR_INVALID_ARG), or SWA_ERR_CUDA if the synchronize or
 * the read fails (the CUDA error string is then in swa_last_error()).
 */
int swa_device_status(void* stream);

/* swa_last_error: message for the calling thread's last non-OK return ("" if none).
 * The pointer stays valid until the thread's next call into the library. */
const char* swa_last_error(void);

/*
 * swa_decode_noalloc: swa_decode without any device allocation by the library.
 *
 * The source pages describe no counterpart of this entry point; it exists for callers
 * that cannot let a library call cudaMalloc. Their device memory is owned end to end by
 * another allocator (a framework's caching allocator, or a serving runtime that carves a
 * fixed arena at start-up and counts any other allocation as a leak), or they run a
 * latency-bound decode step that must not take the implicit device-wide synchronisation
 * of cudaMalloc. Arguments, layout, results and errors are those of swa_decode, except:
 *  - The split partial states and ticket counters live in one file-scope device array
 *    of 4 MiB, which every GPU that loads the library holds until the process exits. The
 *    library's own split plan (about 16 CTAs per SM) needs at most 2.5 MB for any size;
 *    a request that would need more (B*H streams x splits x (D+2) floats plus B*H
 *    counters, possible only when the SWA_DECODE_CHUNK environment variable forces a
 *    small chunk) returns SWA_ERR_UNSUPPORTED with the byte count in swa_last_error()
 *    and enqueues nothing; use swa_decode for it.
 *  - The first call on a device looks up the array's device address and sets kernel
 *    attributes (no allocation); make that first call before any stream capture.
 *  - Every call shares the array and clears the counters it needs (cudaMemsetAsync on
 *    `stream`). Calls whose kernels overlap on the GPU race on the array: keep them on one
 *    stream, or otherwise ordered.
 * The caller still owns and passes every input and output buffer.
 */
int swa_decode_noalloc(const void* q, const void* kring, const void* vring, const int64_t* pos,
                       void* out, int64_t B, int64_t H, int64_t D, int64_t W, void* stream);

/* ---- Host-side work planning (no GPU needed; the kernels use the same code) ---- */

/*
 * swa_prefill_tile_class: how the tensor-core prefill treats the key tile kt for
 * the query tile qt, with query tiles of bm rows and key tiles of bn keys:
 *   0 - not visited (no query row of the tile has a key of the tile in its band),
 *   1 - edge tile (visited and masked element by element),
 *   2 - full tile (every (i, j) pair of the tile is in the band and j < T; no mask).
 * Visited tiles are kt_first .. kt_last with kt_first = max(0, qt*bm - W + 1) / bn and
 * kt_last = min(T - 1, qt*bm + bm - 1) / bn: only the tiles that meet the band, as
 * "NNX Sliding-Window Attention" (A local mask is not a sparse implementation) asks
 * of an implementation that does O(T * min(W, T) * D) work. The kernels use bm = bn = 128.
 * Returns -1 for invalid arguments (T < 1, W < 1, bm or bn < 1, qt or kt < 0,
 * qt*bm >= T).
 */
int swa_prefill_tile_class(int64_t T, int64_t W, int64_t bm, int64_t bn, int64_t qt, int64_t kt);

/*
 * swa_prefill_work_item: the u-th work item of the tensor-core prefill (bf16, D 64 or
 * 128) for sizes B, H, T and window W: the pair of 128-row query tiles (2*pair,
 * 2*pair+1) of head (b, h). Items 0 .. B*H*ceil(ceil(T/128)/2) - 1 cover every pair
 * once. First come the pairs of which both tiles exist and every row sees a whole
 * window (256*pair >= min(W,T) - 1): all the same work, head after head, so that the
 * CTAs at work together share a few heads' key and value tiles in L2. Then the lighter
 * pairs, heaviest first, head-minor. The persistent CTAs take items in a snake order
 * (CTA g of G: items g, 2G-1-g, 2G+g, ...). Writes *b, *h, *pair and returns 0, or
 * returns -1 for invalid arguments (B, H, T or W < 1, u out of range, null pointers).
 */
int swa_prefill_work_item(int64_t u, int64_t B, int64_t H, int64_t T, int64_t W, int64_t* b,
                          int64_t* h, int64_t* pair);

/*
 * swa_backward_cta_tile: the resident tile of the u-th CTA of the tensor-core backward
 * (bf16, D 64 or 128) for sizes B, H, T and window W. kv != 0: the key-tile kernel
 * (dK, dV), whose key tile kt meets min(n_t - kt, a + 1) query tiles; kv == 0: the
 * query-tile kernel (dQ), whose query tile qt meets min(qt, a) + 1 key tiles; n_t =
 * ceil(T/128) and a = ceil((min(W,T) - 1)/128). CTAs 0 .. B*H*n_t - 1 cover every
 * (b, h, tile) once: first the tiles that meet a + 1 tiles, head after head, then the
 * others heaviest first, head-minor, so that the last CTAs to start are the lightest.
 * Writes *b, *h, *tile and returns 0, or returns -1 for invalid arguments (B, H, T or
 * W < 1, u out of range, null pointers).
 */
int swa_backward_cta_tile(int64_t u, int64_t B, int64_t H, int64_t T, int64_t W, int kv, int64_t* b,
                          int64_t* h, int64_t* tile);

/*
 * swa_decode_valid_slots: number n of ring slots that hold in-window positions for a
 * stream at position pos: n = min(pos + 1, W); the valid slots are 0 .. n-1.
 * Returns -1 if pos < 0 or W < 1.
 */
int64_t swa_decode_valid_slots(int64_t pos, int64_t W);

/*
 * swa_decode_split_plan: how swa_decode splits each stream's ring for B*H streams:
 * writes the number of chunks per (b,h) and the chunk length in slots. Returns
 * SWA_OK or SWA_ERR_INVALID_ARG.
 */
int swa_decode_split_plan(int64_t B, int64_t H, int64_t D, int64_t W,
                          int32_t* splits, int32_t* chunk);

/* ---- Diagnostics ---- */

/*
 * Prefill modes (swa_set_prefill_mode), for the bf16 tensor-core prefill with D 64 or 128
 * (swa_forward, swa_forward_ex, swa_forward_lse, swa_forward_host, swa_mha_forward).
 * Every mode meets the same bound on |output - exact|; they differ in how:
 *   SWA_PREFILL_FAST: P (the softmax weights) is one bf16 value per key on every tile past
 *     a head's first 128 rows (bands longer than 144 keys). A row in which one key ends up
 *     above a quarter of the weight and some output reaches 1 in magnitude is recomputed
 *     in fp32 by one warp per SM, over its whole band. Fastest on inputs where such rows
 *     are rare (N(0,1) scores); inputs whose rows are mostly dominated by a few keys make
 *     almost every row such a row and run 100 to 1000 times slower.
 *   SWA_PREFILL_ADAPTIVE: a tile carries P as two bf16 parts (hi + lo, and a second P.V
 *     product) for every warp of 32 rows in which a key could end up above a quarter of its
 *     row's weight; no row needs recomputing. About an eighth slower than FAST on N(0,1)
 *     inputs, and within a few times of it on any input.
 *   SWA_PREFILL_AUTO (the default): FAST until a launch meets more than a few such rows in
 *     one SM's work, then ADAPTIVE for every later launch on that device (see
 *     swa_prefill_auto_state). Results are within the bound either way, but not bitwise the
 *     same across the switch.
 * The modes are process-wide settings read at each launch; a CUDA graph that captured a
 * prefill keeps the kernel chosen when it was captured.
 */
#define SWA_PREFILL_AUTO 0
#define SWA_PREFILL_ADAPTIVE 1
#define SWA_PREFILL_FAST 2

/*
 * swa_set_prefill_mode: set the prefill mode (above) for later launches; returns the
 * previous mode, or -1 (and sets the last error) for an unknown mode.
 */
int swa_set_prefill_mode(int mode);

/*
 * swa_prefill_auto_state: whether SWA_PREFILL_AUTO has switched to adaptive on the current
 * device (1) or not (0); clear != 0 switches it back. Synchronous (a copy from or to the
 * device). Returns -1 (and sets the last error) if the copy fails.
 */
int swa_prefill_auto_state(int clear);

/*
 * swa_set_wait_limit_ns: time limit of every bounded wait inside the kernels, in
 * nanoseconds (default 2e9, or the SWA_WAIT_LIMIT_NS environment variable). A wait
 * that runs past it makes the kernel record SWA_ERR_TIMEOUT, let its in-flight copies
 * and tensor-core operations finish, free its tensor memory and return. 0 restores
 * the default. Returns the previous limit.
 */
uint64_t swa_set_wait_limit_ns(uint64_t ns);

/*
 * swa_timeout_probe: launch one CTA that waits on an mbarrier nothing ever arrives on,
 * under the current wait limit, so that the timeout path can be tested without a
 * fault or a hang. Afterwards swa_device_status() returns SWA_ERR_TIMEOUT.
 */
int swa_timeout_probe(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SWA_H */
