/*
 * swa_oracle.c: float64 CPU oracle for sliding-window causal attention.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load this code. It shares no source, header,
 * helper or constant with the CUDA library, and the CUDA library never calls it.
 *
 * What it computes: the plain definition, written out with no blocking, fusion
 * or reordering. For every batch b, head h and query position i:
 *
 *   band(i) = { j : max(0, i-W+1) <= j <= i }
 *       "27. Sliding-Window Attention", Step-by-Step Approach, step 2: a key is
 *       kept when it is not after the query and fewer than W positions behind it.
 *       "25. Sliding-Window Causal Attention for Streaming Inference",
 *       Step-by-Step Approach, step 3: the same two bounds, the lower one strict
 *       (j > i - W).
 *       "NNX Sliding-Window Attention", opening paragraph: keys from
 *       max(0, i - W + 1) through i.
 *   s_j    = (sum_d q[b,h,i,d] * k[b,h,j,d]) / sqrt(D)       for j in band(i)
 *       "27. Sliding-Window Attention", Step-by-Step Approach, step 1.
 *   m      = max_j s_j
 *   e_j    = exp(s_j - m)
 *       "Mistral Architecture > Implementation: Sliding Window Attention",
 *       Step 2 (stable softmax: subtract the row maximum before exponentiating).
 *   out[b,h,i,:] = (sum_j e_j * v[b,h,j,:]) / (sum_j e_j)
 *       "27. Sliding-Window Attention", Step-by-Step Approach, step 5
 *       (softmax over the keys, then weights @ v).
 *
 * Keys outside band(i) are never read: a masked score has exactly zero weight
 * after the softmax, so leaving it out of the sums is the same result
 * ("27. Sliding-Window Attention", step 3). The loops run in plain order:
 * j ascending, d ascending. All arithmetic is IEEE float64. There is no -ffast-math.
 *
 * Layout: every tensor is row-major contiguous [B, H, T, D], so element
 * (b,h,t,d) sits at ((b*H + h)*T + t)*D + d ("27. Sliding-Window Attention",
 * reference solution: the queries are laid out batch, then head, then position, then
 * feature).
 *
 * Decode: the rolling buffer keeps the last W positions of each stream. Position
 * p lives in slot p mod W ("25. Sliding-Window Causal Attention for Streaming
 * Inference", Problem: a bounded KV cache that evicts anything older than the
 * window). For stream b at absolute position P the query attends to positions
 * max(0, P-W+1) .. P, in ascending position order, read from slot p mod W.
 *
 * Scale: the *_scaled entry points multiply the dot products by a caller-given
 * factor instead of 1/sqrt(D) ("Mistral Architecture > Implementation: Sliding
 * Window Attention", Step 2: the caller may pass the scale; 1/sqrt(D) when absent).
 * The plain entry points are those with scale = 1/sqrt(D).
 *
 * Return codes: 0 on success, 1 for an invalid argument (W < 1, a negative size,
 * a null pointer, a negative position, a non-finite scale). On error nothing is
 * written.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_INVALID 1

/* One query row of the prefill definition. qi: [D]. kh, vh: [T, D] for one (b,h).
 * out: [D]. scores: scratch of at least min(i+1, W) doubles. */
static void oracle_row(const double* qi, const double* kh, const double* vh,
                       int64_t i, int64_t D, int64_t W, double scale, double* scores,
                       double* out) {
    int64_t lo = i - W + 1;
    if (lo < 0) lo = 0;

    /* scores over the band, j ascending */
    double m = -INFINITY;
    for (int64_t j = lo; j <= i; ++j) {
        const double* kj = kh + j * D;
        double dot = 0.0;
        for (int64_t d = 0; d < D; ++d) dot += qi[d] * kj[d];
        double s = dot * scale;
        scores[j - lo] = s;
        if (s > m) m = s;
    }

    /* e_j = exp(s_j - m); numerator and denominator, j ascending */
    for (int64_t d = 0; d < D; ++d) out[d] = 0.0;
    double denom = 0.0;
    for (int64_t j = lo; j <= i; ++j) {
        double e = exp(scores[j - lo] - m);
        denom += e;
        const double* vj = vh + j * D;
        for (int64_t d = 0; d < D; ++d) out[d] += e * vj[d];
    }
    for (int64_t d = 0; d < D; ++d) out[d] = out[d] / denom;
}

static int check_sizes(int64_t B, int64_t H, int64_t T, int64_t D, int64_t W) {
    if (W < 1 || B < 0 || H < 0 || T < 0 || D < 1) return ORACLE_INVALID;
    return ORACLE_OK;
}

/* Full prefill: out[B,H,T,D] for every row, scores scaled by `scale`. */
int swa_oracle_forward_scaled(const double* q, const double* k, const double* v, double* out,
                              int64_t B, int64_t H, int64_t T, int64_t D, int64_t W,
                              double scale) {
    if (check_sizes(B, H, T, D, W) != ORACLE_OK || !isfinite(scale)) return ORACLE_INVALID;
    if (B * H * T == 0) return ORACLE_OK;
    if (!q || !k || !v || !out) return ORACLE_INVALID;
    const int64_t nrows = B * H * T;
    const int64_t band_max = (W < T) ? W : T;
    int bad = 0;
#pragma omp parallel
    {
        double* scores = (double*)malloc((size_t)band_max * sizeof(double));
        if (!scores) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 64)
            for (int64_t r = 0; r < nrows; ++r) {
                const int64_t bh = r / T, i = r % T;
                const double* kh = k + bh * T * D;
                const double* vh = v + bh * T * D;
                oracle_row(q + r * D, kh, vh, i, D, W, scale, scores, out + r * D);
            }
            free(scores);
        }
    }
    return bad ? ORACLE_INVALID : ORACLE_OK;
}

/* Full prefill with the default scale 1/sqrt(D). */
int swa_oracle_forward(const double* q, const double* k, const double* v, double* out,
                       int64_t B, int64_t H, int64_t T, int64_t D, int64_t W) {
    if (D < 1) return ORACLE_INVALID;
    return swa_oracle_forward_scaled(q, k, v, out, B, H, T, D, W, 1.0 / sqrt((double)D));
}

/* Selected rows only: rows[n] holds flattened row indices r = (b*H + h)*T + i.
 * out_rows: [n, D], row t of it is the output of query row rows[t]. */
int swa_oracle_forward_rows(const double* q, const double* k, const double* v,
                            int64_t B, int64_t H, int64_t T, int64_t D, int64_t W,
                            const int64_t* rows, int64_t n, double* out_rows) {
    if (check_sizes(B, H, T, D, W) != ORACLE_OK || n < 0) return ORACLE_INVALID;
    if (n == 0) return ORACLE_OK;
    if (!q || !k || !v || !rows || !out_rows) return ORACLE_INVALID;
    for (int64_t t = 0; t < n; ++t)
        if (rows[t] < 0 || rows[t] >= B * H * T) return ORACLE_INVALID;
    const int64_t band_max = (W < T) ? W : T;
    int bad = 0;
#pragma omp parallel
    {
        double* scores = (double*)malloc((size_t)band_max * sizeof(double));
        if (!scores) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (int64_t t = 0; t < n; ++t) {
                const int64_t r = rows[t];
                const int64_t bh = r / T, i = r % T;
                oracle_row(q + r * D, k + bh * T * D, v + bh * T * D, i, D, W,
                           1.0 / sqrt((double)D), scores, out_rows + t * D);
            }
            free(scores);
        }
    }
    return bad ? ORACLE_INVALID : ORACLE_OK;
}

/* Attention weights of the definition, for checking probabilities on small
 * inputs: weights[B,H,T,T], zero outside the band, e_j / sum e_j inside, with the
 * scores scaled by `scale`. */
int swa_oracle_weights_scaled(const double* q, const double* k, double* weights,
                              int64_t B, int64_t H, int64_t T, int64_t D, int64_t W,
                              double scale) {
    if (check_sizes(B, H, T, D, W) != ORACLE_OK || !isfinite(scale)) return ORACLE_INVALID;
    if (B * H * T == 0) return ORACLE_OK;
    if (!q || !k || !weights) return ORACLE_INVALID;
    for (int64_t bh = 0; bh < B * H; ++bh) {
        for (int64_t i = 0; i < T; ++i) {
            double* wrow = weights + (bh * T + i) * T;
            for (int64_t j = 0; j < T; ++j) wrow[j] = 0.0;
            int64_t lo = i - W + 1;
            if (lo < 0) lo = 0;
            const double* qi = q + (bh * T + i) * D;
            double m = -INFINITY;
            for (int64_t j = lo; j <= i; ++j) {
                const double* kj = k + (bh * T + j) * D;
                double dot = 0.0;
                for (int64_t d = 0; d < D; ++d) dot += qi[d] * kj[d];
                wrow[j] = dot * scale;
                if (wrow[j] > m) m = wrow[j];
            }
            double denom = 0.0;
            for (int64_t j = lo; j <= i; ++j) {
                wrow[j] = exp(wrow[j] - m);
                denom += wrow[j];
            }
            for (int64_t j = lo; j <= i; ++j) wrow[j] = wrow[j] / denom;
        }
    }
    return ORACLE_OK;
}

/* Attention weights with the default scale 1/sqrt(D). */
int swa_oracle_weights(const double* q, const double* k, double* weights,
                       int64_t B, int64_t H, int64_t T, int64_t D, int64_t W) {
    if (D < 1) return ORACLE_INVALID;
    return swa_oracle_weights_scaled(q, k, weights, B, H, T, D, W, 1.0 / sqrt((double)D));
}

/* Decode over a rolling buffer. q: [B,H,D]; kring, vring: [B,H,W,D]; pos: [B];
 * out: [B,H,D]. Stream b attends to positions max(0, P-W+1)..P (P = pos[b]),
 * ascending, each read from slot p mod W; the same formula as a prefill row. */
static void oracle_decode_one(const double* qv, const double* kr, const double* vr,
                              int64_t P, int64_t D, int64_t W, double* scores, double* out) {
    int64_t first = P - W + 1;
    if (first < 0) first = 0;
    const double inv_sqrt_d = 1.0 / sqrt((double)D);
    double m = -INFINITY;
    for (int64_t p = first; p <= P; ++p) {
        const double* kp = kr + (p % W) * D;
        double dot = 0.0;
        for (int64_t d = 0; d < D; ++d) dot += qv[d] * kp[d];
        double s = dot * inv_sqrt_d;
        scores[p - first] = s;
        if (s > m) m = s;
    }
    for (int64_t d = 0; d < D; ++d) out[d] = 0.0;
    double denom = 0.0;
    for (int64_t p = first; p <= P; ++p) {
        double e = exp(scores[p - first] - m);
        denom += e;
        const double* vp = vr + (p % W) * D;
        for (int64_t d = 0; d < D; ++d) out[d] += e * vp[d];
    }
    for (int64_t d = 0; d < D; ++d) out[d] = out[d] / denom;
}

int swa_oracle_decode(const double* q, const double* kring, const double* vring,
                      const int64_t* pos, double* out,
                      int64_t B, int64_t H, int64_t D, int64_t W) {
    if (W < 1 || B < 0 || H < 0 || D < 1) return ORACLE_INVALID;
    if (B * H == 0) return ORACLE_OK;
    if (!q || !kring || !vring || !pos || !out) return ORACLE_INVALID;
    for (int64_t b = 0; b < B; ++b)
        if (pos[b] < 0) return ORACLE_INVALID;
    int bad = 0;
#pragma omp parallel
    {
        double* scores = (double*)malloc((size_t)W * sizeof(double));
        if (!scores) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t bh = 0; bh < B * H; ++bh) {
                const int64_t b = bh / H;
                oracle_decode_one(q + bh * D, kring + bh * W * D, vring + bh * W * D,
                                  pos[b], D, W, scores, out + bh * D);
            }
            free(scores);
        }
    }
    return bad ? ORACLE_INVALID : ORACLE_OK;
}

/* Chunked streaming prefill. Stream b has seen positions 0 .. pos[b]-1; the ring
 * holds the last min(pos[b], W) of them, position p in slot p mod W
 * ("25. Sliding-Window Causal Attention for Streaming Inference", Problem: a bounded
 * KV cache that keeps only the window; "Sliding Window Attention", Advantages: a KV
 * cache of size W). A chunk of C new tokens takes positions pos[b] .. pos[b]+C-1:
 * q, kc, vc, out are [B,H,C,D], kring, vring [B,H,W,D]. Query c, at position
 * P = pos[b] + c, attends to positions max(0, P-W+1) .. P in ascending order, with
 * the same formula as a prefill row: a position p < pos[b] is read from ring slot
 * p mod W, a position p >= pos[b] from chunk row p - pos[b]. */
static void oracle_chunk_one(const double* qc, const double* kcs, const double* vcs,
                             const double* kr, const double* vr, int64_t pos0, int64_t c,
                             int64_t D, int64_t W, double* scores, double* out) {
    const int64_t P = pos0 + c;
    int64_t first = P - W + 1;
    if (first < 0) first = 0;
    const double inv_sqrt_d = 1.0 / sqrt((double)D);
    double m = -INFINITY;
    for (int64_t p = first; p <= P; ++p) {
        const double* kp = (p < pos0) ? kr + (p % W) * D : kcs + (p - pos0) * D;
        double dot = 0.0;
        for (int64_t d = 0; d < D; ++d) dot += qc[d] * kp[d];
        double s = dot * inv_sqrt_d;
        scores[p - first] = s;
        if (s > m) m = s;
    }
    for (int64_t d = 0; d < D; ++d) out[d] = 0.0;
    double denom = 0.0;
    for (int64_t p = first; p <= P; ++p) {
        double e = exp(scores[p - first] - m);
        denom += e;
        const double* vp = (p < pos0) ? vr + (p % W) * D : vcs + (p - pos0) * D;
        for (int64_t d = 0; d < D; ++d) out[d] += e * vp[d];
    }
    for (int64_t d = 0; d < D; ++d) out[d] = out[d] / denom;
}

int swa_oracle_chunk(const double* q, const double* kc, const double* vc,
                     const double* kring, const double* vring, const int64_t* pos,
                     double* out, int64_t B, int64_t H, int64_t C, int64_t D, int64_t W) {
    if (W < 1 || B < 0 || H < 0 || C < 0 || D < 1) return ORACLE_INVALID;
    if (B * H * C == 0) return ORACLE_OK;
    if (!q || !kc || !vc || !kring || !vring || !pos || !out) return ORACLE_INVALID;
    for (int64_t b = 0; b < B; ++b)
        if (pos[b] < 0) return ORACLE_INVALID;
    const int64_t nrows = B * H * C;
    int bad = 0;
#pragma omp parallel
    {
        double* scores = (double*)malloc((size_t)W * sizeof(double));
        if (!scores) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t r = 0; r < nrows; ++r) {
                const int64_t bh = r / C, c = r % C, b = bh / H;
                oracle_chunk_one(q + r * D, kc + bh * C * D, vc + bh * C * D,
                                 kring + bh * W * D, vring + bh * W * D, pos[b], c, D, W,
                                 scores, out + r * D);
            }
            free(scores);
        }
    }
    return bad ? ORACLE_INVALID : ORACLE_OK;
}

/* Ring append: the chunk's positions pos[b] .. pos[b]+C-1 enter the ring in order,
 * position p into slot p mod W, each overwriting what the slot held. kc, vc:
 * [B,H,C,D]; kring, vring: [B,H,W,D], updated in place. */
int swa_oracle_ring_append(const double* kc, const double* vc, double* kring, double* vring,
                           const int64_t* pos, int64_t B, int64_t H, int64_t C, int64_t D,
                           int64_t W) {
    if (W < 1 || B < 0 || H < 0 || C < 0 || D < 1) return ORACLE_INVALID;
    if (B * H * C == 0) return ORACLE_OK;
    if (!kc || !vc || !kring || !vring || !pos) return ORACLE_INVALID;
    for (int64_t b = 0; b < B; ++b)
        if (pos[b] < 0) return ORACLE_INVALID;
    for (int64_t bh = 0; bh < B * H; ++bh) {
        const int64_t b = bh / H;
        for (int64_t c = 0; c < C; ++c) {
            const int64_t slot = (pos[b] + c) % W;
            for (int64_t d = 0; d < D; ++d) {
                kring[(bh * W + slot) * D + d] = kc[(bh * C + c) * D + d];
                vring[(bh * W + slot) * D + d] = vc[(bh * C + c) * D + d];
            }
        }
    }
    return ORACLE_OK;
}

/* Backward pass: the gradients of the prefill definition with respect to q, k and v,
 * given the gradient dout of the output ("NNX Sliding-Window Attention", Mask before
 * softmax: with the band masked to -inf before the softmax, the gradients are well
 * defined for finite allowed scores). They follow from the chain rule through the
 * definition above, row by row, with c = 1/sqrt(D):
 *
 *   p_j   = e_j / sum_l e_l                     for j in band(i)   (the forward weights)
 *   dv_j += p_j * dout_i
 *   dp_j  = dout_i . v_j
 *   ds_j  = p_j * (dp_j - sum_l p_l dp_l)       (softmax Jacobian)
 *   dq_i  = c * sum_j ds_j k_j
 *   dk_j += c * ds_j q_i
 *
 * Keys outside band(i) receive nothing from row i. Layout and loop order as the forward;
 * rows i ascending within each (b,h), so every sum has one fixed order. q, k, v, dout,
 * dq, dk, dv: [B,H,T,D]. */
int swa_oracle_backward(const double* q, const double* k, const double* v, const double* dout,
                        double* dq, double* dk, double* dv,
                        int64_t B, int64_t H, int64_t T, int64_t D, int64_t W) {
    if (check_sizes(B, H, T, D, W) != ORACLE_OK) return ORACLE_INVALID;
    if (B * H * T == 0) return ORACLE_OK;
    if (!q || !k || !v || !dout || !dq || !dk || !dv) return ORACLE_INVALID;
    const int64_t band_max = (W < T) ? W : T;
    const double c = 1.0 / sqrt((double)D);
    int bad = 0;
#pragma omp parallel
    {
        double* p = (double*)malloc((size_t)band_max * sizeof(double));
        double* dp = (double*)malloc((size_t)band_max * sizeof(double));
        if (!p || !dp) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t bh = 0; bh < B * H; ++bh) {
                const double* qh = q + bh * T * D;
                const double* kh = k + bh * T * D;
                const double* vh = v + bh * T * D;
                const double* doh = dout + bh * T * D;
                double* dqh = dq + bh * T * D;
                double* dkh = dk + bh * T * D;
                double* dvh = dv + bh * T * D;
                for (int64_t x = 0; x < T * D; ++x) {
                    dkh[x] = 0.0;
                    dvh[x] = 0.0;
                }
                for (int64_t i = 0; i < T; ++i) {
                    int64_t lo = i - W + 1;
                    if (lo < 0) lo = 0;
                    const double* qi = qh + i * D;
                    const double* doi = doh + i * D;
                    /* forward weights of row i */
                    double m = -INFINITY;
                    for (int64_t j = lo; j <= i; ++j) {
                        double dot = 0.0;
                        for (int64_t d = 0; d < D; ++d) dot += qi[d] * kh[j * D + d];
                        p[j - lo] = dot * c;
                        if (p[j - lo] > m) m = p[j - lo];
                    }
                    double denom = 0.0;
                    for (int64_t j = lo; j <= i; ++j) {
                        p[j - lo] = exp(p[j - lo] - m);
                        denom += p[j - lo];
                    }
                    for (int64_t j = lo; j <= i; ++j) p[j - lo] = p[j - lo] / denom;
                    /* dp_j and the weighted sum of dp */
                    double pdp = 0.0;
                    for (int64_t j = lo; j <= i; ++j) {
                        double dot = 0.0;
                        for (int64_t d = 0; d < D; ++d) dot += doi[d] * vh[j * D + d];
                        dp[j - lo] = dot;
                        pdp += p[j - lo] * dot;
                    }
                    for (int64_t d = 0; d < D; ++d) dqh[i * D + d] = 0.0;
                    for (int64_t j = lo; j <= i; ++j) {
                        const double ds = p[j - lo] * (dp[j - lo] - pdp);
                        for (int64_t d = 0; d < D; ++d) {
                            dqh[i * D + d] += c * ds * kh[j * D + d];
                            dkh[j * D + d] += c * ds * qi[d];
                            dvh[j * D + d] += p[j - lo] * doi[d];
                        }
                    }
                }
            }
        }
        free(p);
        free(dp);
    }
    return bad ? ORACLE_INVALID : ORACLE_OK;
}

/* The number of threads an OpenMP parallel region of this library runs with: what the
 * timings of these functions are reported against. */
int swa_oracle_max_threads(void) { return omp_get_max_threads(); }

/* Team size of the parallel loops that follow (for timing the oracle on fewer threads). */
void swa_oracle_set_threads(int n) {
    if (n > 0) omp_set_num_threads(n);
}
