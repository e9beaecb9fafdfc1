"""float64 CPU oracle for sliding-window causal attention.

TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the benchmark's
CPU-baseline leg may import this package. The CUDA library never imports it, shares
no code with it and never falls back to it.

What it computes is written out in swa_oracle.c (plain float64 loops, OpenMP over
rows). This module only marshals numpy arrays into that library with ctypes.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def _load(path=None):
    global _lib
    if path is not None:
        lib = ctypes.CDLL(path)
    else:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(_build.build())
    d = ctypes.POINTER(ctypes.c_double)
    i64 = ctypes.c_int64
    pi64 = ctypes.POINTER(ctypes.c_int64)
    lib.swa_oracle_forward.argtypes = [d, d, d, d, i64, i64, i64, i64, i64]
    lib.swa_oracle_forward_rows.argtypes = [d, d, d, i64, i64, i64, i64, i64, pi64, i64, d]
    lib.swa_oracle_weights.argtypes = [d, d, d, i64, i64, i64, i64, i64]
    lib.swa_oracle_decode.argtypes = [d, d, d, pi64, d, i64, i64, i64, i64]
    lib.swa_oracle_forward_scaled.argtypes = [d, d, d, d, i64, i64, i64, i64, i64, ctypes.c_double]
    lib.swa_oracle_weights_scaled.argtypes = [d, d, d, i64, i64, i64, i64, i64, ctypes.c_double]
    lib.swa_oracle_chunk.argtypes = [d, d, d, d, d, pi64, d, i64, i64, i64, i64, i64]
    lib.swa_oracle_backward.argtypes = [d, d, d, d, d, d, d, i64, i64, i64, i64, i64]
    lib.swa_oracle_ring_append.argtypes = [d, d, d, d, pi64, i64, i64, i64, i64, i64]
    for f in (lib.swa_oracle_forward, lib.swa_oracle_forward_rows, lib.swa_oracle_weights,
              lib.swa_oracle_decode, lib.swa_oracle_forward_scaled, lib.swa_oracle_weights_scaled,
              lib.swa_oracle_chunk, lib.swa_oracle_ring_append, lib.swa_oracle_backward):
        f.restype = ctypes.c_int
    if path is None:
        _lib = lib
    return lib


def _f64(a):
    a = np.ascontiguousarray(a, dtype=np.float64)
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _i64(a):
    a = np.ascontiguousarray(a, dtype=np.int64)
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))


class OracleError(ValueError):
    pass


def forward(q, k, v, W, lib=None, scale=None):
    """out[B,H,T,D] (float64) for q, k, v of shape [B,H,T,D] and window W. scale=None is
    the default 1/sqrt(D); a number multiplies the dot products instead."""
    lib = lib or _load()
    q, pq = _f64(q)
    k, pk = _f64(k)
    v, pv = _f64(v)
    if q.ndim != 4 or k.shape != q.shape or v.shape != q.shape:
        raise OracleError("q, k, v must share one [B,H,T,D] shape")
    B, H, T, D = q.shape
    out = np.empty_like(q)
    _, po = _f64(out)
    if scale is None:
        rc = lib.swa_oracle_forward(pq, pk, pv, po, B, H, T, D, int(W))
    else:
        rc = lib.swa_oracle_forward_scaled(pq, pk, pv, po, B, H, T, D, int(W), float(scale))
    if rc != 0:
        raise OracleError(f"oracle forward rejected its arguments (rc={rc})")
    return out


def max_threads(lib=None):
    """Threads the oracle's parallel loops run with (OpenMP's team size)."""
    return int((lib or _load()).swa_oracle_max_threads())


def set_threads(n, lib=None):
    """Run the oracle's later parallel loops on n threads (OpenMP's team size)."""
    lib = lib or _load()
    lib.swa_oracle_set_threads.argtypes = [ctypes.c_int]
    lib.swa_oracle_set_threads.restype = None
    lib.swa_oracle_set_threads(int(n))


def forward_rows(q, k, v, W, rows, lib=None):
    """Outputs [n, D] of the flattened query rows r = (b*H + h)*T + i listed in rows."""
    lib = lib or _load()
    q, pq = _f64(q)
    k, pk = _f64(k)
    v, pv = _f64(v)
    B, H, T, D = q.shape
    rows, pr = _i64(rows)
    out = np.empty((rows.shape[0], D), dtype=np.float64)
    _, po = _f64(out)
    rc = lib.swa_oracle_forward_rows(pq, pk, pv, B, H, T, D, int(W), pr, rows.shape[0], po)
    if rc != 0:
        raise OracleError(f"oracle forward_rows rejected its arguments (rc={rc})")
    return out


def weights(q, k, W, lib=None, scale=None):
    """Attention weights [B,H,T,T] of the definition (small inputs only); scale as forward."""
    lib = lib or _load()
    q, pq = _f64(q)
    k, pk = _f64(k)
    B, H, T, D = q.shape
    w = np.empty((B, H, T, T), dtype=np.float64)
    _, pw = _f64(w)
    if scale is None:
        rc = lib.swa_oracle_weights(pq, pk, pw, B, H, T, D, int(W))
    else:
        rc = lib.swa_oracle_weights_scaled(pq, pk, pw, B, H, T, D, int(W), float(scale))
    if rc != 0:
        raise OracleError(f"oracle weights rejected its arguments (rc={rc})")
    return w


def decode(q, kring, vring, pos, W, lib=None):
    """out[B,H,D] for one query per stream over the rolling buffer (slot = pos mod W)."""
    lib = lib or _load()
    q, pq = _f64(q)
    kring, pk = _f64(kring)
    vring, pv = _f64(vring)
    pos, pp = _i64(pos)
    B, H, D = q.shape
    if kring.shape != (B, H, W, D) or vring.shape != (B, H, W, D) or pos.shape != (B,):
        raise OracleError("rings must be [B,H,W,D] and pos [B]")
    out = np.empty_like(q)
    _, po = _f64(out)
    rc = lib.swa_oracle_decode(pq, pk, pv, pp, po, B, H, D, int(W))
    if rc != 0:
        raise OracleError(f"oracle decode rejected its arguments (rc={rc})")
    return out


def chunk(q, kc, vc, kring, vring, pos, W, lib=None):
    """out[B,H,C,D] for a chunk of C new tokens per stream (positions pos[b] ..
    pos[b]+C-1) over the rolling buffer that holds the positions before it."""
    lib = lib or _load()
    q, pq = _f64(q)
    kc, pkc = _f64(kc)
    vc, pvc = _f64(vc)
    kring, pkr = _f64(kring)
    vring, pvr = _f64(vring)
    pos, pp = _i64(pos)
    B, H, C, D = q.shape
    if kc.shape != q.shape or vc.shape != q.shape or kring.shape != (B, H, W, D) or \
            vring.shape != (B, H, W, D) or pos.shape != (B,):
        raise OracleError("chunk: q/k/v [B,H,C,D], rings [B,H,W,D], pos [B]")
    out = np.empty_like(q)
    _, po = _f64(out)
    rc = lib.swa_oracle_chunk(pq, pkc, pvc, pkr, pvr, pp, po, B, H, C, D, int(W))
    if rc != 0:
        raise OracleError(f"oracle chunk rejected its arguments (rc={rc})")
    return out


def ring_append(kc, vc, kring, vring, pos, W, lib=None):
    """New (kring, vring) after the chunk's positions pos[b] .. pos[b]+C-1 enter the
    ring, position p into slot p mod W (the inputs are not modified)."""
    lib = lib or _load()
    kc, pkc = _f64(kc)
    vc, pvc = _f64(vc)
    kring = np.array(kring, dtype=np.float64, copy=True, order="C")
    vring = np.array(vring, dtype=np.float64, copy=True, order="C")
    pkr = kring.ctypes.data_as(ctypes.POINTER(ctypes.c_double))
    pvr = vring.ctypes.data_as(ctypes.POINTER(ctypes.c_double))
    pos, pp = _i64(pos)
    B, H, C, D = kc.shape
    if vc.shape != kc.shape or kring.shape != (B, H, W, D) or vring.shape != (B, H, W, D):
        raise OracleError("ring_append: k/v [B,H,C,D], rings [B,H,W,D]")
    rc = lib.swa_oracle_ring_append(pkc, pvc, pkr, pvr, pp, B, H, C, D, int(W))
    if rc != 0:
        raise OracleError(f"oracle ring_append rejected its arguments (rc={rc})")
    return kring, vring


def backward(q, k, v, dout, W, lib=None):
    """Gradients (dq, dk, dv), each [B,H,T,D] float64, of the prefill output with respect
    to q, k and v, given the output gradient dout [B,H,T,D]."""
    lib = lib or _load()
    q, pq = _f64(q)
    k, pk = _f64(k)
    v, pv = _f64(v)
    dout, pdo = _f64(dout)
    if q.ndim != 4 or any(t.shape != q.shape for t in (k, v, dout)):
        raise OracleError("q, k, v, dout must share one [B,H,T,D] shape")
    B, H, T, D = q.shape
    grads = [np.empty_like(q) for _ in range(3)]
    ptrs = [_f64(g)[1] for g in grads]
    rc = lib.swa_oracle_backward(pq, pk, pv, pdo, *ptrs, B, H, T, D, int(W))
    if rc != 0:
        raise OracleError(f"oracle backward rejected its arguments (rc={rc})")
    return tuple(grads)


def mha(x, wq, bq, wk, bk, wv, bv, wo, bo, H, W, lib=None):
    """The sliding-window multi-head attention module of "NNX Sliding-Window Attention"
    (A complete example with moving averages), in float64: each projection is
    y = x @ kernel + bias with a [d, d] (in x out) kernel; q, k and v are split into H
    heads of Dh = d / H columns (head h is columns h*Dh .. h*Dh+Dh-1); every head runs
    the sliding-window attention of forward() above; the heads are concatenated in head
    order and projected by wo, bo. x is [B, T, d] or [T, d]; a bias may be None (zero).
    The projections are numpy matmuls (a library step); the attention is the C oracle."""
    x = np.asarray(x, dtype=np.float64)
    squeeze = x.ndim == 2
    if squeeze:
        x = x[None]
    B, T, d = x.shape
    if H < 1 or d % H:
        raise OracleError("d_model must be a multiple of the head count")
    Dh = d // H

    def linear(a, w, b):
        y = np.matmul(a, np.asarray(w, dtype=np.float64))
        return y if b is None else y + np.asarray(b, dtype=np.float64)

    heads = lambda y: y.reshape(B, T, H, Dh).transpose(0, 2, 1, 3)
    q, k, v = heads(linear(x, wq, bq)), heads(linear(x, wk, bk)), heads(linear(x, wv, bv))
    o = forward(q, k, v, W, lib=lib)
    concat = o.transpose(0, 2, 1, 3).reshape(B, T, d)
    out = linear(concat, wo, bo)
    return out[0] if squeeze else out


def load_variant(path):
    """Load another build of swa_oracle.c (used by the mutation tests)."""
    return _load(path)
