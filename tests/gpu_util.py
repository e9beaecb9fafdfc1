"""Helpers shared by the GPU parity tests: oracle comparisons on host copies."""
import numpy as np
import torch

import oracle

# Tolerances on max |GPU - float64 oracle| over compared elements: fp32 in/out 1e-5,
# bf16 in/out with fp32 accumulation 1e-2 (the oracle runs on the same bf16-rounded
# inputs, widened exactly to float64).
TOL = {torch.float32: 1e-5, torch.bfloat16: 1e-2}


def f64(t):
    return t.detach().to("cpu").to(torch.float64).numpy()


def max_err(gpu_out, ref):
    return float(np.abs(f64(gpu_out) - ref).max()) if ref.size else 0.0


def sample_rows(T, W, n_random=96, seed=0):
    """Query rows that exercise every kind of position: the first rows (short
    windows), both sides of every multiple of 128 near the start and near W, rows
    around W-1 (first full window), the last rows, and random rows."""
    rng = np.random.default_rng(seed)
    rows = set(range(min(T, 130)))
    for c in (127, 128, 129, 255, 256, 257, W - 2, W - 1, W, W + 1, W + 127, W + 128,
              T // 2, T - 129, T - 128, T - 127, T - 2, T - 1):
        if 0 <= c < T:
            rows.add(c)
    rows.update(int(x) for x in rng.integers(0, T, size=n_random))
    return np.array(sorted(rows), dtype=np.int64)


def oracle_rows(q, k, v, W, heads, rows):
    """Oracle outputs for the given (b, h) heads and query rows; returns
    {(b, h): array [len(rows), D]}."""
    out = {}
    for (b, h) in heads:
        qh, kh, vh = (f64(t[b:b + 1, h:h + 1]) for t in (q, k, v))
        out[(b, h)] = oracle.forward_rows(qh, kh, vh, W, rows)
    return out
