"""Brute-force enumerators for tiny inputs (test infrastructure only).

These are deliberately naive and independent of swa_oracle.c: they build the
band mask pair by pair and evaluate attention as a dense masked matrix, the way
the pages' reference solutions do, so that the C oracle can be checked against a
second, differently structured computation.
"""
import numpy as np


def band_mask(T, W):
    """Boolean (T,T) mask, True where query i may attend key j.

    Built by a double loop over every pair, blocking a pair when the key lies in
    the future (j > i) or at least W steps in the past (i - j >= W), as in
    "Mistral Architecture > Implementation: Sliding Window Attention", Step 1:
    Building the Attention Mask.
    """
    m = np.ones((T, T), dtype=bool)
    for i in range(T):
        for j in range(T):
            if j > i:
                m[i, j] = False
            elif i - j >= W:
                m[i, j] = False
    return m


def dense_masked_attention(q, k, v, W):
    """float64 dense attention with the band applied by -inf replacement.

    Scores for every (i, j) pair, masked by where(), softmax with the row max
    subtracted, then weights @ v; "NNX Sliding-Window Attention", Mask before
    softmax, and "27. Sliding-Window Attention", reference solution.
    Returns (out, weights).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    T, D = q.shape[-2], q.shape[-1]
    scores = np.matmul(q, np.swapaxes(k, -1, -2)) / np.sqrt(D)
    mask = band_mask(T, W)
    scores = np.where(mask, scores, -np.inf)
    mx = scores.max(axis=-1, keepdims=True)
    e = np.exp(scores - mx)
    w = e / e.sum(axis=-1, keepdims=True)
    return np.matmul(w, v), w


def ring_positions(pos, W):
    """Positions held in a W-slot rolling buffer when the stream is at position pos,
    with the slot each one occupies: every position p in (pos-W, pos], p >= 0,
    lives in slot p mod W. Enumerated one position at a time."""
    out = []
    p = pos
    while p >= 0 and pos - p < W:
        out.append((p, p % W))
        p -= 1
    return sorted(out)
