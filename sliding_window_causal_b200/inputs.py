"""Seeded synthetic inputs and the named workloads.

This module draws random numbers and nothing else: it holds none of the attention
arithmetic. The tests feed the same host tensors to the float64 oracle and to the
CUDA library; the benchmark uses the same recipes.

Recipe: one CPU torch.Generator per workload, seeded with 1000 + the workload's index.
torch.randn in float32 is drawn in the order q, k, v (then the rings and positions for
the streaming workloads),
and rounded to bfloat16 (round to nearest even, torch's .to()) when the workload is
bf16. Tensors larger than CHUNK elements are drawn one leading index at a time, so
the host never holds a float32 copy of a multi-gigabyte ring.
"""
from dataclasses import dataclass, field

import torch

CHUNK = 1 << 26


@dataclass(frozen=True)
class Prefill:
    name: str
    B: int
    H: int
    T: int
    D: int
    W: int
    dtype: torch.dtype
    seed: int


@dataclass(frozen=True)
class Decode:
    name: str
    B: int
    H: int
    D: int
    W: int
    pos_max: int
    dtype: torch.dtype
    seed: int


@dataclass(frozen=True)
class Chunk:
    name: str
    B: int
    H: int
    C: int
    D: int
    W: int
    pos_max: int
    dtype: torch.dtype
    seed: int


# The five workloads, in order; seed = 1000 + index.
TINY = [Prefill(f"tiny fp32 B1 H2 T6 D4 W{w}", 1, 2, 6, 4, w, torch.float32, 1000) for w in (3, 6, 1)]
SMALL = Prefill("small bf16 B1 H8 T512 D64 W128", 1, 8, 512, 64, 128, torch.bfloat16, 1001)
MISTRAL = Prefill("mistral-shaped bf16 B1 H32 T16384 D128 W4096", 1, 32, 16384, 128, 4096,
                  torch.bfloat16, 1002)
SWEEP = [Prefill(f"window sweep bf16 B2 H16 T8192 D128 W{w}", 2, 16, 8192, 128, w, torch.bfloat16, 1003)
         for w in (1, 256, 1024, 4096, 8192)]
DECODE = Decode("streaming decode bf16 B64 H32 D128 W4096", 64, 32, 128, 4096, 100000,
                torch.bfloat16, 1004)
# Chunked streaming prefill: the decode workload's streams and rings, each taking a chunk of
# 128 new tokens at once instead of one (seed 1005).
CHUNKED = Chunk("streaming chunk bf16 B64 H32 C128 D128 W4096", 64, 32, 128, 128, 4096, 100000,
                torch.bfloat16, 1005)


def _randn(gen, shape, dtype):
    n = 1
    for s in shape:
        n *= s
    if n <= CHUNK or len(shape) == 1:
        return torch.randn(shape, generator=gen, dtype=torch.float32).to(dtype)
    out = torch.empty(shape, dtype=dtype)
    for i in range(shape[0]):
        out[i] = _randn(gen, shape[1:], dtype)
    return out


def prefill_inputs(B, H, T, D, dtype, seed):
    """q, k, v of shape [B,H,T,D] on the CPU, i.i.d. N(0,1), rounded to dtype."""
    gen = torch.Generator().manual_seed(seed)
    q = _randn(gen, (B, H, T, D), dtype)
    k = _randn(gen, (B, H, T, D), dtype)
    v = _randn(gen, (B, H, T, D), dtype)
    return q, k, v


def peaked_prefill_inputs(B, H, T, D, seed, kind):
    """bf16 q, k, v of shape [B,H,T,D] on the CPU whose rows a few keys dominate: q is all
    ones and every key row is a base value (the same in each of its D elements) plus
    N(0, 0.01^2) noise. "growing": base 0.05*t, so the newest keys of each band dominate;
    "falling": -0.05*t, so the oldest do; "spikes": T // 50 keys at random positions get
    base 1, the rest 0. v ~ N(0, 1)."""
    gen = torch.Generator().manual_seed(seed)
    q = torch.ones(B, H, T, D)
    t = torch.arange(T, dtype=torch.float32)
    if kind == "growing":
        base = 0.05 * t
    elif kind == "falling":
        base = -0.05 * t
    elif kind == "spikes":
        base = torch.zeros(T)
        base[torch.randint(0, T, (T // 50,), generator=gen)] = 1.0
    else:
        raise ValueError(f"unknown kind {kind!r}")
    k = base[None, None, :, None].expand(B, H, T, D).clone() + 0.01 * torch.randn(B, H, T, D, generator=gen)
    v = torch.randn(B, H, T, D, generator=gen)
    return tuple(x.to(torch.bfloat16) for x in (q, k, v))


def decode_inputs(B, H, D, W, pos_max, dtype, seed):
    """q [B,H,D], kring and vring [B,H,W,D] i.i.d. N(0,1) rounded to dtype, and
    pos [B] int64 uniform in [0, pos_max), all on the CPU."""
    gen = torch.Generator().manual_seed(seed)
    q = _randn(gen, (B, H, D), dtype)
    kring = _randn(gen, (B, H, W, D), dtype)
    vring = _randn(gen, (B, H, W, D), dtype)
    pos = torch.randint(0, pos_max, (B,), generator=gen, dtype=torch.int64)
    return q, kring, vring, pos


def chunk_inputs(B, H, C, D, W, pos_max, dtype, seed):
    """q, k, v [B,H,C,D] (the chunk), kring and vring [B,H,W,D] i.i.d. N(0,1) rounded to
    dtype, and pos [B] int64 uniform in [0, pos_max), all on the CPU."""
    gen = torch.Generator().manual_seed(seed)
    q = _randn(gen, (B, H, C, D), dtype)
    k = _randn(gen, (B, H, C, D), dtype)
    v = _randn(gen, (B, H, C, D), dtype)
    kring = _randn(gen, (B, H, W, D), dtype)
    vring = _randn(gen, (B, H, W, D), dtype)
    pos = torch.randint(0, pos_max, (B,), generator=gen, dtype=torch.int64)
    return q, k, v, kring, vring, pos


def for_workload(wl):
    if isinstance(wl, Prefill):
        return prefill_inputs(wl.B, wl.H, wl.T, wl.D, wl.dtype, wl.seed)
    if isinstance(wl, Chunk):
        return chunk_inputs(wl.B, wl.H, wl.C, wl.D, wl.W, wl.pos_max, wl.dtype, wl.seed)
    return decode_inputs(wl.B, wl.H, wl.D, wl.W, wl.pos_max, wl.dtype, wl.seed)
