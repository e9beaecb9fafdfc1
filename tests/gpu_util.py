"""Helpers shared by the GPU parity tests: oracle comparisons on host copies."""
import numpy as np
import torch

# Tolerances on max |GPU - float64 oracle| over compared elements: fp32 in/out 1e-5,
# bf16 in/out with fp32 accumulation 1e-2 (the oracle runs on the same bf16-rounded
# inputs, widened exactly to float64).
TOL = {torch.float32: 1e-5, torch.bfloat16: 1e-2}


def f64(t):
    return t.detach().to("cpu").to(torch.float64).numpy()


def max_err(gpu_out, ref):
    return float(np.abs(f64(gpu_out) - ref).max()) if ref.size else 0.0


def sharp_inputs(B, H, T, D, seed, kind):
    """Inputs whose rows are dominated by a few keys: "growing" (scores rise along the
    sequence, so the newest keys dominate), "falling" (they fall, so the oldest keys of
    each band dominate) or "spikes" (a few keys with large scores anywhere). v ~ N(0,1)."""
    gen = torch.Generator().manual_seed(seed)
    q = torch.ones(B, H, T, D)
    t = torch.arange(T, dtype=torch.float32)
    if kind == "growing":
        base = 0.05 * t
    elif kind == "falling":
        base = -0.05 * t
    else:
        base = torch.zeros(T)
        base[torch.randint(0, T, (T // 50,), generator=gen)] = 1.0
    k = base[None, None, :, None].expand(B, H, T, D).clone() + 0.01 * torch.randn(B, H, T, D, generator=gen)
    v = torch.randn(B, H, T, D, generator=gen)
    return tuple(x.to(torch.bfloat16) for x in (q, k, v))
