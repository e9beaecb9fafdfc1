"""Helpers shared by the GPU parity tests: oracle comparisons on host copies."""
import numpy as np
import torch

# Tolerances on max |GPU - float64 oracle| over compared elements: fp32 in/out 1e-5,
# bf16 in/out with fp32 accumulation 1e-2 (the oracle runs on the same bf16-rounded
# inputs, widened exactly to float64). A bf16 output cannot come closer to a real number
# than half the bf16 spacing there, which exceeds 1e-2 from magnitude 4 on (spacing 2^-5);
# so a bf16 element that is one of the two bf16 values bracketing the oracle's value also
# passes. Below magnitude 4 some bf16 value always lies within 1e-2, and the bar is 1e-2.
TOL = {torch.float32: 1e-5, torch.bfloat16: 1e-2}


def f64(t):
    return t.detach().to("cpu").to(torch.float64).numpy()


def bf16_bracket(r):
    """The largest and smallest bf16 values with lo <= r <= hi (equal when r is one),
    for finite float64 r in bf16's normal range: bf16 has 8 significand bits, so its
    spacing at |r| in [2^e, 2^(e+1)) is 2^(e-7)."""
    a = np.abs(r)
    ulp = np.exp2(np.floor(np.log2(np.where(a > 0, a, 1.0))) - 7)
    return np.floor(r / ulp) * ulp, np.ceil(r / ulp) * ulp


def max_err(gpu_out, ref):
    if not ref.size:
        return 0.0
    g = f64(gpu_out)
    e = np.abs(g - ref)
    if gpu_out.dtype == torch.bfloat16:
        lo, hi = bf16_bracket(ref)
        e = np.where((e > TOL[torch.bfloat16]) & ((g == lo) | (g == hi)), 0.0, e)
    return float(e.max())


def sharp_inputs(B, H, T, D, seed, kind):
    """Inputs whose rows are dominated by a few keys: "growing" (scores rise along the
    sequence, so the newest keys dominate), "falling" (they fall, so the oldest keys of
    each band dominate) or "spikes" (a few keys with large scores anywhere). v ~ N(0,1)."""
    from sliding_window_causal_b200 import inputs
    return inputs.peaked_prefill_inputs(B, H, T, D, seed, kind)
