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
