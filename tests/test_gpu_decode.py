"""GPU rolling-buffer decode (swa_decode through the C ABI) against the float64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import sliding_window_causal_b200 as swa
from sliding_window_causal_b200 import inputs
from gpu_util import TOL, f64, max_err

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL_BF16 = TOL[torch.bfloat16]


def run(q, kr, vr, pos, W):
    out = swa.decode(q.to(DEV), kr.to(DEV), vr.to(DEV), pos.to(DEV), W)
    swa.device_status()
    return out


def positions(W, B, seed):
    """Positions covering the start of a stream, the fill-up edge and wrapped rings."""
    fixed = [0, 1, max(0, W - 2), W - 1, W, W + 1, 3 * W + 5, 99_999]
    rng = np.random.default_rng(seed)
    extra = rng.integers(0, 4 * W + 10, size=max(0, B - len(fixed)))
    return torch.tensor((fixed + list(extra))[:B], dtype=torch.int64)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("W", [1, 5, 64, 300, 2048])
def test_decode_parity(D, W):
    B, H = 8, 3
    q, kr, vr, _ = inputs.decode_inputs(B, H, D, W, 10, torch.bfloat16, 100 + W + D)
    pos = positions(W, B, W)
    out = run(q, kr, vr, pos, W)
    ref = oracle.decode(f64(q), f64(kr), f64(vr), pos.numpy(), W)
    assert max_err(out, ref) <= TOL_BF16


def test_decode_equals_last_prefill_row():
    """Write a seeded history into the ring (slot = position mod W, later positions
    overwrite earlier ones): decode at position P matches row P of the prefill over
    the history, on the GPU and in the oracle."""
    D, H, W, P = 128, 2, 200, 777
    q, k, v = inputs.prefill_inputs(1, H, P + 1, D, torch.bfloat16, 41)
    kr = torch.zeros(1, H, W, D, dtype=torch.bfloat16)
    vr = torch.zeros_like(kr)
    for p in range(P + 1):
        kr[:, :, p % W] = k[:, :, p]
        vr[:, :, p % W] = v[:, :, p]
    pos = torch.tensor([P], dtype=torch.int64)
    dec = run(q[:, :, P].contiguous(), kr, vr, pos, W)
    pre = swa.forward(q.to(DEV), k.to(DEV), v.to(DEV), W)[:, :, P]
    swa.device_status()
    ref = oracle.forward(f64(q), f64(k), f64(v), W)[:, :, P]
    assert max_err(dec, ref) <= TOL_BF16
    assert max_err(pre, ref) <= TOL_BF16


def test_invalid_slots_are_never_read():
    """Slots past min(pos+1, W) may hold anything, NaN included: output unchanged."""
    B, H, D, W = 4, 2, 128, 512
    q, kr, vr, _ = inputs.decode_inputs(B, H, D, W, 10, torch.bfloat16, 43)
    pos = torch.tensor([0, 5, 300, 510], dtype=torch.int64)
    base = run(q, kr, vr, pos, W).cpu()
    kr2, vr2 = kr.clone(), vr.clone()
    for b in range(B):
        n = min(int(pos[b]) + 1, W)
        kr2[b, :, n:] = float("nan")
        vr2[b, :, n:] = float("inf")
    out = run(q, kr2, vr2, pos, W).cpu()
    assert torch.equal(out, base)


def test_decode_deterministic():
    B, H, D, W = 16, 4, 128, 4096
    q, kr, vr, pos = inputs.decode_inputs(B, H, D, W, 100000, torch.bfloat16, 47)
    a = run(q, kr, vr, pos, W)
    b = run(q, kr, vr, pos, W)
    assert torch.equal(a, b)


def test_negative_position_reported():
    B, H, D, W = 2, 2, 64, 16
    q, kr, vr, _ = inputs.decode_inputs(B, H, D, W, 10, torch.bfloat16, 53)
    pos = torch.tensor([-1, 3], dtype=torch.int64)
    out = swa.decode(q.to(DEV), kr.to(DEV), vr.to(DEV), pos.to(DEV), W)
    with pytest.raises(swa.SwaError) as ei:
        swa.device_status()
    assert ei.value.code == 1
    assert bool((out[0] == 0).all())
    ref = oracle.decode(f64(q[1:]), f64(kr[1:]), f64(vr[1:]), pos[1:].numpy(), W)
    assert max_err(out[1:], ref) <= TOL_BF16


def test_decode_argument_errors():
    q = torch.zeros(1, 1, 96, dtype=torch.bfloat16, device=DEV)
    r = torch.zeros(1, 1, 4, 96, dtype=torch.bfloat16, device=DEV)
    pos = torch.zeros(1, dtype=torch.int64, device=DEV)
    with pytest.raises(swa.SwaError) as ei:
        swa.decode(q, r, r, pos, 4)
    assert ei.value.code == 2
    q = torch.zeros(1, 1, 64, dtype=torch.bfloat16, device=DEV)
    r = torch.zeros(1, 1, 4, 64, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ValueError):
        swa.decode(q, r, r, pos, 5)
    swa.device_status()


def test_workspace_reuse_across_sizes():
    """Calls of different sizes on one stream share the library's workspace: a large
    call followed by smaller ones (fewer streams, other split counts) stays exact."""
    cases = [(24, 3, 128, 3000), (2, 1, 128, 200), (5, 2, 64, 700), (1, 2, 128, 4096),
             (24, 3, 128, 3000)]
    for i, (B, H, D, W) in enumerate(cases):
        q, kr, vr, pos = inputs.decode_inputs(B, H, D, W, 5 * W, torch.bfloat16, 60 + i)
        out = run(q, kr, vr, pos, W)
        ref = oracle.decode(f64(q), f64(kr), f64(vr), pos.numpy(), W)
        assert max_err(out, ref) <= TOL_BF16, (B, H, D, W)
