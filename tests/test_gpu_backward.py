"""Gradients of the prefill (swa_backward through the C ABI) against the float64 oracle.

Tolerances, from the arithmetic: fp32 operands (CUDA cores), every gradient a sum of at
most 2*W products formed and added in fp32 with expf-based weights: 1e-4 absolute on O(1)
values. bf16 operands (the oracle sees the same bf16 values widened): on the tensor cores
P and dS are rounded to bf16 before their products, the forward output that delta is
formed from is bf16, and each gradient is rounded once to bf16; each rounding is at most
2^-9 relative and unbiased, so the bar is 1e-2 * max|gradient| + 2e-3."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import sliding_window_causal_b200 as swa
from sliding_window_causal_b200 import _native, inputs
from gpu_util import f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def grads_gpu(q, k, v, do, W):
    out = swa.backward(q.to(DEV), k.to(DEV), v.to(DEV), do.to(DEV), W)
    swa.device_status()
    return out


def check(B, H, T, D, W, dtype, seed):
    q, k, v = inputs.prefill_inputs(B, H, T, D, dtype, seed)
    g = torch.Generator().manual_seed(seed + 1)
    do = torch.randn(B, H, T, D, generator=g).to(dtype)
    got = grads_gpu(q, k, v, do, W)
    ref = oracle.backward(f64(q), f64(k), f64(v), f64(do), W)
    for name, a, b in zip(("dq", "dk", "dv"), got, ref):
        err = float(np.abs(f64(a) - b).max())
        tol = 1e-4 if dtype == torch.float32 else 1e-2 * float(np.abs(b).max()) + 2e-3
        assert err <= tol, f"{name}: max err {err} > {tol}"


@pytest.mark.parametrize("B,H,T,D,W", [(1, 2, 50, 16, 7), (2, 1, 130, 64, 40), (1, 2, 200, 33, 300),
                                       (1, 1, 64, 8, 1), (1, 3, 97, 128, 32), (1, 1, 45, 300, 9),
                                       (1, 1, 40, 512, 40)])
def test_backward_fp32(B, H, T, D, W):
    check(B, H, T, D, W, torch.float32, 11 + T + W)


@pytest.mark.parametrize("B,H,T,D,W", [(1, 2, 300, 64, 77), (1, 2, 257, 128, 128), (2, 1, 129, 128, 1000),
                                       (1, 1, 200, 32, 50), (2, 2, 640, 128, 1), (1, 2, 1000, 64, 300),
                                       (1, 1, 65, 128, 64), (1, 2, 191, 64, 63), (1, 1, 384, 128, 65),
                                       (1, 1, 2048, 64, 700)])
def test_backward_bf16(B, H, T, D, W):
    check(B, H, T, D, W, torch.bfloat16, 23 + T + W)


def test_backward_mid_size_bf16():
    """Two heads of a long sequence (T 4096, D 128, W 1024): every element."""
    check(1, 2, 4096, 128, 1024, torch.bfloat16, 31)


def test_backward_matches_gpu_forward_differences():
    """The gradients give the directional derivative of the GPU fp32 forward itself:
    sum(dout * (f(x + h u) - f(x - h u))) / 2h against sum(grad * u)."""
    B, H, T, D, W = 1, 2, 120, 32, 20
    q, k, v = (t.to(DEV).double().float() for t in inputs.prefill_inputs(B, H, T, D, torch.float32, 41))
    do = torch.randn(B, H, T, D, device=DEV)
    grads = swa.backward(q, k, v, do, W)
    h = 1e-2
    for which in range(3):
        u = torch.randn(B, H, T, D, device=DEV)
        args_p = [q, k, v]
        args_m = [q, k, v]
        args_p[which] = args_p[which] + h * u
        args_m[which] = args_m[which] - h * u
        fd = float(((swa.forward(*args_p, W) - swa.forward(*args_m, W)) * do).double().sum()) / (2 * h)
        an = float((grads[which] * u).double().sum())
        assert abs(fd - an) <= 2e-3 * max(1.0, abs(an)), f"operand {which}: {fd} vs {an}"
    swa.device_status()


def test_backward_deterministic():
    q, k, v = (t.to(DEV) for t in inputs.prefill_inputs(1, 2, 300, 64, torch.bfloat16, 43))
    do = torch.randn(1, 2, 300, 64, device=DEV).to(torch.bfloat16)
    a = swa.backward(q, k, v, do, 100)
    b = swa.backward(q, k, v, do, 100)
    swa.device_status()
    assert all(torch.equal(x, y) for x, y in zip(a, b))


def test_backward_outputs_complete_for_the_next_work_on_the_stream():
    """The query-tile kernel starts while the key-tile kernel's last CTAs run (a
    programmatic dependent launch) and waits for it before it ends: work enqueued on the
    stream right after the backward must see all three gradients complete. Sums taken on
    the stream with no synchronize in between equal the sums taken after one."""
    q, k, v = (t.to(DEV) for t in inputs.prefill_inputs(1, 16, 4096, 128, torch.bfloat16, 808))
    do = inputs.prefill_inputs(1, 16, 4096, 128, torch.bfloat16, 809)[0].to(DEV)
    out, lse = swa.forward_lse(q, k, v, 1024)
    for _ in range(3):
        dq, dk, dv = swa.backward(q, k, v, do, 1024, out=out, lse=lse)
        early = torch.stack([g.float().sum() for g in (dq, dk, dv)])  # same stream, no sync
        swa.device_status()
        late = torch.stack([g.float().sum() for g in (dq, dk, dv)])
        assert torch.equal(early, late)


@pytest.mark.parametrize("D,W", [(64, 50), (128, 6)])
def test_lse_matches_oracle_weights(D, W):
    """forward_lse's lse is log of the sum of exp(scaled score) over each band (W = 6:
    the bf16 CUDA-core kernel for short bands)."""
    B, H, T = 1, 2, 200
    for dtype in (torch.float32, torch.bfloat16):
        q, k, v = inputs.prefill_inputs(B, H, T, D, dtype, 47)
        out, lse = swa.forward_lse(q.to(DEV), k.to(DEV), v.to(DEV), W)
        swa.device_status()
        qd, kd = f64(q), f64(k)
        s = np.einsum("bhid,bhjd->bhij", qd, kd) / np.sqrt(D)
        i, j = np.arange(T)[:, None], np.arange(T)[None, :]
        s = np.where((i - j >= 0) & (i - j < W), s, -np.inf)
        ref = np.log(np.exp(s - s.max(-1, keepdims=True)).sum(-1)) + s.max(-1)
        tol = 1e-4 if dtype == torch.float32 else 2e-2
        assert float(np.abs(f64(lse) - ref).max()) <= tol
        assert torch.equal(out, swa.forward(q.to(DEV), k.to(DEV), v.to(DEV), W))


def test_backward_errors():
    lib = _native.lib()
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    t = torch.zeros(1, 1, 16, 513, device=DEV)
    need = lib.swa_backward_workspace_bytes(1, 1, 16)
    assert need == 128 * 8  # rows padded to a whole 128-row tile
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    lse = torch.zeros(1, 1, 16, device=DEV)
    p, w = t.data_ptr(), ws.data_ptr()
    outs = [torch.empty_like(t).data_ptr() for _ in range(3)]
    f = lambda *a: lib.swa_backward(p, p, p, p, p, lse.data_ptr(), *outs, *a)
    assert f(w, need, 1, 1, 16, 64, 4, 0.125, 0, s) == 0
    assert f(w, need - 8, 1, 1, 16, 64, 4, 0.125, 0, s) == 1     # short workspace
    assert f(w, need, 1, 1, 16, 64, 0, 0.125, 0, s) == 1         # W < 1
    assert f(w, need, 1, 1, 16, 64, 4, float("nan"), 0, s) == 1  # scale
    assert f(None, need, 1, 1, 16, 64, 4, 0.125, 0, s) == 1      # no workspace
    assert f(w, need, 1, 1, 16, 513, 4, 0.125, 0, s) == 2        # D above 512
    assert lib.swa_backward_workspace_bytes(-1, 1, 1) == -1
    swa.device_status()
