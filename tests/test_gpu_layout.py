"""Strided operands, a caller-given scale and the band weights (swa_forward_ex,
swa_band_weights through the C ABI) against the float64 oracle.

The [B,T,H,D] layout and the optional scale are those of "Mistral Architecture >
Implementation: Sliding Window Attention" (Step 2), which also returns the weights."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import sliding_window_causal_b200 as swa
from sliding_window_causal_b200 import _native, inputs
from gpu_util import TOL, f64, max_err, sharp_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def bthd_views(B, H, T, D, dtype, seed):
    """q, k, v stored as contiguous [B,T,H,D] on the device, returned as [B,H,T,D] views
    (strides (T*H*D, D, H*D, 1)), plus contiguous host copies for the oracle."""
    q, k, v = inputs.prefill_inputs(B, H, T, D, dtype, seed)  # [B,H,T,D] host
    dev = [t.transpose(1, 2).contiguous().to(DEV).transpose(1, 2) for t in (q, k, v)]
    for t in dev:
        assert not t.is_contiguous() or H == 1 or T == 1
    return dev, (q, k, v)


LAYOUT_SHAPES = [
    # B, H, T, D, W, dtype
    (1, 4, 300, 64, 77, torch.bfloat16), (2, 3, 1000, 128, 129, torch.bfloat16),
    (1, 2, 777, 128, 5000, torch.bfloat16), (1, 8, 512, 64, 128, torch.bfloat16),
    (2, 3, 50, 4, 6, torch.float32), (1, 2, 257, 33, 40, torch.float32),
    # short bands: the bf16 CUDA-core kernel reads the same strides
    (2, 3, 200, 128, 5, torch.bfloat16), (1, 4, 77, 64, 1, torch.bfloat16),
]


@pytest.mark.parametrize("B,H,T,D,W,dtype", LAYOUT_SHAPES)
def test_bthd_layout_matches_oracle(B, H, T, D, W, dtype):
    (dq, dk, dv), (q, k, v) = bthd_views(B, H, T, D, dtype, 100 + T + W)
    out = swa.forward(dq, dk, dv, W)
    swa.device_status()
    assert out.stride() == dq.stride(), "out keeps the [B,T,H,D] layout"
    ref = oracle.forward(f64(q), f64(k), f64(v), W)
    err = max_err(out, ref)
    assert err <= TOL[dtype], f"max err {err}"


def test_bthd_equals_contiguous_bitwise():
    """The same values through either layout give identical bits: the layout only
    changes addressing."""
    B, H, T, D, W = 1, 4, 700, 128, 200
    (dq, dk, dv), (q, k, v) = bthd_views(B, H, T, D, torch.bfloat16, 5)
    a = swa.forward(dq, dk, dv, W)
    b = swa.forward(q.to(DEV), k.to(DEV), v.to(DEV), W)
    swa.device_status()
    assert torch.equal(a.contiguous(), b)


def test_mixed_strides_and_strided_out():
    """Each operand with its own layout: q [B,T,H,D], k contiguous, v a slice of a wider
    buffer (head-dimension padding), out written into a [B,T,H,D] buffer."""
    B, H, T, D, W = 2, 2, 400, 64, 100
    q, k, v = inputs.prefill_inputs(B, H, T, D, torch.bfloat16, 9)
    dq = q.transpose(1, 2).contiguous().to(DEV).transpose(1, 2)
    dk = k.to(DEV)
    wide = torch.zeros(B, H, T, D + 64, dtype=torch.bfloat16, device=DEV)
    wide[..., :D] = v.to(DEV)
    dv = wide[..., :D]
    obuf = torch.full((B, T, H, D), float("nan"), dtype=torch.bfloat16, device=DEV)
    out = obuf.transpose(1, 2)
    swa.forward(dq, dk, dv, W, out=out)
    swa.device_status()
    ref = oracle.forward(f64(q), f64(k), f64(v), W)
    assert max_err(out, ref) <= TOL[torch.bfloat16]
    assert not torch.isnan(obuf).any()


SCALE_CASES = [(torch.bfloat16, 64, sc) for sc in (0.05, 0.3, 1.0)] + \
              [(torch.bfloat16, 128, sc) for sc in (0.02, 0.2)] + \
              [(torch.float32, 24, sc) for sc in (0.05, 0.3, -0.2, 0.0)]


@pytest.mark.parametrize("dtype,D,scale", SCALE_CASES)
def test_scale_matches_oracle(dtype, D, scale):
    B, H, T, W = 1, 2, 333, 90
    q, k, v = inputs.prefill_inputs(B, H, T, D, dtype, 17 + D)
    out = swa.forward(q.to(DEV), k.to(DEV), v.to(DEV), W, scale=scale)
    swa.device_status()
    ref = oracle.forward(f64(q), f64(k), f64(v), W, scale=scale)
    err = max_err(out, ref)
    assert err <= TOL[dtype], f"scale={scale} max err {err}"


def test_default_scale_is_swa_forward_bitwise():
    B, H, T, D, W = 1, 2, 500, 128, 200
    q, k, v = (t.to(DEV) for t in inputs.prefill_inputs(B, H, T, D, torch.bfloat16, 21))
    a = swa.forward(q, k, v, W)
    b = swa.forward(q, k, v, W, scale=1.0 / np.sqrt(D))
    swa.device_status()
    assert torch.equal(a, b)


def band_of(dense, Wo):
    """Gather the band [.., T, Wo] out of dense weights [.., T, T]: column c of row i is
    key j = i - Wo + 1 + c, zero where j < 0."""
    T = dense.shape[-1]
    out = np.zeros(dense.shape[:-1] + (Wo,))
    for i in range(T):
        for c in range(Wo):
            j = i - Wo + 1 + c
            if j >= 0:
                out[..., i, c] = dense[..., i, j]
    return out


@pytest.mark.parametrize("B,H,T,D,W,dtype", [
    (1, 2, 70, 16, 9, torch.float32), (2, 1, 40, 64, 40, torch.float32),
    (1, 2, 50, 8, 200, torch.float32), (1, 3, 90, 64, 33, torch.bfloat16),
    (1, 1, 37, 128, 1, torch.bfloat16)])
def test_band_weights_match_oracle(B, H, T, D, W, dtype):
    q, k, _ = inputs.prefill_inputs(B, H, T, D, dtype, 31 + T)
    w = swa.band_weights(q.to(DEV), k.to(DEV), W)
    swa.device_status()
    Wo = min(W, T)
    assert w.shape == (B, H, T, Wo) and w.dtype == torch.float32
    ref = band_of(oracle.weights(f64(q), f64(k), W), Wo)
    err = float(np.abs(f64(w) - ref).max())
    assert err <= 1e-5, f"weights max err {err}"
    assert float(np.abs(f64(w).sum(-1) - 1.0).max()) <= 1e-5


def test_band_weights_scale_and_layout():
    B, H, T, D, W = 1, 2, 60, 32, 12
    (dq, dk, _), (q, k, _) = bthd_views(B, H, T, D, torch.float32, 44)
    for sc in (0.0, 0.4, -0.9):
        w = swa.band_weights(dq, dk, W, scale=sc)
        swa.device_status()
        ref = band_of(oracle.weights(f64(q), f64(k), W, scale=sc), W)
        assert float(np.abs(f64(w) - ref).max()) <= 1e-5, f"scale={sc}"


def test_band_weights_times_v_is_forward():
    """The band weights applied to v reproduce the fp32 forward."""
    B, H, T, D, W = 1, 2, 80, 16, 10
    q, k, v = (t.to(DEV) for t in inputs.prefill_inputs(B, H, T, D, torch.float32, 55))
    w = swa.band_weights(q, k, W)
    out = swa.forward(q, k, v, W)
    swa.device_status()
    vb = torch.zeros(B, H, T, W, D, device=DEV)
    for c in range(W):
        shift = W - 1 - c  # key j = i - shift
        vb[:, :, shift:, c, :] = v[:, :, : T - shift, :]
    rec = torch.einsum("bhtc,bhtcd->bhtd", w, vb)
    assert float((rec - out).abs().max()) <= 1e-5


def test_layout_errors():
    lib = _native.lib()
    q = torch.zeros(1, 2, 64, 64, dtype=torch.bfloat16, device=DEV)
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ok = (ctypes.c_int64 * 12)(*([2 * 64 * 64, 64 * 64, 64] * 4))
    o = torch.empty_like(q)
    p, po = q.data_ptr(), o.data_ptr()
    assert lib.swa_forward_ex(p, p, p, po, 1, 2, 64, 64, 8, 0.125, ok, 1, s) == 0
    assert lib.swa_forward_ex(p, p, p, po, 1, 2, 64, 64, 8, float("nan"), ok, 1, s) == 1
    assert lib.swa_forward_ex(p, p, p, po, 1, 2, 64, 64, 8, float("inf"), ok, 1, s) == 1
    bad = (ctypes.c_int64 * 12)(*ok)
    bad[2] = 68  # t stride of q: not a multiple of 8 elements
    assert lib.swa_forward_ex(p, p, p, po, 1, 2, 64, 64, 8, 0.125, bad, 1, s) == 3
    neg = (ctypes.c_int64 * 12)(*ok)
    neg[4] = -64
    assert lib.swa_forward_ex(p, p, p, po, 1, 2, 64, 64, 8, 0.125, neg, 1, s) == 1
    # the tensor-core path takes positive scales only
    assert lib.swa_forward_ex(p, p, p, po, 1, 2, 64, 64, 8, 0.0, ok, 1, s) == 2
    assert lib.swa_forward_ex(p, p, p, po, 1, 2, 64, 64, 8, -0.5, ok, 1, s) == 2
    w = torch.empty(1, 2, 64, 8, device=DEV)
    assert lib.swa_band_weights(p, p, w.data_ptr(), 1, 2, 64, 64, 0, 0.1, None, 1, s) == 1
    assert lib.swa_band_weights(p, p, w.data_ptr(), 1, 2, 64, 64, 8, float("nan"), None, 1, s) == 1
    assert lib.swa_band_weights(p, p, None, 1, 2, 64, 64, 8, 0.1, None, 1, s) == 1
    swa.device_status()


def test_mistral_bthd_full_size_equals_contiguous():
    """The Mistral-shaped prefill (B1 H32 T16384 D128 W4096) with q, k, v and out in the
    [B,T,H,D] layout gives, in every element, the bits of the contiguous layout (whose
    every element test_gpu_fullsize.py compares with the oracle)."""
    wl = inputs.MISTRAL
    (dq, dk, dv), (q, k, v) = bthd_views(wl.B, wl.H, wl.T, wl.D, wl.dtype, wl.seed)
    a = swa.forward(dq, dk, dv, wl.W)
    b = swa.forward(q.to(DEV), k.to(DEV), v.to(DEV), wl.W)
    swa.device_status()
    assert a.stride() == dq.stride()
    assert torch.equal(a.contiguous(), b)


@pytest.mark.parametrize("kind", ["growing", "falling", "spikes"])
@pytest.mark.parametrize("D,W,scale", [(128, 600, None), (64, 300, 0.2), (128, 4096, None)])
def test_sharp_rows_bthd_and_scale(kind, D, W, scale):
    """Rows that a few keys dominate (recomputed in fp32 by the kernel) in the [B,T,H,D]
    layout and with a caller-given scale still match the oracle; so does the training
    forward's log-sum-exp of those rows."""
    B, H, T = 1, 3, 1300
    q, k, v = sharp_inputs(B, H, T, D, 90 + W + D, kind)
    dev = [x.transpose(1, 2).contiguous().to(DEV).transpose(1, 2) for x in (q, k, v)]
    out = swa.forward(*dev, W, scale=scale) if scale is not None else swa.forward(*dev, W)
    swa.device_status()
    ref = oracle.forward(f64(q), f64(k), f64(v), W, scale=scale)
    assert max_err(out, ref) <= TOL[torch.bfloat16]
    if scale is None:
        out2, lse = swa.forward_lse(q.to(DEV), k.to(DEV), v.to(DEV), W)
        swa.device_status()
        assert max_err(out2, ref) <= TOL[torch.bfloat16]
        # natural log-sum-exp of each row's scaled scores, from the float64 definition
        qd, kd = f64(q), f64(k)
        s = np.einsum("bhid,bhjd->bhij", qd, kd) / np.sqrt(D)
        i = np.arange(T)[:, None]
        j = np.arange(T)[None, :]
        s = np.where((i - j >= 0) & (i - j < W), s, -np.inf)
        mx = s.max(-1, keepdims=True)
        ref_lse = (mx + np.log(np.exp(s - mx).sum(-1, keepdims=True)))[..., 0]
        assert float(np.abs(f64(lse) - ref_lse).max()) <= 2e-2  # the bar of test_gpu_backward.py
