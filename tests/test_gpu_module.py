"""The sliding-window multi-head attention module (swa_mha_forward through the C ABI):
cuBLASLt projections around the attention kernels, against the float64 oracle.

Tolerance for bf16: 2e-2. Beyond the attention's own bf16 error (the 1e-2 bar), four
intermediates are rounded to bf16 (q, k, v and the concatenated heads, each by at most
2^-9 relative): with unit-variance projections the rounding of q and k moves the scores
by about 2^-9 * |s|, and the rounding of the heads reaches the output through the output
kernel's sum over d terms of variance 1/d, a further ~2^-9. fp32 keeps the 1e-5 bar."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import sliding_window_causal_b200 as swa
from sliding_window_causal_b200 import _native
from golden import read_moving_average
from gpu_util import f64, max_err

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL_MODULE = {torch.float32: 1e-5, torch.bfloat16: 2e-2}


def params(d, dtype, seed, bias=True):
    """Unit-variance projections: kernels N(0, 1/d), biases N(0, 0.1^2), on the host."""
    g = torch.Generator().manual_seed(seed)
    ws = [(torch.randn(d, d, generator=g) / d ** 0.5).to(dtype) for _ in range(4)]
    bs = [(torch.randn(d, generator=g) * 0.1).to(dtype) if bias else None for _ in range(4)]
    return ws, bs


def run_module(x, ws, bs, H, W):
    dv = lambda t: None if t is None else t.to(DEV)
    out = swa.mha_forward(x.to(DEV), dv(ws[0]), dv(bs[0]), dv(ws[1]), dv(bs[1]), dv(ws[2]), dv(bs[2]),
                          dv(ws[3]), dv(bs[3]), H, W)
    swa.device_status()
    return out


def oracle_module(x, ws, bs, H, W):
    o = lambda t: None if t is None else f64(t)
    return oracle.mha(f64(x), o(ws[0]), o(bs[0]), o(ws[1]), o(bs[1]), o(ws[2]), o(bs[2]), o(ws[3]),
                      o(bs[3]), H, W)


def test_worked_example_exact():
    """The page's module example: zero query/key kernels, identity value/output kernels,
    zero biases, two heads of width 1, window 3: the printed trailing means, exactly."""
    g = read_moving_average()
    x = torch.tensor(g["x"], dtype=torch.float32)
    z, eye = torch.zeros(2, 2), torch.eye(2)
    out = run_module(x, [z, z, eye, eye], [None] * 4, 2, g["W"]).cpu()
    assert torch.equal(out, torch.tensor(g["y"], dtype=torch.float32))
    row, vals = g["changed_row"]
    x2 = x.clone()
    x2[row] = torch.tensor(vals)
    out2 = run_module(x2, [z, z, eye, eye], [None] * 4, 2, g["W"]).cpu()
    u = g["unchanged_from"]
    assert torch.equal(out2[u:], out[u:])


@pytest.mark.parametrize("B,T,d,H,W,dtype", [
    (2, 50, 24, 3, 7, torch.float32), (1, 130, 64, 2, 40, torch.float32), (1, 9, 6, 6, 100, torch.float32),
    (2, 300, 256, 2, 100, torch.bfloat16), (1, 257, 256, 4, 64, torch.bfloat16),
    (1, 1000, 512, 4, 300, torch.bfloat16), (3, 129, 128, 2, 1, torch.bfloat16)])
def test_module_matches_oracle(B, T, d, H, W, dtype):
    g = torch.Generator().manual_seed(B * 1000 + T + d)
    x = torch.randn(B, T, d, generator=g).to(dtype)
    ws, bs = params(d, dtype, T + d)
    out = run_module(x, ws, bs, H, W)
    err = max_err(out, oracle_module(x, ws, bs, H, W))
    assert err <= TOL_MODULE[dtype], f"module max err {err}"


def test_no_bias_equals_zero_bias():
    B, T, d, H, W = 1, 200, 256, 2, 50
    x = torch.randn(B, T, d).to(torch.bfloat16)
    ws, _ = params(d, torch.bfloat16, 5, bias=False)
    zeros = [torch.zeros(d, dtype=torch.bfloat16)] * 4
    a = run_module(x, ws, [None] * 4, H, W)
    b = run_module(x, ws, zeros, H, W)
    assert torch.equal(a, b)


def test_module_is_its_steps_full_size():
    """Mistral-shaped module (B1 T16384 d4096, 32 heads of 128, W4096) equals torch's
    matmuls (cuBLAS) around swa_forward on the same bf16 inputs: the wrapper reads and
    writes the [B,T,H,Dh] layouts it claims."""
    B, T, d, H, W = 1, 16384, 4096, 32, 4096
    g = torch.Generator().manual_seed(77)
    x = torch.randn(B, T, d, generator=g).to(torch.bfloat16).to(DEV)
    ws, bs = params(d, torch.bfloat16, 78)
    ws = [w.to(DEV) for w in ws]
    bs = [b.to(DEV) for b in bs]
    out = swa.mha_forward(x, ws[0], bs[0], ws[1], bs[1], ws[2], bs[2], ws[3], bs[3], H, W)
    proj = [(x.float() @ ws[i].float() + bs[i].float()).to(torch.bfloat16) for i in range(3)]
    q, k, v = (p.view(B, T, H, d // H).transpose(1, 2) for p in proj)
    o = swa.forward(q, k, v, W)  # strided [B,H,T,Dh] views
    ref = (o.transpose(1, 2).reshape(B, T, d).float() @ ws[3].float() + bs[3].float())
    swa.device_status()
    diff = (out.float() - ref).abs()
    assert torch.isfinite(out.float()).all()
    assert float(diff.max()) <= TOL_MODULE[torch.bfloat16], f"max diff {float(diff.max())}"


def test_module_errors():
    lib = _native.lib()
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    d = 128
    x = torch.zeros(1, 8, d, dtype=torch.bfloat16, device=DEV)
    w = torch.zeros(d, d, dtype=torch.bfloat16, device=DEV)
    need = lib.swa_mha_workspace_bytes(1, 8, d, 1)
    assert need == 4 * 2048 + (32 << 20)  # four 2 KiB parts and the GEMM scratch
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    o = torch.empty_like(x)
    p, wp, op, wsp = x.data_ptr(), w.data_ptr(), o.data_ptr(), ws.data_ptr()
    f = lambda *a: lib.swa_mha_forward(p, wp, None, wp, None, wp, None, wp, None, op, *a)
    assert f(wsp, need, 1, 8, d, 1, 4, 1, s) == 0             # one head of 128
    assert f(wsp, need, 1, 8, d, 3, 4, 1, s) == 1             # d_model % H != 0
    assert f(wsp, need, 1, 8, d, 4, 4, 1, s) == 2             # bf16 head width 32
    assert f(wsp, need - 1, 1, 8, d, 1, 4, 1, s) == 1         # short workspace
    assert f(None, need, 1, 8, d, 1, 4, 1, s) == 1            # no workspace
    assert f(wsp + 16, need, 1, 8, d, 1, 4, 1, s) == 3        # misaligned workspace (refused before use)
    assert f(wsp, need, 1, 8, d, 1, 0, 1, s) == 1             # W < 1
    assert f(wsp, need, 0, 8, d, 1, 4, 1, s) == 0             # empty batch: no-op
    assert lib.swa_mha_workspace_bytes(1, 8, 0, 1) == -1
    swa.device_status()
