"""swa_forward_host (host buffers in and out, copies overlapped with the attention on the
library's own streams) against swa_forward on device copies, bit for bit."""
import ctypes

import pytest
import torch

import oracle
import sliding_window_causal_b200 as swa
from sliding_window_causal_b200 import _native, inputs
from gpu_util import TOL, f64, max_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("hpg", [0, 1, 4, 6, 100])
def test_host_pipeline_equals_device_forward(hpg):
    B, H, T, D, W = 2, 3, 1000, 128, 300
    q, k, v = inputs.prefill_inputs(B, H, T, D, torch.bfloat16, 300 + hpg)
    ref = swa.forward(q.to(DEV), k.to(DEV), v.to(DEV), W).cpu()
    pq, pk, pv = (t.pin_memory() for t in (q, k, v))
    out = swa.forward_host(pq, pk, pv, W, heads_per_group=hpg)
    swa.device_status()
    assert torch.equal(out, ref)
    assert max_err(out, oracle.forward(f64(q), f64(k), f64(v), W)) <= TOL[torch.bfloat16]


def test_host_pipeline_fp32_and_pageable_memory():
    B, H, T, D, W = 1, 5, 200, 33, 40
    q, k, v = inputs.prefill_inputs(B, H, T, D, torch.float32, 310)
    ref = swa.forward(q.to(DEV), k.to(DEV), v.to(DEV), W).cpu()
    out = torch.empty_like(q)  # pageable
    swa.forward_host(q, k, v, W, out=out, heads_per_group=2)
    swa.device_status()
    assert torch.equal(out, ref)


def test_host_pipeline_orders_after_the_stream_and_reuses_staging():
    """Two calls on one stream with the same staging buffers and a kernel of the caller's
    between them: each result is that of its own inputs."""
    B, H, T, D, W = 1, 8, 700, 64, 128
    a = inputs.prefill_inputs(B, H, T, D, torch.bfloat16, 320)
    b = inputs.prefill_inputs(B, H, T, D, torch.bfloat16, 321)
    staging = tuple(torch.empty(B, H, T, D, dtype=torch.bfloat16, device=DEV) for _ in range(4))
    ra = swa.forward(*(t.to(DEV) for t in a), W).cpu()
    rb = swa.forward(*(t.to(DEV) for t in b), W).cpu()
    # the host tensors must outlive the copies the calls enqueue: keep them until the sync
    pa = [t.pin_memory() for t in a]
    pb = [t.pin_memory() for t in b]
    oa = swa.forward_host(*pa, W, staging=staging)
    staging[0].fill_(7.0)  # the caller's own work on a staging buffer, in stream order
    ob = swa.forward_host(*pb, W, staging=staging)
    swa.device_status()
    assert torch.equal(oa, ra) and torch.equal(ob, rb)


def test_host_pipeline_argument_errors():
    h = _native.lib()
    d = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16, device=DEV).data_ptr()
    x = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16).pin_memory()
    p = x.data_ptr()
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert h.swa_forward_host(None, p, p, p, d, d, d, d, 1, 1, 8, 64, 4, 0, 1, s) == 1
    assert h.swa_forward_host(p, p, p, p, d, d, d, d, 1, 1, 8, 64, 4, -1, 1, s) == 1
    assert h.swa_forward_host(p, p, p, p, d, d, d, d, 1, 1, 8, 64, 0, 0, 1, s) == 1
    assert h.swa_forward_host(p, p, p, p, d, d, d, d, 1, 1, 8, 96, 4, 0, 1, s) == 2
    assert h.swa_forward_host(p, p, p, p, d, d, d, d, 0, 1, 8, 64, 4, 0, 1, s) == 0
    swa.device_status()
