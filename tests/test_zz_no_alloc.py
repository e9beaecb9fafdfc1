"""The allocation-free decode entry point against the allocating one.

swa_decode_noalloc serves callers that cannot let a library call cudaMalloc (device
memory owned end to end by another allocator, or a latency-bound decode step that must
not take cudaMalloc's device-wide synchronisation): it keeps its split partial states in
a fixed 4 MiB array compiled into the library instead of a cudaMalloc'd workspace. It
runs swa_decode's kernel with swa_decode's split plan, so its results must equal
swa_decode's bit for bit, call after call, although every call shares that array.
This file is collected last, so that a run which stops at the first failure has already
run every other test; it also passes on its own in a fresh process.
"""
import ctypes
import os

import pytest
import torch

import oracle
import sliding_window_causal_b200 as swa
from sliding_window_causal_b200 import _native, inputs
from gpu_util import TOL, f64, max_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def noalloc(q, kr, vr, pos, W, out):
    B, H, D = q.shape
    rc = _native.lib().swa_decode_noalloc(
        q.data_ptr(), kr.data_ptr(), vr.data_ptr(), pos.data_ptr(), out.data_ptr(), B, H, D, W,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc


CASES = [
    # B, H, D, W, positions drawn from [0, pos_max)
    (4, 2, 128, 300, 2000),     # many splits per stream
    (3, 5, 64, 77, 500),
    (16, 8, 128, 4096, 100000),  # two splits per stream
    (64, 40, 64, 256, 1000),    # enough streams for a single split (no scratch)
]


@pytest.mark.parametrize("B,H,D,W,pos_max", CASES)
def test_noalloc_matches_decode_on_consecutive_calls(B, H, D, W, pos_max):
    """Two calls in a row share the fixed array. Both run the same kernel with the same
    split plan as swa_decode, so their outputs equal its output bit for bit; the first is
    also checked against the float64 oracle."""
    qh, krh, vrh, posh = inputs.decode_inputs(B, H, D, W, pos_max, torch.bfloat16, 90 + W)
    q, kr, vr, pos = (t.to(DEV) for t in (qh, krh, vrh, posh))
    ref = swa.decode(q, kr, vr, pos, W)
    swa.device_status()
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        assert noalloc(q, kr, vr, pos, W, out) == 0, _native.lib().swa_last_error()
        swa.device_status()
        assert torch.equal(out, ref), f"call {call}"
        if call == 0:
            err = max_err(out, oracle.decode(f64(qh), f64(krh), f64(vrh), posh.numpy(), W))
            assert err <= TOL[torch.bfloat16], err


def test_noalloc_after_a_call_of_another_size():
    """A call that leaves other partial states and counters in the array, then the first
    size again: stale contents would change the bits."""
    sizes = [(4, 2, 128, 300, 2000), (16, 8, 128, 4096, 100000), (3, 5, 64, 77, 500), (4, 2, 128, 300, 2000)]
    outs = []
    for i, (B, H, D, W, pos_max) in enumerate(sizes):
        q, kr, vr, pos = (t.to(DEV) for t in inputs.decode_inputs(B, H, D, W, pos_max, torch.bfloat16, 90 + W))
        ref = swa.decode(q, kr, vr, pos, W)
        out = torch.full_like(q, float("nan"))
        assert noalloc(q, kr, vr, pos, W, out) == 0, _native.lib().swa_last_error()
        swa.device_status()
        assert torch.equal(out, ref), (B, H, D, W)
        outs.append(out)
    assert torch.equal(outs[0], outs[-1])


def test_noalloc_rejects_requests_beyond_the_array(monkeypatch):
    """A forced small chunk makes the partial states outgrow the fixed array: the call
    is refused before anything is enqueued, with the sizes in the message."""
    monkeypatch.setenv("SWA_DECODE_CHUNK", "32")
    # 256 streams x 32 splits x 130 floats = 4.3 MB of partial states > 4 MiB. The buffers
    # have their full sizes, so the call would be safe even if it were not refused.
    B, H, D, W = 8, 32, 128, 1024
    q = torch.zeros(B, H, D, dtype=torch.bfloat16, device=DEV)
    r = torch.zeros(B, H, W, D, dtype=torch.bfloat16, device=DEV)
    pos = torch.zeros(B, dtype=torch.int64, device=DEV)
    out = torch.full_like(q, float("nan"))
    assert noalloc(q, r, r, pos, W, out) == 2
    assert b"scratch" in _native.lib().swa_last_error()
    swa.device_status()
    assert bool(torch.isnan(out).all()), "a refused call enqueues nothing"

