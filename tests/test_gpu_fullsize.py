"""Every output element of the full-size workloads against the float64 oracle: the
Mistral-shaped prefill, each window of the sweep, the streaming decode and the chunked
streaming step (with its rings after the append, bit for bit). The oracle runs head by
head (stream by stream for the rings), on the same bf16-rounded inputs widened to
float64, so the host never holds a float64 copy of a whole multi-gigabyte tensor."""
import numpy as np
import pytest
import torch

import oracle
import sliding_window_causal_b200 as swa
from sliding_window_causal_b200 import inputs
from gpu_util import TOL, f64, max_err

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
DEV = "cuda"
BF = torch.bfloat16


def prefill_every_element(wl):
    q, k, v = inputs.for_workload(wl)
    out = swa.forward(q.to(DEV), k.to(DEV), v.to(DEV), wl.W).cpu()
    swa.device_status()
    worst = 0.0
    for b in range(wl.B):
        for h in range(wl.H):
            sl = (slice(b, b + 1), slice(h, h + 1))
            ref = oracle.forward(f64(q[sl]), f64(k[sl]), f64(v[sl]), wl.W)
            err = max_err(out[sl], ref)
            assert err <= TOL[wl.dtype], f"{wl.name}: head ({b},{h}) max err {err}"
            worst = max(worst, err)
    return worst


def test_mistral_shaped_every_element():
    prefill_every_element(inputs.MISTRAL)


@pytest.mark.parametrize("wl", inputs.SWEEP, ids=lambda w: w.name)
def test_window_sweep_every_element(wl):
    prefill_every_element(wl)


def test_streaming_decode_every_element():
    wl = inputs.DECODE
    q, kr, vr, pos = inputs.for_workload(wl)
    out = swa.decode(q.to(DEV), kr.to(DEV), vr.to(DEV), pos.to(DEV), wl.W).cpu()
    swa.device_status()
    for b in range(wl.B):
        ref = oracle.decode(f64(q[b:b + 1]), f64(kr[b:b + 1]), f64(vr[b:b + 1]), pos[b:b + 1].numpy(), wl.W)
        err = max_err(out[b:b + 1], ref)
        assert err <= TOL[BF], f"stream {b} (pos {int(pos[b])}): max err {err}"


def test_chunk_workload_every_element():
    wl = inputs.CHUNKED
    q, k, v, kr, vr, pos = inputs.for_workload(wl)
    dk, dv = kr.to(DEV), vr.to(DEV)
    out = swa.chunk_forward(q.to(DEV), k.to(DEV), v.to(DEV), dk, dv, pos.to(DEV), wl.W).cpu()
    swa.device_status()
    for b in range(wl.B):
        s = slice(b, b + 1)
        p = pos.numpy()[s]
        ref = oracle.chunk(f64(q[s]), f64(k[s]), f64(v[s]), f64(kr[s]), f64(vr[s]), p, wl.W)
        err = max_err(out[s], ref)
        assert err <= TOL[BF], f"stream {b} (pos {int(pos[b])}): max err {err}"
        ek, ev = oracle.ring_append(f64(k[s]), f64(v[s]), f64(kr[s]), f64(vr[s]), p, wl.W)
        assert np.array_equal(f64(dk[s]), ek) and np.array_equal(f64(dv[s]), ev), f"stream {b}: ring"
