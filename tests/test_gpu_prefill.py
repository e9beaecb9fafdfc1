"""GPU prefill (swa_forward through the C ABI) against the float64 oracle."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import sliding_window_causal_b200 as swa
from sliding_window_causal_b200 import _native, inputs
from golden import read_moving_average
from gpu_util import TOL, f64, max_err, sharp_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run(q, k, v, W):
    out = swa.forward(q.to(DEV), k.to(DEV), v.to(DEV), W)
    swa.device_status()
    return out


def full_parity(B, H, T, D, W, dtype, seed):
    q, k, v = inputs.prefill_inputs(B, H, T, D, dtype, seed)
    out = run(q, k, v, W)
    ref = oracle.forward(f64(q), f64(k), f64(v), W)
    err = max_err(out, ref)
    assert err <= TOL[dtype], f"max err {err} (B{B} H{H} T{T} D{D} W{W} {dtype})"
    return err


@pytest.mark.parametrize("wl", inputs.TINY, ids=lambda w: w.name)
def test_tiny_fp32_workload(wl):
    full_parity(wl.B, wl.H, wl.T, wl.D, wl.W, wl.dtype, wl.seed)


def test_small_bf16_workload():
    wl = inputs.SMALL
    full_parity(wl.B, wl.H, wl.T, wl.D, wl.W, wl.dtype, wl.seed)


BF16_SHAPES = [
    # B, H, T, D, W: ragged T, W below/at/above a tile, W >= T, single rows
    (1, 2, 300, 64, 1), (1, 2, 300, 64, 77), (2, 2, 1000, 128, 128), (1, 3, 1000, 128, 127),
    (1, 2, 1000, 128, 129), (1, 2, 777, 128, 300), (1, 1, 1000, 128, 1000),
    (1, 1, 1000, 128, 5000), (1, 2, 129, 64, 2), (1, 1, 1, 128, 1), (1, 1, 5, 64, 3),
    (2, 3, 400, 64, 256), (1, 1, 2000, 128, 640), (1, 2, 1280, 64, 1),
    # either side of the band length (1024 keys) where the kernel moves from two MMA
    # issuers to one
    (1, 2, 3000, 128, 1024), (1, 2, 3000, 128, 1025), (1, 2, 2000, 64, 1500),
    # bands of at most 7 keys take the CUDA-core kernel (32 rows a CTA): ragged and short
    # T, band lengths up to 7, and 8 and 9, the first bands of the tensor-core kernel
    (2, 2, 333, 128, 8), (1, 3, 95, 64, 5), (1, 2, 33, 128, 4), (1, 1, 7, 128, 8),
    (2, 1, 500, 64, 7), (1, 2, 64, 128, 6), (1, 2, 300, 128, 9), (1, 1, 31, 64, 8),
    (1, 2, 200, 64, 7),
    # either side of the band length (144 keys) up to which every tile carries P as hi + lo
    (1, 2, 700, 128, 33), (1, 2, 600, 64, 48), (2, 1, 900, 128, 64), (1, 2, 500, 128, 129),
    (1, 2, 600, 128, 144), (1, 2, 500, 64, 145), (1, 2, 500, 128, 160),
]


@pytest.mark.parametrize("B,H,T,D,W", BF16_SHAPES)
def test_bf16_parity(B, H, T, D, W):
    full_parity(B, H, T, D, W, torch.bfloat16, 7 + T + W)


FP32_SHAPES = [(1, 2, 6, 4, 3), (2, 3, 100, 1, 7), (1, 2, 257, 33, 40), (1, 1, 300, 128, 300),
               (1, 2, 70, 200, 1000), (1, 1, 40, 1100, 9)]


@pytest.mark.parametrize("B,H,T,D,W", FP32_SHAPES)
def test_fp32_parity(B, H, T, D, W):
    full_parity(B, H, T, D, W, torch.float32, 3 + T + W)


def test_moving_average_example_exact():
    """The printed moving-average example (two heads of width 1, window 3, zero q and
    k) comes out exactly, and changing input row 0 leaves rows 3+ unchanged."""
    g = read_moving_average()
    x = torch.tensor(g["x"], dtype=torch.float32)
    T, Hn = x.shape
    v = x.t().reshape(1, Hn, T, 1).contiguous()
    z = torch.zeros_like(v)
    out = run(z, z, v, g["W"])[0, :, :, 0].t().cpu()
    assert torch.equal(out, torch.tensor(g["y"], dtype=torch.float32))
    row, vals = g["changed_row"]
    x2 = x.clone()
    x2[row] = torch.tensor(vals)
    v2 = x2.t().reshape(1, Hn, T, 1).contiguous()
    out2 = run(z, z, v2, g["W"])[0, :, :, 0].t().cpu()
    u = g["unchanged_from"]
    assert torch.equal(out2[u:], out[u:])


@pytest.mark.parametrize("dtype,D", [(torch.bfloat16, 64), (torch.bfloat16, 128), (torch.float32, 5)])
def test_window_one_returns_v_bitwise(dtype, D):
    q, k, v = inputs.prefill_inputs(2, 2, 333, D, dtype, 11)
    out = run(q, k, v, 1).cpu()
    assert torch.equal(out, v)


def test_window_at_least_T_is_causal():
    """W >= T equals ordinary causal attention (the oracle with W = T), and every
    W >= T gives the same bits."""
    q, k, v = inputs.prefill_inputs(1, 2, 500, 128, torch.bfloat16, 13)
    ref = oracle.forward(f64(q), f64(k), f64(v), 500)
    a = run(q, k, v, 500)
    b = run(q, k, v, 10**9)
    assert max_err(a, ref) <= TOL[torch.bfloat16]
    assert torch.equal(a, b)


@pytest.mark.parametrize("D", [64, 128])
def test_out_of_band_corruption_bitwise(D):
    """Corrupt-and-compare: changing k and v (finite values) at positions j <= i0 - W
    leaves every row i >= i0 bitwise unchanged."""
    T, W, i0 = 1000, 100, 700
    q, k, v = inputs.prefill_inputs(1, 2, T, D, torch.bfloat16, 17)
    base = run(q, k, v, W).cpu()
    k2, v2 = k.clone(), v.clone()
    k2[:, :, : i0 - W + 1] = 100.0
    v2[:, :, : i0 - W + 1] = -200.0
    out = run(q, k2, v2, W).cpu()
    assert torch.equal(out[:, :, i0:], base[:, :, i0:])
    assert not torch.equal(out[:, :, :i0], base[:, :, :i0])


def test_deterministic():
    q, k, v = inputs.prefill_inputs(1, 4, 1500, 128, torch.bfloat16, 19)
    a = run(q, k, v, 600)
    b = run(q, k, v, 600)
    assert torch.equal(a, b)


def test_three_dim_input_is_one_head():
    q = torch.randn(1, 5, 3, generator=torch.Generator().manual_seed(5))
    out = swa.forward(q.to(DEV), q.to(DEV), q.to(DEV), 2)
    swa.device_status()
    assert out.shape == (1, 5, 3)
    ref = oracle.forward(f64(q)[:, None], f64(q)[:, None], f64(q)[:, None], 2)[:, 0]
    assert max_err(out, ref) <= TOL[torch.float32]


def test_empty_inputs_are_noops():
    for shape in [(0, 2, 16, 64), (1, 0, 16, 64), (1, 2, 0, 64)]:
        q = torch.zeros(shape, dtype=torch.bfloat16, device=DEV)
        out = swa.forward(q, q, q, 4)
        assert out.shape == shape
    swa.device_status()


def test_argument_errors():
    h = _native.lib()
    q = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16, device=DEV)
    p = q.data_ptr()
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert h.swa_forward(p, p, p, p, 1, 1, 8, 64, 0, 1, s) == 1  # W < 1
    assert b"W=0" in h.swa_last_error()
    assert h.swa_forward(p, p, p, p, 1, 1, 8, 64, 3, 7, s) == 1  # dtype
    assert h.swa_forward(p, p, p, p, -1, 1, 8, 64, 3, 1, s) == 1  # negative size
    assert h.swa_forward(None, p, p, p, 1, 1, 8, 64, 3, 1, s) == 1  # null
    assert h.swa_forward(p, p, p, p, 1, 1, 8, 96, 3, 1, s) == 2  # bf16 D=96
    assert h.swa_forward(p + 2, p, p, p, 1, 1, 4, 64, 3, 1, s) == 3  # misaligned
    with pytest.raises(swa.SwaError):
        swa.forward(q, q, q, 0)
    swa.device_status()


def test_timeout_path_reports_and_recovers():
    """A wait that nothing completes runs out and is reported, and the context
    stays usable for the next calls."""
    prev = swa.set_wait_limit_ns(20_000_000)
    try:
        swa.timeout_probe()
        with pytest.raises(swa.SwaError) as ei:
            swa.device_status()
        assert ei.value.code == 5
    finally:
        swa.set_wait_limit_ns(0)
    full_parity(1, 2, 300, 128, 100, torch.bfloat16, 23)
    swa.device_status()


# ---------------------------------------------------------------- full-size workloads
# Every element of the full-size workloads is compared in test_gpu_fullsize.py; here the
# properties that hold at any size, over every output of the Mistral-shaped workload.

@pytest.mark.parametrize("D", [64, 128])
def test_score_jump_in_a_later_key_tile(D):
    """One key whose scaled score exceeds every earlier key of the band by far more than
    fp32's exponent range (about 650 in log2 units): the rows whose band holds it, and
    which met ordinary keys in earlier key tiles first, must come out as that key's v, as
    the oracle's max-subtracted softmax gives, not overflow."""
    B, H, T, W = 1, 2, 1000, 600
    q, k, v = inputs.prefill_inputs(B, H, T, D, torch.bfloat16, 301 + D)
    q = torch.ones_like(q)
    k = (0.01 * k.float()).to(torch.bfloat16)
    k[:, :, 300] = 40.0 * 128.0 / D  # q . k_300 = 5120: 653 log2 units after the scale at D = 128
    out = run(q, k, v, W)
    ref = oracle.forward(f64(q), f64(k), f64(v), W)
    err = max_err(out, ref)
    assert err <= TOL[torch.bfloat16], f"max err {err}"
    assert torch.equal(out.cpu()[:, :, 300:900], v[:, :, 300:301].expand(B, H, 600, D))


@pytest.mark.parametrize("H", [147, 148, 149])
def test_work_items_either_side_of_the_sm_count(H):
    """Fewer pairs of query tiles than SMs make each work item a single query tile; at or
    above the SM count (148 on a B200) items are pairs. Two tiles per head (T = 256), so
    H is the number of pairs: every row against the oracle on either side of the switch."""
    B, T, D, W = 1, 256, 64, 100
    q, k, v = inputs.prefill_inputs(B, H, T, D, torch.bfloat16, 400 + H)
    out = run(q, k, v, W)
    ref = oracle.forward(f64(q), f64(k), f64(v), W)
    err = max_err(out, ref)
    assert err <= TOL[torch.bfloat16], f"H {H}: max err {err}"


def test_mistral_shaped_properties():
    wl = inputs.MISTRAL
    q, k, v = inputs.for_workload(wl)
    out = swa.forward(q.to(DEV), k.to(DEV), v.to(DEV), wl.W)
    swa.device_status()
    # finite, and each output a convex combination of v rows, so no larger in magnitude
    # than the largest |v|
    assert bool(torch.isfinite(out).all())
    vmax = v.abs().max().item()
    assert out.abs().max().item() <= vmax * (1 + 2 ** -8)


@pytest.mark.parametrize("D,W", [(128, 4096), (64, 700), (128, 200)])
def test_growing_scores_move_the_reference(D, W):
    """Scores that grow steadily along the sequence (q . k_j grows with j) push every
    row's running maximum up by far more than the lazy-rescale threshold, tile after
    tile; the output must still match.

    A handful of keys dominate every row, so |out| comes close to a single |v| and can
    pass 2, where the bf16 output spacing alone costs up to 0.0078 of the 1e-2 budget.
    These are the rows the kernel recomputes in fp32 (a key of a single-bf16 tile holds
    more than 1/16 of the row's weight); v is drawn at full scale, N(0, 1)."""
    T = 1500
    gen = torch.Generator().manual_seed(71)
    q = torch.ones(1, 2, T, D)
    k = (torch.arange(T, dtype=torch.float32) * 0.05)[None, None, :, None].expand(1, 2, T, D).clone()
    k += 0.01 * torch.randn(1, 2, T, D, generator=gen)
    v = torch.randn(1, 2, T, D, generator=gen)
    q, k, v = (t.to(torch.bfloat16) for t in (q, k, v))
    out = run(q, k, v, W)
    ref = oracle.forward(f64(q), f64(k), f64(v), W)
    assert max_err(out, ref) <= TOL[torch.bfloat16]


@pytest.mark.parametrize("kind", ["growing", "falling", "spikes"])
@pytest.mark.parametrize("D,W", [(128, 4096), (64, 300), (128, 600)])
def test_adaptive_mode_on_rows_a_few_keys_dominate(kind, D, W):
    """Adaptive P (hi + lo parts on the tiles where a key of one of a warp's rows could end
    up above a quarter of its row's weight, and a second P.V product for those warps'
    rows): the inputs that make the fast mode recompute nearly every row match the oracle
    without recomputing any, in the plain and the training forward."""
    B, H, T = 1, 3, 1300
    q, k, v = sharp_inputs(B, H, T, D, 50 + W + D, kind)
    prev = swa.set_prefill_mode(swa.PREFILL_ADAPTIVE)
    try:
        out = run(q, k, v, W)
        out2, _ = swa.forward_lse(q.to(DEV), k.to(DEV), v.to(DEV), W)
        swa.device_status()
    finally:
        swa.set_prefill_mode(prev)
    ref = oracle.forward(f64(q), f64(k), f64(v), W)
    assert max_err(out, ref) <= TOL[torch.bfloat16]
    assert max_err(out2, ref) <= TOL[torch.bfloat16]


@pytest.mark.parametrize("B,H,T,D,W", [(1, 2, 3000, 128, 1500), (2, 2, 1000, 128, 300), (1, 3, 777, 64, 200)])
def test_adaptive_mode_parity(B, H, T, D, W):
    """Adaptive P on N(0,1) inputs: one and two MMA issuers, D 64 and 128, ragged T."""
    prev = swa.set_prefill_mode(swa.PREFILL_ADAPTIVE)
    try:
        full_parity(B, H, T, D, W, torch.bfloat16, 11 + T + W)
    finally:
        swa.set_prefill_mode(prev)


def test_auto_mode_switches_after_many_sharp_rows():
    """In the default mode a launch whose inputs make many rows sharp (here the oldest key
    of every band dominates) is computed with single-bf16 P and those rows recomputed; it
    switches the device to adaptive P for later launches, which still match the oracle."""
    prev = swa.set_prefill_mode(swa.PREFILL_AUTO)
    try:
        assert swa.prefill_auto_state() == 0
        full_parity(1, 2, 1000, 128, 700, torch.bfloat16, 5)
        assert swa.prefill_auto_state() == 0, "N(0,1) inputs make almost no row sharp"
        q, k, v = sharp_inputs(1, 3, 1300, 128, 7, "falling")
        out = run(q, k, v, 600)
        assert max_err(out, oracle.forward(f64(q), f64(k), f64(v), 600)) <= TOL[torch.bfloat16]
        assert swa.prefill_auto_state() == 1
        full_parity(1, 2, 1000, 128, 700, torch.bfloat16, 6)
        assert swa.prefill_auto_state(clear=True) == 1
        assert swa.prefill_auto_state() == 0
    finally:
        swa.set_prefill_mode(prev)


def test_fast_mode_never_switches():
    prev = swa.set_prefill_mode(swa.PREFILL_FAST)
    try:
        q, k, v = sharp_inputs(1, 3, 1300, 128, 7, "falling")
        out = run(q, k, v, 600)
        assert max_err(out, oracle.forward(f64(q), f64(k), f64(v), 600)) <= TOL[torch.bfloat16]
        assert swa.prefill_auto_state() == 0
    finally:
        swa.set_prefill_mode(prev)
