"""Argument validation at the C ABI, on the CPU: every call checks its arguments before it
touches the device, so a refused call returns its status here without a GPU. The pointers
are dummies that a valid call would have to dereference; every call here is refused or is
a no-op (an empty batch), so none of them launches anything, on a machine with a GPU too."""
import ctypes

import pytest

from sliding_window_causal_b200 import _native, build

DUMMY = 0x10000  # 64 KiB-aligned, never dereferenced
OK, INVALID, UNSUPPORTED, MISALIGNED = 0, 1, 2, 3


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _native.lib()


def strides(*vals):
    return (ctypes.c_int64 * len(vals))(*vals)


def test_forward_errors(lib):
    p = DUMMY
    f = lib.swa_forward
    assert f(p, p, p, p, 1, 2, 8, 64, 0, 1, None) == INVALID       # W < 1
    assert f(p, p, p, p, 1, -2, 8, 64, 4, 1, None) == INVALID      # negative size
    assert f(p, p, p, p, 1, 2, 8, 0, 4, 1, None) == INVALID        # D < 1
    assert f(p, p, p, p, 1, 2, 8, 64, 4, 7, None) == INVALID       # dtype
    assert f(None, p, p, p, 1, 2, 8, 64, 4, 1, None) == INVALID    # null pointer
    assert f(p, p, p, p, 1, 2, 8, 64, 4, 7, None) == INVALID
    assert lib.swa_last_error()                                     # a refusal leaves a message
    assert f(None, None, None, None, 0, 2, 8, 64, 4, 1, None) == OK  # empty: no-op


def test_forward_ex_errors(lib):
    p = DUMMY
    f = lib.swa_forward_ex
    good = strides(*([2 * 8 * 64, 8 * 64, 64] * 4))
    assert f(p, p, p, p, 1, 2, 8, 64, 4, float("nan"), good, 1, None) == INVALID
    assert f(p, p, p, p, 1, 2, 8, 64, 4, float("inf"), good, 1, None) == INVALID
    neg = strides(*([2 * 8 * 64, -8 * 64, 64] + [2 * 8 * 64, 8 * 64, 64] * 3))
    assert f(p, p, p, p, 1, 2, 8, 64, 4, 0.125, neg, 1, None) == INVALID
    huge = strides(*([1 << 39, 8 * 64, 64] + [2 * 8 * 64, 8 * 64, 64] * 3))
    assert f(p, p, p, p, 2, 2, 8, 64, 4, 0.125, huge, 1, None) == INVALID
    assert b"stride" in lib.swa_last_error()


def test_band_weights_errors(lib):
    p = DUMMY
    f = lib.swa_band_weights
    assert f(p, p, p, 1, 2, 8, 64, 0, 0.1, None, 1, None) == INVALID
    assert f(p, p, None, 1, 2, 8, 64, 4, 0.1, None, 1, None) == INVALID
    assert f(p, p, p, 1, 2, 8, 64, 4, float("nan"), None, 1, None) == INVALID
    assert f(p, p, p, 1, 2, 8, 5000, 4, 0.1, None, 0, None) == UNSUPPORTED  # D > 4096
    assert f(p, p, p, 1, 1 << 27, 1 << 7, 4, 1, 0.5, None, 0, None) == UNSUPPORTED  # 2^32 rows
    assert b"too many rows" in lib.swa_last_error()


def test_decode_and_streaming_errors(lib):
    p = DUMMY
    for f in (lib.swa_decode, lib.swa_decode_noalloc):
        assert f(p, p, p, p, p, 2, 2, 64, 0, None) == INVALID           # W < 1
        assert f(p, p, p, p, p, 2, 2, 96, 16, None) == UNSUPPORTED      # D = 96
        assert f(p + 2, p, p, p, p, 2, 2, 64, 16, None) == MISALIGNED   # q not 16-byte aligned
        assert f(p, p, p, None, p, 2, 2, 64, 16, None) == INVALID       # null pos
        assert f(p, p, p, p, p, 0, 2, 64, 16, None) == OK               # no streams: no-op
    c = lib.swa_chunk_forward
    assert c(p, p, p, p, p, p, p, 1, 1, 8, 64, 0, None) == INVALID
    assert c(p, p, p, p, p, p, p, 1, 1, 8, 96, 16, None) == UNSUPPORTED
    assert c(p, p, p, p + 8, p, p, p, 1, 1, 8, 64, 16, None) == MISALIGNED
    assert c(p, p, p, p, p, p, p, 1, 1, 0, 64, 16, None) == OK         # empty chunk
    a = lib.swa_ring_append
    assert a(p, p, p, p, p, 1, 1, 8, 64, 0, None) == INVALID
    assert a(p, p, p, p, None, 1, 1, 8, 64, 16, None) == INVALID


def test_module_and_backward_errors(lib):
    p = DUMMY
    need = lib.swa_mha_workspace_bytes(1, 8, 128, 1)
    m = lambda *a: lib.swa_mha_forward(p, p, None, p, None, p, None, p, None, p, *a)
    assert m(p, need, 1, 8, 128, 3, 4, 1, None) == INVALID        # d_model % H
    assert m(p, need, 1, 8, 128, 4, 4, 1, None) == UNSUPPORTED    # bf16 head width 32
    assert m(p, need - 1, 1, 8, 128, 1, 4, 1, None) == INVALID    # short workspace
    assert m(p + 16, need, 1, 8, 128, 1, 4, 1, None) == MISALIGNED
    assert m(p, need, 1, 8, 128, 1, 4, 9, None) == INVALID        # dtype
    wb = lib.swa_backward_workspace_bytes(1, 1, 16)
    b = lambda *a: lib.swa_backward(p, p, p, p, p, p, p, p, p, *a)
    assert b(p, wb - 8, 1, 1, 16, 64, 4, 0.125, 1, None) == INVALID   # short workspace
    assert b(p, wb, 1, 1, 16, 64, 0, 0.125, 1, None) == INVALID       # W < 1
    assert b(p, wb, 1, 1, 16, 64, 4, float("nan"), 1, None) == INVALID
    assert b(p, wb, 1, 1, 16, 513, 4, 0.125, 0, None) == UNSUPPORTED  # CUDA-core D limit
    assert b(p + 64, wb, 1, 1, 16, 64, 4, 0.125, 1, None) == MISALIGNED  # bf16 workspace 256
    assert b(p, wb, 1, 1, 16, 64, 4, -0.5, 1, None) == UNSUPPORTED    # bf16 scale > 0
    lse_none = lib.swa_backward(p, p, p, p, p, None, p, p, p, p, wb, 1, 1, 16, 64, 4, 0.125, 1, None)
    assert lse_none == INVALID                                        # tensor-core path needs lse
    assert lib.swa_forward_lse(p, p, p, p, None, 1, 1, 16, 64, 4, 0.125, 1, None) == INVALID
    assert lib.swa_forward_lse(p, p, p, p, p + 2, 1, 1, 16, 64, 4, 0.125, 1, None) == MISALIGNED
    assert b(p + 2, wb, 1, 1, 16, 64, 4, 0.125, 0, None) == MISALIGNED  # fp32 workspace 8
    assert b(p, wb, 0, 1, 16, 64, 4, 0.125, 1, None) == OK              # empty batch: no-op


def test_forward_refusals_need_no_device(lib):
    """Every refusal of the prefill, the dtype-specific ones included, is decided on the
    host before the library asks the runtime for a device."""
    p = DUMMY
    f = lib.swa_forward
    assert f(p, p, p, p, 1, 2, 8, 96, 4, 1, None) == UNSUPPORTED       # bf16 D = 96
    assert f(p, p, p, p, 1, 2, 8, 5000, 4, 0, None) == UNSUPPORTED     # fp32 D > 4096
    assert f(p + 8, p, p, p, 1, 2, 8, 64, 4, 1, None) == MISALIGNED    # bf16 16-byte rule
    assert f(p + 2, p, p, p, 1, 2, 8, 64, 4, 0, None) == MISALIGNED    # fp32 4-byte rule
    g = lib.swa_forward_ex
    odd = strides(*([2 * 8 * 64, 8 * 64, 68] + [2 * 8 * 64, 8 * 64, 64] * 3))
    assert g(p, p, p, p, 1, 2, 8, 64, 4, 0.125, odd, 1, None) == MISALIGNED
    assert b"multiples of 8" in lib.swa_last_error()
    assert g(p, p, p, p, 1, 2, 8, 64, 4, -1.0, None, 1, None) == UNSUPPORTED


def test_module_refuses_before_its_first_gemm(lib):
    """The module checks the attention's limits before it enqueues a projection: a
    [B, T, H, Dh] stride T*d_model above 2^38 elements is refused as the attention would
    refuse it, without the runtime being asked for a device."""
    p = DUMMY
    B, T, d, H = 1, 1 << 20, 1 << 19, 1 << 13
    need = lib.swa_mha_workspace_bytes(B, T, d, 1)
    assert need > 0
    rc = lib.swa_mha_forward(p, p, None, p, None, p, None, p, None, p, p, need, B, T, d, H, 4, 1, None)
    assert rc == INVALID
    assert b"stride" in lib.swa_last_error()


def test_decode_refuses_more_splits_than_the_grid_holds(lib, monkeypatch):
    """A forced small chunk over a long ring would need more than 65535 splits (the grid's
    y limit): refused before anything is enqueued. The library's own plan stays far below."""
    from sliding_window_causal_b200 import split_plan
    p = DUMMY
    W = 1 << 24
    assert split_plan(1, 1, 64, W)[0] <= 148 * 16
    monkeypatch.setenv("SWA_DECODE_CHUNK", "1")
    splits, chunk = split_plan(1, 1, 64, W)
    assert splits > 65535 and splits * chunk >= W
    for f in (lib.swa_decode, lib.swa_decode_noalloc):
        assert f(p, p, p, p, p, 1, 1, 64, W, None) == UNSUPPORTED
        assert b"65535" in lib.swa_last_error()


def test_backward_refuses_grids_it_cannot_launch(lib):
    """Sizes whose statistics grid (one warp per padded row) would not fit a launch are
    refused before the device is touched, not truncated."""
    p = DUMMY
    B, H, T = 1, 1 << 20, 1 << 15
    wb = lib.swa_backward_workspace_bytes(B, H, T)
    assert lib.swa_backward(p, p, p, p, p, p, p, p, p, p, wb, B, H, T, 64, 4, 0.125, 1, None) == UNSUPPORTED
    assert b"too many tiles" in lib.swa_last_error()
    B, H, T = 1, 1 << 27, 1 << 7  # CUDA-core path: 2^31 row blocks
    wb = lib.swa_backward_workspace_bytes(B, H, T)
    assert lib.swa_backward(p, p, p, p, p, None, p, p, p, p, wb, B, H, T, 32, 4, 0.125, 0, None) == UNSUPPORTED
    assert b"too many rows" in lib.swa_last_error()
