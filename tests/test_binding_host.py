"""The Python binding's argument checks (host only): shapes, dtypes and devices are refused
before anything reaches the library, so these run without a GPU."""
import pytest
import torch

import sliding_window_causal_b200 as swa


def cpu(*shape, dtype=torch.bfloat16):
    return torch.zeros(*shape, dtype=dtype)


def test_forward_refuses_host_tensors_and_bad_shapes():
    q = cpu(1, 2, 8, 64)
    with pytest.raises(ValueError, match="CUDA"):
        swa.forward(q, q, q, 4)
    with pytest.raises(ValueError, match="shape"):
        swa.forward(q, cpu(1, 2, 9, 64), q, 4)
    with pytest.raises(TypeError, match="dtype"):
        swa.forward(q, q.float(), q, 4)


def test_decode_checks_ring_and_positions():
    q = cpu(2, 3, 64)
    ring = cpu(2, 3, 16, 64)
    with pytest.raises(ValueError, match="rings"):
        swa.decode(q, cpu(2, 3, 15, 64), ring, torch.zeros(2, dtype=torch.int64), 16)
    with pytest.raises(ValueError, match="pos"):
        swa.decode(q, ring, ring, torch.zeros(2, dtype=torch.int32), 16)
    with pytest.raises(TypeError, match="bf16"):
        swa.decode(q.float(), ring.float(), ring.float(), torch.zeros(2, dtype=torch.int64), 16)


def test_streaming_calls_check_shapes():
    k = cpu(2, 3, 5, 64)
    ring = cpu(2, 3, 16, 64)
    pos = torch.zeros(2, dtype=torch.int64)
    with pytest.raises(ValueError, match="rings"):
        swa.chunk_forward(k, k, k, cpu(2, 3, 8, 64), ring, pos, 16)
    with pytest.raises(ValueError, match="pos"):
        swa.ring_append(k, k, ring, ring, torch.zeros(3, dtype=torch.int64), 16)
    with pytest.raises(ValueError, match="CUDA"):
        swa.ring_append(k, k, ring, ring, pos, 16)


def test_module_and_backward_check_shapes():
    x = cpu(1, 8, 64)
    w = cpu(64, 64)
    with pytest.raises(ValueError, match="kernels"):
        swa.mha_forward(x, cpu(64, 32), None, w, None, w, None, w, None, 2, 4)
    with pytest.raises(TypeError, match="dtype"):
        swa.mha_forward(x, w.float(), None, w, None, w, None, w, None, 2, 4)
    q = cpu(1, 2, 8, 64)
    with pytest.raises(ValueError, match="shape"):
        swa.backward(q, q, q, cpu(1, 2, 8, 32), 4)
    with pytest.raises(ValueError, match="CUDA"):
        swa.backward(q, q, q, q, 4)


def test_host_planning_needs_no_gpu():
    # the planners the kernels use are callable without a device
    assert swa.tile_class(300, 77, 128, 128, 1, 0) in (0, 1, 2)
    assert swa.valid_slots(5, 16) == 6 and swa.valid_slots(100, 16) == 16
    splits, chunk = swa.split_plan(64, 32, 128, 4096)
    assert splits >= 1 and splits * chunk >= 4096
