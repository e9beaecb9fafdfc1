"""The bench's work accounting (host only): band FLOPs, decode bytes and chunk work against
brute-force enumeration of the band pairs."""
import os
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from sliding_window_causal_b200 import inputs  # noqa: E402


def brute_pairs(T, W):
    return sum(1 for i in range(T) for j in range(T) if 0 <= i - j < W)


def test_band_flops_counts_band_pairs():
    for (B, H, T, D, W) in ((1, 1, 1, 4, 1), (2, 3, 17, 8, 5), (1, 2, 40, 16, 40), (1, 1, 33, 2, 100),
                            (3, 1, 64, 128, 1)):
        assert bench.band_flops(B, H, T, D, W) == 4 * B * H * D * brute_pairs(T, W)


def test_band_flops_of_the_named_workloads():
    # Mistral-shaped: 43.75 % of the causal triangle; the sweep's W = 4096 case: 75 %
    causal = lambda T: T * (T + 1) // 2
    f = bench.band_flops(1, 32, 16384, 128, 4096)
    assert f == 962106228736
    assert abs(f / (4 * 32 * 128 * causal(16384)) - 0.4375) < 1e-3
    g = bench.band_flops(2, 16, 8192, 128, 4096)
    assert abs(g / (4 * 2 * 16 * 128 * causal(8192)) - 0.75) < 1e-3


def test_decode_bytes_counts_valid_slots():
    B, H, D, W = 3, 2, 8, 5
    pos = torch.tensor([0, 3, 100], dtype=torch.int64)
    slots = sum(min(int(p) + 1, W) for p in pos)
    assert bench.decode_bytes(B, H, D, W, pos) == slots * H * D * 2 * 2 + 2 * B * H * D * 2 + 8 * B


def test_chunk_work_against_enumeration():
    B, H, C, D, W = 2, 3, 5, 8, 4
    pos = torch.tensor([0, 7], dtype=torch.int64)
    flops, nbytes = bench.chunk_work(B, H, C, D, W, pos)
    pairs = 0
    ring = 0
    for p0 in pos.tolist():
        for c in range(C):
            P = p0 + c
            pairs += sum(1 for p in range(P + 1) if P - p < W)
        ring += len([p for p in range(p0) if p >= p0 - W + 1])
    assert flops == 4 * H * D * pairs
    assert nbytes == H * ring * D * 2 * 2 + B * H * C * D * 2 * 4 + B * H * min(C, W) * D * 2 * 2 + 8 * B


def test_measured_traffic_matches_the_recorded_sources():
    """Each recorded DRAM traffic figure is reported only for the sources it was captured
    from; the records hold one entry per bench leg that reports traffic."""
    assert set(bench.MEASURED_TRAFFIC) == set(bench.KERNEL_SOURCES)
    for kind in bench.MEASURED_TRAFFIC:
        v = bench.measured_traffic(kind)
        assert v is None or v == bench.MEASURED_TRAFFIC[kind]["bytes"]


def _skip_randn(gen, shape):
    """Advance gen exactly as the input generator does for a tensor of this shape (the
    same per-leading-index split), without keeping the numbers."""
    n = 1
    for s in shape:
        n *= s
    if n <= inputs.CHUNK or len(shape) == 1:
        torch.randn(shape, generator=gen, dtype=torch.float32)
        return
    for _ in range(shape[0]):
        _skip_randn(gen, shape[1:])


def _positions(shapes, B, pos_max, seed):
    gen = torch.Generator().manual_seed(seed)
    for shp in shapes:
        _skip_randn(gen, shp)
    return torch.randint(0, pos_max, (B,), generator=gen, dtype=torch.int64)


@pytest.mark.slow
def test_sampled_traffic_is_scaled_by_the_workloads_algorithmic_bytes():
    """The decode and chunk captures ran 16 of the 64 streams; the recorded (sample, full)
    algorithmic byte counts that scale them are those of the seeded workloads."""
    d, c = inputs.DECODE, inputs.CHUNKED
    dshapes = lambda B: [(B, d.H, d.D), (B, d.H, d.W, d.D), (B, d.H, d.W, d.D)]
    cshapes = lambda B: [(B, c.H, c.C, c.D)] * 3 + [(B, c.H, c.W, c.D)] * 2
    # the walk reproduces the generator's positions
    p16 = _positions(dshapes(16), 16, d.pos_max, d.seed)
    assert torch.equal(p16, inputs.decode_inputs(16, d.H, d.D, d.W, d.pos_max, d.dtype, d.seed)[3])
    q16 = _positions(cshapes(16), 16, c.pos_max, c.seed)
    assert torch.equal(q16, inputs.chunk_inputs(16, c.H, c.C, c.D, c.W, c.pos_max, c.dtype, c.seed)[5])

    got = {"decode": [], "chunk": []}
    for B in (16, 64):
        pd = _positions(dshapes(B), B, d.pos_max, d.seed)
        got["decode"].append(bench.decode_bytes(B, d.H, d.D, d.W, pd))
        pc = _positions(cshapes(B), B, c.pos_max, c.seed)
        append_writes = B * c.H * min(c.C, c.W) * c.D * 2 * 2
        got["chunk"].append(bench.chunk_work(B, c.H, c.C, c.D, c.W, pc)[1] - append_writes)
    for kind in ("decode", "chunk"):
        assert tuple(got[kind]) == bench.SAMPLE_ALGORITHMIC_BYTES[kind], kind


def test_cpu_baseline_sample_is_described_as_taken():
    """The CPU baseline reports the oracle's own thread count and a sample description that
    matches the rows it ran, including when the sample wraps around the heads."""
    import oracle
    for wl, budget in ((inputs.SMALL, 0.3), (inputs.TINY[0], 0.05)):
        q, k, v = inputs.for_workload(wl)
        rate, desc, threads = bench.cpu_baseline_prefill(wl, budget, q, k, v)
        assert rate > 0 and threads == oracle.max_threads()
        rows = int(desc.split()[0])
        assert rows > 0 and "in the oracle" in desc
        if rows > wl.H * wl.T:
            assert "round again" in desc
        else:
            assert "round again" not in desc
