"""The tcgen05 descriptor encoders agree bit for bit with CUTLASS's descriptor unions
(compiled as host code here; no GPU)."""
import os
import subprocess
import tempfile

import pytest

from sliding_window_causal_b200 import build

HERE = os.path.dirname(os.path.abspath(__file__))
CANDIDATES = [
    "/opt/prime-rl/.venv/lib/python3.12/site-packages/flashinfer/data/cutlass/include",
    "/opt/prime-rl/.venv/lib/python3.12/site-packages/tilelang/3rdparty/cutlass/include",
]


@pytest.mark.parametrize("inc", CANDIDATES)
def test_descriptors_match_cutlass_unions(inc):
    if not os.path.isdir(inc):
        pytest.skip(f"no CUTLASS headers at {inc}")
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "check")
        subprocess.run([build.nvcc(), "-std=c++17", "-x", "cu", "-I", inc, "-I", build.CSRC,
                        os.path.join(HERE, "cpp", "umma_desc_check.cu"), "-o", exe], check=True)
        r = subprocess.run([exe], capture_output=True, text=True)
        assert r.returncode == 0 and r.stdout.strip().endswith("OK"), r.stdout
