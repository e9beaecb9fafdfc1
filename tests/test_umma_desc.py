"""The tcgen05 descriptor encoders agree bit for bit with CUTLASS's descriptor unions
(compiled as host code here; no GPU)."""
import importlib.util
import os
import subprocess
import tempfile

import pytest

from sliding_window_causal_b200 import build

HERE = os.path.dirname(os.path.abspath(__file__))


def cutlass_include_dirs():
    """CUTLASS/CuTe header trees shipped inside installed Python packages (found by
    importing the packages' locations, never from a fixed path), plus any directory
    named by the CUTLASS_INCLUDE environment variable."""
    dirs = []
    env = os.environ.get("CUTLASS_INCLUDE")
    if env:
        dirs.append(env)
    for pkg, rel in (("flashinfer", ("data", "cutlass", "include")),
                     ("tilelang", ("3rdparty", "cutlass", "include"))):
        spec = importlib.util.find_spec(pkg)
        if spec is not None and spec.submodule_search_locations:
            for loc in spec.submodule_search_locations:
                d = os.path.join(loc, *rel)
                if os.path.isdir(os.path.join(d, "cute")):
                    dirs.append(d)
    return dirs or ["(none found)"]


CANDIDATES = cutlass_include_dirs()


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
