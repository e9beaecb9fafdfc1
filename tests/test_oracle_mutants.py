"""Mutation check of the pins: each plausible mistake planted in a copy of the oracle's
C source, on the CPU, must make at least one pin fail.

Each mutant is compiled and checked in a child process, so a mutant that corrupts
memory cannot take the test session down with it (a crash is reported, not counted
as caught).
"""
import json
import os
import subprocess
import sys
import tempfile

import pytest

from oracle import build as obuild

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

# The scratch for scores holds min(W, T) entries (W for decode); mutants that visit
# one more key widen it too, so that they stay in bounds and fail on values alone.
WIDER_SCRATCH = [("const int64_t band_max = (W < T) ? W : T;", "const int64_t band_max = W + 1;"),
                 ("malloc((size_t)W * sizeof(double))", "malloc((size_t)(W + 1) * sizeof(double))")]

# (name, list of (text to find, replacement))
MUTANTS = [
    ("band one key wider (the [i-W, i] reading)",
     [("int64_t lo = i - W + 1;", "int64_t lo = i - W;")] + WIDER_SCRATCH),
    ("band one key narrower", [("int64_t lo = i - W + 1;", "int64_t lo = i - W + 2;")]),
    ("scale 1/D instead of 1/sqrt(D)", [("1.0 / sqrt((double)D)", "1.0 / (double)D")]),
    ("prefill ignores the scale", [("double s = dot * scale;", "double s = dot;")]),
    ("decode ignores the scale", [("double s = dot * inv_sqrt_d;", "double s = dot;")]),
    ("weights ignore the scale", [("wrow[j] = dot * scale;", "wrow[j] = dot;")]),
    ("scale applied twice", [("double s = dot * scale;", "double s = dot * scale * scale;")]),
    ("scores read v instead of k",
     [("const double* kj = kh + j * D;", "const double* kj = vh + j * D;")]),
    ("exponent sign flipped", [("exp(scores[j - lo] - m)", "exp(m - scores[j - lo])")]),
    ("denominator dropped", [("out[d] = out[d] / denom;", "out[d] = out[d];")]),
    ("value row fixed at the band start",
     [("const double* vj = vh + j * D;", "const double* vj = vh + lo * D;")]),
    ("decode wrong slot", [("(p % W) * D", "((p + 1) % W) * D")]),
    ("decode one extra position",
     [("int64_t first = P - W + 1;", "int64_t first = P - W;")] + WIDER_SCRATCH),
    ("chunk reads its own first position from the ring",
     [("(p < pos0) ? kr + (p % W) * D", "(p <= pos0) ? kr + (p % W) * D")]),
    ("chunk band one key wider",
     [("int64_t first = P - W + 1;\n    if (first < 0) first = 0;\n    const double inv_sqrt_d = 1.0 / sqrt((double)D);\n    double m = -INFINITY;\n    for (int64_t p = first; p <= P; ++p) {\n        const double* kp = (p < pos0)",
       "int64_t first = P - W;\n    if (first < 0) first = 0;\n    const double inv_sqrt_d = 1.0 / sqrt((double)D);\n    double m = -INFINITY;\n    for (int64_t p = first; p <= P; ++p) {\n        const double* kp = (p < pos0)")] + WIDER_SCRATCH),
    ("ring append one slot late", [("(pos[b] + c) % W", "(pos[b] + c + 1) % W")]),
    ("backward drops the softmax Jacobian's mean term",
     [("const double ds = p[j - lo] * (dp[j - lo] - pdp);", "const double ds = p[j - lo] * dp[j - lo];")]),
    ("backward dk without the scale",
     [("dkh[j * D + d] += c * ds * qi[d];", "dkh[j * D + d] += ds * qi[d];")]),
    ("backward dv weighted by ds", [("dvh[j * D + d] += p[j - lo] * doi[d];", "dvh[j * D + d] += ds * doi[d];")]),
    ("weights unnormalised", [("wrow[j] = wrow[j] / denom;", "wrow[j] = wrow[j];")]),
    ("backward dq built from query rows",
     [("dqh[i * D + d] += c * ds * kh[j * D + d];", "dqh[i * D + d] += c * ds * qh[j * D + d];")]),
    ("backward dp against k instead of v",
     [("for (int64_t d = 0; d < D; ++d) dot += doi[d] * vh[j * D + d];",
       "for (int64_t d = 0; d < D; ++d) dot += doi[d] * kh[j * D + d];")]),
    ("backward dk built from dout", [("dkh[j * D + d] += c * ds * qi[d];", "dkh[j * D + d] += c * ds * doi[d];")]),
]

_CHILD = r"""
import json, sys
sys.path[:0] = [{root!r}, {here!r}]
import oracle
from oracle_pins import ALL_PINS
lib = oracle.load_variant({so!r})
failed = []
for pin in ALL_PINS:
    try:
        pin(lib)
    except AssertionError:
        failed.append(pin.__name__)
print(json.dumps(failed))
"""


@pytest.mark.parametrize("name,edits", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, edits):
    src = open(obuild.SRC).read()
    for old, new in edits:
        assert old in src, f"mutation anchor missing: {old}"
        src = src.replace(old, new)
    with tempfile.TemporaryDirectory() as d:
        cpath = os.path.join(d, "mutant.c")
        with open(cpath, "w") as f:
            f.write(src)
        so = obuild.build(src=cpath, out=os.path.join(d, "mutant.so"), force=True)
        code = _CHILD.format(root=ROOT, here=HERE, so=so)
        r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                           timeout=300)
        assert r.returncode == 0, f"mutant child crashed: {r.stderr[-2000:]}"
        failed = json.loads(r.stdout.strip().splitlines()[-1])
        assert failed, f"no pin caught mutant: {name}"


# Mistakes planted in a copy of the module oracle's Python source (oracle.mha), on the
# CPU; the copy replaces oracle.mha for the duration of the test only.
PY_MUTANTS = [
    ("module heads interleaved",
     [("y.reshape(B, T, H, Dh).transpose(0, 2, 1, 3)", "y.reshape(B, T, Dh, H).transpose(0, 3, 1, 2)")]),
    ("module bias dropped", [("return y if b is None else y + np.asarray(b, dtype=np.float64)", "return y")]),
    ("module kernel transposed",
     [("np.matmul(a, np.asarray(w, dtype=np.float64))", "np.matmul(a, np.asarray(w, dtype=np.float64).T)")]),
    ("module output projection skipped", [("out = linear(concat, wo, bo)", "out = concat")]),
    ("module heads concatenated in reverse order",
     [("concat = o.transpose(0, 2, 1, 3)", "concat = o[:, ::-1].transpose(0, 2, 1, 3)")]),
    ("module window one key wider", [("o = forward(q, k, v, W, lib=lib)", "o = forward(q, k, v, W + 1, lib=lib)")]),
    ("module keys projected by the query kernel",
     [("heads(linear(x, wk, bk))", "heads(linear(x, wq, bq))")]),
]


@pytest.mark.parametrize("name,edits", PY_MUTANTS, ids=[m[0] for m in PY_MUTANTS])
def test_module_mutant_is_caught(name, edits, monkeypatch):
    import inspect
    import textwrap

    import oracle
    from oracle_pins import ALL_PINS

    src = textwrap.dedent(inspect.getsource(oracle.mha))
    for old, new in edits:
        assert old in src, f"mutation anchor missing: {old}"
        src = src.replace(old, new)
    ns = dict(vars(oracle))
    exec(compile(src, "<mutated oracle.mha>", "exec"), ns)
    monkeypatch.setattr(oracle, "mha", ns["mha"])
    lib = oracle._load()
    failed = []
    for pin in ALL_PINS:
        try:
            pin(lib)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught mutant: {name}"
