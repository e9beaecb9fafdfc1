"""C-ABI library on the CPU: it loads, exports every symbol include/swa.h declares, and
its host-side work planning (tile classification, ring slots, decode splits) is
bit-exact against brute-force enumeration. No GPU compute is called here."""
import heapq
import itertools
import os
import re

import numpy as np
import pytest

import sliding_window_causal_b200 as swa
from sliding_window_causal_b200 import _native, build
from oracle import brute

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built_library():
    build.build()


def header_symbols():
    text = open(os.path.join(ROOT, "include", "swa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(swa_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_symbol():
    names = header_symbols()
    assert set(names) == set(_native.EXPORTS), "binding list and header disagree"
    h = _native.lib()
    for n in names:
        assert hasattr(h, n), f"{n} not exported"


def test_exports_are_c_linkage():
    out = os.popen(f"nm -D --defined-only {_native.LIB_PATH}").read()
    for n in header_symbols():
        assert re.search(rf"\sT {n}$", out, flags=re.M), f"{n} missing or mangled"


def _brute_tile_class(T, W, bm, bn, qt, kt):
    """Enumerate every (i, j) pair of the tile: band membership for real rows decides
    'visited', and 'full' means every pair of the tile (padding rows included) is in
    the band with j < T."""
    mask = brute.band_mask(max(T, (qt + 1) * bm, (kt + 1) * bn), W)
    rows = range(qt * bm, qt * bm + bm)
    cols = range(kt * bn, kt * bn + bn)
    visited = any(mask[i, j] for i in rows if i < T for j in cols if j < T)
    if not visited:
        return 0
    full = all(mask[i, j] and j < T for i in rows for j in cols)
    return 2 if full else 1


@pytest.mark.parametrize("bm,bn", [(4, 4), (4, 8), (8, 4), (3, 5)])
def test_tile_class_matches_brute_force(bm, bn):
    for T in (1, 2, 5, 8, 13, 24):
        for W in (1, 2, 3, 4, 7, 8, 9, 16, 30):
            for qt in range((T + bm - 1) // bm):
                for kt in range((T + bn - 1) // bn + 1):
                    got = swa.tile_class(T, W, bm, bn, qt, kt)
                    assert got == _brute_tile_class(T, W, bm, bn, qt, kt), (T, W, bm, bn, qt, kt)


def test_tile_class_kernel_tiles():
    """The kernels' 128 x 128 tiles: every in-band pair lies in a visited tile, and
    tiles flagged full hold only in-band pairs (checked by counting)."""
    bm = bn = 128
    for T, W in [(130, 1), (300, 129), (1000, 128), (1000, 127), (520, 4096), (777, 300)]:
        mask = brute.band_mask(T, W) if T <= 1000 else None
        nq = (T + bm - 1) // bm
        covered = np.zeros((T, T), dtype=bool)
        for qt in range(nq):
            for kt in range(nq):
                c = swa.tile_class(T, W, bm, bn, qt, kt)
                r = slice(qt * bm, min(T, qt * bm + bm))
                s = slice(kt * bn, min(T, kt * bn + bn))
                if c:
                    covered[r, s] = True
                    assert mask[r, s].any(), "visited tile without an in-band pair"
                if c == 2:
                    assert mask[r, s].all() and kt * bn + bn <= T
        assert not (mask & ~covered).any(), "in-band pair outside the visited tiles"


def test_tile_class_rejects_bad_args():
    assert swa.tile_class(0, 3, 128, 128, 0, 0) == -1
    assert swa.tile_class(100, 0, 128, 128, 0, 0) == -1
    assert swa.tile_class(100, 3, 128, 128, 1, 0) == -1


def _pair_tiles(T, W, p):
    """Visited 128 x 128 tiles of the pair of query tiles (2p, 2p+1), by enumeration."""
    n_qt = (T + 127) // 128
    return sum(1 for qt in (2 * p, 2 * p + 1) if qt < n_qt
               for kt in range(n_qt) if swa.tile_class(T, W, 128, 128, qt, kt) > 0)


@pytest.mark.parametrize("B,H,T,W", [(1, 32, 16384, 4096), (2, 16, 8192, 1), (2, 16, 8192, 1024),
                                     (2, 16, 8192, 8192), (1, 8, 512, 128), (1, 3, 1000, 129),
                                     (2, 3, 1300, 5000), (1, 2, 129, 64), (3, 1, 640, 300)])
def test_work_items_cover_every_pair_once_heads_grouped(B, H, T, W):
    """The prefill's work items are a permutation of all (b, h, pair); the equal-work
    pairs come first, head after head; the rest follow with non-increasing work; and the
    snake assignment over min(items, 148) CTAs gives every CTA about the mean work."""
    n_qt = (T + 127) // 128
    n_pairs = (n_qt + 1) // 2
    n = B * H * n_pairs
    items = [swa.work_item(u, B, H, T, W) for u in range(n)]
    assert sorted(items) == sorted((b, h, p) for b in range(B) for h in range(H) for p in range(n_pairs))
    assert swa.work_item(n, B, H, T, W) is None and swa.work_item(-1, B, H, T, W) is None
    w = min(W, T)
    full = [(b, h, p) for (b, h, p) in items if 256 * p >= w - 1 and 2 * p + 1 < n_qt]
    nf = len(full)
    assert items[:nf] == full, "the whole-window pairs come first"
    heads = [b * H + h for (b, h, _) in full]
    assert heads == sorted(heads), "head after head"
    work = {p: _pair_tiles(T, W, p) for p in range(n_pairs)}
    assert len({work[p] for (_, _, p) in full}) <= 1, "the first section is equal work"
    rest = [work[p] for (_, _, p) in items[nf:]]
    assert rest == sorted(rest, reverse=True), "the rest heaviest first"
    G = min(n, 148)
    per_cta = np.zeros(G)
    for g in range(G):
        r = 0
        while True:
            u = r * G + ((G - 1 - g) if r & 1 else g)
            if u >= n:
                break
            per_cta[g] += work[items[u][2]]
            r += 1
    if n >= 4 * G:  # several items per CTA
        assert per_cta.max() <= 1.08 * per_cta.mean()


def test_work_item_rejects_bad_args():
    assert swa.work_item(0, 0, 1, 10, 3) is None
    assert swa.work_item(0, 1, 1, 0, 3) is None
    assert swa.work_item(0, 1, 1, 10, 0) is None


def _streamed_tiles(T, W, tile, kv):
    """Tiles the backward streams past a resident tile, by enumeration: the query tiles
    that visit key tile `tile` (kv), or the key tiles that query tile `tile` visits."""
    n = (T + 127) // 128
    if kv:
        return sum(1 for qt in range(n) if swa.tile_class(T, W, 128, 128, qt, tile) > 0)
    return sum(1 for kt in range(n) if swa.tile_class(T, W, 128, 128, tile, kt) > 0)


@pytest.mark.parametrize("kv", [True, False])
@pytest.mark.parametrize("B,H,T,W", [(1, 32, 16384, 4096), (2, 16, 8192, 1), (2, 16, 8192, 1024),
                                     (2, 16, 8192, 8192), (1, 8, 512, 128), (1, 3, 1000, 129),
                                     (2, 3, 1300, 5000), (1, 2, 129, 64), (3, 1, 640, 300), (1, 1, 100, 7)])
def test_backward_ctas_cover_every_tile_once_lightest_last(B, H, T, W, kv):
    """The backward's CTAs are a permutation of all (b, h, tile); the tiles that stream the
    most tiles come first, head after head and in order within a head; the rest follow
    with non-increasing work; and CTAs dealt in that order to whichever of 148 SMs is free
    first (a fixed cost of 1.5 tiles each) finish within 2 % of the mean."""
    n_t = (T + 127) // 128
    n = B * H * n_t
    ctas = [swa.backward_cta_tile(u, B, H, T, W, kv) for u in range(n)]
    assert sorted(ctas) == [(b, h, t) for b in range(B) for h in range(H) for t in range(n_t)]
    assert swa.backward_cta_tile(n, B, H, T, W, kv) is None and swa.backward_cta_tile(-1, B, H, T, W, kv) is None
    work = {t: _streamed_tiles(T, W, t, kv) for t in range(n_t)}
    top = max(work.values())
    nf = next((u for u, c in enumerate(ctas) if work[c[2]] != top), n)
    assert all(work[t] != top for (_, _, t) in ctas[nf:]) or nf == 0, "the heaviest tiles come first"
    head_order = [(b * H + h, t) for (b, h, t) in ctas[:nf]]
    assert head_order == sorted(head_order), "head after head, tiles in order"
    rest = [work[t] for (_, _, t) in ctas[nf:]]
    assert rest == sorted(rest, reverse=True), "the rest heaviest first"
    if n >= 8 * 148:
        free = [0.0] * 148
        heapq.heapify(free)
        for (_, _, t) in ctas:
            heapq.heappush(free, heapq.heappop(free) + work[t] + 1.5)
        mean = sum(work[t] + 1.5 for (_, _, t) in ctas) / 148
        assert max(free) <= 1.02 * mean


def test_backward_cta_tile_rejects_bad_args():
    assert swa.backward_cta_tile(0, 0, 1, 10, 3, True) is None
    assert swa.backward_cta_tile(0, 1, 1, 0, 3, False) is None
    assert swa.backward_cta_tile(0, 1, 1, 10, 0, True) is None


def test_valid_slots_match_ring_enumeration():
    for W in (1, 2, 3, 7, 64):
        for pos in list(range(0, 3 * W + 2)) + [W - 2, W - 1, W, 10**6 + 3]:
            if pos < 0:
                continue
            n = swa.valid_slots(pos, W)
            held = brute.ring_positions(pos, W)
            slots = sorted(s for _, s in held)
            assert slots == list(range(n)), (pos, W)
            assert n == min(pos + 1, W)
    assert swa.valid_slots(-1, 4) == -1
    assert swa.valid_slots(3, 0) == -1


def test_split_plan_covers_window():
    for (B, H, D, W) in itertools.product((1, 3, 64), (1, 32), (64, 128), (1, 31, 4096, 5000)):
        S, chunk = swa.split_plan(B, H, D, W)
        assert S >= 1 and chunk >= 1
        assert (S - 1) * chunk < W <= S * chunk
    with pytest.raises(swa.SwaError):
        swa.split_plan(1, 1, 96, 10)


def test_workspace_sizes():
    """The workspace queries (host only): the backward's rows are padded to whole 128-row
    tiles, two fp32 values each; the module's four [B*T, d] parts are rounded up to 256
    bytes, plus 32 MiB of GEMM scratch. Invalid sizes give -1."""
    lib = _native.lib()
    for (B, H, T) in ((1, 1, 1), (2, 3, 128), (1, 32, 16384), (4, 2, 129), (0, 5, 7)):
        tpad = (T + 127) // 128 * 128
        assert lib.swa_backward_workspace_bytes(B, H, T) == 8 * B * H * tpad
    assert lib.swa_backward_workspace_bytes(-1, 1, 1) == -1
    for (B, T, d, dt, esz) in ((1, 5, 2, 0, 4), (1, 16384, 4096, 1, 2), (2, 300, 256, 1, 2)):
        part = (B * T * d * esz + 255) // 256 * 256
        assert lib.swa_mha_workspace_bytes(B, T, d, dt) == 4 * part + (32 << 20)
    assert lib.swa_mha_workspace_bytes(1, 5, 0, 1) == -1
    assert lib.swa_mha_workspace_bytes(1, 5, 8, 7) == -1


def _c_prototypes():
    """name -> (return type, [parameter types]) for every function swa.h declares."""
    text = open(os.path.join(ROOT, "include", "swa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    protos = {}
    for m in re.finditer(r"([A-Za-z_][\w \*]*?)\b(swa_[a-z0-9_]+)\s*\(([^)]*)\)\s*;", text):
        ret, name, params = m.group(1).strip(), m.group(2), m.group(3).strip()
        types = []
        if params and params != "void":
            for p in params.split(","):
                p = " ".join(p.split())
                # drop the parameter name: the last identifier not part of the type
                t = re.sub(r"\s*\b[A-Za-z_]\w*$", "", p) if not p.endswith("*") else p
                types.append(t.replace(" *", "*").replace("const ", "").strip())
        protos[name] = (ret.replace("const ", "").strip(), types)
    return protos


def _kind(ct):
    """Class of a ctypes type as the C ABI sees it."""
    import ctypes
    if ct is None:
        return "void"
    if ct in (ctypes.c_void_p, ctypes.c_char_p) or hasattr(ct, "_type_") and isinstance(ct._type_, type):
        return "ptr"
    return {ctypes.c_int64: "i64", ctypes.c_int32: "i32", ctypes.c_uint64: "u64",
            ctypes.c_double: "f64"}[ct]


def _c_kind(t):
    if t.endswith("*"):
        return "ptr"
    return {"int64_t": "i64", "int": "i32", "uint64_t": "u64", "double": "f64", "void": "void"}[t]


def test_ctypes_signatures_match_the_header():
    """Every binding declares exactly the header's parameter list (count and ABI class of
    each argument) and return type: a mismatch would pass arguments in the wrong
    registers without any error."""
    h = _native.lib()
    protos = _c_prototypes()
    assert set(protos) == set(_native.EXPORTS)
    for name, (ret, params) in protos.items():
        f = getattr(h, name)
        assert f.argtypes is not None, name
        got = [_kind(a) for a in f.argtypes]
        want = [_c_kind(t) for t in params]
        assert got == want, f"{name}: binding {got} vs header {want}"
        assert _kind(f.restype) == _c_kind(ret), f"{name}: return {f.restype} vs {ret}"


def test_prefill_mode_setting():
    """swa_set_prefill_mode returns the previous mode and refuses unknown ones (host only)."""
    prev = swa.set_prefill_mode(swa.PREFILL_FAST)
    try:
        assert swa.set_prefill_mode(swa.PREFILL_ADAPTIVE) == swa.PREFILL_FAST
        assert swa.set_prefill_mode(swa.PREFILL_AUTO) == swa.PREFILL_ADAPTIVE
        with pytest.raises(swa.SwaError):
            swa.set_prefill_mode(3)
        with pytest.raises(swa.SwaError):
            swa.set_prefill_mode(-1)
        assert swa.set_prefill_mode(swa.PREFILL_AUTO) == swa.PREFILL_AUTO
    finally:
        swa.set_prefill_mode(prev)
