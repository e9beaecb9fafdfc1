"""Pins that tie the float64 oracle to what the pages and the mathematics fix.

Each pin takes an oracle library handle so that the same checks can run against
deliberately broken builds of the oracle (tests/test_oracle_mutants.py): every
plausible mistake there must make at least one pin fail.

None of these pins re-types the oracle's formula. They compare it with printed
values, with torch's own scaled-dot-product attention (a library routine), with
a dense masked computation built a different way, with closed forms, and with
invariants.
"""
import numpy as np
import torch

import oracle
from oracle import brute

from golden import read_band, read_moving_average

TIGHT = 1e-12


def _sdpa(q, k, v, mask=None, causal=False, scale=None):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))
    out = torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), attn_mask=None if mask is None else torch.from_numpy(mask),
        dropout_p=0.0, is_causal=causal, scale=scale)
    return out.numpy()


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def pin_band_masks(lib):
    """q = k = 0 and v = identity (D = T) make output row i equal to
    1/|band(i)| on the band's columns and 0 elsewhere, so the oracle's own band
    can be read off its output. It must equal the two printed masks bit for bit,
    and the brute-force pair enumeration for every small (T, W)."""
    def oracle_band(T, W):
        q = np.zeros((1, 1, T, T))
        v = np.eye(T).reshape(1, 1, T, T)
        out = oracle.forward(q, q, v, W, lib=lib)[0, 0]
        mask = out > 0
        counts = mask.sum(axis=1)
        # within the band every weight is exactly 1/count (exp(0) = 1, exact division)
        assert np.array_equal(out[mask], np.repeat(1.0 / counts, counts)), "band weights"
        return mask

    for name in ("nnx_band_T5_W3.txt", "mistral_impl_band_T8_W4.txt"):
        T, W, printed = read_band(name)
        assert np.array_equal(oracle_band(T, W), printed), f"printed mask {name}"
    for T in (1, 2, 3, 7, 16, 33):
        for W in (1, 2, 3, 5, 8, 15, 16, 17, 40):
            m = oracle_band(T, W)
            assert np.array_equal(m, brute.band_mask(T, W)), f"band T={T} W={W}"
            assert np.array_equal(m.sum(axis=1), np.minimum(np.arange(T) + 1, W))


def pin_moving_average(lib):
    """The worked example with zero q/k projections prints exact trailing means,
    and changing input row 0 leaves rows 3 and later unchanged."""
    g = read_moving_average()
    W, x = g["W"], g["x"]
    T, Hn = x.shape
    v = x.T.reshape(1, Hn, T, 1).copy()
    z = np.zeros_like(v)
    out = oracle.forward(z, z, v, W, lib=lib)[0, :, :, 0].T
    assert np.array_equal(out, g["y"]), "moving average printed values"
    row, vals = g["changed_row"]
    x2 = x.copy()
    x2[row] = vals
    v2 = x2.T.reshape(1, Hn, T, 1).copy()
    out2 = oracle.forward(z, z, v2, W, lib=lib)[0, :, :, 0].T
    u = g["unchanged_from"]
    assert np.array_equal(out2[u:], out[u:]), "rows past the window unchanged"
    assert not np.array_equal(out2[:u], out[:u])


def pin_trailing_mean_any_k(lib):
    """Generalisation of the worked example: q = 0 gives the trailing mean of v over
    the band whatever k holds (every score is 0, so all weights are equal)."""
    rng = np.random.default_rng(7)
    for (T, D, W) in ((9, 3, 4), (20, 5, 1), (12, 2, 30)):
        q = np.zeros((1, 2, T, D))
        k = _rand(rng, 1, 2, T, D)
        v = _rand(rng, 1, 2, T, D)
        out = oracle.forward(q, k, v, W, lib=lib)
        for i in range(T):
            lo = max(0, i - W + 1)
            ref = v[:, :, lo:i + 1, :].mean(axis=2)
            assert np.abs(out[:, :, i, :] - ref).max() <= TIGHT, "trailing mean"


def pin_causal_reduction(lib):
    """W >= T is ordinary causal attention: compare with torch's scaled dot-product
    attention (is_causal=True) in float64."""
    rng = np.random.default_rng(11)
    for (B, H, T, D) in ((1, 2, 6, 4), (2, 3, 17, 8), (1, 1, 40, 1)):
        q, k, v = (_rand(rng, B, H, T, D) for _ in range(3))
        ref = _sdpa(q, k, v, causal=True)
        for W in (T, T + 1, 3 * T):
            out = oracle.forward(q, k, v, W, lib=lib)
            assert np.abs(out - ref).max() <= TIGHT, f"causal W={W}"


def pin_general_band(lib):
    """Random inputs, general W: compare with torch's scaled dot-product attention
    given the brute-force boolean band mask, and with the dense masked computation."""
    rng = np.random.default_rng(13)
    for (B, H, T, D, W) in ((1, 2, 6, 4, 3), (2, 2, 19, 5, 4), (1, 3, 33, 16, 7),
                            (1, 1, 12, 2, 11), (1, 2, 25, 3, 2)):
        q, k, v = (_rand(rng, B, H, T, D) * 2.0 for _ in range(3))
        out = oracle.forward(q, k, v, W, lib=lib)
        ref = _sdpa(q, k, v, mask=brute.band_mask(T, W))
        assert np.abs(out - ref).max() <= TIGHT, f"sdpa band T={T} W={W}"
        ref2, _ = brute.dense_masked_attention(q, k, v, W)
        assert np.abs(out - ref2).max() <= TIGHT, f"dense band T={T} W={W}"


def pin_window_one(lib):
    """W = 1 keeps only the diagonal, so the output is v exactly."""
    rng = np.random.default_rng(17)
    q, k, v = (_rand(rng, 2, 3, 10, 6) for _ in range(3))
    assert np.array_equal(oracle.forward(q, k, v, 1, lib=lib), v), "W=1 returns v"


def pin_independence(lib):
    """Corrupt-and-compare: changing k and v at positions j <= i - W leaves row i
    unchanged exactly; changing a position inside the window changes it."""
    rng = np.random.default_rng(19)
    B, H, T, D, W = 1, 2, 24, 4, 5
    q, k, v = (_rand(rng, B, H, T, D) for _ in range(3))
    base = oracle.forward(q, k, v, W, lib=lib)
    for i in (W, 11, T - 1):
        k2, v2 = k.copy(), v.copy()
        k2[:, :, : i - W + 1, :] = 100.0
        v2[:, :, : i - W + 1, :] = 200.0
        out = oracle.forward(q, k2, v2, W, lib=lib)
        assert np.array_equal(out[:, :, i, :], base[:, :, i, :]), f"row {i} independent"
        k3 = k.copy()
        k3[:, :, i - W + 1, :] += 1.0
        out3 = oracle.forward(q, k3, v, W, lib=lib)
        assert not np.array_equal(out3[:, :, i, :], base[:, :, i, :]), f"row {i} sees j=i-W+1"


def pin_weights(lib):
    """Probabilities: zero outside the band, each row sums to 1, weights @ v is the output."""
    rng = np.random.default_rng(23)
    B, H, T, D, W = 1, 2, 16, 32, 4
    q, k, v = (_rand(rng, B, H, T, D) for _ in range(3))
    w = oracle.weights(q, k, W, lib=lib)
    mask = brute.band_mask(T, W)
    assert np.all(w[:, :, ~mask] == 0.0), "off-band weights are zero"
    assert np.all(w[:, :, mask] > 0.0)
    assert np.abs(w.sum(axis=-1) - 1.0).max() <= TIGHT, "rows sum to 1"
    out = oracle.forward(q, k, v, W, lib=lib)
    assert np.abs(np.matmul(w, v) - out).max() <= TIGHT
    _, wref = brute.dense_masked_attention(q, k, v, W)
    assert np.abs(w - wref).max() <= TIGHT


def pin_rows_subset(lib):
    """forward_rows returns exactly the rows of the full forward."""
    rng = np.random.default_rng(29)
    B, H, T, D, W = 2, 2, 21, 5, 6
    q, k, v = (_rand(rng, B, H, T, D) for _ in range(3))
    full = oracle.forward(q, k, v, W, lib=lib).reshape(-1, D)
    rows = np.array([0, 5, 20, 21, 40, 63, B * H * T - 1])
    sub = oracle.forward_rows(q, k, v, W, rows, lib=lib)
    assert np.array_equal(sub, full[rows])


def _ring_from_history(kh, vh, P, W):
    """Write positions 0..P of a history [P+1, D] into a W-slot ring, slot p mod W,
    later positions overwriting earlier ones (brute force, position by position)."""
    D = kh.shape[-1]
    kr = np.zeros((W, D))
    vr = np.zeros((W, D))
    for p in range(P + 1):
        kr[p % W] = kh[p]
        vr[p % W] = vh[p]
    return kr, vr


def pin_decode(lib):
    """Decode over a ring built from a seeded history equals the last row of the
    prefill over that history; for P >= W-1 the answer depends only on the ring."""
    rng = np.random.default_rng(31)
    D, H = 6, 2
    for W in (1, 3, 8):
        for P in sorted({0, 1, max(0, W - 2), W - 1, W, W + 1, 2 * W + 3, 3 * W}):
            B = 2
            kh = _rand(rng, B, H, P + 1, D)
            vh = _rand(rng, B, H, P + 1, D)
            qh = _rand(rng, B, H, P + 1, D)
            kr = np.zeros((B, H, W, D))
            vr = np.zeros((B, H, W, D))
            for b in range(B):
                for h in range(H):
                    kr[b, h], vr[b, h] = _ring_from_history(kh[b, h], vh[b, h], P, W)
            pos = np.array([P, P])
            out = oracle.decode(qh[:, :, P, :], kr, vr, pos, W, lib=lib)
            ref = oracle.forward(qh, kh, vh, W, lib=lib)[:, :, P, :]
            assert np.abs(out - ref).max() <= TIGHT, f"decode W={W} P={P}"
            if P >= W - 1:
                out2 = oracle.decode(qh[:, :, P, :], kr, vr, pos + 3 * W, W, lib=lib)
                assert np.abs(out2 - out).max() <= TIGHT, "full ring independent of P"


def pin_shapes(lib):
    """Printed shapes: (1,2,6,4) with window 3 keeps its shape; the 3-D (1,5,3)
    case with window 2 is one head."""
    rng = np.random.default_rng(37)
    q = _rand(rng, 1, 2, 6, 4)
    assert oracle.forward(q, q, q, 3, lib=lib).shape == (1, 2, 6, 4)
    q3 = _rand(rng, 1, 5, 3)
    out = oracle.forward(q3[:, None], q3[:, None], q3[:, None], 2, lib=lib)[:, 0]
    assert out.shape == (1, 5, 3)


def pin_scaled(lib):
    """A caller-given scale ("Mistral Architecture > Implementation: Sliding Window
    Attention", Step 2): torch's scaled dot-product attention with the same scale and the
    brute-force band mask agrees; scale 0 gives the trailing mean of v whatever q and k
    hold; scaling q by a and the scale by 1/a changes nothing; and the default scale is
    1/sqrt(D)."""
    rng = np.random.default_rng(41)
    for (B, H, T, D, W) in ((1, 2, 9, 4, 3), (2, 1, 20, 8, 6), (1, 2, 14, 3, 20)):
        q, k, v = (_rand(rng, B, H, T, D) for _ in range(3))
        for sc in (0.05, 0.5, 1.0, 2.0, -0.7):
            out = oracle.forward(q, k, v, W, lib=lib, scale=sc)
            ref = _sdpa(q, k, v, mask=brute.band_mask(T, W), scale=sc)
            assert np.abs(out - ref).max() <= TIGHT, f"sdpa scale={sc} T={T} W={W}"
        out0 = oracle.forward(q, k, v, W, lib=lib, scale=0.0)
        for i in range(T):
            lo = max(0, i - W + 1)
            assert np.abs(out0[:, :, i, :] - v[:, :, lo:i + 1, :].mean(axis=2)).max() <= TIGHT
        a = 3.0
        o1 = oracle.forward(q * a, k, v, W, lib=lib, scale=0.25 / a)
        o2 = oracle.forward(q, k, v, W, lib=lib, scale=0.25)
        assert np.abs(o1 - o2).max() <= TIGHT, "homogeneity in q and the scale"
        d = oracle.forward(q, k, v, W, lib=lib, scale=1.0 / np.sqrt(D))
        assert np.array_equal(d, oracle.forward(q, k, v, W, lib=lib)), "default scale"


def pin_weights_scaled(lib):
    """Weights with a caller-given scale equal torch's softmax of the scaled, band-masked
    score matrix built with torch.matmul; scale 0 spreads each row evenly over its band."""
    rng = np.random.default_rng(43)
    B, H, T, D, W = 1, 2, 13, 5, 4
    q, k = (_rand(rng, B, H, T, D) for _ in range(2))
    mask = brute.band_mask(T, W)
    for sc in (0.3, 1.7, -1.1):
        w = oracle.weights(q, k, W, lib=lib, scale=sc)
        sco = torch.matmul(torch.from_numpy(q), torch.from_numpy(k).transpose(-1, -2)) * sc
        sco = sco.masked_fill(~torch.from_numpy(mask), float("-inf"))
        ref = torch.softmax(sco, dim=-1).numpy()
        assert np.abs(w - ref).max() <= TIGHT, f"weights scale={sc}"
    w0 = oracle.weights(q, k, W, lib=lib, scale=0.0)
    counts = np.minimum(np.arange(T) + 1, W)
    even = np.where(mask, 1.0 / counts[:, None], 0.0)
    assert np.abs(w0 - even).max() <= TIGHT, "scale 0 gives even weights"


def pin_chunk_stream(lib):
    """A stream fed chunk by chunk: each chunk's outputs over the ring (built position by
    position from the history) equal the same rows of torch's scaled dot-product
    attention over the whole history with the brute-force band mask; a chunk of one
    token equals decode."""
    rng = np.random.default_rng(47)
    D, H, B = 4, 2, 1
    for W in (1, 3, 8):
        for (pos0, C) in ((0, 5), (0, 1), (2, 4), (W - 1, 3), (W, 1), (W + 2, 2 * W + 1),
                          (3 * W + 1, W), (5, 12)):
            T = pos0 + C
            qh, kh, vh = (_rand(rng, B, H, T, D) for _ in range(3))
            ref = _sdpa(qh, kh, vh, mask=brute.band_mask(T, W))[:, :, pos0:, :]
            kr = np.zeros((B, H, W, D))
            vr = np.zeros((B, H, W, D))
            if pos0 > 0:
                for h in range(H):
                    kr[0, h], vr[0, h] = _ring_from_history(kh[0, h], vh[0, h], pos0 - 1, W)
            pos = np.array([pos0])
            out = oracle.chunk(qh[:, :, pos0:], kh[:, :, pos0:], vh[:, :, pos0:], kr, vr, pos, W,
                               lib=lib)
            assert np.abs(out - ref).max() <= TIGHT, f"chunk W={W} pos={pos0} C={C}"
            if C == 1:
                kr2, vr2 = kr.copy(), vr.copy()
                kr2[:, :, pos0 % W], vr2[:, :, pos0 % W] = kh[:, :, pos0], vh[:, :, pos0]
                dec = oracle.decode(qh[:, :, pos0], kr2, vr2, pos, W, lib=lib)
                assert np.abs(out[:, :, 0] - dec).max() <= TIGHT, "one-token chunk is decode"


def pin_ring_append(lib):
    """Appending a history in chunks of any sizes leaves the ring that writing it
    position by position leaves (brute force), whatever the chunking."""
    rng = np.random.default_rng(53)
    D, H = 3, 2
    for W in (1, 4, 7):
        T = 3 * W + 5
        kh, vh = _rand(rng, 1, H, T, D), _rand(rng, 1, H, T, D)
        for sizes in ([T], [1] * T, [W + 2, 1, T - W - 3], [2, W, W, T - 2 - 2 * W]):
            kr = np.full((1, H, W, D), np.nan)
            vr = np.full((1, H, W, D), np.nan)
            p = 0
            for c in sizes:
                kr, vr = oracle.ring_append(kh[:, :, p:p + c], vh[:, :, p:p + c], kr, vr,
                                            np.array([p]), W, lib=lib)
                p += c
                for h in range(H):
                    ek, ev = _ring_from_history(kh[0, h], vh[0, h], p - 1, W)
                    n = min(p, W)
                    slots = [q % W for q in range(p - n, p)]
                    assert np.array_equal(kr[0, h, slots], ek[slots]), f"ring k W={W} {sizes}"
                    assert np.array_equal(vr[0, h, slots], ev[slots]), f"ring v W={W} {sizes}"


def pin_module_worked_example(lib):
    """The module's printed example: d_model 2, two heads, window 3, zero query and key
    kernels, identity value and output kernels, zero biases, gives the printed trailing
    means exactly; replacing input row 0 leaves rows 3 and later unchanged."""
    g = read_moving_average()
    x = np.array(g["x"])
    z, eye = np.zeros((2, 2)), np.eye(2)
    out = oracle.mha(x, z, None, z, None, eye, None, eye, None, 2, g["W"], lib=lib)
    assert np.array_equal(out, np.array(g["y"])), "printed module output"
    row, vals = g["changed_row"]
    x2 = x.copy()
    x2[row] = vals
    out2 = oracle.mha(x2, z, None, z, None, eye, None, eye, None, 2, g["W"], lib=lib)
    u = g["unchanged_from"]
    assert np.array_equal(out2[u:], out[u:])


def pin_module_vs_torch(lib):
    """Random kernels and biases: the module equals torch's linear layers around its
    scaled dot-product attention with the brute-force band mask, in float64."""
    rng = np.random.default_rng(59)
    F = torch.nn.functional
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    for (B, T, d, H, W) in ((2, 13, 12, 3, 4), (1, 20, 8, 2, 1), (1, 9, 6, 1, 30)):
        x = _rand(rng, B, T, d)
        ws = [_rand(rng, d, d) / np.sqrt(d) for _ in range(4)]
        bs = [_rand(rng, d) * 0.1 for _ in range(4)]
        out = oracle.mha(x, ws[0], bs[0], ws[1], bs[1], ws[2], bs[2], ws[3], bs[3], H, W, lib=lib)
        proj = [F.linear(t(x), t(ws[i]).T, t(bs[i])) for i in range(3)]
        Dh = d // H
        q, k, v = (p.reshape(B, T, H, Dh).transpose(1, 2) for p in proj)
        o = F.scaled_dot_product_attention(q, k, v, attn_mask=torch.from_numpy(brute.band_mask(T, W)))
        ref = F.linear(o.transpose(1, 2).reshape(B, T, d), t(ws[3]).T, t(bs[3])).numpy()
        assert np.abs(out - ref).max() <= TIGHT, f"module B={B} T={T} d={d} H={H} W={W}"


def pin_backward_autograd(lib):
    """The gradients equal torch autograd through its scaled dot-product attention with
    the brute-force band mask, in float64, for several windows including W = 1 and
    W >= T."""
    rng = np.random.default_rng(61)
    for (B, H, T, D, W) in ((1, 2, 9, 4, 3), (2, 1, 17, 6, 5), (1, 2, 12, 3, 1), (1, 1, 10, 5, 40)):
        q, k, v, do = (_rand(rng, B, H, T, D) for _ in range(4))
        dq, dk, dv = oracle.backward(q, k, v, do, W, lib=lib)
        tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
        out = torch.nn.functional.scaled_dot_product_attention(
            tq, tk, tv, attn_mask=torch.from_numpy(brute.band_mask(T, W)))
        out.backward(torch.from_numpy(do))
        for name, a, b in (("dq", dq, tq.grad), ("dk", dk, tk.grad), ("dv", dv, tv.grad)):
            assert np.abs(a - b.numpy()).max() <= TIGHT, f"{name} T={T} W={W}"


def pin_backward_finite_differences(lib):
    """Central differences of the forward oracle (a different code path) in random
    directions agree with the directional derivative sum(dout * d out) given by the
    gradients."""
    rng = np.random.default_rng(67)
    B, H, T, D, W = 1, 2, 11, 4, 4
    q, k, v, do = (_rand(rng, B, H, T, D) for _ in range(4))
    grads = oracle.backward(q, k, v, do, W, lib=lib)
    h = 1e-5
    for which in range(3):
        for _ in range(3):
            u = _rand(rng, B, H, T, D)
            args = [q, k, v]
            plus = list(args)
            minus = list(args)
            plus[which] = args[which] + h * u
            minus[which] = args[which] - h * u
            fd = (np.sum(do * oracle.forward(*plus, W, lib=lib)) -
                  np.sum(do * oracle.forward(*minus, W, lib=lib))) / (2 * h)
            an = np.sum(grads[which] * u)
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), f"finite differences, operand {which}"


ALL_PINS = [pin_band_masks, pin_moving_average, pin_trailing_mean_any_k, pin_causal_reduction,
            pin_general_band, pin_window_one, pin_independence, pin_weights, pin_rows_subset,
            pin_decode, pin_shapes, pin_scaled, pin_weights_scaled, pin_chunk_stream,
            pin_ring_append, pin_module_worked_example, pin_module_vs_torch, pin_backward_autograd,
            pin_backward_finite_differences]
