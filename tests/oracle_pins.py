"""Pins that tie the float64 oracle to something other than itself.

Each pin takes an ``oracle.Oracle`` instance and raises AssertionError when
the oracle disagrees with: a hand-derived worked example (tests/golden), a
closed form, an invariant the operator must satisfy, a library special case
(numpy.fft for the hand-written FFT), or the direct definition on small
inputs.  ``test_oracle.py`` runs every pin against the committed oracle and
``test_oracle_mutations.py`` runs them against deliberately broken builds to
show that a plausible mistake fails at least one pin.
"""
from __future__ import annotations

import json
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _close(a, b, tol=1e-12, what=""):
    a = np.asarray(a)
    b = np.asarray(b)
    if not (np.iscomplexobj(a) or np.iscomplexobj(b)):
        a = a.astype(np.float64)
        b = b.astype(np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= tol * scale, f"{what}: max abs err {err:.3e} > {tol:.1e} * {scale:.3e}"


# ------------------------------------------------------------------ FFT ---
def pin_fft_matches_numpy(orc):
    """The hand-written radix-2 FFT against numpy.fft (library special case)."""
    rng = np.random.default_rng(1)
    for m in range(0, 15):
        n = 1 << m
        z = rng.standard_normal(n) + 1j * rng.standard_normal(n)
        _close(orc.fft(z), np.fft.fft(z), 1e-11, f"fft n={n}")
        _close(orc.fft(z, inverse=True), np.fft.ifft(z) * n, 1e-11, f"ifft n={n}")


def pin_fft_delta_and_parseval(orc):
    n = 1024
    d = np.zeros(n, complex); d[0] = 1.0
    _close(orc.fft(d), np.ones(n), 1e-14, "fft(delta) = 1")
    d2 = np.zeros(n, complex); d2[1] = 1.0
    f = np.arange(n)
    _close(orc.fft(d2), np.exp(-2j * np.pi * f / n), 1e-13, "fft(delta_1) = exp(-2 pi i f/n)")
    z = np.random.default_rng(2).standard_normal(n) + 0j
    Z = orc.fft(z)
    assert abs(np.sum(np.abs(Z) ** 2) / n - np.sum(np.abs(z) ** 2)) < 1e-9 * np.sum(np.abs(z) ** 2)


# ------------------------------------------------------------ worked examples
def pin_golden_shortconv(orc):
    g = _golden("shortconv_len4.json")
    _close(orc.shortconv(g["u"], g["w"], g["bias"]), g["expected"], 1e-15, "shortconv golden")


def pin_golden_fftconv(orc):
    g = _golden("fftconv_len4.json")
    _close(orc.causal_conv_direct(g["k"], g["D"], g["x"]), g["expected"], 1e-15, "direct golden")
    _close(orc.causal_conv_fft(g["k"], g["D"], g["x"]), g["expected"], 1e-13, "fft golden")


def pin_golden_operator_order2(orc):
    g = _golden("operator_order2_len4.json")
    u = np.array(g["u"], float)[None]
    k = np.array(g["k"], float)[None]
    D = np.array(g["D"], float)[None]
    for method in (1, 2):
        _close(orc.hyena_rows(u, k, D, method=method)[0], g["expected"], 1e-13,
               f"operator order 2 golden, method {method}")


def pin_golden_operator_order3(orc):
    g = _golden("operator_order3_len3.json")
    u = np.array(g["u"], float)[None]
    k = np.array(g["k"], float)[None]
    D = np.array(g["D"], float)[None]
    for method in (1, 2):
        _close(orc.hyena_rows(u, k, D, method=method)[0], g["expected"], 1e-13,
               f"operator order 3 golden, method {method}")


def pin_golden_conv2d(orc):
    g = _golden("conv2d_2x2.json")
    _close(orc.conv2d_direct(g["K"], g["D"], g["x"]), g["expected"], 1e-15, "conv2d direct golden")
    _close(orc.conv2d_fft(g["K"], g["D"], g["x"]), g["expected"], 1e-13, "conv2d fft golden")


def pin_golden_operator2d(orc):
    g = _golden("operator2d_order2_2x2.json")
    u = np.array(g["u"], float)[None]
    k = np.array(g["k"], float)[None]
    D = np.array(g["D"], float)[None]
    for method in (1, 2):
        _close(orc.hyena_rows(u, k, D, ndim=2, method=method)[0], g["expected"], 1e-13,
               f"2-D operator golden, method {method}")


def pin_golden_split_order3(orc):
    """Stacked [B, (order+1) C, L] -> chunk j of channel c is channel j*C + c."""
    g = _golden("operator_split_order3_c2.json")
    u = np.array(g["u"], float)
    k = np.array(g["k"], float)
    D = np.array(g["D"], float)
    want = np.array(g["expected"], float).reshape(g["B"] * g["C"], -1)
    for method in (1, 2):
        y = orc.hyena_stacked(u, k, D, B=g["B"], C=g["C"], order=g["order"], shape=u.shape[2:], method=method)
        _close(y, want, 1e-13, f"split golden (order 3), method {method}")


def pin_golden_split_taps(orc):
    """Short-conv taps and bias of chunk j of channel c are those of channel j*C + c."""
    g = _golden("operator_split_taps_order2_c2.json")
    u = np.array(g["u"], float)
    want = np.array(g["expected"], float).reshape(g["B"] * g["C"], -1)
    for method in (1, 2):
        y = orc.hyena_stacked(u, np.array(g["k"], float), np.array(g["D"], float), np.array(g["sc_w"], float),
                              np.array(g["sc_b"], float), B=g["B"], C=g["C"], order=g["order"],
                              shape=u.shape[2:], method=method)
        _close(y, want, 1e-13, f"split taps golden, method {method}")


def pin_split_batches_rows_and_storage(orc):
    """Batch b of a stacked call equals a call on u[b] alone; a row subset
    equals those rows of the full call; bf16 bit patterns decode to the same
    values as float32 (values chosen exactly representable in bf16)."""
    rng = np.random.default_rng(21)
    B, C, order, L = 3, 4, 3, 32
    u = rng.integers(-8, 9, size=(B, (order + 1) * C, L)).astype(np.float32) / 4
    k = rng.integers(-8, 9, size=(order - 1, C, L)).astype(np.float32) / 8
    D = rng.standard_normal((order - 1, C))
    w = rng.standard_normal(((order + 1) * C, 3))
    bias = rng.standard_normal((order + 1) * C)
    kw = dict(C=C, order=order, shape=(L,), method=1)
    full = orc.hyena_stacked(u, k, D, w, bias, B=B, **kw).reshape(B, C, L)
    for b in range(B):
        one = orc.hyena_stacked(u[b:b + 1], k, D, w, bias, B=1, **kw).reshape(C, L)
        _close(full[b], one, 0.0, f"batch {b} on its own")
    rows = np.array([7, 0, 11, 5])
    sub = orc.hyena_stacked(u, k, D, w, bias, B=B, rows=rows, **kw)
    _close(sub, full.reshape(B * C, L)[rows], 0.0, "row subset")
    ubits = (u.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    kbits = (k.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    assert np.array_equal((ubits.astype(np.uint32) << np.uint32(16)).view(np.float32), u)
    viabits = orc.hyena_stacked(ubits, kbits, D, w, bias, B=B, **kw).reshape(B, C, L)
    _close(viabits, full, 0.0, "bf16 bit patterns")


def pin_split_per_sample_filters(orc):
    """Per-sample filters: row (b, c) takes filter b*C + c.  Filters repeated
    over the batch give the shared-filter result, and batch b equals a
    shared-filter call with the filters of sample b."""
    rng = np.random.default_rng(22)
    B, C, order, L = 2, 3, 3, 16
    u = rng.standard_normal((B, (order + 1) * C, L))
    k = rng.standard_normal((order - 1, B * C, L))
    D = rng.standard_normal((order - 1, B * C))
    w = rng.standard_normal(((order + 1) * C, 3))
    kw = dict(C=C, order=order, shape=(L,), method=1)
    ps = orc.hyena_stacked(u, k, D, w, B=B, per_sample=True, **kw).reshape(B, C, L)
    for b in range(B):
        shared = orc.hyena_stacked(u[b:b + 1], k[:, b * C:(b + 1) * C], D[:, b * C:(b + 1) * C], w, B=1,
                                   **kw).reshape(C, L)
        _close(ps[b], shared, 0.0, f"per-sample filters of sample {b}")
    k_rep = np.concatenate([k[:, :C]] * B, axis=1)
    D_rep = np.concatenate([D[:, :C]] * B, axis=1)
    _close(orc.hyena_stacked(u, k_rep, D_rep, w, B=B, per_sample=True, **kw),
           orc.hyena_stacked(u, k[:, :C], D[:, :C], w, B=B, **kw), 0.0, "repeated per-sample = shared")


def pin_golden_projections(orc):
    """in_proj with its 'b l d -> b d l' rearrangement and out_proj on the
    rearranged y, against a hand-derived example."""
    g = _golden("projections_2x2.json")
    a = g["in_proj"]
    _close(orc.in_proj(np.array(a["x"], float), np.array(a["W"], float), np.array(a["bias"], float)),
           a["expected"], 1e-15, "in_proj golden")
    b = g["out_proj"]
    _close(orc.out_proj(np.array(b["y"], float), np.array(b["W"], float), np.array(b["bias"], float)),
           b["expected"], 1e-15, "out_proj golden")


def pin_projections_match_numpy(orc):
    """Random shapes against numpy's matmul (a library special case), with and
    without bias, and bf16 bit patterns decoded exactly."""
    rng = np.random.default_rng(31)
    for B, L, D, J in ((1, 5, 3, 7), (2, 16, 8, 24), (3, 9, 16, 16)):
        x = rng.standard_normal((B, L, D)); W = rng.standard_normal((J, D)); bias = rng.standard_normal(J)
        _close(orc.in_proj(x, W, bias), np.einsum("bld,jd->bjl", x, W) + bias[None, :, None], 1e-12, "in_proj")
        _close(orc.in_proj(x, W), np.matmul(x, W.T).transpose(0, 2, 1), 1e-12, "in_proj no bias")
        y = rng.standard_normal((B, D, L)); W2 = rng.standard_normal((J, D))
        _close(orc.out_proj(y, W2, bias), np.matmul(y.transpose(0, 2, 1), W2.T) + bias, 1e-12, "out_proj")
    xq = (rng.integers(-64, 64, size=(2, 8, 4)) / 16).astype(np.float32)
    Wq = (rng.integers(-64, 64, size=(6, 4)) / 16).astype(np.float32)
    bits = lambda a: (a.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    _close(orc.in_proj(bits(xq), bits(Wq)), orc.in_proj(xq, Wq), 0.0, "in_proj on bf16 bits")


def pin_layer_with_identity_projections(orc):
    """W_in = [I; I; I] copies x into every chunk and W_out = I: the layer is
    then the operator on the stacked x^T (the projections compose with the
    split in the order [P4] 二.1 gives)."""
    rng = np.random.default_rng(32)
    B, L, D, order = 2, 16, 3, 2
    x = rng.standard_normal((B, L, D))
    W_in = np.concatenate([np.eye(D)] * (order + 1), axis=0)
    k = rng.standard_normal((order - 1, D, L)); Dk = rng.standard_normal((order - 1, D))
    u = orc.in_proj(x, W_in)
    _close(u, np.concatenate([x.transpose(0, 2, 1)] * (order + 1), axis=1), 0.0, "identity in_proj")
    y = orc.hyena_stacked(u, k, Dk, B=B, C=D, order=order, shape=(L,), method=1).reshape(B, D, L)
    out = orc.out_proj(y, np.eye(D))
    _close(out, y.transpose(0, 2, 1), 0.0, "identity out_proj")


# ---------------------------------------------------------- closed forms ---
def pin_geometric_filter_closed_form(orc):
    """k[t] = r^t, x = 1  ->  out[t] = (1 - r^(t+1)) / (1 - r) + D."""
    L, r, D = 257, 0.97, -0.75
    t = np.arange(L)
    k = r ** t
    want = (1 - r ** (t + 1)) / (1 - r) + D
    _close(orc.causal_conv_direct(k, D, np.ones(L)), want, 1e-12, "geometric direct")
    _close(orc.causal_conv_fft(k, D, np.ones(L)), want, 1e-11, "geometric fft")


def pin_delta_invariant(orc):
    """x0 = x1 = 1, v = delta_0, no short conv  ->  y = k + D delta_0 (order 2)."""
    rng = np.random.default_rng(3)
    for L in (16, 1024, 8192):
        k = rng.standard_normal(L)
        D = 0.625
        u = np.ones((1, 3, L)); u[0, 2] = 0.0; u[0, 2, 0] = 1.0
        want = k.copy(); want[0] += D
        for method in (1, 2):
            if method == 1 and L > 1024:
                continue
            y = orc.hyena_rows(u, k[None, None], np.array([[D]]), method=method)[0]
            _close(y, want, 1e-12, f"delta invariant L={L} method {method}")


# ------------------------------------------------------------ invariants ---
def _rand_rows(rng, R, order, L, shortconv=True, bias=False):
    u = rng.standard_normal((R, order + 1, L))
    k = rng.standard_normal((R, order - 1, L)) * np.exp(-3.0 * np.arange(L) / L)
    D = rng.standard_normal((R, order - 1))
    w = rng.standard_normal((R, order + 1, 3)) * np.sqrt(1 / 3) if shortconv else None
    b = rng.standard_normal((R, order + 1)) if (shortconv and bias) else None
    return u, k, D, w, b


def pin_fft_conv_equals_direct(orc):
    rng = np.random.default_rng(4)
    for L in (1, 2, 3, 5, 8, 17, 64, 100, 1024, 4096):
        k = rng.standard_normal(L); x = rng.standard_normal(L); D = float(rng.standard_normal())
        _close(orc.causal_conv_fft(k, D, x), orc.causal_conv_direct(k, D, x), 1e-11, f"L={L}")


def pin_conv2d_fft_equals_direct(orc):
    rng = np.random.default_rng(5)
    for H, W in ((1, 1), (1, 8), (3, 5), (8, 8), (16, 32), (32, 32)):
        K = rng.standard_normal((H, W)); x = rng.standard_normal((H, W))
        _close(orc.conv2d_fft(K, 0.3, x), orc.conv2d_direct(K, 0.3, x), 1e-11, f"{H}x{W}")


def pin_conv2d_single_row_is_1d(orc):
    rng = np.random.default_rng(6)
    W = 64
    K = rng.standard_normal((1, W)); x = rng.standard_normal((1, W))
    _close(orc.conv2d_direct(K, 0.5, x)[0], orc.causal_conv_direct(K[0], 0.5, x[0]), 1e-12, "H=1")
    Kc = rng.standard_normal((W, 1)); xc = rng.standard_normal((W, 1))
    _close(orc.conv2d_direct(Kc, 0.5, xc)[:, 0], orc.causal_conv_direct(Kc[:, 0], 0.5, xc[:, 0]),
           1e-12, "W=1")


def pin_operator_direct_equals_fft(orc):
    rng = np.random.default_rng(7)
    for order in (2, 3, 4):
        u, k, D, w, b = _rand_rows(rng, 3, order, 300, bias=True)
        y1 = orc.hyena_rows(u, k, D, w, b, method=1)
        y2 = orc.hyena_rows(u, k, D, w, b, method=2)
        _close(y2, y1, 1e-10, f"order {order}")


def pin_causality(orc):
    """Perturbing any chunk at t > s leaves y[0..s] bitwise unchanged."""
    rng = np.random.default_rng(8)
    L, s = 200, 117
    for order in (2, 3):
        u, k, D, w, b = _rand_rows(rng, 1, order, L, bias=True)
        y = orc.hyena_rows(u, k, D, w, b, method=1)
        u2 = u.copy()
        u2[:, :, s + 1:] += rng.standard_normal(u2[:, :, s + 1:].shape)
        y2 = orc.hyena_rows(u2, k, D, w, b, method=1)
        assert np.array_equal(y[:, :s + 1], y2[:, :s + 1]), f"order {order}: not causal"
        assert not np.array_equal(y[:, s + 1:], y2[:, s + 1:])


def pin_linearity_in_v(orc):
    """Order 2, no short conv: y is linear in the value chunk v."""
    rng = np.random.default_rng(9)
    L = 512
    u, k, D, _, _ = _rand_rows(rng, 1, 2, L, shortconv=False)
    a, c = rng.standard_normal(L), rng.standard_normal(L)
    alpha, beta = 1.75, -0.5

    def run(v):
        uu = u.copy(); uu[0, 2] = v
        return orc.hyena_rows(uu, k, D, method=2)[0]

    _close(run(alpha * a + beta * c), alpha * run(a) + beta * run(c), 1e-11, "linearity")


def pin_gating(orc):
    """Order 2, no short conv: scaling x0 or x1 by alpha scales y by alpha; y/x0 is gate-free."""
    rng = np.random.default_rng(10)
    L = 256
    u, k, D, _, _ = _rand_rows(rng, 1, 2, L, shortconv=False)
    y = orc.hyena_rows(u, k, D, method=1)[0]
    for j in (0, 1):
        uu = u.copy(); uu[0, j] *= -2.5
        _close(orc.hyena_rows(uu, k, D, method=1)[0], -2.5 * y, 1e-12, f"scale x{j}")
    # y / x0 equals the ungated long conv of x1*v
    conv = orc.causal_conv_direct(k[0, 0], D[0, 0], u[0, 1] * u[0, 2])
    _close(y, u[0, 0] * conv, 1e-12, "output gate")


def pin_order3_step_pairing(orc):
    """Order 3 with one step made the identity isolates the other step's pairing."""
    rng = np.random.default_rng(11)
    L = 64
    u, k, D, _, _ = _rand_rows(rng, 1, 3, L, shortconv=False)
    delta = np.zeros(L); delta[0] = 1.0
    # step 2 (gate x1, k[1], D[1]) is the identity: x1 = 1, k[1] = delta, D[1] = 0
    u1 = u.copy(); u1[0, 1] = 1.0
    k1 = k.copy(); k1[0, 1] = delta
    D1 = D.copy(); D1[0, 1] = 0.0
    want = u[0, 0] * orc.causal_conv_direct(k[0, 0], D[0, 0], u[0, 3] * u[0, 2])
    _close(orc.hyena_rows(u1, k1, D1, method=1)[0], want, 1e-12, "step 1 = (x2, k[0], D[0])")
    # step 1 (gate x2, k[0], D[0]) is the identity
    u2 = u.copy(); u2[0, 2] = 1.0
    k2 = k.copy(); k2[0, 0] = delta
    D2 = D.copy(); D2[0, 0] = 0.0
    want = u[0, 0] * orc.causal_conv_direct(k[0, 1], D[0, 1], u[0, 3] * u[0, 1])
    _close(orc.hyena_rows(u2, k2, D2, method=1)[0], want, 1e-12, "step 2 = (x1, k[1], D[1])")


def pin_shortconv_feeds_every_chunk(orc):
    """With taps (0, 0, c_j) the short conv is a per-chunk scale c_j + bias b_j."""
    rng = np.random.default_rng(12)
    L = 128
    u, k, D, _, _ = _rand_rows(rng, 1, 2, L, shortconv=False)
    c = np.array([1.5, -0.5, 2.0]); bias = np.array([0.25, -1.0, 0.5])
    w = np.zeros((1, 3, 3)); w[0, :, 2] = c
    y = orc.hyena_rows(u, k, D, w, bias[None], method=1)[0]
    us = u * c[None, :, None] + bias[None, :, None]
    _close(y, orc.hyena_rows(us, k, D, method=1)[0], 1e-12, "per-chunk scale")


# ------------------------------------------------- 2-D circular form ---
# [P5] 边界处理: the circular (periodic) convolution, no padding.
def pin_conv2d_circ_matches_numpy(orc):
    """Direct sum and FFT form against numpy's unpadded FFT2 product (library
    special case of circular convolution)."""
    rng = np.random.default_rng(21)
    for H, W in ((1, 8), (4, 4), (8, 16), (16, 8), (32, 32)):
        K = rng.standard_normal((H, W)); x = rng.standard_normal((H, W))
        ref = np.fft.ifft2(np.fft.fft2(K) * np.fft.fft2(x)).real + 0.7 * x
        _close(orc.conv2d_circ_direct(K, 0.7, x), ref, 1e-11, f"direct {H}x{W}")
        _close(orc.conv2d_circ_fft(K, 0.7, x), ref, 1e-11, f"fft {H}x{W}")


def pin_conv2d_circ_delta_and_shift(orc):
    """A delta at (0, 0) returns K + D delta; a cyclic shift of the input
    shifts the output by the same amount (both the direct and the FFT form)."""
    rng = np.random.default_rng(22)
    H, W = 8, 16
    K = rng.standard_normal((H, W))
    d = np.zeros((H, W)); d[0, 0] = 1.0
    want = K.copy(); want[0, 0] += 0.4
    for f in (orc.conv2d_circ_direct, orc.conv2d_circ_fft):
        _close(f(K, 0.4, d), want, 1e-12, "delta")
        x = rng.standard_normal((H, W))
        _close(f(K, 0.4, np.roll(x, (3, 5), axis=(0, 1))), np.roll(f(K, 0.4, x), (3, 5), axis=(0, 1)),
               1e-11, "shift")


def pin_conv2d_circ_without_wrap_is_linear(orc):
    """Kernel and input supported in the top-left quarter never wrap, so the
    circular form equals the zero-padded (non-circular) one; the whole
    operator too."""
    rng = np.random.default_rng(23)
    H, W = 16, 32
    K = np.zeros((H, W)); K[: H // 2, : W // 2] = rng.standard_normal((H // 2, W // 2))
    x = np.zeros((H, W)); x[: H // 2, : W // 2] = rng.standard_normal((H // 2, W // 2))
    _close(orc.conv2d_circ_direct(K, 0.3, x), orc.conv2d_direct(K, 0.3, x), 1e-12, "conv")
    u = np.zeros((2, 3, H, W)); u[:, :, : H // 2, : W // 2] = rng.standard_normal((2, 3, H // 2, W // 2))
    k = np.zeros((2, 1, H, W)); k[:, :, : H // 2, : W // 2] = rng.standard_normal((2, 1, H // 2, W // 2))
    D = rng.standard_normal((2, 1))
    _close(orc.hyena_rows(u, k, D, ndim=2, method=1, circular=True), orc.hyena_rows(u, k, D, ndim=2, method=1),
           1e-12, "operator")
    _close(orc.hyena_rows(u, k, D, ndim=2, method=2, circular=True), orc.hyena_rows(u, k, D, ndim=2, method=1),
           1e-11, "operator fft")


def pin_operator2d_circ_direct_equals_fft_and_numpy(orc):
    """The circular operator (order 2, full-support data that wraps): direct
    sums equal the FFT form, and both equal gating around numpy's circular
    FFT2 product."""
    rng = np.random.default_rng(25)
    H, W = 8, 16
    u = rng.standard_normal((3, 3, H, W)); k = rng.standard_normal((3, 1, H, W))
    D = rng.standard_normal((3, 1))
    yd = orc.hyena_rows(u, k, D, ndim=2, method=1, circular=True)
    yf = orc.hyena_rows(u, k, D, ndim=2, method=2, circular=True)
    _close(yd, yf, 1e-11, "direct vs fft")
    for r in range(3):
        w = u[r, 1] * u[r, 2]
        v = np.fft.ifft2(np.fft.fft2(k[r, 0]) * np.fft.fft2(w)).real + D[r, 0] * w
        _close(yd[r], u[r, 0] * v, 1e-11, "numpy composition")


def pin_operator2d_circ_wraps(orc):
    """With a kernel at the last row and column only, the circular operator
    differs from the padded one exactly by the wrapped terms: the padded form
    sees K[H-1][W-1] only at (H-1, W-1), the circular one at every output."""
    rng = np.random.default_rng(24)
    H, W = 8, 8
    K = np.zeros((H, W)); K[H - 1, W - 1] = 2.0
    x = rng.standard_normal((H, W))
    circ = orc.conv2d_circ_direct(K, 0.0, x)
    _close(circ, 2.0 * np.roll(x, (H - 1, W - 1), axis=(0, 1)), 1e-12, "wrapped shift")
    lin = orc.conv2d_direct(K, 0.0, x)
    want = np.zeros((H, W)); want[H - 1, W - 1] = 2.0 * x[0, 0]
    _close(lin, want, 1e-12, "padded")


# -------------------------------------------------------------- 3-D form ---
# [P5] 原生 ND 卷积 / 边界处理: N-D global convolution, zero padded per axis.
def _np_linear3(K, x):
    n = [2 * s for s in x.shape]
    ax = (0, 1, 2)
    y = np.fft.ifftn(np.fft.fftn(K, n, axes=ax) * np.fft.fftn(x, n, axes=ax), axes=ax).real
    return y[: x.shape[0], : x.shape[1], : x.shape[2]]


def pin_conv3d_matches_numpy(orc):
    """Direct sum and FFT form against numpy's zero-padded fftn product."""
    rng = np.random.default_rng(31)
    for shape in ((1, 4, 8), (4, 4, 4), (2, 8, 4), (8, 4, 16)):
        K = rng.standard_normal(shape); x = rng.standard_normal(shape)
        ref = _np_linear3(K, x) + 0.6 * x
        _close(orc.conv3d_direct(K, 0.6, x), ref, 1e-11, f"direct {shape}")
        _close(orc.conv3d_fft(K, 0.6, x), ref, 1e-11, f"fft {shape}")


def pin_conv3d_single_slice_is_2d(orc):
    """N1 = 1 reduces to the 2-D form, and the delta returns K + D delta."""
    rng = np.random.default_rng(32)
    K = rng.standard_normal((1, 8, 16)); x = rng.standard_normal((1, 8, 16))
    _close(orc.conv3d_direct(K, 0.2, x)[0], orc.conv2d_direct(K[0], 0.2, x[0]), 1e-12, "N1=1")
    K = rng.standard_normal((4, 4, 8))
    d = np.zeros((4, 4, 8)); d[0, 0, 0] = 1.0
    want = K.copy(); want[0, 0, 0] += 0.2
    _close(orc.conv3d_direct(K, 0.2, d), want, 1e-12, "delta direct")
    _close(orc.conv3d_fft(K, 0.2, d), want, 1e-12, "delta fft")


def pin_operator3d(orc):
    """The 3-D operator: direct equals FFT (orders 2 and 3), and one slice
    equals the 2-D operator."""
    rng = np.random.default_rng(33)
    for order in (2, 3):
        u = rng.standard_normal((2, order + 1, 2, 4, 8)); k = rng.standard_normal((2, order - 1, 2, 4, 8))
        D = rng.standard_normal((2, order - 1))
        _close(orc.hyena_rows3(u, k, D, method=1), orc.hyena_rows3(u, k, D, method=2), 1e-11, f"order {order}")
    u = rng.standard_normal((2, 3, 1, 8, 8)); k = rng.standard_normal((2, 1, 1, 8, 8)); D = rng.standard_normal((2, 1))
    _close(orc.hyena_rows3(u, k, D, method=1)[:, 0], orc.hyena_rows(u[:, :, 0], k[:, :, 0], D, ndim=2, method=1),
           1e-12, "N1=1 operator")


ALL_PINS = [v for n, v in sorted(globals().items()) if n.startswith("pin_")]
