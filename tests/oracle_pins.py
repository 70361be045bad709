"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each ``pin_*`` raises AssertionError when the oracle disagrees with what the method's
definition, the mathematics or a library routine fixes: a hand-derived worked case, numpy's own
bit packing, exact rational arithmetic, closed forms (equal-scale averages, constant-gradient
Adam), invariants (error-feedback identity, norm preservation, telescoping sums, worker
permutation, chunk independence, frozen variance) and degenerate cases (W = 1, zero chunks,
NaN, the ragged tail chunk). The pins are plain functions so that the mutation test can run all
of them against copies of the oracle with a planted mistake.
"""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction as F

import numpy as np

import oracle
from exact import exact_compressed_step, fr, r32, r32_sqrt, ulp32

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _numpy_pack(x: np.ndarray) -> np.ndarray:
    """Reference packing with numpy: bit = x >= 0 (NaN -> 0), little-endian bit order."""
    bits = np.asarray(x >= 0, dtype=np.uint8)
    nbytes = ((x.size + 31) // 32) * 4
    b = np.packbits(bits, bitorder="little")
    b = np.concatenate([b, np.zeros(nbytes - b.size, dtype=np.uint8)])
    return b.view("<u4")


def _numpy_unpack(words: np.ndarray, n: int) -> np.ndarray:
    return np.unpackbits(words.astype("<u4").view(np.uint8), bitorder="little")[:n].astype(bool)


def _fresh(d, W):
    return (np.zeros(d, np.float32), np.zeros(d, np.float32), np.ones(d, np.float32),
            np.zeros((W, d), np.float32), np.zeros(d, np.float32))


# ----------------------------------------------------------------------------------------------

def pin_hand_case():
    """The d=8, W=2, C=4 step worked by hand (tests/golden/hand_case_d8_w2.json)."""
    with open(os.path.join(GOLDEN, "hand_case_d8_w2.json")) as f:
        case = json.load(f)
    inp, exp = case["inputs"], case["expected"]
    g = np.array(inp["g"], dtype=np.float32)
    x = np.array(inp["x"], dtype=np.float32)
    m = np.array(inp["m"], dtype=np.float32)
    v = np.array(inp["v"], dtype=np.float32)
    e_w = np.zeros_like(g)
    e_s = np.zeros_like(x)
    C = inp["C"]
    s, bits_w = oracle.worker(m, g, e_w, C, inp["beta1"])
    np.testing.assert_array_equal(s, np.array(exp["s"], np.float32))
    np.testing.assert_array_equal(bits_w, np.array(exp["bits_w"], np.uint32))
    np.testing.assert_array_equal(e_w, np.array(exp["e_w"], np.float32))
    S, bits_s, z, inexact = oracle.server(s, bits_w, e_s, C)
    assert inexact == 0
    np.testing.assert_array_equal(z, np.array(exp["z"], np.float32))
    S_exp = np.array([r32_sqrt(F(str(q))) for q in exp["S_exact_squares"]], np.float32)
    np.testing.assert_array_equal(S, S_exp)
    np.testing.assert_array_equal(bits_s, np.array(exp["bits_s"], np.uint32))
    S0, S1 = S_exp
    f = np.float32
    es_exp = np.array([S0 - f(0.5), f(2.5) - S0, f(2.5) - S0, S0 - f(0.5),
                       f(1) - S1, -S1, f(1) - S1, -S1], np.float32)
    np.testing.assert_array_equal(e_s, es_exp)
    oracle.apply(bits_s, S, v, m, x, C, inp["eps"], inp["lr"])
    m_exp = np.array([-S0, S0, S0, -S0, S1, S1, S1, S1], np.float32)
    np.testing.assert_array_equal(m, m_exp)
    np.testing.assert_array_equal(x, -m_exp)


def pin_pack_matches_numpy():
    """Packing equals numpy.packbits(x >= 0, bitorder='little') for ragged n, +-0 and NaN."""
    rng = np.random.default_rng(1)
    for n in (1, 31, 32, 33, 1000, 4097):
        x = rng.standard_normal(n).astype(np.float32)
        x[rng.random(n) < 0.05] = 0.0
        x[rng.random(n) < 0.05] = -0.0
        x[rng.random(n) < 0.02] = np.nan
        np.testing.assert_array_equal(oracle.pack(x), _numpy_pack(x))


def pin_unpack_matches_numpy():
    """Decompression equals +-scales[i // C] with numpy.unpackbits (little bit order)."""
    rng = np.random.default_rng(2)
    for n, C in ((777, 64), (100, 100), (4096, 32), (65, 1000)):
        words = rng.integers(0, 2**32, size=(n + 31) // 32, dtype=np.uint64).astype(np.uint32)
        scales = rng.random((n + C - 1) // C).astype(np.float32)
        bits = _numpy_unpack(words, n)
        sc = scales[np.arange(n) // C]
        np.testing.assert_array_equal(oracle.unpack(words, scales, n, C), np.where(bits, sc, -sc))


def pin_round_trip_exhaustive():
    """unpack(pack(b)) == b for every sign pattern of length <= 12 (unit scale)."""
    for n in range(1, 13):
        pats = ((np.arange(2 ** n)[:, None] >> np.arange(n)) & 1).astype(bool)
        for b in pats:
            x = np.where(b, 1.0, -1.0).astype(np.float32)
            words = oracle.pack(x)
            assert words.size == 1
            assert int(words[0]) >> n == 0, "padding bits must be 0"
            np.testing.assert_array_equal(oracle.unpack(words, np.ones(1, np.float32), n, 32), x)


def pin_scale_and_error_feedback():
    """With beta1 = 0 and zero state, x_w = g_w exactly. Then per chunk: the scale is the
    correctly rounded sqrt of the exact mean square (within 1 ulp, fp64 summation); the sign
    plane is numpy's; the residual is x - (+-s) rounded once (exact identity); the decompressed
    chunk keeps the l2 norm; inside the Sterbenz range the residual adds back to x exactly."""
    rng = np.random.default_rng(3)
    for d, W, C in ((96, 3, 32), (200, 2, 64), (1000, 1, 1000)):
        g = (rng.standard_normal((W, d)) * 10.0 ** rng.uniform(-3, 1, (W, 1))).astype(np.float32)
        x_exp = g.copy()
        m, _, _, e_w, _ = _fresh(d, W)
        s, bits = oracle.worker(m, g, e_w, C, 0.0)
        for w in range(W):
            np.testing.assert_array_equal(bits[w], _numpy_pack(x_exp[w]))
            for k in range((d + C - 1) // C):
                lo, hi = k * C, min(d, (k + 1) * C)
                xs = x_exp[w, lo:hi]
                exact = sum((F(float(t)) ** 2 for t in xs), F(0)) / (hi - lo)
                s_true = r32_sqrt(exact)
                assert abs(float(s[w, k]) - float(s_true)) <= ulp32(s_true), (s[w, k], s_true)
                q = np.where(xs >= 0, s[w, k], -s[w, k]).astype(np.float32)
                # residual: one correctly rounded subtraction
                e_exp = np.array([r32(fr(a) - fr(b)) for a, b in zip(xs, q)], np.float32)
                np.testing.assert_array_equal(e_w[w, lo:hi], e_exp)
                # norm preservation of the decompressed chunk
                n_q = math.sqrt(math.fsum(float(t) ** 2 for t in q))
                n_x = math.sqrt(math.fsum(float(t) ** 2 for t in xs))
                assert abs(n_q - n_x) <= 2 ** -22 * n_x
                # Sterbenz range: e + q == x exactly
                st = (np.abs(xs) >= s[w, k] / 2) & (np.abs(xs) <= 2 * s[w, k])
                np.testing.assert_array_equal((e_w[w, lo:hi] + q)[st], xs[st])


def pin_tail_chunk_true_length():
    """The last, shorter chunk is scaled by its own length, not by C."""
    d, C = 100, 64
    g = np.ones((1, d), np.float32)
    g[0, 64:] = 3.0
    m, _, _, e_w, _ = _fresh(d, 1)
    s, _ = oracle.worker(m, g, e_w, C, 0.0)
    np.testing.assert_array_equal(s, np.array([[1.0, 3.0]], np.float32))
    np.testing.assert_array_equal(e_w, np.zeros((1, d), np.float32))


def pin_zero_chunk_and_nan():
    """An all-zero chunk has scale 0, all bits 1 (0 >= 0) and residual +0; NaN takes bit 0."""
    d, C = 64, 32
    g = np.zeros((1, d), np.float32)
    g[0, 32:] = np.linspace(-1, 1, 32, dtype=np.float32)
    g[0, 40] = np.nan
    m, _, _, e_w, _ = _fresh(d, 1)
    s, bits = oracle.worker(m, g, e_w, C, 0.0)
    assert s[0, 0] == 0.0
    assert int(bits[0, 0]) == 0xFFFFFFFF
    assert not np.signbit(e_w[0, :32]).any() and (e_w[0, :32] == 0).all()
    assert (int(bits[0, 1]) >> 8) & 1 == 0
    assert np.isnan(s[0, 1])


def pin_w1_reduces_to_scaled_sign():
    """W = 1 with zero residuals: the server's average is the worker's own message, so its
    bits equal the worker's, its scale equals the worker's (exactly for power-of-two scales),
    its residual is zero, and m = s * sign(beta1*m + (1-beta1)*g): scaled sign-SGD with momentum
    under the frozen preconditioner."""
    rng = np.random.default_rng(4)
    d, C = 256, 64
    mag = np.repeat(2.0 ** rng.integers(-6, 2, size=d // C), C).astype(np.float32)
    g = (np.where(rng.random(d) < 0.5, -1.0, 1.0) * mag).astype(np.float32)[None, :]
    x0 = rng.uniform(-0.05, 0.05, d).astype(np.float32)
    x, m, v, e_w, e_s = x0.copy(), *(_fresh(d, 1)[1:])
    v = rng.uniform(0.5, 2.0, d).astype(np.float32)
    out = oracle.compressed_step(x, m, v, e_w, e_s, g, C, 0.0, 1e-8, 1e-3)
    np.testing.assert_array_equal(out["bits_s"], out["bits_w"][0])
    np.testing.assert_array_equal(out["S"], out["s"][0])
    np.testing.assert_array_equal(out["S"], mag[::C])
    np.testing.assert_array_equal(e_s, np.zeros(d, np.float32))
    np.testing.assert_array_equal(m, g[0])
    np.testing.assert_array_equal(e_w, np.zeros((1, d), np.float32))


def pin_equal_scales_closed_form():
    """Workers whose chunk values all have magnitude c (a power of two) have scale c, and the
    server's average of element i is c * (2 * #positive - W) / W rounded once."""
    rng = np.random.default_rng(5)
    W, d, C = 5, 96, 32
    c = np.repeat(2.0 ** rng.integers(-4, 3, size=d // C), C)
    sgn = np.where(rng.random((W, d)) < 0.5, -1.0, 1.0)
    g = (sgn * c).astype(np.float32)
    m, _, _, e_w, e_s = _fresh(d, W)
    s, bits = oracle.worker(m, g, e_w, C, 0.0)
    np.testing.assert_array_equal(s, np.tile(c[::C].astype(np.float32), (W, 1)))
    _, _, z, _ = oracle.server(s, bits, e_s, C)
    npos = (sgn > 0).sum(axis=0)
    z_exp = np.array([r32(F(float(ci)) * (2 * int(p) - W) / W) for ci, p in zip(c, npos)],
                     np.float32)
    np.testing.assert_array_equal(z, z_exp)


def pin_worker_permutation_invariance():
    """Reordering the workers leaves every server output bit-identical (exact fp64 sum)."""
    rng = np.random.default_rng(6)
    W, d, C = 6, 320, 64
    g = (rng.standard_normal((W, d)) * 1e-2).astype(np.float32)
    xv = rng.uniform(-0.05, 0.05, d).astype(np.float32)
    v = rng.uniform(1e-6, 1e-4, d).astype(np.float32)
    m0 = (rng.standard_normal(d) * 1e-3).astype(np.float32)
    res = []
    for perm in (np.arange(W), rng.permutation(W), rng.permutation(W)):
        x, m = xv.copy(), m0.copy()
        e_w = np.zeros((W, d), np.float32)
        e_s = np.zeros(d, np.float32)
        out = oracle.compressed_step(x, m, v, e_w, e_s, np.ascontiguousarray(g[perm]), C,
                                     0.9, 1e-8, 1e-4)
        assert out["inexact"] == 0
        res.append((x, m, e_s, out["S"], out["bits_s"]))
    for r in res[1:]:
        for a, b in zip(res[0], r):
            np.testing.assert_array_equal(a, b)


def pin_chunk_independence():
    """Changing the inputs of one chunk changes no output of any other chunk."""
    rng = np.random.default_rng(7)
    W, d, C = 3, 300, 100
    g = (rng.standard_normal((W, d)) * 1e-2).astype(np.float32)
    g2 = g.copy()
    g2[:, 100:200] = (rng.standard_normal((W, 100)) * 5.0).astype(np.float32)
    outs = []
    for gg in (g, g2):
        x = np.full(d, 0.01, np.float32)
        m = np.zeros(d, np.float32)
        v = np.ones(d, np.float32)
        e_w = np.zeros((W, d), np.float32)
        e_s = np.zeros(d, np.float32)
        for _ in range(3):
            out = oracle.compressed_step(x, m, v, e_w, e_s, gg, C, 0.9, 1e-8, 1e-2)
        outs.append((x.copy(), m.copy(), e_w.copy(), e_s.copy(), out["s"], out["S"]))
    keep = np.r_[0:100, 200:300]
    for a, b in zip(outs[0], outs[1]):
        if a.ndim == 1 and a.size == d:
            np.testing.assert_array_equal(a[keep], b[keep])
        elif a.ndim == 2 and a.shape[1] == d:
            np.testing.assert_array_equal(a[:, keep], b[:, keep])
        elif a.ndim == 2:
            np.testing.assert_array_equal(a[:, [0, 2]], b[:, [0, 2]])
        else:
            np.testing.assert_array_equal(a[[0, 2]], b[[0, 2]])
    assert not np.array_equal(outs[0][0][100:200], outs[1][0][100:200])


def pin_error_feedback_telescopes():
    """Error feedback loses nothing over time: for every worker element the messages sent over
    T steps sum to the inputs compressed minus the final residual, sum_t q_t = sum_t u_t - e_T
    (u_t = g_t when beta1 = 0), up to one rounding per step; the same holds on the server with
    y_t the average of the workers' decompressed messages."""
    rng = np.random.default_rng(8)
    W, d, C, T = 4, 256, 64, 25
    m = np.zeros(d, np.float32)
    e_w = np.zeros((W, d), np.float32)
    e_s = np.zeros(d, np.float32)
    sum_q = np.zeros((W, d))
    sum_u = np.zeros((W, d))
    sum_Q = np.zeros(d)
    sum_y = np.zeros(d)
    bound_w = np.zeros((W, d))
    bound_s = np.zeros(d)
    for _ in range(T):
        g = (rng.standard_normal((W, d)) * 1e-2).astype(np.float32)
        s, bits = oracle.worker(m, g, e_w, C, 0.0)
        q = np.stack([oracle.unpack(bits[w], s[w], d, C) for w in range(W)]).astype(np.float64)
        sum_q += q
        sum_u += g
        y = q.mean(axis=0)
        sum_y += y
        bound_w += 2 * np.abs(q) * 2.0 ** -24 + np.abs(g) * 2.0 ** -23
        S, bits_s, z, _ = oracle.server(s, bits, e_s, C)
        Q = oracle.unpack(bits_s, S, d, C).astype(np.float64)
        sum_Q += Q
        bound_s += 4 * np.abs(Q) * 2.0 ** -24 + np.abs(y) * 2.0 ** -23
    assert (np.abs(sum_q - (sum_u - e_w)) <= bound_w + 1e-30).all()
    assert (np.abs(sum_Q - (sum_y - e_s)) <= bound_s + 1e-30).all()


def pin_exact_rederivation():
    """Brute force on tiny inputs: an exact-rational re-derivation of the whole step (every
    fp32 operation rounded once from the exact value, exact norms, correctly rounded square
    roots) agrees with the oracle: sign planes bit for bit except where |x| < 1e-6 * scale,
    scales within 1 ulp, and every other output within the ulps a 1-ulp scale difference moves."""
    rng = np.random.default_rng(9)
    cases = 0
    for d in (8, 40, 64):
        for W in (1, 2, 3, 4):
            for C in sorted({32, d, 8}):
                x = rng.uniform(-0.05, 0.05, d).astype(np.float32)
                m = (rng.standard_normal(d) * 1e-2).astype(np.float32)
                v = rng.uniform(1e-5, 1e-3, d).astype(np.float32)
                e_w = (rng.standard_normal((W, d)) * 1e-3).astype(np.float32)
                e_s = (rng.standard_normal(d) * 1e-3).astype(np.float32)
                g = (rng.standard_normal((W, d)) * 1e-2).astype(np.float32)
                ex = exact_compressed_step(x, m, v, e_w, e_s, g, C, 0.9, 1e-8, 1e-4)
                xo, mo, ewo, eso = x.copy(), m.copy(), e_w.copy(), e_s.copy()
                out = oracle.compressed_step(xo, mo, v, ewo, eso, g, C, 0.9, 1e-8, 1e-4)
                nch = (d + C - 1) // C
                sc_w = np.repeat(ex["s"], C, axis=1)[:, :d]
                tie = np.abs(ex["xw"]) < 1e-6 * sc_w
                bits_o = np.stack([_numpy_unpack(out["bits_w"][w], d) for w in range(W)])
                assert ((bits_o == ex["bits_w"]) | tie).all()
                assert (np.abs(out["s"] - ex["s"]) <= np.vectorize(ulp32)(ex["s"])).all()
                assert (np.abs(ewo - ex["e_w"]) <= 2 * np.vectorize(ulp32)(sc_w)).all()
                sc_s = np.repeat(ex["S"], C)[:d]
                assert (np.abs(out["S"] - ex["S"]) <= 2 * np.vectorize(ulp32)(ex["S"])).all()
                tie_s = np.abs(ex["z"]) < 1e-6 * sc_s
                assert ((_numpy_unpack(out["bits_s"], d) == ex["bits_s"]) | tie_s).all()
                tol_s = 4 * np.vectorize(ulp32)(sc_s)
                assert (np.abs(eso - ex["e_s"]) <= tol_s).all()
                assert (np.abs(mo - ex["m"]) <= tol_s).all()
                tol_x = 2 * np.vectorize(ulp32)(ex["x"]) + 1e-4 * tol_s / np.sqrt(v)
                assert (np.abs(xo - ex["x"]) <= tol_x).all()
                assert nch == ex["S"].size
                cases += 1
    assert cases == 32


def pin_frozen_variance():
    """Compressed steps never write the frozen variance."""
    rng = np.random.default_rng(10)
    W, d, C = 2, 128, 64
    st = oracle.OracleState(rng.uniform(-0.05, 0.05, d), W, C)
    for _ in range(3):
        st.warmup_step((rng.standard_normal((W, d)) * 1e-2).astype(np.float32), 1e-3)
    st.freeze()
    v0 = st.v.copy()
    for _ in range(4):
        st.compressed_step((rng.standard_normal((W, d)) * 1e-2).astype(np.float32), 1e-3)
    np.testing.assert_array_equal(st.v.view(np.uint32), v0.view(np.uint32))


def pin_warmup_constant_gradient_closed_form():
    """Plain Adam without bias correction under a constant averaged gradient c:
    m_T = c (1 - beta1^T), v_T = c^2 (1 - beta2^T), x_T = x_0 - lr sum_t m_t / (sqrt(v_t) + eps).
    The workers' gradients are c +- delta in pairs, so their average is exactly c."""
    W, d, T = 4, 64, 30
    rng = np.random.default_rng(11)
    c = (rng.standard_normal(d) * 1e-2).astype(np.float32)
    delta = np.float32(2.0 ** -12)
    g = np.stack([c + delta, c - delta, c + 2 * delta, c - 2 * delta]).astype(np.float32)
    gbar = g.astype(np.float64).mean(axis=0)
    b1, b2, eps, lr = 0.9, 0.999, 1e-8, 1e-3
    x0 = rng.uniform(-0.05, 0.05, d).astype(np.float32)
    st = oracle.OracleState(x0, W, 64, b1, b2, eps)
    for _ in range(T):
        st.warmup_step(g, lr)
    b1f, b2f = float(np.float32(b1)), float(np.float32(b2))
    m_T = gbar * (1 - b1f ** T)
    v_T = gbar ** 2 * (1 - b2f ** T)
    upd = sum(lr * gbar * (1 - b1f ** t) / (np.sqrt(gbar ** 2 * (1 - b2f ** t)) + eps)
              for t in range(1, T + 1))
    np.testing.assert_allclose(st.m, m_T, rtol=2e-5)
    np.testing.assert_allclose(st.v, v_T, rtol=2e-5)
    np.testing.assert_allclose(st.x - x0.astype(np.float64), -upd, rtol=1e-4, atol=1e-9)


def pin_server_exactness_report():
    """The server reports a chunk whose worker scales are too far apart for an exact fp64
    sum, and reports none for comparable scales."""
    W, d, C = 2, 64, 32
    s = np.array([[1.0, 1.0], [2.0 ** -40, 0.75]], np.float32)
    bits = np.zeros((W, 2), np.uint32)
    _, _, _, inexact = oracle.server(s, bits, np.zeros(d, np.float32), C)
    assert inexact == 1


PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
