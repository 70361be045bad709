"""Pins for the 0/1 Adam variant's CPU oracle (``oracle.zo_*``, readings Z1-Z7): checks against
things other than that oracle itself -- the 1-bit Adam oracle (independently pinned) through the
exact scaling identity that ties the two together, a case worked by hand, an independent exact
rational re-derivation, and the closed form of momentum SGD under the stale preconditioner when
the 1-bit messages are lossless.

Like ``oracle_pins``, the pins are plain functions so that the mutation test can run all of them
against copies of the oracle with a planted mistake.
"""
from __future__ import annotations

import json
import os
from fractions import Fraction as F

import numpy as np

import oracle
from exact import exact_zero_one_run, fr, r32, r32_sqrt

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _warm_state(d, W, seed):
    """A state at the freeze: two warm-up steps of the (pinned) 1-bit Adam oracle."""
    rng = np.random.default_rng(seed)
    x = rng.uniform(-0.05, 0.05, d).astype(np.float32)
    st = oracle.OracleState(x, W, 32, 0.9, 0.999, 1e-8)
    for _ in range(2):
        st.warmup_step((rng.standard_normal((W, d)) * 1e-2).astype(np.float32), 1e-3)
    return st.x, st.m, st.v


def pin01_hand_case():
    """The d=8, W=2, C=4, H=2, K=1 case worked by hand (tests/golden)."""
    with open(os.path.join(GOLDEN, "zero_one_hand_case_d8_w2.json")) as f:
        case = json.load(f)
    inp, exp = case["inputs"], case["expected"]
    st = oracle.ZeroOneState(np.array(inp["x"], np.float32), inp["W"], inp["C"], inp["H"],
                             inp["K"], inp["beta1"], inp["beta2"], inp["eps"])
    st.m = np.array(inp["m"], np.float32)
    st.v = np.array(inp["v"], np.float32)
    st.freeze()
    g = [np.array(a, np.float32) for a in inp["g"]]
    assert st.step(g[0], inp["lr"]) is None
    e1 = exp["after_step_1"]
    np.testing.assert_array_equal(st.m_w, np.array(e1["m_w"], np.float32))
    np.testing.assert_array_equal(st.u_w, np.array(e1["u_w"], np.float32))
    np.testing.assert_array_equal(st.local_model(0), np.array(e1["local_model_0"], np.float32))
    out = st.step(g[1], inp["lr"])
    e2 = exp["sync_after_step_2"]
    assert out is not None and out["refresh"]
    np.testing.assert_array_equal(out["s"], np.array(e2["s"], np.float32))
    np.testing.assert_array_equal(out["bits_w"], np.array(e2["bits_w"], np.uint32))
    np.testing.assert_array_equal(st.e_w, np.array(e2["e_w"], np.float32))
    np.testing.assert_array_equal(out["S"], np.array(e2["S"], np.float32))
    np.testing.assert_array_equal(out["bits_s"], np.array(e2["bits_s"], np.uint32))
    np.testing.assert_array_equal(st.e_s, np.array(e2["e_s"], np.float32))
    np.testing.assert_array_equal(st.x, np.array(e2["x"], np.float32))
    np.testing.assert_array_equal(out["mbar"], np.array(e2["mbar"], np.float32))
    np.testing.assert_array_equal(st.v, np.array(e2["v"], np.float32))
    assert not st.u_w.any()
    assert st.step(g[2], inp["lr"]) is None
    e3 = exp["after_step_3"]
    np.testing.assert_array_equal(st.m_w, np.array(e3["m_w"], np.float32))
    np.testing.assert_array_equal(st.u_w, np.array(e3["u_w"], np.float32))


def pin01_reduces_to_onebit_adam():
    """With a synchronisation every step (H = 1), the variance frozen (K = 0) and a power-of-two
    learning rate, every quantity of the variant is lr times its 1-bit Adam counterpart, exactly
    (scaling by a power of two commutes with every rounding), so both give the same parameters
    and messages bit for bit, step after step, and the momentum estimate is 1-bit Adam's m."""
    d, W, C = 150, 3, 64                        # a ragged last chunk of 22
    x, m, v = _warm_state(d, W, 11)
    lr = 2.0 ** -9
    a = oracle.OracleState(x, W, C, 0.9, 0.999, 1e-8)
    a.m, a.v = m.copy(), v.copy()
    a.freeze()
    b = oracle.ZeroOneState(x, W, C, 1, 0, 0.9, 0.999, 1e-8)
    b.m, b.v = m.copy(), v.copy()
    b.freeze()
    rng = np.random.default_rng(12)
    for _ in range(6):
        g = (rng.standard_normal((W, d)) * 1e-2).astype(np.float32)
        ra = a.compressed_step(g, lr)
        rb = b.step(g, lr)
        np.testing.assert_array_equal(rb["bits_w"], ra["bits_w"])
        np.testing.assert_array_equal(rb["bits_s"], ra["bits_s"])
        np.testing.assert_array_equal(rb["s"], np.float32(lr) * ra["s"])
        np.testing.assert_array_equal(rb["S"], np.float32(lr) * ra["S"])
        np.testing.assert_array_equal(b.e_w, np.float32(lr) * a.e_w)
        np.testing.assert_array_equal(b.e_s, np.float32(lr) * a.e_s)
        np.testing.assert_array_equal(rb["mbar"], a.m)
        np.testing.assert_array_equal(b.x.view(np.uint32), a.x.view(np.uint32))
    np.testing.assert_array_equal(b.v, a.v)


def pin01_exact_rederivation():
    """Bit-for-bit agreement with an independent exact-rational re-derivation (every fp32
    operation the exact result rounded once, norms summed exactly) over local steps,
    synchronisations, variance refreshes and a ragged chunk, with learning rates that are not
    powers of two."""
    cases = ((37, 2, 16, 3, 1), (24, 3, 24, 2, 2), (40, 1, 8, 1, 0))
    for n, (d, W, C, H, K) in enumerate(cases):
        x, m, v = _warm_state(d, W, 20 + n)
        rng = np.random.default_rng(30 + n)
        steps = 2 * H + 1
        gs = [(rng.standard_normal((W, d)) * 1e-2).astype(np.float32) for _ in range(steps)]
        lrs = [float(np.float32(0.3 + 0.1 * t)) for t in range(steps)]
        ref = exact_zero_one_run(x, m, v, gs, lrs, C, H, K, 0.9, 0.999, 1e-8)
        st = oracle.ZeroOneState(x, W, C, H, K, 0.9, 0.999, 1e-8)
        st.m, st.v = m.copy(), v.copy()
        st.freeze()
        syncs = []
        for g, lr in zip(gs, lrs):
            out = st.step(g, lr)
            if out is not None:
                syncs.append(out)
        assert len(syncs) == len(ref["syncs"])
        for got, want in zip(syncs, ref["syncs"]):
            np.testing.assert_array_equal(got["s"], want["s"])
            np.testing.assert_array_equal(got["S"], want["S"])
            np.testing.assert_array_equal(got["mbar"], want["mbar"])
            w = np.asarray(want["bits_w"])
            for r in range(W):
                bits = np.unpackbits(got["bits_w"][r].view(np.uint8), bitorder="little")[:d]
                np.testing.assert_array_equal(bits.astype(bool), w[r])
            bits = np.unpackbits(got["bits_s"].view(np.uint8), bitorder="little")[:d]
            np.testing.assert_array_equal(bits.astype(bool), np.asarray(want["bits_s"]))
            assert got["refresh"] == want["refresh"]
        for nm in ("x", "v", "m_w", "u_w", "e_w", "e_s"):
            np.testing.assert_array_equal(getattr(st, nm), ref[nm], err_msg=nm)


def pin01_lossless_interval_is_momentum_sgd():
    """One worker, constant gradient magnitude with fixed signs and a momentum of the same
    signs: every element of a chunk then has the same |u|, so the 1-bit messages are lossless
    (zero residuals, ubar = u exactly) and the synchronised step must be momentum SGD under the
    stale preconditioner over the interval -- x_H = x_0 - sum_t lr_t * m_t / (sqrt(v) + eps) and
    mbar = sum_t lr_t * m_t / sum_t lr_t, both within a few roundings of the closed form -- and
    the local model after H - 1 local steps must follow the same closed form over those
    steps."""
    d, C, H = 64, 32, 4
    rng = np.random.default_rng(5)
    sgn = np.where(rng.random(d) < 0.5, -1.0, 1.0).astype(np.float32)
    v = (rng.uniform(0.5, 2.0, d) ** 2).astype(np.float32) * np.float32(1e-4)
    x0 = rng.uniform(-0.05, 0.05, d).astype(np.float32)
    m0, gmag, b1, eps = 0.03, 0.02, 0.9, 1e-8
    lrs = [0.1, 0.25, 0.05, 0.2]
    st = oracle.ZeroOneState(x0, 1, C, H, 0, b1, 0.999, eps)
    st.m = (np.float32(m0) * sgn).astype(np.float32)
    st.v = v.copy()
    st.freeze()
    mt, usum, gam = F(m0), F(0), F(0)
    for t, lr in enumerate(lrs, start=1):
        if t == H:
            before, usum_before = st.local_model(0), usum
        mt = F(b1) * mt + (1 - F(b1)) * F(gmag)
        usum += F(lr) * mt
        gam += F(lr)
        out = st.step((np.float32(gmag) * sgn).reshape(1, d), lr)
    assert out is not None and not st.e_w.any() and not st.e_s.any()
    den = np.sqrt(v.astype(np.float64)) + eps
    x_ref = x0.astype(np.float64) - float(usum) * sgn / den
    tol = 16 * np.abs(x_ref) * 2.0 ** -24 + 1e-12
    assert np.all(np.abs(st.x - x_ref) <= tol), np.max(np.abs(st.x - x_ref) / tol)
    m_ref = float(usum / gam) * sgn
    assert np.all(np.abs(out["mbar"] - m_ref) <= 16 * np.abs(m_ref) * 2.0 ** -24)
    # the local model after H - 1 steps: x0 - u/(sqrt(v)+eps), the same closed form
    x_before = x0.astype(np.float64) - float(usum_before) * sgn / den
    assert np.all(np.abs(before - x_before) <= 16 * np.abs(x_before) * 2.0 ** -24 + 1e-12)


def pin01_variance_refresh():
    """A refresh is v = beta2*v + (1-beta2)*mbar^2 with the step taken on the old v: with
    beta2 = 1/2 and power-of-two magnitudes everything is exact, so the refreshed v and the
    parameters can be written down; without the refresh (K = 0) v stays bitwise frozen."""
    d, C = 32, 32
    for K in (0, 1):
        st = oracle.ZeroOneState(np.zeros(d, np.float32), 1, C, 1, K, 0.5, 0.5, 0.0)
        st.m = np.zeros(d, np.float32)
        st.v = np.full(d, 4.0, np.float32)
        st.freeze()
        g = np.full((1, d), 8.0, np.float32)          # m = 4, u = lr*m = 2 (lr = 1/2)
        out = st.step(g, 0.5)
        np.testing.assert_array_equal(out["S"], np.float32([2.0]))
        np.testing.assert_array_equal(st.x, np.full(d, -1.0, np.float32))   # 0 - 2/sqrt(4)
        np.testing.assert_array_equal(out["mbar"], np.full(d, 4.0, np.float32))  # 2 / (1/2)
        want = 4.0 / 2 + 16.0 / 2 if K else 4.0
        np.testing.assert_array_equal(st.v, np.full(d, want, np.float32))


def pin01_schedule():
    """Synchronisations fall on every H-th step and refreshes on every K-th synchronisation;
    Gamma restarts after each synchronisation (checked through mbar = ubar / Gamma on a
    lossless case with lr = 1: Gamma = H)."""
    d, C, H, K = 32, 32, 3, 2
    st = oracle.ZeroOneState(np.zeros(d, np.float32), 1, C, H, K, 0.5, 0.5, 0.0)
    st.m = np.zeros(d, np.float32)
    st.v = np.ones(d, np.float32)
    st.freeze()
    pattern = []
    for t in range(1, 13):
        out = st.step(np.full((1, d), 2.0, np.float32), 1.0)
        pattern.append(None if out is None else bool(out["refresh"]))
        if out is not None:
            ubar = out["S"][0]
            np.testing.assert_array_equal(out["mbar"], np.full(d, ubar / np.float32(H), np.float32))
    assert pattern == [None, None, False, None, None, True, None, None, False, None, None, True]


PINS01 = [pin01_hand_case, pin01_reduces_to_onebit_adam, pin01_exact_rederivation,
          pin01_lossless_interval_is_momentum_sgd, pin01_variance_refresh, pin01_schedule]
