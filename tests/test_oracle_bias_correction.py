"""The optional bias-corrected warm-up of the oracle (reading B1, oracle/bias_corrected_oracle.c)
against closed forms: Adam with bias correction under a constant gradient steps by
lr * g / (|g| + eps) from its very first step; the stored moments stay those of the uncorrected
warm-up; the freeze divides them by the corrections of the last step; the corrections are
1 - beta^t. Planted mistakes in copies of the file must each fail one of these pins."""
import os
import subprocess
from fractions import Fraction as F

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(oracle.__file__)
SRCBC = os.path.join(HERE, "bias_corrected_oracle.c")


def pin_bc_constant_gradient():
    """Every worker sends the same constant gradient g: m_t = (1 - b1^t) g and
    v_t = (1 - b2^t) g^2 exactly in real arithmetic, so each corrected step moves x by
    lr * g / (|g| + eps); after t steps x = x0 - t * lr * g / (|g| + eps) within the
    steps' roundings."""
    d, W, T, lr, eps = 96, 3, 12, 1e-3, 1e-8
    rng = np.random.default_rng(3)
    g1 = (rng.standard_normal(d) * 1e-2).astype(np.float32)
    g = np.ascontiguousarray(np.broadcast_to(g1, (W, d)), dtype=np.float32)
    x0 = rng.uniform(-0.05, 0.05, d).astype(np.float32)
    st = oracle.OracleState(x0, W, 32, 0.9, 0.999, eps, bias_correction=True)
    step = lr * g1.astype(np.float64) / (np.abs(g1.astype(np.float64)) + eps)
    for t in range(1, T + 1):
        st.warmup_step(g, lr)
        ref = x0.astype(np.float64) - t * step
        err = np.abs(st.x - ref)
        assert np.all(err <= 2e-6 * np.abs(step) * t + 4 * t * np.abs(ref) * 2.0 ** -24), t


def pin_bc_first_step_exact():
    """Step 1 from m = v = 0: the update is lr * (omb1 g / c1) / (sqrt(omb2 g^2 / c2) + eps)
    with every operation rounded once; checked against exact rationals rounded the same way
    (c1 = 1 - b1 and c2 = 1 - b2 in fp32)."""
    from exact import fr, r32, r32_sqrt
    d, lr, eps = 40, 1e-3, 1e-8
    rng = np.random.default_rng(4)
    g = (rng.standard_normal((1, d)) * 1e-2).astype(np.float32)
    x0 = rng.uniform(-0.05, 0.05, d).astype(np.float32)
    st = oracle.OracleState(x0, 1, 32, 0.9, 0.999, eps, bias_correction=True)
    st.warmup_step(g, lr)
    b1, b2 = fr(0.9), fr(0.999)
    c1, c2 = r32(1 - b1), r32(1 - b2)
    for i in range(d):
        m = r32(fr(r32(b1 * 0)) + fr(r32(fr(c1) * fr(g[0, i]))))
        v = r32(fr(r32(b2 * 0)) + fr(r32(fr(c2) * fr(r32(fr(g[0, i]) ** 2)))))
        mh, vh = r32(fr(m) / fr(c1)), r32(fr(v) / fr(c2))
        den = r32(fr(r32_sqrt(fr(vh))) + fr(eps))
        x = r32(fr(x0[i]) - fr(r32(fr(lr) * fr(r32(fr(mh) / fr(den))))))
        assert st.x[i] == x and st.m[i] == m and st.v[i] == v, i


def pin_bc_moments_and_freeze():
    """The correction changes the steps only: m and v equal the uncorrected warm-up's bit for
    bit; the freeze then continues from m / c1_T and v / c2_T (numpy's IEEE division)."""
    d, W, T = 200, 4, 7
    rng = np.random.default_rng(5)
    gs = [(rng.standard_normal((W, d)) * 1e-2).astype(np.float32) for _ in range(T)]
    x0 = rng.uniform(-0.05, 0.05, d).astype(np.float32)
    a = oracle.OracleState(x0, W, 64, 0.9, 0.999, 1e-8, bias_correction=True)
    b = oracle.OracleState(x0, W, 64, 0.9, 0.999, 1e-8)
    for g in gs:
        a.warmup_step(g, 1e-3)
        b.warmup_step(g, 1e-3)
    np.testing.assert_array_equal(a.m, b.m)
    np.testing.assert_array_equal(a.v, b.v)
    assert not np.array_equal(a.x, b.x)
    c1, c2 = oracle.bias_corrections(0.9, 0.999, T)
    a.freeze()
    np.testing.assert_array_equal(a.m, b.m / np.float32(c1))
    np.testing.assert_array_equal(a.v, b.v / np.float32(c2))


def pin_bc_corrections():
    """c_t = 1 - beta^t correctly rounded to fp32 (exact rationals), and exact for beta = 1/2."""
    from exact import r32
    for beta in (0.9, 0.999, 0.5):
        bf = F(float(np.float32(beta)))
        for t in (1, 2, 5, 20, 100):
            c1, c2 = oracle.bias_corrections(beta, beta, t)
            assert c1 == c2 == float(r32(1 - bf ** t)), (beta, t)
    assert oracle.bias_corrections(0.5, 0.5, 3) == (0.875, 0.875)


PINS_BC = [pin_bc_constant_gradient, pin_bc_first_step_exact, pin_bc_moments_and_freeze,
           pin_bc_corrections]

MUTANTS_BC = {
    "variance_uses_c1": ("float vh = v[i] / c2;", "float vh = v[i] / c1;"),
    "momentum_uncorrected": ("float mh = m[i] / c1;", "float mh = m[i];"),
    "stored_momentum_corrected": ("        m[i] = b1m + tg;\n", "        m[i] = (b1m + tg) / c1;\n"),
    "freeze_keeps_v": ("        v[i] = v[i] / c2;\n    }", "        v[i] = v[i];\n    }"),
    "variance_squared_correction": ("float vh = v[i] / c2;", "float vh = v[i] / (c2 * c2);"),
}


@pytest.mark.parametrize("pin", PINS_BC, ids=[p.__name__ for p in PINS_BC])
def test_bias_corrected_warmup_pin(pin):
    pin()


@pytest.mark.parametrize("name", sorted(MUTANTS_BC))
def test_pins_catch_planted_mistake(name, tmp_path):
    src = open(SRCBC).read()
    old, new = MUTANTS_BC[name]
    assert src.count(old) == 1, name
    c = tmp_path / "mutant_bc.c"
    c.write_text(src.replace(old, new))
    so = tmp_path / "mutant_bc.so"
    others = [s for s in oracle.SOURCES if s != SRCBC]
    subprocess.check_call(["gcc", *oracle.CFLAGS, "-o", str(so), *others, str(c), "-lm"])
    caught = []
    with oracle.use_library(str(so)):
        for pin in PINS_BC:
            try:
                pin()
            except AssertionError:
                caught.append(pin.__name__)
    assert caught, "no pin caught the planted mistake %s" % name
