"""The 0/1 Adam variant's oracle against its pins, and planted mistakes that the pins must
catch (each mutant is a copy of zero_one_oracle.c with one plausible error, built with the
oracle's other, unchanged files; the mistakes are planted on the CPU only)."""
import os
import subprocess

import pytest

import oracle
from oracle01_pins import PINS01

SRC01 = os.path.join(os.path.dirname(oracle.__file__), "zero_one_oracle.c")

MUTANTS01 = {
    "accumulate_drops_lr": ("float step = lr * m_w[j];", "float step = m_w[j];"),
    "local_momentum_drops_old_m": ("m_w[j] = b1m + tg;", "m_w[j] = tg;"),
    "compress_drops_residual": ("for (int64_t i = 0; i < d; ++i) e[i] = u[i] + e[i];",
                                "for (int64_t i = 0; i < d; ++i) e[i] = u[i];"),
    "compress_residual_sign": ("e[i] = e[i] - (e[i] >= 0.0f ? s : -s);",
                               "e[i] = e[i] + (e[i] >= 0.0f ? s : -s);"),
    "momentum_estimate_not_divided": ("mbar[i] = ubar / gamma;", "mbar[i] = ubar;"),
    "step_applies_lr_again": ("x[i] = x[i] - q;", "x[i] = x[i] - q * gamma;"),
    "step_wrong_direction": ("x[i] = x[i] - q;", "x[i] = x[i] + q;"),
    "refresh_uses_message": ("float sq = mbar[i] * mbar[i];", "float sq = ubar * ubar;"),
    "refresh_drops_old_v": ("v[i] = b2v + tv;", "v[i] = tv;"),
    "workers_keep_own_momentum": ("m_w[(int64_t)w * d + i] = mbar[i];", "(void)0;"),
    "accumulator_not_reset": ("u_w[(int64_t)w * d + i] = 0.0f;", "(void)0;"),
    "local_model_sign": ("out[i] = x[i] - q;", "out[i] = x[i] + q;"),
}


@pytest.mark.parametrize("pin", PINS01, ids=[p.__name__ for p in PINS01])
def test_zero_one_oracle_pin(pin):
    pin()


@pytest.fixture(scope="module")
def src01_text():
    with open(SRC01) as f:
        return f.read()


@pytest.mark.parametrize("name", sorted(MUTANTS01))
def test_pins_catch_planted_mistake(name, src01_text, tmp_path):
    old, new = MUTANTS01[name]
    assert src01_text.count(old) == 1, "mutation site not unique: %s" % name
    c = tmp_path / "mutant01.c"
    c.write_text(src01_text.replace(old, new))
    so = tmp_path / "mutant01.so"
    others = [src for src in oracle.SOURCES if src != SRC01]
    subprocess.check_call(["gcc", *oracle.CFLAGS, "-o", str(so), *others, str(c), "-lm"])
    caught = []
    with oracle.use_library(str(so)):
        for pin in PINS01:
            try:
                pin()
            except (AssertionError, FloatingPointError, ValueError):
                caught.append(pin.__name__)
    assert caught, "no pin caught the planted mistake %s" % name
