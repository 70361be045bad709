"""Planted mistakes: each mutant is a copy of the oracle's C file with one plausible error (a
dropped term, a wrong sign or index, a transposed operand, a wrong constant). Every mutant must
fail at least one pin; a mutant that passes them all would mean the pins cannot tell that
mistake from the method. The mistakes are planted in the oracle on the CPU only."""
import os
import subprocess

import pytest

import oracle
from oracle_pins import PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "onebit_oracle.c")

MUTANTS = {
    "worker_drops_residual": ("e[i] = mw + e[i];", "e[i] = mw;"),
    "worker_residual_sign": ("e[i] = e[i] - (sign_bit(e[i]) ? s : -s);",
                             "e[i] = e[i] + (sign_bit(e[i]) ? s : -s);"),
    "momentum_wrong_coefficient": ("float tg = omb1 * gf;", "float tg = beta1 * gf;"),
    "momentum_drops_old_m": ("float mw = b1m + tg;", "float mw = tg;"),
    "scale_uses_padded_length": ("return (float)sqrt(ss / (double)len);",
                                 "return (float)sqrt(ss / (double)((len + 31) / 32 * 32));"),
    "scale_is_mean_abs_squared": ("ss += (double)x[i] * (double)x[i];",
                                  "ss += fabs((double)x[i]) * 1.0;"),
    "sign_zero_negative": ("static int sign_bit(float x) { return x >= 0.0f; }",
                           "static int sign_bit(float x) { return x > 0.0f; }"),
    "pack_msb_first": ("words[i / 32] |= (1u << (i % 32));",
                       "words[i / 32] |= (1u << (31 - i % 32));"),
    "server_average_off_by_one": ("float y = (float)(acc / (double)W);",
                                  "float y = (float)(acc / (double)(W + 1));"),
    "server_drops_error": ("z_tmp[i] = y + e_s[i];", "z_tmp[i] = y;"),
    "server_residual_sign": ("e_s[i] = z_tmp[i] - (sign_bit(z_tmp[i]) ? S : -S);",
                             "e_s[i] = z_tmp[i] + (sign_bit(z_tmp[i]) ? S : -S);"),
    "server_reads_worker_zero_only": ("double sw = (double)s[(int64_t)w * nch + k];",
                                      "double sw = (double)s[k];"),
    "apply_wrong_direction": ("        x[i] = x[i] - upd;\n    }\n}\n\n/*\n * One whole",
                              "        x[i] = x[i] + upd;\n    }\n}\n\n/*\n * One whole"),
    "apply_eps_inside_sqrt": ("        float den = sqrtf(v[i]) + eps;\n        float q = m[i] / den;\n"
                              "        float upd = lr * q;\n        x[i] = x[i] - upd;\n    }\n}\n\n/*\n * One",
                              "        float den = sqrtf(v[i] + eps);\n        float q = m[i] / den;\n"
                              "        float upd = lr * q;\n        x[i] = x[i] - upd;\n    }\n}\n\n/*\n * One"),
    "unpack_transposed_index": ("float s = scales[i / C];", "float s = scales[i % C];"),
    "warmup_v_uses_g_not_g2": ("float tv = omb2 * g2;", "float tv = omb2 * gbar;"),
    "warmup_drops_one_minus_beta1": ("float tg = omb1 * gbar;", "float tg = gbar;"),
    "warmup_sums_instead_of_averaging": ("float gbar = (float)(acc / (double)W);",
                                         "float gbar = (float)acc;"),
}


@pytest.fixture(scope="module")
def src_text():
    with open(SRC) as f:
        return f.read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, src_text, tmp_path):
    old, new = MUTANTS[name]
    assert src_text.count(old) == 1, "mutation site not unique: %s" % name
    mutated = src_text.replace(old, new)
    c = tmp_path / "mutant.c"
    c.write_text(mutated)
    so = tmp_path / "mutant.so"
    # the mutant is linked with the oracle's other files, unchanged
    others = [src for src in oracle.SOURCES if src != SRC]
    subprocess.check_call(["gcc", *oracle.CFLAGS, "-o", str(so), str(c), *others, "-lm"])
    caught = []
    with oracle.use_library(str(so)):
        for pin in PINS:
            try:
                pin()
            except (AssertionError, FloatingPointError, ValueError) as e:  # noqa: PERF203
                caught.append(pin.__name__)
                del e
    assert caught, "no pin caught the planted mistake %s" % name
