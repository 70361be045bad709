"""Randomised small-problem parity: vector lengths, chunk lengths, worker counts (up to the
library's 256), gradient types, distributions and beta1 drawn from a seeded generator. Each case
runs warm-up steps (the last one bit-exact) and compressed steps teacher forced against the
oracle, plus the oracle free running from the post-warm-up state."""
import dataclasses

import numpy as np
import pytest

from communication_compressed_optimizer_momentum_b200 import workloads as wls
from gpu_helpers import run_parity

pytestmark = pytest.mark.gpu

_BASE = wls.WORKLOADS["smoke_1m"]


def _cases(n=24, seed=20260):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        W = int(rng.choice([1, 2, 3, 5, 7, 8, 9, 12, 16, 17, 24, 31, 32, 48, 64, 100, 129, 256]))
        d = int(rng.integers(1, 120_000 if W <= 64 else 30_000))
        C = int(rng.choice([32, 64, 2048, 4096, 4128, 8192, 65_536, ((d + 31) // 32) * 32]))
        out.append(dataclasses.replace(
            _BASE, name="rand%02d_d%d_W%d_C%d" % (i, d, W, C), d=d, W=W, C=C,
            grad_dtype=str(rng.choice(["f32", "bf16"])),
            grad_kind=str(rng.choice(["normal", "outlier_normal", "student_t", "edge_normal"])),
            sigma=float(10.0 ** rng.uniform(-4, -1)), beta1=float(rng.choice([0.0, 0.5, 0.9, 0.99])),
            warmup_steps=2, compressed_steps=3, seed=int(rng.integers(1, 1 << 30)),
            layer_sizes=()))
    return out


CASES = _cases()


@pytest.mark.parametrize("wl", CASES, ids=[w.name for w in CASES])
def test_random_case(wl):
    st = run_parity(wl, chunks=None, teacher_steps=(1, 2, 3), free_steps=3)
    assert st["status_flags"] == 0
