"""Parity at the full workload sizes, in the launch configuration the benchmark times.

Chunks are independent (the chunk-independence pin), so a sample of whole chunks (the first, the
second, the last -- which holds any ragged tail -- and a seeded random one) checks every output
that depends on them. For each workload: the last warm-up step bit-exact on the sampled chunks,
compressed steps teacher forced against the oracle (the GPU's pre-step state of the chunk in,
the GPU's post-step state compared), and the oracle free running from the GPU's post-warm-up
state on the sampled chunks. The gradients are generated on the device per step and the oracle
gets the exact bytes the GPU consumed.
"""
import dataclasses

import pytest
import torch

from communication_compressed_optimizer_momentum_b200 import workloads as wls
from gpu_helpers import run_parity

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _free_gb():
    free, _ = torch.cuda.mem_get_info()
    return free / 1e9


def _need(gb):
    if _free_gb() < gb:
        pytest.skip("needs %.0f GB of free device memory, %.0f GB free" % (gb, _free_gb()))


def test_bert_base_bucket():
    wl = wls.WORKLOADS["bert_base_bucket"]
    _need(12)
    st = run_parity(wl, chunks=wls.sample_chunks(wl), teacher_steps=(1, 2, 10, "last"),
                    free_steps=10)
    assert st["inexact_chunks"] == 0 and st["status_flags"] == 0


def test_bert_large_bucket():
    wl = wls.WORKLOADS["bert_large_bucket"]
    _need(42)
    st = run_parity(wl, chunks=[0, wl.nch - 1], teacher_steps=(1, "last"), free_steps=10,
                    free_chunks=[0])
    assert st["inexact_chunks"] == 0 and st["status_flags"] == 0


def test_gpt2_xl_bucket():
    wl = wls.WORKLOADS["gpt2_xl_bucket"]
    _need(110)
    ks = wls.sample_chunks(wl)
    st = run_parity(wl, chunks=ks, teacher_steps=(1, 2, "last"), free_steps=10,
                    free_chunks=[ks[0], ks[-1]])
    assert st["inexact_chunks"] == 0 and st["status_flags"] == 0


SWEEP = wls.sweep_points()


@pytest.mark.parametrize("W,C", SWEEP, ids=["W%d_C%s" % (w, c or "dW") for w, c in SWEEP])
def test_sweep_point(W, C):
    # full sizes and the benchmark's launch configuration; 3 warm-up steps instead of 20 keep
    # the 24 points affordable (the warm-up count does not change what the compressed path does)
    wl = dataclasses.replace(wls.sweep_workload(W, C), warmup_steps=3)
    _need(2.2 * W * wl.d * 4 / 1e9 + 8)
    if wl.nch > 4:
        chunks = sorted({0, 1, wl.nch - 1, wl.nch // 2})
    else:
        chunks = [wl.nch - 1]                  # chunks of 2^28 / W elements: the last one
    free = 10 if wl.C <= (1 << 20) else 0
    st = run_parity(wl, chunks=chunks, teacher_steps=(1, 10), free_steps=free,
                    free_chunks=[chunks[0], chunks[-1]])
    assert st["inexact_chunks"] == 0 and st["status_flags"] == 0
