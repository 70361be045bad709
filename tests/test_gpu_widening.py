"""Every bf16 bit pattern through the warm-up kernels.

The warm-up kernels widen bf16 gradients to fp64 with integer operations for normal values and
zeros and through fp32 for subnormal, infinite and NaN ones. Here each of W workers holds a
different permutation of all 65,536 bf16 patterns (d = 65,536, a multiple of 8, so the 16-byte
path with four workers' loads in flight runs, and W = 5 also runs the remainder loop), and one
warm-up step of the single-GPU handle and of 5 emulated data-parallel ranks (one worker each:
k_warmup_partial and k_warmup_reduce) must give the oracle's m, v and x bit for bit (NaN
compares equal to NaN: payloads of NaN results are not part of the arithmetic). A second step
runs from the first step's state so that nonzero m and v take part too.
"""
import numpy as np
import pytest
import torch

import communication_compressed_optimizer_momentum_b200 as ob
import oracle
from communication_compressed_optimizer_momentum_b200 import dp
from gpu_helpers import DEV

pytestmark = pytest.mark.gpu

D, W = 65_536, 5
B1, B2, EPS, LR = 0.9, 0.999, 1e-8, 1e-3


def _patterns(seed):
    rng = np.random.default_rng(seed)
    return np.stack([rng.permutation(65_536).astype(np.uint16) for _ in range(W)])


def _same(a, b):
    """Bitwise equality, with any NaN equal to any NaN."""
    a = np.asarray(a, np.float32)
    b = np.asarray(b, np.float32)
    nan = np.isnan(a) & np.isnan(b)
    return bool((nan | (a.view(np.uint32) == b.view(np.uint32))).all())


def _to_dev(g16):
    return torch.from_numpy(g16.view(np.int16)).to(DEV).view(torch.bfloat16)


def test_every_bf16_pattern_through_the_warmup():
    steps = [_patterns(7), _patterns(8)]
    # the patterns that are not finite make some elements NaN or infinite; keep x finite where
    # the oracle's is, and compare everything bitwise
    x0 = np.random.default_rng(3).uniform(-0.05, 0.05, D).astype(np.float32)

    xo, mo, vo = x0.copy(), np.zeros(D, np.float32), np.zeros(D, np.float32)
    x1 = torch.from_numpy(x0).to(DEV)
    single = ob.OneBitAdam(D, W, 4096, B1, B2, EPS, grad_dtype=torch.bfloat16, device=DEV)
    em = dp.EmulatedRanks(D, W, 4096, W, B1, B2, EPS, grad_dtype=torch.bfloat16, device=DEV)
    xs = [torch.from_numpy(x0).to(DEV) for _ in range(W)]
    for g in steps:
        oracle.warmup_step(xo, mo, vo, g, B1, B2, EPS, LR)
        gd = _to_dev(g)
        single.warmup_step(x1, gd, LR)
        em.warmup_step(xs, [_to_dev(np.ascontiguousarray(g[r:r + 1])) for r in range(W)], LR)
        torch.cuda.synchronize()
        for name, got, ref in (("x", x1.cpu().numpy(), xo),
                               ("m", single.get_state("m").cpu().numpy(), mo),
                               ("v", single.get_state("v").cpu().numpy(), vo)):
            assert _same(got, ref), "single-GPU warm-up %s differs at %d elements" % (
                name, int((~(np.isnan(got) & np.isnan(ref)) &
                           (got.view(np.uint32) != ref.view(np.uint32))).sum()))
        for r in range(W):
            assert _same(xs[r].cpu().numpy(), xo), "rank %d's x" % r
        assert _same(em.ranks[0].get_state("m").cpu().numpy(), mo)
        assert _same(em.ranks[0].get_state("v").cpu().numpy(), vo)
    # the inputs hold every finite bf16 value, so the step did real arithmetic on all of them
    assert np.isfinite(xo).sum() > D // 2
    single.close()
    em.close()
