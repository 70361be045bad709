"""Data-parallel ranks of the 0/1 Adam variant on the GPU: R ranks emulated as R handles on this
GPU, each step driven phase by phase across the ranks, against one single-GPU 0/1 handle with all
W workers -- bit for bit after every step: every rank's x, its workers' momenta and accumulated
updates, residuals, scales and sign planes, the server state, v (refreshed at synchronisations)
and a local model. Also the whole-step entry point at R = 1 (its barriers signal and wait in one
launch) and the phase rules of a 0/1 rank."""
import dataclasses

import pytest
import torch

import communication_compressed_optimizer_momentum_b200 as ob
from communication_compressed_optimizer_momentum_b200 import dp
from communication_compressed_optimizer_momentum_b200 import workloads as wls
from gpu_helpers import DEV

pytestmark = pytest.mark.gpu

F32 = wls.WORKLOADS["smoke_1m"]
BF16 = wls.WORKLOADS["bert_large_bucket"]


def _wl(base, d, W, C, **kw):
    return dataclasses.replace(base, name="zo_dp_%d_%d_%d" % (d, W, C), d=d, W=W, C=C,
                               layer_sizes=(), **kw)


# (workload, R, H, K, compressed steps)
CASES = {
    "r2_h3_k2": (_wl(F32, 65_536, 4, 8192), 2, 3, 2, 7),
    "r4_bf16_h2_k1": (_wl(BF16, 262_144, 16, 16_384, grad_kind="normal"), 4, 2, 1, 5),
    "r3_ragged_h4_k0": (_wl(F32, 98_321, 6, 4096), 3, 4, 0, 9),       # d % 4 != 0, 2 workers each
    "r2_h1": (_wl(F32, 40_000, 8, 2048), 2, 1, 0, 3),                  # every step synchronises
    "r2_w64_bank_private": (_wl(F32, 300_000, 64, 131_072), 2, 2, 1, 4),
}

NAMES = ("v", "e_w", "e_s", "s", "S", "bits_w", "bits_s")


def _same(a, b):
    if a.dtype == torch.float32:
        return torch.equal(a.view(torch.int32), b.view(torch.int32))
    return torch.equal(a, b)


def _rank_grads(g, R):
    Wl = g.shape[0] // R
    out = []
    for r in range(R):
        v = g[r * Wl:(r + 1) * Wl]
        out.append(v if v.data_ptr() % 16 == 0 else v.clone())
    return out


def _assert_same(em, single, xs, x1, where):
    R = em.R
    for r, xr in enumerate(xs):
        assert _same(xr, x1), "%s: rank %d's x" % (where, r)
    Wl = single.W // R
    for which in ("m_w", "u_w"):
        ref = single.get_worker_state(which)
        for r, o in enumerate(em.ranks):
            assert _same(o.get_worker_state(which), ref[r * Wl:(r + 1) * Wl]), \
                "%s: rank %d's %s" % (where, r, which)
    st = {nm: em.ranks[0].get_state(nm) for nm in ("v", "S", "bits_s")}
    for nm in ("e_w", "s", "bits_w", "e_s"):
        st[nm] = torch.cat([o.get_state(nm) for o in em.ranks])
    for nm in NAMES:
        assert _same(st[nm], single.get_state(nm)), "%s: state %s" % (where, nm)
    for r, o in enumerate(em.ranks):
        for nm in ("v", "S", "bits_s"):
            assert _same(o.get_state(nm), st[nm]), "%s: rank %d's %s" % (where, r, nm)
    # the last worker of the last rank: its local model
    lm = em.ranks[-1].local_model(Wl - 1, xs[-1])
    assert _same(lm, single.local_model(single.W - 1, x1)), "%s: local model" % where


def run_against_single(wl, R, H, K, steps, warm=3):
    dt = wls.torch_dtype(wl)
    x1 = wls.torch_params(wl, DEV)
    xs = [x1.clone() for _ in range(R)]
    g = torch.empty((wl.W, wl.d), dtype=dt, device=DEV)
    single = ob.ZeroOneAdam(wl.d, wl.W, wl.C, H, K, wl.beta1, wl.beta2, wl.eps, grad_dtype=dt,
                            device=DEV)
    em = dp.EmulatedRanks(wl.d, wl.W, wl.C, R, wl.beta1, wl.beta2, wl.eps, grad_dtype=dt,
                          device=DEV, zero_one=(H, K))
    for t in range(warm):
        wls.torch_fill_grads(wl, g, 0, t)
        single.warmup_step(x1, g, wl.lr)
        em.warmup_step(xs, _rank_grads(g, R), wl.lr)
    single.freeze()
    em.freeze()
    for t in range(1, steps + 1):
        lr = wl.lr * (1.0 + 0.25 * (t % 3))
        wls.torch_fill_grads(wl, g, 1, t)
        single.step(x1, g, lr)
        em.step(xs, _rank_grads(g, R), lr)
        _assert_same(em, single, xs, x1, "0/1 step %d" % t)
    infos = [o.zo_info() for o in em.ranks]
    assert all(i == single.zo_info() for i in infos)
    assert infos[0]["syncs"] == steps // H
    assert em.status() == 0 and single.status() == 0
    em.close()
    single.close()


@pytest.mark.parametrize("case", list(CASES))
def test_zero_one_ranks_match_single_handle(case):
    wl, R, H, K, steps = CASES[case]
    run_against_single(wl, R, H, K, steps)


def test_zero_one_whole_step_one_rank():
    """R = 1 through onebit01_step (the whole step: the three phases, each barrier one launch
    that signals and waits) equals the single 0/1 handle."""
    wl = _wl(F32, 70_000, 4, 8192)
    H, K = 3, 1
    x1 = wls.torch_params(wl, DEV)
    x2 = x1.clone()
    g = torch.empty((wl.W, wl.d), dtype=torch.float32, device=DEV)
    single = ob.ZeroOneAdam(wl.d, wl.W, wl.C, H, K, wl.beta1, wl.beta2, wl.eps, device=DEV)
    opt = dp.ZeroOneAdamRank(wl.d, wl.W, wl.C, 1, 0, H, K, wl.beta1, wl.beta2, wl.eps,
                             device=DEV)
    opt.connect()
    for t in range(2):
        wls.torch_fill_grads(wl, g, 0, t)
        single.warmup_step(x1, g, wl.lr)
        opt.warmup_step(x2, g, wl.lr)
    single.freeze()
    opt.freeze()
    for t in range(1, 8):
        wls.torch_fill_grads(wl, g, 1, t)
        single.step(x1, g, wl.lr)
        opt.step(x2, g, wl.lr)
        assert _same(x1, x2), "step %d" % t
    for which in ("m_w", "u_w"):
        assert _same(opt.get_worker_state(which), single.get_worker_state(which))
    assert opt.status() == 0
    opt.close()
    single.close()


def test_zero_one_rank_phase_rules():
    """A 0/1 rank steps only through its own phases, in order; a 1-bit rank's compressed phases
    refuse it, and a synchronisation whose Gamma is 0 is refused before any launch."""
    wl = _wl(F32, 20_000, 4, 2048)
    em = dp.EmulatedRanks(wl.d, wl.W, wl.C, 2, device=DEV, zero_one=(2, 0))
    xs = [wls.torch_params(wl, DEV) for _ in range(2)]
    g = _rank_grads(torch.zeros((wl.W, wl.d), device=DEV), 2)
    r0 = em.ranks[0]
    with pytest.raises(ob.OneBitError):            # before the freeze
        r0.zo_phase(0, xs[0], g[0], 1e-3)
    em.warmup_step(xs, g, 1e-3)
    em.freeze()
    with pytest.raises(ob.OneBitError):            # phase 1 before phase 0
        r0.zo_phase(1, xs[0], g[0], 1e-3)
    with pytest.raises(ob.OneBitError):            # a 1-bit Adam phase on a 0/1 rank
        r0.compressed_phase(0, xs[0], g[0], 1e-3)
    em.step(xs, g, 1e-3)                           # local step
    with pytest.raises(ob.OneBitError):            # synchronisation with Gamma = 1e-3 - 1e-3 = 0
        r0.zo_phase(0, xs[0], g[0], -1e-3)
    em.step(xs, g, 2e-3)                           # the synchronisation
    assert r0.zo_info()["syncs"] == 1
    assert em.status() == 0
    em.close()
