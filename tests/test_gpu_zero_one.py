"""GPU parity of the 0/1 Adam variant (``onebit01_*``) against its CPU oracle (``oracle.zo_*``).

Every step is checked teacher forced: the GPU's state before the step (x, v, every worker's m_w
and u_w, the residuals) goes to the oracle, which takes the same step (local, or local plus the
synchronisation and, on its schedule, the variance refresh); the GPU's state after the step is
compared with the oracle's. Tolerances are those of the 1-bit Adam parity tests
(``gpu_helpers``): the local step's m_w and u_w are elementwise with the same operation order
on both sides and must match bit for bit; sign words bit-exact outside ties; scales relative
1e-5 (their fp64 norms are summed in another order); residuals within 1e-5 of the chunk scale;
parameters within relative 1e-5. Chunks are independent, so the full-size workload is checked
on sampled chunks.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import pytest
import torch

import communication_compressed_optimizer_momentum_b200 as ob
import oracle
from communication_compressed_optimizer_momentum_b200 import workloads as wls
from gpu_helpers import (DEV, RTOL, TIE, expand, padding_is_zero, record_stats, rel_x, to_np,
                         unpack_bits)

pytestmark = pytest.mark.gpu


def _state(opt, x, k=None):
    """The GPU's state of the whole vector (k None) or of chunk k, as numpy arrays."""
    if k is None:
        lo, hi = 0, opt.d
        get = opt.get_state
        wk = -1
    else:
        lo, hi = k * opt.C, min(opt.d, (k + 1) * opt.C)
        get = lambda nm: opt.get_chunk_state(nm, k)  # noqa: E731
        wk = k
    return {"x": to_np(x[lo:hi]), "v": to_np(get("v")), "e_w": to_np(get("e_w")),
            "e_s": to_np(get("e_s")), "m_w": to_np(opt.get_worker_state("m_w", wk)),
            "u_w": to_np(opt.get_worker_state("u_w", wk))}


def _messages(opt, k=None):
    get = opt.get_state if k is None else (lambda nm: opt.get_chunk_state(nm, k))
    return {nm: to_np(get(nm)) for nm in ("s", "S", "bits_w", "bits_s")}


def _check_step(pre, g, post, msg, C, H, K, beta1, beta2, eps, lr, gamma, sync, refresh,
                stats):
    """One oracle step from the GPU's pre-step state, compared with the GPU's post-step state."""
    st = {nm: np.ascontiguousarray(a).copy() for nm, a in pre.items()}
    out = oracle.zo_step(st["x"], st["m_w"], st["u_w"], st["v"], st["e_w"], st["e_s"], g, C,
                         beta1, beta2, eps, lr, gamma, sync, refresh)
    W, n = g.shape
    if not sync:
        for nm in ("m_w", "u_w"):
            np.testing.assert_array_equal(post[nm].view(np.uint32), st[nm].view(np.uint32),
                                          err_msg=nm)
        for nm in ("x", "v", "e_w", "e_s"):
            np.testing.assert_array_equal(post[nm], pre[nm], err_msg=nm + " changed")
        stats["local"] += 1
        return
    stats["sync"] += 1
    s_el = expand(out["s"], C, n)
    xw = st["e_w"] + np.where(unpack_bits(out["bits_w"], n), s_el, -s_el)
    tie_w = np.abs(xw) < TIE * s_el
    stats["ties_w"] += int(tie_w.sum())
    bad = (unpack_bits(msg["bits_w"], n) != unpack_bits(out["bits_w"], n)) & ~tie_w
    assert not bad.any(), "worker sign bits differ at %d non-tie elements" % bad.sum()
    assert padding_is_zero(msg["bits_w"], n)
    s_g = msg["s"].reshape(out["s"].shape)
    assert (np.abs(s_g - out["s"]) <= RTOL * np.abs(out["s"])).all(), "worker scales differ"
    stats["s_exact"] += int((s_g == out["s"]).sum())
    stats["s_total"] += s_g.size
    bad = (np.abs(post["e_w"] - st["e_w"]) > RTOL * s_el) & ~tie_w
    assert not bad.any(), "worker residuals differ at %d elements" % bad.sum()
    S_el = expand(out["S"], C, n)
    S_g = msg["S"].reshape(out["S"].shape)
    assert (np.abs(S_g - out["S"]) <= RTOL * np.abs(out["S"])).all(), "server scales differ"
    stats["S_exact"] += int((S_g == out["S"]).sum())
    stats["S_total"] += S_g.size
    z = st["e_s"] + np.where(unpack_bits(out["bits_s"], n), S_el, -S_el)
    tie_s = (np.abs(z) < TIE * S_el) | tie_w.any(axis=0)
    stats["ties_s"] += int((np.abs(z) < TIE * S_el).sum())
    bad = (unpack_bits(msg["bits_s"], n) != unpack_bits(out["bits_s"], n)) & ~tie_s
    assert not bad.any(), "server sign bits differ at %d non-tie elements" % bad.sum()
    bad = (np.abs(post["e_s"] - st["e_s"]) > RTOL * S_el) & ~tie_s
    assert not bad.any(), "server residuals differ at %d elements" % bad.sum()
    # every worker restarts from mbar = ubar / Gamma, u_w = 0
    for w in range(W):
        bad = (np.abs(post["m_w"][w] - out["mbar"]) > RTOL * S_el / gamma) & ~tie_s
        assert not bad.any(), "momentum estimate differs at %d elements" % bad.sum()
    assert not post["u_w"].any(), "accumulated updates not restarted"
    rel = rel_x(post["x"], st["x"])
    bad = (rel > RTOL) & ~tie_s
    assert not bad.any(), "parameters differ at %d elements (max rel %g)" % (bad.sum(), rel.max())
    stats["x_exact"] += int(((post["x"] == st["x"]) & ~tie_s).sum())
    stats["x_total"] += int((~tie_s).sum())
    if refresh:
        stats["refresh"] += 1
        relv = np.abs(post["v"] - st["v"]) / np.maximum(np.abs(st["v"]), 1e-30)
        assert ((relv <= 2 * RTOL) | tie_s).all(), "refreshed variance differs"
    else:
        np.testing.assert_array_equal(post["v"], pre["v"], err_msg="v changed without a refresh")


def _run(wl, H, K, steps, chunks=None, lr_scale=1.0):
    """Warm-up, freeze, then `steps` steps of the variant on the GPU, each checked teacher
    forced against the oracle on `chunks` (the whole vector when None)."""
    torch.cuda.synchronize()
    dt = wls.torch_dtype(wl)
    x = wls.torch_params(wl, DEV)
    g = torch.empty((wl.W, wl.d), dtype=dt, device=DEV)
    opt = ob.ZeroOneAdam(wl.d, wl.W, wl.C, H, K, wl.beta1, wl.beta2, wl.eps, grad_dtype=dt,
                         device=DEV)
    for t in range(wl.warmup_steps):
        wls.torch_fill_grads(wl, g, 0, t)
        opt.warmup_step(x, g, wl.lr)
    opt.freeze()
    stats = {"local": 0, "sync": 0, "refresh": 0, "ties_w": 0, "ties_s": 0, "s_exact": 0,
             "s_total": 0, "S_exact": 0, "S_total": 0, "x_exact": 0, "x_total": 0}
    gamma = np.float32(0.0)
    syncs = 0
    keys = [None] if chunks is None else list(chunks)
    for t in range(1, steps + 1):
        lr = float(np.float32(wl.lr * lr_scale * (1.0 + 0.25 * (t % 3))))
        wls.torch_fill_grads(wl, g, 1, t)
        gamma = np.float32(gamma + np.float32(lr))
        sync = t % H == 0
        refresh = sync and K > 0 and (syncs + 1) % K == 0
        pre = {k: _state(opt, x, k) for k in keys}
        gk = {}
        for k in keys:
            lo, hi = (0, wl.d) if k is None else (k * wl.C, min(wl.d, (k + 1) * wl.C))
            gk[k] = to_np(g[:, lo:hi])
        info = opt.zo_info()
        assert info["launches_next_step"] == (5 if sync else 1)
        opt.step(x, g, lr)
        for k in keys:
            post = _state(opt, x, k)
            msg = _messages(opt, k) if sync else None
            _check_step(pre[k], gk[k], post, msg, wl.C, H, K, wl.beta1, wl.beta2, wl.eps, lr,
                        float(gamma), sync, refresh, stats)
        if sync:
            syncs += 1
            gamma = np.float32(0.0)
    # a worker's local model against the oracle's (on the checked chunks)
    lm = opt.local_model(wl.W - 1, x)
    for k in keys:
        lo, hi = (0, wl.d) if k is None else (k * wl.C, min(wl.d, (k + 1) * wl.C))
        st = _state(opt, x, k)
        np.testing.assert_array_equal(
            to_np(lm[lo:hi]), oracle.zo_local_model(st["x"], st["u_w"][-1], st["v"], wl.eps))
    assert opt.zo_info()["syncs"] == steps // H
    flags = opt.status()
    opt.close()
    del g, x
    torch.cuda.empty_cache()
    assert flags == 0, flags
    print("0/1 parity %s H=%d K=%d: %s" % (wl.name, H, K, stats))
    record_stats("zero_one_%s_H%d_K%d" % (wl.name, H, K), stats)
    return stats


SMALL = [
    # (d, W, C, grads, H, K)
    (10_000, 3, 4096, "f32", 3, 1),
    (65_536, 4, 16_384, "f32", 4, 2),
    (50_017, 16, 8192, "bf16", 2, 1),
    (33_000, 8, 33_024, "bf16", 1, 0),
    (20_000, 64, 4096, "f32", 3, 0),
]


@pytest.mark.parametrize("d,W,C,grads,H,K", SMALL,
                         ids=["d%d_W%d_C%d_%s_H%d_K%d" % c for c in SMALL])
def test_zero_one_parity_small(d, W, C, grads, H, K):
    base = wls.WORKLOADS["smoke_1m"]
    wl = wls.scaled(base, d, W=W, C=C)
    wl = dataclasses.replace(wl, grad_dtype=grads, warmup_steps=3)
    steps = 2 * H + 1
    st = _run(wl, H, K, steps=steps)
    assert st["sync"] == steps // H and st["local"] == steps - steps // H


def test_zero_one_bert_large_bucket_sampled_chunks():
    wl = dataclasses.replace(wls.WORKLOADS["bert_large_bucket"], warmup_steps=3)
    free, _ = torch.cuda.mem_get_info()
    if free < 100e9:
        pytest.skip("needs 100 GB of free device memory")
    st = _run(wl, 4, 2, steps=9, chunks=[0, wl.nch - 1])
    assert st["sync"] == 2 * 2 and st["refresh"] == 2


def test_zero_one_reduces_to_onebit_adam_on_the_gpu():
    """With a synchronisation every step, the variance frozen and a power-of-two lr, the
    variant's CUDA path gives the 1-bit Adam CUDA path's parameters bit for bit."""
    d, W, C = 300_001, 4, 65_536
    gen = torch.Generator(device=DEV)
    gen.manual_seed(7)
    x0 = (torch.rand(d, device=DEV, generator=gen) - 0.5) * 0.1
    gs = [torch.randn(W, d, device=DEV, generator=gen) * 1e-2 for _ in range(6)]
    a = ob.OneBitAdam(d, W, C, device=DEV)
    b = ob.ZeroOneAdam(d, W, C, 1, 0, device=DEV)
    xa, xb = x0.clone(), x0.clone()
    for g in gs[:2]:
        a.warmup_step(xa, g, 1e-3)
        b.warmup_step(xb, g, 1e-3)
    a.freeze()
    b.freeze()
    lr = 2.0 ** -10
    for g in gs[2:]:
        a.step(xa, g, lr)
        b.step(xb, g, lr)
        torch.cuda.synchronize()
        assert torch.equal(xa.view(torch.int32), xb.view(torch.int32))
    assert torch.equal(a.get_state("bits_s"), b.get_state("bits_s"))
    assert torch.equal(a.get_state("m"), b.get_worker_state("m_w")[0])
    assert a.status() == 0 and b.status() == 0
    a.close()
    b.close()


def test_zero_one_rejects_the_onebit_step_and_vice_versa():
    d, W, C = 4096, 2, 1024
    x = torch.zeros(d, device=DEV)
    g = torch.zeros(W, d, device=DEV)
    b = ob.ZeroOneAdam(d, W, C, 2, 0, device=DEV)
    b.freeze()
    with pytest.raises(ob.OneBitError) as e:
        ob.onebit_adam_compressed_step(b.h, x, g, 1e-3)
    assert e.value.code == -3
    with pytest.raises(ob.OneBitError) as e:
        b.get_state("m")
    assert e.value.code == -1
    b.close()
    a = ob.OneBitAdam(d, W, C, device=DEV)
    a.freeze()
    with pytest.raises(ob.OneBitError) as e:
        ob.onebit01_step(a.h, x, g, 1e-3)
    assert e.value.code == -3
    a.close()


def test_bench_zero_one_line():
    """bench.py --variant zero_one prints one JSON line: every step counted (local and
    synchronising), one launch per local step and five per synchronising step, the roofline over
    the interval's average bytes."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--workload", "smoke_1m",
                        "--variant", "zero_one", "--sync-every", "3", "--refresh-every", "1",
                        "--steps", "6", "--warmup", "3", "--no-e2e", "--no-cpu-baseline"],
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["config"]["variant"] == "0/1 Adam" and j["config"]["sync_every"] == 3
    assert j["gpu_launches"] == 6 + 4 * 2
    assert j["value"] > 0 and j["status_flags"] == 0
    roof = j["roofline"]
    assert roof["bound"] == "hbm" and abs(roof["frac"] - roof["achieved"] / roof["peak"]) < 1e-9


@pytest.mark.parametrize("resume_after", [3, 4, 5], ids=["after_sync", "after_first_local",
                                                         "after_second_local"])
def test_zero_one_checkpoint_resume_bit_identical(resume_after):
    """A frozen 0/1 handle restored from another's checkpoint (v, residuals, every worker's
    momentum and accumulated update, the schedule) continues bit for bit like it, whatever form
    the saved state had: right after a synchronisation (momentum estimate from the server plane,
    update zero), after the interval's first step (update not stored), after its second."""
    import dataclasses
    wl = dataclasses.replace(wls.WORKLOADS["smoke_1m"], name="zo_ckpt", d=70_003, W=5, C=16_384,
                             grad_dtype="bf16", layer_sizes=())
    H, K = 3, 2
    dt = wls.torch_dtype(wl)
    g = torch.empty((wl.W, wl.d), dtype=dt, device=DEV)
    a = ob.ZeroOneAdam(wl.d, wl.W, wl.C, H, K, wl.beta1, wl.beta2, wl.eps, grad_dtype=dt,
                       device=DEV)
    xa = wls.torch_params(wl, DEV)
    for t in range(3):
        wls.torch_fill_grads(wl, g, 0, t)
        a.warmup_step(xa, g, wl.lr)
    a.freeze()
    lrs = [wl.lr * (1.0 + 0.25 * (t % 3)) for t in range(1, resume_after + 7)]
    for t in range(1, resume_after + 1):
        wls.torch_fill_grads(wl, g, 1, t)
        a.step(xa, g, lrs[t - 1])
    ck = a.checkpoint()
    xb = xa.clone()
    b = ob.ZeroOneAdam(wl.d, wl.W, wl.C, H, K, wl.beta1, wl.beta2, wl.eps, grad_dtype=dt,
                       device=DEV)
    b.freeze()
    b.restore(ck)
    assert b.schedule() == a.schedule()

    def same(u, v):
        return torch.equal(u.view(torch.int32), v.view(torch.int32))

    for t in range(resume_after + 1, resume_after + 7):
        wls.torch_fill_grads(wl, g, 1, t)
        a.step(xa, g, lrs[t - 1])
        b.step(xb, g, lrs[t - 1])
        assert same(xa, xb), "x after step %d" % t
        for nm in ("v", "e_w", "e_s"):
            assert same(a.get_state(nm), b.get_state(nm)), "%s after step %d" % (nm, t)
        for nm in ("m_w", "u_w"):
            assert same(a.get_worker_state(nm), b.get_worker_state(nm)), "%s, step %d" % (nm, t)
        assert a.schedule() == b.schedule()
    assert a.status() == 0 and b.status() == 0
    a.close()
    b.close()
