"""Helpers for the GPU parity tests: run the CUDA path through the C ABI, hand the exact bytes
it consumed to the CPU oracle, and compare.

Tolerances (stated once, used by every parity test):
  - packed sign words: bit-exact, except elements whose pre-compression value is a tie,
    |x| < 1e-6 * scale (either answer is correct there; the count is reported). Padding bits
    past the end of the vector must be 0.
  - scales s and S: relative 1e-5.
  - residuals e_w, e_s and the momentum m: |diff| <= 1e-5 * the chunk's scale (they are
    multiples-of-scale quantities; a 1-ulp difference of the scale moves them by ulp(scale)).
  - parameters x: |diff| <= 1e-5 * max(|x_ref|, 1e-3 * rms(x_ref)) after one step (teacher
    forced, and free running after 1 step); 1e-4 after 10 free-running steps. Elements that
    were a tie at any step are excluded and counted.
  - warm-up (plain Adam, elementwise, same operation order on both sides): bit-exact.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import numpy as np
import torch

import communication_compressed_optimizer_momentum_b200 as ob
import oracle
from communication_compressed_optimizer_momentum_b200 import workloads as wls

TIE = 1e-6
RTOL = 1e-5
RTOL_10 = 1e-4
DEV = "cuda:0"


def to_np(t: torch.Tensor) -> np.ndarray:
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16).copy()
    if t.dtype == torch.int32:
        return t.numpy().view(np.uint32).copy()
    return t.numpy().copy()


def unpack_bits(words: np.ndarray, n: int) -> np.ndarray:
    w = np.ascontiguousarray(words, dtype=np.uint32)
    return np.unpackbits(w.view(np.uint8), bitorder="little", axis=-1)[..., :n].astype(bool)


def padding_is_zero(words: np.ndarray, n: int) -> bool:
    r = n % 32
    if r == 0:
        return True
    last = np.asarray(words)[..., -1].astype(np.uint64)
    return bool(((last >> r) == 0).all())


def expand(scales: np.ndarray, C: int, n: int) -> np.ndarray:
    if scales.shape[-1] == 1:          # one chunk: broadcast instead of materialising W x n
        return np.broadcast_to(scales, scales.shape[:-1] + (n,))
    return np.repeat(scales, C, axis=-1)[..., :n]


@dataclasses.dataclass
class StepReport:
    ties_w: int = 0
    ties_s: int = 0
    s_exact: int = 0
    s_total: int = 0
    S_exact: int = 0
    S_total: int = 0
    ew_exact: int = 0
    ew_total: int = 0
    es_exact: int = 0
    es_total: int = 0
    m_exact: int = 0
    m_total: int = 0
    max_rel_x: float = 0.0
    inexact_chunks: int = 0


def check_compressed_step(pre: Dict[str, np.ndarray], g: np.ndarray, post: Dict[str, np.ndarray],
                          C: int, beta1: float, eps: float, lr: float,
                          tie_mask: Optional[np.ndarray] = None) -> StepReport:
    """Run the oracle for one compressed step from the GPU's pre-step state `pre` (x, m, v,
    e_w, e_s; one chunk or a whole vector) and compare with the GPU's post-step state `post`
    (x, m, e_w, e_s, s, S, bits_w, bits_s). `tie_mask` (optional, length n) accumulates the
    elements that were ties."""
    W, n = g.shape
    x, m = pre["x"].copy(), pre["m"].copy()
    e_w, e_s = pre["e_w"].copy(), pre["e_s"].copy()
    out = oracle.compressed_step(x, m, pre["v"], e_w, e_s, g, C, beta1, eps, lr)
    rep = StepReport(inexact_chunks=out["inexact"])
    s_el = expand(out["s"], C, n)
    bits_o = unpack_bits(out["bits_w"], n)
    xw = e_w + np.where(bits_o, s_el, -s_el)
    tie_w = np.abs(xw) < TIE * s_el
    rep.ties_w = int(tie_w.sum())
    any_tie_w = tie_w.any(axis=0)

    bits_g = unpack_bits(post["bits_w"], n)
    bad = (bits_g != bits_o) & ~tie_w
    assert not bad.any(), "worker sign bits differ at %d non-tie elements (first %s)" % (
        bad.sum(), np.argwhere(bad)[:5].tolist())
    assert padding_is_zero(post["bits_w"], n), "worker padding bits not zero"

    s_g = post["s"].reshape(out["s"].shape)
    assert (np.abs(s_g - out["s"]) <= RTOL * np.abs(out["s"])).all(), "worker scales differ"
    rep.s_exact, rep.s_total = int((s_g == out["s"]).sum()), out["s"].size
    d_ew = np.abs(post["e_w"] - e_w)
    bad = (d_ew > RTOL * s_el) & ~tie_w
    assert not bad.any(), "worker residuals differ at %d elements" % bad.sum()
    # the tolerance is the assertion; how many non-tie values matched bit for bit is reported
    rep.ew_exact = int(((post["e_w"].view(np.uint32) == e_w.view(np.uint32)) & ~tie_w).sum())
    rep.ew_total = int((~tie_w).sum())

    S_el = expand(out["S"], C, n)
    S_g = post["S"].reshape(out["S"].shape)
    assert (np.abs(S_g - out["S"]) <= RTOL * np.abs(out["S"])).all(), "server scales differ"
    rep.S_exact, rep.S_total = int((S_g == out["S"]).sum()), out["S"].size
    bits_so = unpack_bits(out["bits_s"], n)
    z = e_s + np.where(bits_so, S_el, -S_el)
    tie_s = (np.abs(z) < TIE * S_el) | any_tie_w
    rep.ties_s = int((np.abs(z) < TIE * S_el).sum())
    bad = (unpack_bits(post["bits_s"], n) != bits_so) & ~tie_s
    assert not bad.any(), "server sign bits differ at %d non-tie elements" % bad.sum()
    assert padding_is_zero(post["bits_s"], n), "server padding bits not zero"
    bad = (np.abs(post["e_s"] - e_s) > RTOL * S_el) & ~tie_s
    assert not bad.any(), "server residuals differ at %d elements" % bad.sum()
    bad = (np.abs(post["m"] - m) > RTOL * S_el) & ~tie_s
    assert not bad.any(), "momentum differs at %d elements" % bad.sum()
    rep.es_exact = int(((post["e_s"].view(np.uint32) == e_s.view(np.uint32)) & ~tie_s).sum())
    rep.m_exact = int(((post["m"].view(np.uint32) == m.view(np.uint32)) & ~tie_s).sum())
    rep.es_total = rep.m_total = int((~tie_s).sum())
    rel = rel_x(post["x"], x)
    bad = (rel > RTOL) & ~tie_s
    assert not bad.any(), "parameters differ at %d elements (max rel %g)" % (bad.sum(), rel.max())
    rep.max_rel_x = float(rel[~tie_s].max()) if (~tie_s).any() else 0.0
    if tie_mask is not None:
        tie_mask |= tie_s
    return rep


def rel_x(x: np.ndarray, x_ref: np.ndarray) -> np.ndarray:
    rms = float(np.sqrt(np.mean(x_ref.astype(np.float64) ** 2))) if x_ref.size else 0.0
    den = np.maximum(np.abs(x_ref).astype(np.float64), 1e-3 * rms)
    den = np.where(den == 0, 1.0, den)
    return np.abs(x.astype(np.float64) - x_ref) / den


# ----------------------------------------------------------------------------------------------
# driving the CUDA path

def gpu_chunk_state(opt: "ob.OneBitAdam", x: torch.Tensor, k: int, names) -> Dict[str, np.ndarray]:
    lo, hi = k * opt.C, min(opt.d, (k + 1) * opt.C)
    out = {}
    for nm in names:
        if nm == "x":
            out["x"] = to_np(x[lo:hi])
        else:
            out[nm] = to_np(opt.get_chunk_state(nm, k))
    return out


PRE = ("x", "m", "v", "e_w", "e_s")
POST = ("x", "m", "e_w", "e_s", "s", "S", "bits_w", "bits_s")


def run_parity(wl: wls.Workload, chunks: Optional[List[int]] = None,
               teacher_steps=(1, 2), free_steps: int = 0, warm_check: bool = True,
               free_chunks: Optional[List[int]] = None, log=print) -> dict:
    """Run wl's warm-up and compressed steps on the GPU (grads regenerated per step on the
    device); check the last warm-up step bit-exactly and the given compressed steps teacher
    forced against the oracle on `chunks` (all chunks when None); run the oracle free-running
    for `free_steps` steps from the GPU's post-warm-up state on the same chunks."""
    torch.cuda.synchronize()
    dt = wls.torch_dtype(wl)
    x = wls.torch_params(wl, DEV)
    g = torch.empty((wl.W, wl.d), dtype=dt, device=DEV)
    opt = ob.OneBitAdam(wl.d, wl.W, wl.C, wl.beta1, wl.beta2, wl.eps, grad_dtype=dt, device=DEV)
    ks = list(range(wl.nch)) if chunks is None else list(chunks)
    bounds = {k: (k * wl.C, min(wl.d, (k + 1) * wl.C)) for k in ks}
    stats = {"chunks": ks, "ties_w": 0, "ties_s": 0, "s_exact": 0, "s_total": 0, "S_exact": 0,
             "S_total": 0, "ew_exact": 0, "ew_total": 0, "es_exact": 0, "es_total": 0,
             "m_exact": 0, "m_total": 0, "inexact_chunks": 0, "free_excluded": 0,
             "free_rel": {}}

    def grads_of(k):
        lo, hi = bounds[k]
        return to_np(g[:, lo:hi])

    for t in range(wl.warmup_steps):
        wls.torch_fill_grads(wl, g, 0, t)
        last = t == wl.warmup_steps - 1
        if last and warm_check:
            pre = {k: gpu_chunk_state(opt, x, k, ("x", "m", "v")) for k in ks}
            gk = {k: grads_of(k) for k in ks}
        opt.warmup_step(x, g, wl.lr)
        if last and warm_check:
            for k in ks:
                post = gpu_chunk_state(opt, x, k, ("x", "m", "v"))
                xo, mo, vo = pre[k]["x"], pre[k]["m"], pre[k]["v"]
                oracle.warmup_step(xo, mo, vo, gk[k], wl.beta1, wl.beta2, wl.eps, wl.lr)
                for nm, ref in (("x", xo), ("m", mo), ("v", vo)):
                    assert np.array_equal(post[nm].view(np.uint32), ref.view(np.uint32)), \
                        "warm-up %s differs in chunk %d" % (nm, k)
    opt.freeze()
    free = {}
    fks = ks if free_chunks is None else [k for k in free_chunks if k in ks]
    if free_steps:
        for k in fks:
            st = gpu_chunk_state(opt, x, k, ("x", "m", "v"))
            n = st["x"].size
            st["e_w"] = np.zeros((wl.W, n), np.float32)
            st["e_s"] = np.zeros(n, np.float32)
            st["tie"] = np.zeros(n, bool)
            free[k] = st
    last_step = wl.compressed_steps
    for t in range(1, last_step + 1):
        wls.torch_fill_grads(wl, g, 1, t)
        tf = t in teacher_steps or (t == last_step and "last" in teacher_steps)
        need_g = tf or t <= free_steps
        gk = {k: grads_of(k) for k in (ks if tf else fks)} if need_g else None
        pre = {k: gpu_chunk_state(opt, x, k, PRE) for k in ks} if tf else None
        opt.step(x, g, wl.lr)
        if tf:
            for k in ks:
                post = gpu_chunk_state(opt, x, k, POST)
                r = check_compressed_step(pre[k], gk[k], post, wl.C, wl.beta1, wl.eps, wl.lr)
                for f in ("ties_w", "ties_s", "s_exact", "s_total", "S_exact", "S_total",
                          "ew_exact", "ew_total", "es_exact", "es_total", "m_exact", "m_total",
                          "inexact_chunks"):
                    stats[f] += getattr(r, f)
        if t <= free_steps:
            for k in fks:
                st = free[k]
                out = oracle.compressed_step(st["x"], st["m"], st["v"], st["e_w"], st["e_s"],
                                             gk[k], wl.C, wl.beta1, wl.eps, wl.lr)
                n = st["x"].size
                S_el = expand(out["S"], wl.C, n)
                s_el = expand(out["s"], wl.C, n)
                bits_o = unpack_bits(out["bits_w"], n)
                xw = st["e_w"] + np.where(bits_o, s_el, -s_el)
                z = st["e_s"] + np.where(unpack_bits(out["bits_s"], n), S_el, -S_el)
                st["tie"] |= (np.abs(xw) < TIE * s_el).any(axis=0) | (np.abs(z) < TIE * S_el)
                if t in (1, free_steps):
                    xg = to_np(x[bounds[k][0]:bounds[k][1]])
                    rel = rel_x(xg, st["x"])
                    tol = RTOL if t == 1 else RTOL_10
                    ok = rel <= tol
                    bad = ~ok & ~st["tie"]
                    assert not bad.any(), "free-running x after %d steps differs in chunk %d " \
                        "at %d elements (max rel %g)" % (t, k, bad.sum(), rel[~st["tie"]].max())
                    stats["free_rel"]["step%d_chunk%d" % (t, k)] = float(rel[~st["tie"]].max())
                    stats["free_excluded"] = max(stats["free_excluded"], int(st["tie"].sum()))
    flags = opt.status()
    stats["status_flags"] = flags
    opt.close()
    del g, x, opt
    torch.cuda.empty_cache()
    log("parity %s: %s" % (wl.name, stats))
    record_stats(wl.name, stats)
    return stats


def record_stats(name: str, stats: dict) -> None:
    """Append one run's parity counts to the JSON-lines file named by ONEBIT_PARITY_LOG (if
    set), so that a whole test session's exact-match totals can be read afterwards."""
    import json
    import os
    path = os.environ.get("ONEBIT_PARITY_LOG")
    if not path:
        return
    keep = {k: v for k, v in stats.items() if isinstance(v, (int, float))}
    with open(path, "a") as f:
        f.write(json.dumps(dict(keep, workload=name)) + "\n")
