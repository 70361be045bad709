"""Data-parallel ranks as separate processes (two and three), connected through CUDA IPC.

Each rank is its own process with its own CUDA context; the exchange regions are mapped across
the processes with onebit_dp_ipc_handle / onebit_dp_open_peer, so the worker, server and warm-up
kernels store into (and, in the warm-up, load from) the other process's memory and the barrier
kernels publish their flags there. Both processes share this one GPU, so the test host runs the
phases one at a time, in the order of the emulated ranks: phase p of rank 0, then of rank 1,
then phase p + 1, each only after the previous one has finished on the device. Every barrier
wait is therefore launched after the signal it waits for has completed and returns at its first
poll; no kernel ever waits for a kernel that is still running or not yet launched (each rank's
barrier timeout is cut to 2 s, so a missing flag would show up as a status flag, not a stall).
Both ranks' parameters must equal the single-GPU handle's bit for bit.
"""
import multiprocessing as pymp

import numpy as np
import pytest
import torch

import communication_compressed_optimizer_momentum_b200 as ob
from gpu_helpers import DEV

pytestmark = pytest.mark.gpu

D, C = 20_000, 2048
B1, B2, EPS, LR = 0.9, 0.999, 1e-8, 1e-3
WARM, STEPS = 2, 3


def _inputs(W):
    rng = np.random.default_rng(4242 + W)
    x0 = rng.uniform(-0.05, 0.05, D).astype(np.float32)
    gw = [(rng.standard_normal((W, D)) * 1e-2).astype(np.float32) for _ in range(WARM)]
    gc = [(rng.standard_normal((W, D)) * 1e-2).astype(np.float32) for _ in range(STEPS)]
    return x0, gw, gc


def _rank(rank, R, W, cmd, out):
    """Child process: one rank. Runs the commands the test host sends, one at a time."""
    import sys
    import os
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch
    from communication_compressed_optimizer_momentum_b200 import dp
    try:
        torch.cuda.set_device(0)
        x0, gw, gc = _inputs(W)
        Wl = W // R
        opt = dp.OneBitAdamRank(D, W, C, R, rank, B1, B2, EPS, device="cuda:0")
        opt.set_timeout_us(2_000_000)
        x = torch.from_numpy(x0).cuda()
        mine = lambda g: torch.from_numpy(np.ascontiguousarray(g[rank * Wl:(rank + 1) * Wl])).cuda()
        out.put(("handle", rank, opt.ipc_handle()))
        while True:
            msg = cmd.get(timeout=300)
            kind = msg[0]
            if kind == "open":
                for q, h in msg[1]:
                    opt.open_peer(q, h)
                opt.connect()
            elif kind == "warm":
                opt.warmup_phase(msg[2], x, mine(gw[msg[1]]), LR)
            elif kind == "freeze":
                opt.freeze()
            elif kind == "step":
                opt.compressed_phase(msg[2], x, mine(gc[msg[1]]), LR)
            elif kind == "result":
                torch.cuda.synchronize()
                out.put(("result", rank, x.cpu().numpy(), opt.status()))
                continue
            elif kind == "close":
                torch.cuda.synchronize()
                opt.close()
                out.put(("closed", rank))
                return
            torch.cuda.synchronize()
            out.put(("done", rank))
    except Exception as e:  # report instead of leaving the host waiting
        out.put(("error", rank, repr(e)))


def _expect(out, what, rank):
    msg = out.get(timeout=300)
    assert msg[0] != "error", msg
    assert msg[0] == what and msg[1] == rank, msg
    return msg


@pytest.mark.parametrize("R", [2, 3])
def test_rank_processes_over_ipc_match_the_single_handle(R):
    W = 2 * R
    ctx = pymp.get_context("spawn")
    cmds = [ctx.Queue() for _ in range(R)]
    outs = [ctx.Queue() for _ in range(R)]
    procs = [ctx.Process(target=_rank, args=(r, R, W, cmds[r], outs[r])) for r in range(R)]
    for p in procs:
        p.start()
    try:
        handles = [_expect(outs[r], "handle", r)[2] for r in range(R)]
        for r in range(R):
            cmds[r].put(("open", [(q, handles[q]) for q in range(R) if q != r]))
            _expect(outs[r], "done", r)

        def run(kind, t):
            for phase in range(3):
                for r in range(R):          # phase p of every rank, each one finished
                    cmds[r].put((kind, t, phase))
                    _expect(outs[r], "done", r)

        for t in range(WARM):
            run("warm", t)
        for r in range(R):
            cmds[r].put(("freeze",))
            _expect(outs[r], "done", r)
        for t in range(STEPS):
            run("step", t)
        xs = []
        for r in range(R):
            cmds[r].put(("result",))
            msg = _expect(outs[r], "result", r)
            assert msg[3] == 0, "rank %d status flags %d" % (r, msg[3])
            xs.append(msg[2])
        for r in reversed(range(R)):        # every rank waits on the device, then lets go
            cmds[r].put(("close",))
            _expect(outs[r], "closed", r)
    finally:
        for p in procs:
            p.join(timeout=120)
            if p.is_alive():
                p.kill()
    for p in procs:
        assert p.exitcode == 0

    x0, gw, gc = _inputs(W)
    x = torch.from_numpy(x0).to(DEV)
    single = ob.OneBitAdam(D, W, C, B1, B2, EPS, device=DEV)
    for g in gw:
        single.warmup_step(x, torch.from_numpy(g).to(DEV), LR)
    single.freeze()
    for g in gc:
        single.step(x, torch.from_numpy(g).to(DEV), LR)
    ref = x.cpu().numpy()
    single.close()
    for r in range(R):
        assert np.array_equal(xs[r].view(np.uint32), ref.view(np.uint32)), "rank %d" % r
