"""Data-parallel ranks on the GPU: R ranks emulated as R handles on this GPU (their exchange
regions addressed directly, each step driven phase by phase across the ranks) against one
single-GPU handle with all W workers -- bit for bit, every step, in every piece of state -- and
one compressed step against the oracle. Also: the fused-barrier whole-step entry points at R = 1
(alone and through a torch.distributed group, which exercises the IPC handle export), the
phase-order rules, checkpoint/resume of ranks, a barrier whose peer never arrives (it gives up
after its timeout and sets the status flag; nothing hangs), and the BERT-Large bucket at full
size over 4 ranks."""
import dataclasses
import datetime
import os
import socket

import numpy as np
import pytest
import torch

import communication_compressed_optimizer_momentum_b200 as ob
from communication_compressed_optimizer_momentum_b200 import dp
from communication_compressed_optimizer_momentum_b200 import workloads as wls
from gpu_helpers import DEV, check_compressed_step, to_np

pytestmark = pytest.mark.gpu

F32 = wls.WORKLOADS["smoke_1m"]
BF16 = wls.WORKLOADS["bert_large_bucket"]


def _wl(base, d, W, C, **kw):
    return dataclasses.replace(base, name="dp_%d_%d_%d" % (d, W, C), d=d, W=W, C=C,
                               layer_sizes=(), **kw)


CASES = {
    "r1": (_wl(F32, 20_000, 4, 2048), 1),
    "r2": (_wl(F32, 65_536, 4, 8192), 2),
    "r2_ragged_unaligned": (_wl(F32, 100_003, 4, 4096), 2),     # d % 4 != 0: element loads
    "r3_bf16": (_wl(BF16, 98_321, 6, 4096, grad_kind="normal"), 3),
    "r4_w16_bf16": (_wl(BF16, 262_144, 16, 16_384), 4),
    "r4_fewer_chunks": (_wl(F32, 50_000, 8, 32_768), 4),        # 2 chunks: two ranks serve none
    "r8_one_worker_each": (_wl(F32, 131_168, 8, 8192), 8),
    "r2_w64": (_wl(F32, 40_000, 64, 4096), 2),                 # residuals not staged (W > 32)
    "r5_w10": (_wl(F32, 60_000, 10, 2048), 5),                  # W not a power of two
    "r3_spread": (_wl(F32, 30_000, 6, 1024, last_worker_sigma=1e-8), 3),  # in-order decode
    # the single handle's server uses bank-private tables and 16 segments per block; the ranks'
    # server blocks cover the same 16 segments with one-copy tables
    "r2_w64_bank_private": (_wl(F32, 300_000, 64, 131_072), 2),
    "r2_w30_bank_private_bf16": (_wl(BF16, 200_003, 30, 65_536, grad_kind="normal"), 2),
}

NAMES = ("m", "v", "e_w", "e_s", "s", "S", "bits_w", "bits_s")


def _rank_grads(g, R):
    """Rank r's [W / R][d] rows (views when they start 16-byte aligned, else copies)."""
    Wl = g.shape[0] // R
    out = []
    for r in range(R):
        v = g[r * Wl:(r + 1) * Wl]
        out.append(v if v.data_ptr() % 16 == 0 else v.clone())
    return out


def dp_state(em: dp.EmulatedRanks) -> dict:
    """The ranks' state assembled in the single-handle layout: per-worker rows in rank order,
    the server residual from each rank's own chunks, the replicated pieces from rank 0."""
    st = {}
    r0 = em.ranks[0]
    for nm in ("m", "v", "S", "bits_s"):
        st[nm] = r0.get_state(nm)
    for nm in ("e_w", "s", "bits_w"):
        st[nm] = torch.cat([o.get_state(nm) for o in em.ranks])
    st["e_s"] = torch.cat([o.get_state("e_s") for o in em.ranks])
    return st


def _same(a, b):
    if a.dtype == torch.float32:
        return torch.equal(a.view(torch.int32), b.view(torch.int32))
    return torch.equal(a, b)


def _assert_same_state(em, single, xs, x1, where):
    for r, xr in enumerate(xs):
        assert _same(xr, x1), "%s: rank %d's x differs from the single handle's" % (where, r)
    st = dp_state(em)
    for nm in NAMES:
        ref = single.get_state(nm)
        assert _same(st[nm], ref), "%s: state %s differs" % (where, nm)
    for r, o in enumerate(em.ranks):
        if r:
            for nm in ("m", "v", "S", "bits_s"):
                assert _same(o.get_state(nm), st[nm]), "%s: rank %d's %s" % (where, r, nm)


def run_against_single(wl, R, warm=3, steps=4, check_every=True):
    dt = wls.torch_dtype(wl)
    x1 = wls.torch_params(wl, DEV)
    xs = [x1.clone() for _ in range(R)]
    g = torch.empty((wl.W, wl.d), dtype=dt, device=DEV)
    single = ob.OneBitAdam(wl.d, wl.W, wl.C, wl.beta1, wl.beta2, wl.eps, grad_dtype=dt,
                           device=DEV)
    em = dp.EmulatedRanks(wl.d, wl.W, wl.C, R, wl.beta1, wl.beta2, wl.eps, grad_dtype=dt,
                          device=DEV)
    for t in range(warm):
        wls.torch_fill_grads(wl, g, 0, t)
        single.warmup_step(x1, g, wl.lr)
        em.warmup_step(xs, _rank_grads(g, R), wl.lr)
        for r in range(R):
            assert _same(xs[r], x1), "warm-up step %d: rank %d" % (t, r)
    single.freeze()
    em.freeze()
    for t in range(1, steps + 1):
        wls.torch_fill_grads(wl, g, 1, t)
        single.step(x1, g, wl.lr)
        em.step(xs, _rank_grads(g, R), wl.lr)
        if check_every or t == steps:
            _assert_same_state(em, single, xs, x1, "compressed step %d" % t)
    assert em.status() == 0 and single.status() == 0
    em.close()
    single.close()


@pytest.mark.parametrize("case", list(CASES))
def test_ranks_match_single_handle(case):
    wl, R = CASES[case]
    run_against_single(wl, R)


def test_rank_step_against_oracle():
    """One compressed step of 3 emulated ranks checked against the oracle from the ranks' own
    pre-step state (the teacher-forced check of the single-GPU parity tests)."""
    wl, R = _wl(F32, 24_000, 6, 2048), 3
    x = wls.torch_params(wl, DEV)
    xs = [x.clone() for _ in range(R)]
    g = torch.empty((wl.W, wl.d), dtype=torch.float32, device=DEV)
    em = dp.EmulatedRanks(wl.d, wl.W, wl.C, R, wl.beta1, wl.beta2, wl.eps, device=DEV)
    for t in range(2):
        wls.torch_fill_grads(wl, g, 0, t)
        em.warmup_step(xs, _rank_grads(g, R), wl.lr)
    em.freeze()
    for t in range(1, 4):
        wls.torch_fill_grads(wl, g, 1, t)
        pre = {k: to_np(v) for k, v in dp_state(em).items()}
        pre["x"] = to_np(xs[0])
        gn = to_np(g)
        em.step(xs, _rank_grads(g, R), wl.lr)
        post = {k: to_np(v) for k, v in dp_state(em).items()}
        post["x"] = to_np(xs[1])
        rep = check_compressed_step(pre, gn, post, wl.C, wl.beta1, wl.eps, wl.lr)
        assert rep.s_exact == rep.s_total and rep.S_exact == rep.S_total
    em.close()


def _fused_rank(wl, R=1):
    opt = dp.OneBitAdamRank(wl.d, wl.W, wl.C, R, 0, wl.beta1, wl.beta2, wl.eps, device=DEV)
    return opt


def test_whole_step_entry_points_one_rank():
    """R = 1 through onebit_adam_warmup_step / onebit_adam_compressed_step (each barrier is one
    launch that signals and waits) equals the single handle, and the launch count is 7."""
    wl = _wl(F32, 70_000, 4, 8192)
    x1 = wls.torch_params(wl, DEV)
    x2 = x1.clone()
    g = torch.empty((wl.W, wl.d), dtype=torch.float32, device=DEV)
    single = ob.OneBitAdam(wl.d, wl.W, wl.C, wl.beta1, wl.beta2, wl.eps, device=DEV)
    opt = _fused_rank(wl)
    opt.connect()
    assert opt.info()["launches_per_step"] == 7
    for t in range(2):
        wls.torch_fill_grads(wl, g, 0, t)
        single.warmup_step(x1, g, wl.lr)
        opt.warmup_step(x2, g, wl.lr)
    single.freeze()
    opt.freeze()
    opt.timing(3)
    for t in range(1, 4):
        wls.torch_fill_grads(wl, g, 1, t)
        single.step(x1, g, wl.lr)
        opt.step(x2, g, wl.lr)
    assert _same(x1, x2)
    ms, n = opt.timing_read()
    assert n == 3 and all(v > 0 for v in ms.values())
    assert opt.status() == 0
    opt.close()
    single.close()


def test_process_group_connect_world_one():
    """connect_process_group over a one-rank NCCL group: exports the exchange region's IPC
    handle, all-gathers it, connects, and steps."""
    import torch.distributed as dist
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True, timeout=datetime.timedelta(seconds=30))
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device(DEV))
    try:
        wl = _wl(F32, 30_000, 2, 4096)
        opt = _fused_rank(wl)
        h = opt.ipc_handle()
        assert isinstance(h, bytes) and len(h) == 64
        dp.connect_process_group(opt)
        x1 = wls.torch_params(wl, DEV)
        x2 = x1.clone()
        g = torch.empty((wl.W, wl.d), dtype=torch.float32, device=DEV)
        single = ob.OneBitAdam(wl.d, wl.W, wl.C, wl.beta1, wl.beta2, wl.eps, device=DEV)
        wls.torch_fill_grads(wl, g, 0, 0)
        single.warmup_step(x1, g, wl.lr)
        opt.warmup_step(x2, g, wl.lr)
        single.freeze()
        opt.freeze()
        for t in range(1, 3):
            wls.torch_fill_grads(wl, g, 1, t)
            single.step(x1, g, wl.lr)
            opt.step(x2, g, wl.lr)
        assert _same(x1, x2) and opt.status() == 0
        opt.close()
        single.close()
    finally:
        dist.destroy_process_group()


def test_phase_order_rules():
    wl, R = _wl(F32, 10_000, 4, 2048), 2
    x = wls.torch_params(wl, DEV)
    g = torch.zeros((wl.W // R, wl.d), dtype=torch.float32, device=DEV)
    unconnected = dp.OneBitAdamRank(wl.d, wl.W, wl.C, R, 0, device=DEV)
    with pytest.raises(ob.OneBitError) as e:
        unconnected.warmup_phase(0, x, g, 1e-3)
    assert e.value.code == -3                     # not connected
    with pytest.raises(ob.OneBitError):
        unconnected.connect()                     # peer 1 not set
    unconnected.close()
    em = dp.EmulatedRanks(wl.d, wl.W, wl.C, R, device=DEV)
    a = em.ranks[0]
    with pytest.raises(ob.OneBitError) as e:
        a.warmup_phase(1, x, g, 1e-3)             # phase 1 before phase 0
    assert e.value.code == -3
    with pytest.raises(ob.OneBitError) as e:
        a.compressed_phase(0, x, g, 1e-3)         # compressed before the freeze
    assert e.value.code == -3
    xs = [x.clone() for _ in range(R)]
    for r in range(R):
        em.ranks[r].warmup_phase(0, xs[r], g, 1e-3)
    with pytest.raises(ob.OneBitError) as e:
        a.freeze()                                # mid-step
    assert e.value.code == -3
    with pytest.raises(ob.OneBitError) as e:
        a.warmup_step(xs[0], g, 1e-3)             # whole step while a phased one is open
    assert e.value.code == -3
    for p in (1, 2):
        for r in range(R):
            em.ranks[r].warmup_phase(p, xs[r], g, 1e-3)
    em.freeze()
    assert em.status() == 0
    em.close()


def test_barrier_timeout_sets_flag_and_returns():
    """Rank 0 of 2 waits for rank 1, which never signals: the wait gives up after its timeout
    (2 ms here), the status carries ONEBIT_FLAG_TIMEOUT, and the device keeps working."""
    wl, R = _wl(F32, 8192, 2, 2048), 2
    em = dp.EmulatedRanks(wl.d, wl.W, wl.C, R, device=DEV)
    a = em.ranks[0]
    a.set_timeout_us(2000)
    x = wls.torch_params(wl, DEV)
    g = torch.zeros((1, wl.d), dtype=torch.float32, device=DEV)
    a.warmup_phase(0, x, g, 1e-3)
    a.warmup_phase(1, x, g, 1e-3)                 # waits for rank 1's phase 0: never comes
    torch.cuda.synchronize()
    flags = a.status()
    assert flags & 4, flags
    em.close()
    # the context is intact
    y = torch.randn(1000, device=DEV)
    words = ob.onebit_pack(y)
    assert words.numel() == 32


def test_rank_checkpoint_resume():
    wl, R = _wl(BF16, 40_960, 4, 4096, grad_kind="normal"), 2
    dt = torch.bfloat16
    x = wls.torch_params(wl, DEV)
    xa = [x.clone() for _ in range(R)]
    g = torch.empty((wl.W, wl.d), dtype=dt, device=DEV)
    A = dp.EmulatedRanks(wl.d, wl.W, wl.C, R, wl.beta1, wl.beta2, wl.eps, grad_dtype=dt,
                         device=DEV)
    for t in range(2):
        wls.torch_fill_grads(wl, g, 0, t)
        A.warmup_step(xa, _rank_grads(g, R), wl.lr)
    A.freeze()
    for t in range(1, 3):
        wls.torch_fill_grads(wl, g, 1, t)
        A.step(xa, _rank_grads(g, R), wl.lr)
    saved = [{nm: o.get_state(nm) for nm in ("m", "v", "e_w", "e_s")} for o in A.ranks]
    B = dp.EmulatedRanks(wl.d, wl.W, wl.C, R, wl.beta1, wl.beta2, wl.eps, grad_dtype=dt,
                         device=DEV)
    B.freeze()
    for o, st in zip(B.ranks, saved):
        for nm in ("m", "v", "e_w", "e_s"):
            o.set_state(nm, st[nm])
    xb = [t.clone() for t in xa]
    for t in range(3, 5):
        wls.torch_fill_grads(wl, g, 1, t)
        A.step(xa, _rank_grads(g, R), wl.lr)
        B.step(xb, _rank_grads(g, R), wl.lr)
    for r in range(R):
        assert _same(xa[r], xb[r])
    assert A.status() == 0 and B.status() == 0
    A.close()
    B.close()


def test_graph_replay_of_rank_steps():
    """A step of 2 emulated ranks captured in a CUDA graph and replayed equals eager steps: the
    barriers count in device memory, so a replay synchronizes like a new step."""
    wl, R = _wl(F32, 65_536, 4, 8192), 2
    x = wls.torch_params(wl, DEV)
    g = torch.empty((wl.W, wl.d), dtype=torch.float32, device=DEV)
    eager = dp.EmulatedRanks(wl.d, wl.W, wl.C, R, device=DEV)
    graphed = dp.EmulatedRanks(wl.d, wl.W, wl.C, R, device=DEV)
    xe = [x.clone() for _ in range(R)]
    xg = [x.clone() for _ in range(R)]
    wls.torch_fill_grads(wl, g, 0, 0)
    gs = _rank_grads(g, R)
    for em, xs in ((eager, xe), (graphed, xg)):
        em.warmup_step(xs, gs, wl.lr)
        em.freeze()
        em.step(xs, gs, wl.lr)          # the first step reads the explicit warm-up momentum
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        graphed.step(xg, gs, wl.lr)
    torch.cuda.synchronize()
    for t in range(4):
        wls.torch_fill_grads(wl, g, 1, t + 2)    # new values in the captured buffers
        gs2 = _rank_grads(g, R)
        assert all(a.data_ptr() == b.data_ptr() for a, b in zip(gs, gs2))
        eager.step(xe, gs, wl.lr)
        graph.replay()
        torch.cuda.synchronize()
        for r in range(R):
            assert _same(xe[r], xg[r]), "replay %d, rank %d" % (t, r)
    assert eager.status() == 0 and graphed.status() == 0
    del graph
    eager.close()
    graphed.close()


@pytest.mark.slow
def test_bert_large_bucket_four_ranks():
    """The BERT-Large bucket (333.6M parameters, 16 workers, bf16) over 4 emulated ranks equals
    the single handle bit for bit after the warm-up and two compressed steps (x, all state)."""
    wl = dataclasses.replace(BF16, warmup_steps=1, compressed_steps=2)
    free, _ = torch.cuda.mem_get_info()
    if free < 110e9:
        pytest.skip("needs about 110 GB of free device memory")
    run_against_single(wl, 4, warm=1, steps=2, check_every=False)


def test_bench_dp_line():
    """bench.py --dp 2 (two emulated ranks) prints one JSON line with the data-parallel step's
    throughput, its roofline against the data-parallel byte count and the single-GPU step."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--dp", "2",
                        "--workload", "smoke_1m", "--steps", "5", "--warmup", "3"],
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["value"] > 0 and line["status_flags"] == 0
    assert line["config"]["parallelism"] == "dp2 emulated on one GPU"
    assert line["config"]["workers_per_rank"] == 2
    assert line["gpu_launches"] == 9 * 2 * 5
    assert line["single_gpu_ms_per_step"] > 0
    wl = wls.WORKLOADS["smoke_1m"]
    assert line["algorithmic_bytes_per_step"] == wl.dp_algorithmic_bytes_per_param(2) * wl.d
    assert line["nvlink"]["bytes_per_rank_per_step"] == wl.dp_nvlink_bytes_per_rank(2)


def test_bench_dp_under_torchrun_one_process():
    """bench.py --dp under torchrun takes the one-process-per-rank path (NCCL process group,
    IPC handle exchange, whole-step entry points with one barrier launch each), here with one
    rank on this GPU."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
                        "--nproc-per-node", "1", "--master-addr", "127.0.0.1",
                        "--master-port", str(port), os.path.join(root, "bench.py"), "--dp", "1",
                        "--workload", "smoke_1m", "--steps", "5", "--warmup", "3"],
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["config"]["parallelism"] == "dp1" and line["scaling"] == "strong"
    assert line["gpu_launches"] == 7 * 5 and line["status_flags"] == 0
    assert line["value"] > 0 and line["rank0_kernel_ms_per_step"]["worker"] > 0


def test_host_buffer_step_of_a_rank():
    """onebit_adam_compressed_step_host on a one-rank handle (upload, step with its barriers,
    read-back of x) gives the single-GPU handle's x."""
    wl = _wl(F32, 50_000, 4, 8192)
    x1 = wls.torch_params(wl, DEV)
    x2 = x1.clone()
    g = torch.empty((wl.W, wl.d), dtype=torch.float32, device=DEV)
    single = ob.OneBitAdam(wl.d, wl.W, wl.C, wl.beta1, wl.beta2, wl.eps, device=DEV)
    opt = _fused_rank(wl)
    opt.connect()
    wls.torch_fill_grads(wl, g, 0, 0)
    single.warmup_step(x1, g, wl.lr)
    opt.warmup_step(x2, g, wl.lr)
    single.freeze()
    opt.freeze()
    g_host = torch.empty((wl.W, wl.d), dtype=torch.float32, pin_memory=True)
    x_host = torch.empty(wl.d, dtype=torch.float32, pin_memory=True)
    g_dev = torch.empty_like(g)
    for t in range(1, 4):
        wls.torch_fill_grads(wl, g, 1, t)
        g_host.copy_(g)
        single.step(x1, g, wl.lr)
        opt.step_host(x2, g_dev, g_host, x_host, wl.lr)
        opt.host_wait()
        torch.cuda.synchronize()
        assert torch.equal(x_host.view(torch.int32), x1.cpu().view(torch.int32)), t
    assert opt.status() == 0
    opt.close()
    single.close()


def test_empty_vector_ranks():
    """d = 0: every phase and step of the ranks is a no-op that succeeds."""
    em = dp.EmulatedRanks(0, 4, 64, 2, device=DEV)
    xs = [torch.empty(0, device=DEV) for _ in range(2)]
    gs = [torch.empty((2, 0), device=DEV) for _ in range(2)]
    em.warmup_step(xs, gs, 1e-3)
    em.freeze()
    em.step(xs, gs, 1e-3)
    assert em.status() == 0
    assert all(o.info()["steps"] == 1 for o in em.ranks)
    em.close()
