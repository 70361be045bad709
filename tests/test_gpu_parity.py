"""CUDA path vs the CPU oracle through the C ABI, at sizes the oracle finishes in seconds
(several segments and chunks, ragged tails, every code path of the kernels), plus the
library's own properties: determinism, checkpoint/resume, the host-buffer entry point, status
flags, phase and alignment errors, per-kernel timing."""
import dataclasses
import json
import os

import numpy as np
import pytest
import torch

import communication_compressed_optimizer_momentum_b200 as ob
import oracle
from communication_compressed_optimizer_momentum_b200 import workloads as wls
from gpu_helpers import DEV, padding_is_zero, run_parity, to_np

pytestmark = pytest.mark.gpu

BASE = wls.WORKLOADS["smoke_1m"]


def small(d, W, C, dt="f32", kind="normal", warm=3, comp=5, seed=7, **kw):
    name = "small_d%d_W%d_C%d_%s" % (d, W, C, dt) + "".join("_%s%g" % i for i in kw.items())
    return dataclasses.replace(BASE, name=name, d=d, W=W, C=C, grad_dtype=dt, grad_kind=kind,
                               warmup_steps=warm, compressed_steps=comp, seed=seed,
                               layer_sizes=(), **kw)


SMALL = [
    small(50_000, 3, 4096),                   # C does not divide d; many segments
    small(50_001, 2, 8192),                   # d % 4 != 0: scalar gradient loads; d % 32 != 0
    small(70_003, 5, 16_384, "bf16"),         # bf16, ragged
    small(10_000, 1, 32),                     # W = 1, one-word chunks
    small(100_000, 64, 100_000),              # W = 64, one chunk of 25 segments
    small(1000, 7, 1 << 20, "bf16"),          # C > d: one short chunk
    small(262_161, 16, 65_536, "bf16", "outlier_normal"),
    small(33, 4, 32),                         # last chunk of one element
    small(200_000, 8, 8192, "f32", "edge_normal"),
    small(300_000, 4, 1 << 17, "bf16", "student_t"),
    small(60_000, 12, 8192),                  # W > 8, not a power of 2: exact division by W
    small(60_000, 24, 16_384, "bf16"),
    # one worker's scale far below the others' (beta1 = 0, so x_w follows g_w): the server's
    # integer tables no longer fit (fp64 tables), or the fp64 sum is no longer provably exact
    # (in-order decode)
    small(40_000, 16, 8192, beta1=0.0, last_worker_sigma=1e-2),
    small(40_000, 16, 8192, beta1=0.0, last_worker_sigma=1e-10),
    small(40_000, 12, 8192, beta1=0.0, last_worker_sigma=1e-10),
    # bank-private server tables: 4 groups with W not a power of two (8 segments per block),
    # 8 groups with a ragged last chunk (16 segments per block)
    small(150_000, 30, 40_000, "bf16"),
    small(300_007, 60, 69_984),
    # the same bank-private kernel in the fp64-table and in-order decodes
    small(120_000, 30, 40_000, beta1=0.0, last_worker_sigma=1e-2),
    small(120_000, 30, 40_000, beta1=0.0, last_worker_sigma=1e-10),
]


@pytest.mark.parametrize("wl", SMALL, ids=[w.name for w in SMALL])
def test_compressed_parity_small(wl):
    st = run_parity(wl, chunks=None, teacher_steps=tuple(range(1, wl.compressed_steps + 1)),
                    free_steps=wl.compressed_steps)
    if wl.last_worker_sigma < 1e-6:
        # the scale spread breaks the exactness bound: the in-order decode was exercised
        assert st["inexact_chunks"] > 0
    else:
        assert st["inexact_chunks"] == 0
    assert st["status_flags"] == 0


def test_two_group_bank_private_tables_sampled():
    """The bank-private tables of 2 groups need at least 2048 x 8 server segments in all: W = 12
    (not a power of two) over 2^26 + 4099 parameters in 2^18-element chunks (257 chunks of 64
    segments, streamed 16 per block), checked on sampled chunks including the ragged last
    one."""
    wl = small((1 << 26) + 4099, 12, 1 << 18, "bf16", "outlier_normal", warm=2, comp=3)
    free, _ = torch.cuda.mem_get_info()
    if free < 8e9:
        pytest.skip("needs about 8 GB of free device memory")
    assert wl.nch * (((wl.C + 4095) // 4096 + 7) // 8) >= 2048
    st = run_parity(wl, chunks=[0, 1, wl.nch - 1], teacher_steps=(1, 2, 3), free_steps=0)
    assert st["inexact_chunks"] == 0 and st["status_flags"] == 0


def test_smoke_1m_workload():
    """The 1,048,576-parameter W=4 workload in full: 20 warm-up steps (last one bit-exact),
    10 compressed steps, each teacher forced on every chunk, and 10 free-running steps."""
    wl = wls.WORKLOADS["smoke_1m"]
    st = run_parity(wl, chunks=None, teacher_steps=tuple(range(1, 11)), free_steps=10)
    assert st["inexact_chunks"] == 0


def test_exact_zero_edge_cases():
    """No warm-up (m = 0) and zero residuals: exact-zero gradients give x = 0 exactly, which
    takes bit 1; an all-zero chunk has scale 0 and residual +0. None of these are ties, so the
    GPU must match the oracle bit for bit there."""
    d, W, C = 8192, 3, 1024
    g = np.random.default_rng(0).standard_normal((W, d)).astype(np.float32) * 1e-2
    g[:, 1024:2048] = 0.0                     # an all-zero chunk
    g[np.random.default_rng(1).random((W, d)) < 0.05] = 0.0
    g[0, 5000:5010] = -0.0
    x = torch.full((d,), 0.01, device=DEV)
    gt = torch.from_numpy(g).to(DEV)
    opt = ob.OneBitAdam(d, W, C, device=DEV)
    opt.set_state("v", torch.ones(d, device=DEV))
    opt.freeze()
    opt.step(x, gt, 1e-3)
    xo = np.full(d, 0.01, np.float32)
    mo = np.zeros(d, np.float32)
    ew = np.zeros((W, d), np.float32)
    es = np.zeros(d, np.float32)
    out = oracle.compressed_step(xo, mo, np.ones(d, np.float32), ew, es, g, C, 0.9, 1e-8, 1e-3)
    np.testing.assert_array_equal(to_np(opt.get_state("bits_w")), out["bits_w"])
    np.testing.assert_array_equal(to_np(opt.get_state("s")), out["s"])
    assert (to_np(opt.get_state("s"))[:, 1] == 0).all()
    ewg = to_np(opt.get_state("e_w"))
    assert not np.signbit(ewg[:, 1024:2048]).any() and (ewg[:, 1024:2048] == 0).all()
    np.testing.assert_array_equal(to_np(opt.get_state("bits_s")), out["bits_s"])
    np.testing.assert_array_equal(to_np(x), xo)
    opt.close()


def test_hand_case_on_gpu():
    """The hand-derived d=8, W=2 step (tests/golden) through the C ABI."""
    case = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                       "hand_case_d8_w2.json")))
    inp, exp = case["inputs"], case["expected"]
    d, W, C = inp["d"], inp["W"], 32          # the library needs C % 32 == 0; one chunk of 8
    g = torch.tensor(inp["g"], dtype=torch.float32, device=DEV)
    x = torch.zeros(d, device=DEV)
    opt = ob.OneBitAdam(d, W, C, beta1=inp["beta1"], eps=inp["eps"], device=DEV)
    opt.set_state("v", torch.ones(d, device=DEV))
    opt.freeze()
    opt.step(x, g, inp["lr"])
    # with one chunk of 8 the scales differ from the golden C=4 case; check against the oracle
    # on the same single-chunk split and against the C=4 golden words via the oracle pins
    xo = np.zeros(d, np.float32)
    mo = np.zeros(d, np.float32)
    ew = np.zeros((W, d), np.float32)
    es = np.zeros(d, np.float32)
    out = oracle.compressed_step(xo, mo, np.ones(d, np.float32), ew, es,
                                 np.array(inp["g"], np.float32), C, inp["beta1"], inp["eps"],
                                 inp["lr"])
    np.testing.assert_array_equal(to_np(opt.get_state("bits_w")).ravel(), out["bits_w"].ravel())
    np.testing.assert_array_equal(to_np(opt.get_state("bits_w")).ravel(),
                                  np.array(exp["bits_w"], np.uint32).ravel())
    np.testing.assert_array_equal(to_np(opt.get_state("s")), out["s"])
    np.testing.assert_array_equal(to_np(opt.get_state("e_w")), ew)
    np.testing.assert_array_equal(to_np(x), xo)
    opt.close()


@pytest.mark.parametrize("n", [0, 1, 31, 32, 33, 4095, 4097, 100_003, 1 << 20])
def test_pack_unpack_parity(n):
    rng = np.random.default_rng(n)
    x = rng.standard_normal(max(n, 1)).astype(np.float32)[:n]
    if n:
        x[rng.random(n) < 0.05] = 0.0
        x[rng.random(n) < 0.05] = -0.0
        x[rng.random(n) < 0.01] = np.nan
    xt = torch.from_numpy(x).to(DEV)
    words = ob.onebit_pack(xt)
    torch.cuda.synchronize()
    w = to_np(words)
    np.testing.assert_array_equal(w, oracle.pack(x))
    assert padding_is_zero(w, n) or n == 0
    for C in (32, 4096, 1000, max(n, 1)):
        sc = rng.random((n + C - 1) // C).astype(np.float32) if n else np.zeros(1, np.float32)
        out = ob.onebit_unpack(words, torch.from_numpy(sc).to(DEV), n, C)
        np.testing.assert_array_equal(to_np(out), oracle.unpack(w, sc, n, C))


def _run_steps(opt, x, g_list, lr):
    for g in g_list:
        opt.step(x, g, lr)


def _grads(W, d, n, seed, dt=torch.float32):
    gen = torch.Generator(device=DEV)
    gen.manual_seed(seed)
    return [(torch.randn(W, d, device=DEV, generator=gen) * 1e-2).to(dt) for _ in range(n)]


def test_run_to_run_bit_identical():
    d, W, C = 300_000, 8, 65_536
    gl = _grads(W, d, 4, 1)
    res = []
    for _ in range(2):
        x = torch.linspace(-0.05, 0.05, d, device=DEV)
        opt = ob.OneBitAdam(d, W, C, device=DEV)
        opt.warmup_step(x, gl[0], 1e-3)
        opt.freeze()
        _run_steps(opt, x, gl[1:], 1e-3)
        res.append([to_np(x)] + [to_np(opt.get_state(k)) for k in ("m", "e_w", "e_s", "s", "S")])
        opt.close()
    for a, b in zip(*res):
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


def test_checkpoint_resume_bit_identical():
    """A fresh handle given m, v, e_w, e_s of a running one continues bit for bit."""
    d, W, C = 123_457, 5, 32_768
    gl = _grads(W, d, 7, 2, torch.bfloat16)
    x = torch.linspace(-0.05, 0.05, d, device=DEV)
    a = ob.OneBitAdam(d, W, C, grad_dtype=torch.bfloat16, device=DEV)
    a.warmup_step(x, gl[0], 1e-3)
    a.freeze()
    _run_steps(a, x, gl[1:4], 1e-3)
    ck = {k: a.get_state(k) for k in ("m", "v", "e_w", "e_s")}
    x_ck = x.clone()
    b = ob.OneBitAdam(d, W, C, grad_dtype=torch.bfloat16, device=DEV)
    b.freeze()
    for k, t in ck.items():
        b.set_state(k, t)
    _run_steps(a, x, gl[4:], 1e-3)
    _run_steps(b, x_ck, gl[4:], 1e-3)
    assert torch.equal(x, x_ck)
    for k in ("m", "e_w", "e_s", "bits_w", "bits_s"):
        assert torch.equal(a.get_state(k), b.get_state(k)), k
    a.close()
    b.close()


def test_host_entry_matches_device_entry():
    d, W, C = 99_999, 3, 8192
    gl = _grads(W, d, 3, 3)
    xa = torch.linspace(-0.05, 0.05, d, device=DEV)
    xb = xa.clone()
    a = ob.OneBitAdam(d, W, C, device=DEV)
    b = ob.OneBitAdam(d, W, C, device=DEV)
    for o in (a, b):
        o.freeze()
    gdev = torch.empty(W, d, device=DEV)
    x_host = torch.empty(d, pin_memory=True)
    for g in gl:
        a.step(xa, g, 1e-3)
        g_host = g.cpu().pin_memory()
        b.step_host(xb, gdev, g_host, x_host, 1e-3)
        b.host_wait()
        torch.cuda.current_stream().synchronize()
        assert torch.equal(x_host, xa.cpu())
    assert torch.equal(xa, xb)
    # back-to-back host steps: each read-back overlaps the next upload; the results still match
    hosts = [g.cpu().pin_memory() for g in gl]
    outs = [torch.empty(d, pin_memory=True) for _ in gl]
    for g, gh, xo in zip(gl, hosts, outs):
        a.step(xa, g, 1e-3)
        b.step_host(xb, gdev, gh, xo, 1e-3)
    b.host_wait()
    torch.cuda.current_stream().synchronize()
    assert torch.equal(outs[-1], xa.cpu())
    assert torch.equal(xa, xb)
    a.close()
    b.close()


def test_nan_gradient_sets_status_flag():
    d, W, C = 4096, 2, 1024
    g = torch.randn(W, d, device=DEV) * 1e-2
    g[1, 7] = float("nan")
    x = torch.zeros(d, device=DEV)
    opt = ob.OneBitAdam(d, W, C, device=DEV)
    opt.freeze()
    assert opt.status() == 0
    opt.step(x, g, 1e-3)
    flags = opt.status()
    assert flags & ob.FLAG_NAN_WORKER
    bits = to_np(opt.get_state("bits_w"))
    assert (bits[1, 0] >> 7) & 1 == 0
    assert opt.status() == 0        # cleared by the read
    opt.close()


def test_phase_and_alignment_errors():
    d, W, C = 1024, 2, 512
    x = torch.zeros(d + 4, device=DEV)
    g = torch.zeros(W, d, device=DEV)
    opt = ob.OneBitAdam(d, W, C, device=DEV)
    with pytest.raises(ob.OneBitError) as e:
        opt.step(x[:d], g, 1e-3)
    assert e.value.code == -3
    with pytest.raises(ob.OneBitError) as e:
        opt.warmup_step(x[1:d + 1], g, 1e-3)       # 4-byte offset: not 16-byte aligned
    assert e.value.code == -2
    opt.freeze()
    with pytest.raises(ob.OneBitError) as e:
        opt.freeze()
    assert e.value.code == -3
    with pytest.raises(ob.OneBitError) as e:
        opt.warmup_step(x[:d], g, 1e-3)
    assert e.value.code == -3
    opt.step(x[:d], g, 1e-3)
    opt.close()


def test_empty_vector_steps_are_noops():
    opt = ob.OneBitAdam(0, 3, 64, device=DEV)
    x = torch.zeros(4, device=DEV)
    g = torch.zeros(3, 4, device=DEV)
    opt.warmup_step(x, g, 1e-3)
    opt.freeze()
    opt.step(x, g, 1e-3)
    assert opt.info()["steps"] == 1
    opt.close()


def test_timing_reports_each_kernel():
    d, W, C = 1 << 20, 4, 1 << 18
    gl = _grads(W, d, 3, 4)
    x = torch.zeros(d, device=DEV)
    opt = ob.OneBitAdam(d, W, C, device=DEV)
    opt.freeze()
    opt.timing(2)
    _run_steps(opt, x, gl, 1e-3)             # third step is past the window
    per_step = opt.timing_steps()
    ms, n = opt.timing_read()
    assert n == 2 and len(per_step) == 2
    assert all(v > 0 for v in ms.values()), ms
    # a step's first-to-last event time holds its kernels' intervals
    assert abs(sum(per_step) - sum(ms.values())) <= 1e-3 * sum(ms.values()) + 1e-3
    opt.timing(0)
    opt.close()


def test_bounded_wait_gives_up_and_the_context_survives():
    """Failure detection without a GPU fault: a wait on bytes that never arrive expires after
    its bound, the kernel returns, and the device keeps working."""
    assert ob.onebit_selftest_bounded_wait(1000)
    assert ob.onebit_selftest_bounded_wait(20_000)
    x = torch.ones(4096, device=DEV)
    words = ob.onebit_pack(x)
    torch.cuda.synchronize()
    assert int(words[0].item()) == -1          # all 32 signs positive


def test_bench_json_line_contract(tmp_path):
    """bench.py prints one JSON line with the keys the benchmark contract names."""
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--workload", "smoke_1m",
                        "--steps", "3", "--warmup", "3", "--e2e-steps", "1",
                        "--cpu-seconds", "0.2"], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "roofline", "cpu_baseline", "e2e", "clocks", "gpu_launches"):
        assert key in j, key
    assert j["value"] > 0 and j["steps"] == 3 and j["n_gpus"] == 1
    assert j["config"]["workload"] == "smoke_1m"
    # three launches per step: both chunk-scale reductions fold into the server and apply
    # kernels at this size (a chunk has 8 server blocks)
    assert j["gpu_launches"] == 9
    roof = j["roofline"]
    assert roof["bound"] == "hbm" and roof["unit"] == "GB/s" and roof["peak"] > 0
    assert abs(roof["frac"] - roof["achieved"] / roof["peak"]) < 1e-9
    assert j["e2e"]["h2d_bytes_per_step"] == 4 * 1_048_576 * 4
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["cores"] == 1
    dist = j["step_ms_distribution"]
    assert dist["steps"] == 3 and 0 < dist["p10"] <= dist["p50"] <= dist["p90"]
    assert abs(j["compression_ratio"] - 4.0 * 1_048_576 / (1_048_576 / 8 + 4 * 4)) < 1e-9


def test_cuda_graph_replay_matches_eager():
    """A compressed step queues kernels only (no host synchronisation), so it can be captured
    in a CUDA graph. After the first step (which reads the explicit warm-up momentum) every step
    launches the same kernels, so replays of a captured step equal eager steps bit for bit."""
    d, W, C = 200_000, 4, 16_384
    gl = _grads(W, d, 6, 5)
    g_static = torch.empty_like(gl[0])
    xa = torch.linspace(-0.05, 0.05, d, device=DEV)
    xb = xa.clone()
    a = ob.OneBitAdam(d, W, C, device=DEV)
    b = ob.OneBitAdam(d, W, C, device=DEV)
    for o in (a, b):
        o.freeze()
    a.step(xa, gl[0], 1e-3)
    b.step(xb, gl[0], 1e-3)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    g_static.copy_(gl[1])
    torch.cuda.synchronize()
    with torch.cuda.graph(graph, stream=s):
        b.step(xb, g_static, 1e-3)
    # capture records the launches without running them: replay once per step from here on
    for g in gl[1:]:
        a.step(xa, g, 1e-3)
        g_static.copy_(g)
        graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(xa, xb)
    for k in ("m", "e_w", "e_s", "bits_s"):
        assert torch.equal(a.get_state(k), b.get_state(k)), k
    del graph
    a.close()
    b.close()
