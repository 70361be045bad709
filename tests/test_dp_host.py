"""Data-parallel ranks without a GPU: the chunk partition, the host-side checks of the
``onebit_dp_*`` entry points, and -- on gloo ranks -- that splitting the compressed step the way
the ranks do (workers per rank, servers per chunk range, an exchange of plane slices and scales,
a broadcast of the server plane) reproduces the single-process oracle step exactly.

The decomposition test uses the oracle only (the CUDA path needs a GPU); it pins the
decomposition the data-parallel kernels rely on, with the library's own chunk ranges. The last
test runs ``connect_process_group`` on three gloo ranks with a stand-in for the rank handle and
checks that every rank maps every other rank's exchange region from that rank's IPC handle."""
import ctypes
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import communication_compressed_optimizer_momentum_b200 as ob
from communication_compressed_optimizer_momentum_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from communication_compressed_optimizer_momentum_b200 import build
    build.build()
    return _abi.lib()


@pytest.mark.parametrize("R", [1, 2, 3, 5, 8])
def test_chunk_ranges_partition_the_chunks(lib, R):
    for nch in (0, 1, 2, 3, 7, 8, 9, 16, 100, 1001):
        bounds = [ob.onebit_dp_chunk_range(nch, R, q) for q in range(R)]
        assert bounds[0][0] == 0 and bounds[-1][1] == nch
        for (a0, a1), (b0, b1) in zip(bounds, bounds[1:]):
            assert a1 == b0                            # contiguous, in rank order
        sizes = [k1 - k0 for k0, k1 in bounds]
        assert max(sizes) - min(sizes) <= 1            # balanced
        if nch == R:
            assert bounds == [(q, q + 1) for q in range(R)]   # rank r serves chunk r


def test_chunk_range_arguments(lib):
    k0, k1 = ctypes.c_int64(), ctypes.c_int64()
    for args in ((10, 0, 0), (10, 9, 0), (10, 2, 2), (10, 2, -1), (-1, 2, 0)):
        assert lib.onebit_dp_chunk_range(*args, ctypes.byref(k0), ctypes.byref(k1)) == -1, args
    assert lib.onebit_dp_chunk_range(10, 2, 0, None, ctypes.byref(k1)) == -1


def test_dp_init_validates_arguments(lib):
    h = ctypes.c_void_p()
    good = (10_000, 8, 1024, 0.9, 0.999, 1e-8)
    assert lib.onebit_dp_init(ctypes.byref(h), *good, 4, 3) == 0 and h.value
    info = ob.onebit_dp_info(h)
    assert (info["R"], info["rank"], info["W"]) == (4, 3, 8)
    assert ob.onebit_adam_info(h)["W"] == 2            # this rank's own workers
    nch = 10
    assert (info["k0"], info["k1"]) == ob.onebit_dp_chunk_range(nch, 4, 3)
    assert info["e0"] == info["k0"] * 1024
    assert info["d_own"] == 10_000 - info["e0"]        # the last rank holds the ragged tail
    assert info["exchange_bytes"] > 16 * 10_000        # m, v (fp32) and the fp64 sums at least
    lib.onebit_adam_destroy(h)
    bad = [
        (good + (0, 0), -1),        # no ranks
        (good + (9, 0), -1),        # more ranks than the route holds
        (good + (4, 4), -1),        # rank out of range
        (good + (3, 0), -1),        # workers not divisible by ranks
        ((10_000, 8, 100, 0.9, 0.999, 1e-8, 2, 0), -2),   # chunk not a multiple of 32
        ((10_000, 512, 1024, 0.9, 0.999, 1e-8, 2, 0), -1),  # too many workers
    ]
    for args, code in bad:
        h = ctypes.c_void_p()
        assert lib.onebit_dp_init(ctypes.byref(h), *args) == code, args
        assert not h.value


def test_dp_calls_before_bind_and_on_single_handles(lib):
    h = ob.onebit_dp_init(4096, 4, 1024, 0.9, 0.999, 1e-8, 2, 0)
    base, n = ctypes.c_void_p(), ctypes.c_uint64()
    assert lib.onebit_dp_exchange(h, ctypes.byref(base), ctypes.byref(n)) == -3  # no region yet
    assert lib.onebit_dp_ipc_handle(h, ctypes.create_string_buffer(64)) == -3
    assert lib.onebit_dp_connect(h, None) == -3
    assert lib.onebit_dp_set_peer(h, 0, ctypes.c_void_p(0x100000)) == -1   # itself
    assert lib.onebit_dp_set_peer(h, 2, ctypes.c_void_p(0x100000)) == -1   # no such rank
    assert lib.onebit_dp_set_peer(h, 1, ctypes.c_void_p(0x100010)) == -2   # misaligned
    assert lib.onebit_dp_set_timeout(h, 0) == -1
    assert lib.onebit_dp_set_timeout(h, 1000) == 0
    lr = ctypes.c_float(1e-3)
    for fn in (lib.onebit_dp_warmup_phase, lib.onebit_dp_compressed_phase):
        assert fn(h, 0, None, None, lr, None) == -3        # unbound
        assert fn(h, 3, None, None, lr, None) == -1        # no such phase
    assert lib.onebit_adam_compressed_step(h, None, None, lr, None) == -3
    ob.onebit_adam_destroy(h)
    single = ob.onebit_adam_init(4096, 4, 1024)
    assert lib.onebit_dp_info(single, (ctypes.c_int64 * 8)()) == -1
    assert lib.onebit_dp_compressed_phase(single, 0, None, None, lr, None) == -1
    ob.onebit_adam_destroy(single)


def test_dp_state_sizes(lib):
    d, W, C, R = 1000, 4, 256, 2                      # chunks 0,1 | 2,3 (232 elements)
    sizes = {}
    for r in range(R):
        h = ob.onebit_dp_init(d, W, C, 0.9, 0.999, 1e-8, R, r)
        sizes[r] = {k: ob.onebit_adam_state_bytes(h, ob.STATE[k]) for k in ob.STATE}
        ob.onebit_adam_destroy(h)
    for r in range(R):
        assert sizes[r]["m"] == sizes[r]["v"] == d * 4
        assert sizes[r]["e_w"] == (W // R) * d * 4
        assert sizes[r]["s"] == (W // R) * 4 * 4
        assert sizes[r]["S"] == 4 * 4 and sizes[r]["bits_s"] == 32 * 4
    assert sizes[0]["e_s"] == 512 * 4 and sizes[1]["e_s"] == (d - 512) * 4


# ----------------------------------------------------------------------------------------------
# the decomposition on gloo ranks, against the single-process oracle

D, W, C, STEPS = 5000, 4, 384, 3           # 14 chunks, the last one ragged
B1, EPS, LR = 0.9, 1e-8, 1e-3


def _inputs():
    rng = np.random.default_rng(20260402)
    g = (rng.standard_normal((STEPS, W, D)) * 1e-2).astype(np.float32)
    x = rng.standard_normal(D).astype(np.float32)
    m = (rng.standard_normal(D) * 1e-3).astype(np.float32)
    v = (rng.random(D) * 1e-4 + 1e-6).astype(np.float32)
    return g, x, m, v


def _gather(t, world):
    out = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(out, t)
    return out


def _rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import oracle
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    g, x, m, v = _inputs()
    Wl = W // world
    nch = oracle.nchunks(D, C)
    k0, k1 = ob.onebit_dp_chunk_range(nch, world, rank)
    e0, e1 = k0 * C, min(k1 * C, D)
    e_w = np.zeros((Wl, D), np.float32)                 # this rank's workers' residuals
    e_s = np.zeros(e1 - e0, np.float32)                 # this rank's chunks' server residual
    for t in range(STEPS):
        s, bits = oracle.worker(m, g[t, rank * Wl:(rank + 1) * Wl], e_w, C, B1)
        # exchange: every rank's planes and scales; this rank keeps the slice of its chunks
        s_all = torch.cat(_gather(torch.from_numpy(s), world)).numpy()
        b_all = torch.cat(_gather(torch.from_numpy(bits.view(np.int32)), world)).numpy()
        s_own = np.ascontiguousarray(s_all[:, k0:k1])
        b_own = np.ascontiguousarray(b_all[:, e0 // 32:(e1 + 31) // 32]).view(np.uint32)
        if e1 > e0:
            S_own, bs_own, _, _ = oracle.server(s_own, b_own, e_s, C)
        else:
            S_own, bs_own = np.zeros(0, np.float32), np.zeros(0, np.uint32)
        # broadcast of the server plane and scales (uneven pieces: gathered as objects)
        pieces = [None] * world
        dist.all_gather_object(pieces, (k0, S_own, bs_own))
        S = np.zeros(nch, np.float32)
        bits_s = np.zeros(oracle.nwords(D), np.uint32)
        for (p0, Sp, bp) in pieces:
            S[p0:p0 + Sp.size] = Sp
            bits_s[p0 * C // 32:p0 * C // 32 + bp.size] = bp
        oracle.apply(bits_s, S, v, m, x, C, EPS, LR)
    q.put((rank, x.copy(), m.copy(), e_w.copy(), e_s.copy(), e0, e1))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_rank_decomposition_matches_the_single_process_step(lib, world):
    sys.path.insert(0, ROOT)
    import oracle
    g, x, m, v = _inputs()
    e_w = np.zeros((W, D), np.float32)
    e_s = np.zeros(D, np.float32)
    for t in range(STEPS):
        oracle.compressed_step(x, m, v, e_w, e_s, g[t], C, B1, EPS, LR)

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    Wl = W // world
    for rank, xr, mr, ewr, esr, e0, e1 in out:
        assert np.array_equal(xr.view(np.uint32), x.view(np.uint32))   # every replica of x
        assert np.array_equal(mr.view(np.uint32), m.view(np.uint32))
        assert np.array_equal(ewr, e_w[rank * Wl:(rank + 1) * Wl])
        assert np.array_equal(esr, e_s[e0:e1])


# ----------------------------------------------------------------------------------------------
# connect_process_group's exchange of IPC handles, on gloo ranks with a stand-in handle


class _StubRank:
    """Records what connect_process_group asks of a rank's handle (no GPU needed)."""

    def __init__(self, R, rank):
        self.R, self.rank = R, rank
        self.opened = {}
        self.connected = False

    def ipc_handle(self):
        return bytes([self.rank]) * 64

    def open_peer(self, q, handle):
        self.opened[q] = handle

    def connect(self, stream=None):
        self.connected = True


def _connect_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    from communication_compressed_optimizer_momentum_b200 import dp
    torch.cuda.synchronize = lambda *a, **k: None       # no device in this test
    stub = _StubRank(world, rank)
    dp.connect_process_group(stub)
    bad = _StubRank(world + 1, rank)
    try:
        dp.connect_process_group(bad)
        mismatch = False
    except ValueError:
        mismatch = True
    q.put((rank, sorted(stub.opened.items()), stub.connected, mismatch))
    dist.barrier()
    dist.destroy_process_group()


def test_connect_process_group_routes_every_peer_handle(lib):
    world = 3
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    procs = [ctx.Process(target=_connect_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, opened, connected, mismatch in out:
        assert connected and mismatch
        assert opened == [(p, bytes([p]) * 64) for p in range(world) if p != rank]


def test_python_rank_classes_check_arguments_on_the_host(lib):
    """Bad rank counts are refused before any device memory is touched."""
    from communication_compressed_optimizer_momentum_b200 import dp
    with pytest.raises(ValueError):
        dp.EmulatedRanks(1000, 8, 256, 9, device="cpu")
    with pytest.raises(ValueError):
        dp.EmulatedRanks(1000, 8, 256, 0, device="cpu")
    with pytest.raises(ob.OneBitError) as e:
        dp.OneBitAdamRank(1000, 6, 256, 4, 0, device="cpu")     # 6 workers over 4 ranks
    assert e.value.code == -1
    with pytest.raises(ob.OneBitError):
        dp.OneBitAdamRank(1000, 8, 256, 2, 2, device="cpu")     # no rank 2 of 2


# ----------------------------------------------------------------------------------------------
# the 0/1 Adam variant's ranks: local steps on each rank's own workers, and at every H-th step
# the same exchange, server range and broadcast as above

ZH, ZK, ZSTEPS, B2 = 2, 1, 5, 0.999


def _zo_rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import oracle
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    g, x, m, v = _inputs_zo()
    Wl = W // world
    nch = oracle.nchunks(D, C)
    k0, k1 = ob.onebit_dp_chunk_range(nch, world, rank)
    e0, e1 = k0 * C, min(k1 * C, D)
    m_w = np.ascontiguousarray(np.broadcast_to(m, (Wl, D)), dtype=np.float32)
    u_w = np.zeros((Wl, D), np.float32)
    e_w = np.zeros((Wl, D), np.float32)
    e_s = np.zeros(e1 - e0, np.float32)
    gamma, syncs = np.float32(0.0), 0
    for t in range(1, ZSTEPS + 1):
        lr = float(np.float32(LR * (1.0 + 0.25 * (t % 3))))
        gamma = np.float32(gamma + np.float32(lr))
        oracle.zo_local(m_w, u_w, g[t - 1, rank * Wl:(rank + 1) * Wl], B1, lr)
        if t % ZH:
            continue                                   # local step: nothing is exchanged
        refresh = ZK > 0 and (syncs + 1) % ZK == 0
        s, bits = oracle.zo_compress(u_w, e_w, C)
        s_all = torch.cat(_gather(torch.from_numpy(s), world)).numpy()
        b_all = torch.cat(_gather(torch.from_numpy(bits.view(np.int32)), world)).numpy()
        s_own = np.ascontiguousarray(s_all[:, k0:k1])
        b_own = np.ascontiguousarray(b_all[:, e0 // 32:(e1 + 31) // 32]).view(np.uint32)
        if e1 > e0:
            S_own, bs_own, _, _ = oracle.server(s_own, b_own, e_s, C)
        else:
            S_own, bs_own = np.zeros(0, np.float32), np.zeros(0, np.uint32)
        pieces = [None] * world
        dist.all_gather_object(pieces, (k0, S_own, bs_own))
        S = np.zeros(nch, np.float32)
        bits_s = np.zeros(oracle.nwords(D), np.uint32)
        for (p0, Sp, bp) in pieces:
            S[p0:p0 + Sp.size] = Sp
            bits_s[p0 * C // 32:p0 * C // 32 + bp.size] = bp
        mbar = oracle.zo_apply(bits_s, S, v, x, C, EPS, float(gamma), B2, refresh)
        m_w[:] = mbar                                  # every worker restarts from mbar, u_w = 0
        u_w[:] = 0.0
        syncs += 1
        gamma = np.float32(0.0)
    q.put((rank, x.copy(), v.copy(), m_w.copy(), u_w.copy(), e_w.copy(), e_s.copy(), e0, e1))
    dist.barrier()
    dist.destroy_process_group()


def _inputs_zo():
    g, x, m, v = _inputs()
    rng = np.random.default_rng(20261203)
    g = np.concatenate([g, (rng.standard_normal((ZSTEPS - STEPS, W, D)) * 1e-2).astype(
        np.float32)]) if ZSTEPS > STEPS else g
    return g, x, m, v


def test_zero_one_rank_decomposition_matches_the_single_process_variant(lib):
    """Two gloo ranks running the 0/1 variant's decomposition (each rank's own workers' local
    steps; at a synchronisation its workers' messages exchanged, the server stage of its chunk
    range, the server plane broadcast, the synchronised step) reproduce the single-process
    oracle of the variant bit for bit: x, v, every worker's momentum and update, residuals."""
    sys.path.insert(0, ROOT)
    import oracle
    world = 2
    g, x, m, v = _inputs_zo()
    st = oracle.ZeroOneState(x, W, C, ZH, ZK, B1, B2, EPS)
    st.m[:] = m
    st.v[:] = v
    st.freeze()
    for t in range(1, ZSTEPS + 1):
        lr = float(np.float32(LR * (1.0 + 0.25 * (t % 3))))
        st.step(g[t - 1], lr)

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    procs = [ctx.Process(target=_zo_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    Wl = W // world

    def same(a, b):
        return np.array_equal(np.asarray(a).view(np.uint32), np.asarray(b).view(np.uint32))

    for rank, xr, vr, mw, uw, ew, es, e0, e1 in out:
        rows = slice(rank * Wl, (rank + 1) * Wl)
        assert same(xr, st.x) and same(vr, st.v), rank
        assert same(mw, st.m_w[rows]) and same(uw, st.u_w[rows]), rank
        assert same(ew, st.e_w[rows]) and same(es, st.e_s[e0:e1]), rank
