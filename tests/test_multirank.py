"""The benchmark's multi-rank host logic on the CPU: gloo process groups of world size 2 stand
in for one process per GPU. Every rank runs its own replica (no data-path collective); ranks
agree on the slowest rank's time, and the reference arm runs on rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    ms_local = 10.0 + 5.0 * rank           # rank 1 is the slow one
    ms_max = bench.max_over_ranks(ms_local, "cpu")
    rate = bench.whole_job_rate(1000, world, ms_max)
    q.put((rank, ms_max, rate))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_rate_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms_max, rate in out:
        assert ms_max == 15.0                  # every rank sees the slowest rank's time
        assert rate == pytest.approx(2 * 1000 / 0.015)


def _bench_reference(rank, world):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--gpus", str(world), "--steps", "1", "--warmup", "0",
                           "--workload", "smoke_1m"],
                          env=env, capture_output=True, text=True, timeout=600)


def test_reference_arm_runs_on_rank_zero_only():
    r1 = _bench_reference(1, 2)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = _bench_reference(0, 2)
    assert r0.returncode == 0, r0.stderr[-2000:]
    lines = [l for l in r0.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["unit"] == "params*workers/s" and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]


def _dp_rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    from communication_compressed_optimizer_momentum_b200 import workloads as wls
    wl = wls.WORKLOADS["bert_large_bucket"]
    flags = 4 if rank == 1 else 0               # rank 1's barrier wait ran out
    ms_max = bench.max_over_ranks(8.0 + rank, "cpu")
    all_flags = bench.gather_flags(flags, world)
    obj = bench.dp_subobject(wl, world, ms_max, 9.4, all_flags)
    q.put((rank, obj))
    dist.barrier()
    dist.destroy_process_group()


def test_data_parallel_subobject_gloo():
    """Under torchrun with N > 1 the benchmark adds a "dp" object: the data-parallel step timed
    as the max over ranks, its speed-up over the single-GPU step, the bytes a rank stores into
    its peers per step and every rank's status word, gathered in rank order."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dp_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    d, W = 333_563_904, 16
    for rank in (0, 1):
        obj = out[rank]
        assert obj["ranks"] == 2 and obj["workers_per_rank"] == 8
        assert obj["ms_per_step"] == 9.0                       # the slower rank's time
        assert obj["strong_scaling_vs_single"] == pytest.approx(9.4 / 9.0)
        assert obj["nvlink_bytes_per_rank_per_step"] == pytest.approx((W / 2 + 1) * d / 16)
        assert obj["status_flags_per_rank"] == [0, 4]
        assert obj["timeout_seen"] is True


def test_data_parallel_section_only_where_workers_split():
    sys.path.insert(0, ROOT)
    import bench
    from communication_compressed_optimizer_momentum_b200 import workloads as wls
    wl = wls.WORKLOADS["bert_large_bucket"]                    # W = 16
    assert [n for n in range(1, 10) if bench.dp_ranks_supported(wl, n)] == [2, 4, 8]
    assert not bench.dp_ranks_supported(wls.sweep_workload(2, None), 4)
