"""Host-side logic without a GPU: workload shapes, the benchmark's parsing of the committed ncu
summary and of nvidia-smi samples, and its derived figures."""
import hashlib
import json
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from communication_compressed_optimizer_momentum_b200 import workloads as wls  # noqa: E402


def test_bucket_shapes_are_the_sums_of_their_tensors():
    assert wls.transformer_layer_params(768, 3072) == 7_087_872
    assert wls.WORKLOADS["bert_base_bucket"].d == 12 * 7_087_872 + 30522 * 768 == 108_495_360
    assert wls.WORKLOADS["bert_large_bucket"].d == 24 * 12_596_224 + 30522 * 1024 == 333_563_904
    assert wls.WORKLOADS["gpt2_xl_bucket"].d == 48 * 30_740_800 + 50257 * 1600 == 1_555_969_600
    bl = wls.WORKLOADS["bert_large_bucket"]
    assert bl.C * bl.W == bl.d and bl.nch == 16
    g2 = wls.WORKLOADS["gpt2_xl_bucket"]
    assert g2.nch == 371 and g2.d - 370 * g2.C == 4_077_120
    for w in wls.WORKLOADS.values():
        assert w.d % 32 == 0 and w.C % 32 == 0
        assert sum(w.layer_sizes or (w.d,)) == w.d


def test_sweep_points_and_chunk_rounding():
    pts = wls.sweep_points()
    assert len(pts) == 24
    for W, C in pts:
        wl = wls.sweep_workload(W, C)
        assert wl.C % 32 == 0 and wl.d == 1 << 28
        if C is None:
            assert wl.C * W >= wl.d and (wl.C - 32) * W < wl.d


def test_algorithmic_bytes_split_by_kernel():
    for w in list(wls.WORKLOADS.values()) + [wls.sweep_workload(64, None)]:
        kb = w.kernel_bytes_per_param()
        assert sum(kb.values()) == pytest.approx(w.algorithmic_bytes_per_param())
    assert wls.WORKLOADS["bert_large_bucket"].algorithmic_bytes_per_param() == 184.375


def test_data_parallel_byte_counts():
    """One rank is the single-GPU step; each extra rank adds one apply pass (x, v and the server
    plane read, x written) and a copy of the server plane; the NVLink bytes are the sign words
    and server-plane shares that leave a rank."""
    for w in list(wls.WORKLOADS.values()) + [wls.sweep_workload(64, None)]:
        assert w.dp_algorithmic_bytes_per_param(1) == w.algorithmic_bytes_per_param()
        assert w.dp_algorithmic_bytes_per_param(4) - w.dp_algorithmic_bytes_per_param(3) == 12.375
        assert w.dp_nvlink_bytes_per_rank(1) == 0
    bl = wls.WORKLOADS["bert_large_bucket"]                     # W = 16, 8 ranks of 2 workers
    assert bl.dp_nvlink_bytes_per_rank(8) == pytest.approx(3 * bl.d * 7 / 64)


def test_scaled_workload_keeps_segment_proportions():
    wl = wls.scaled(wls.WORKLOADS["bert_base_bucket"], 1 << 20)
    assert wl.d == 1 << 20 and sum(wl.layer_sizes) == wl.d and len(wl.layer_sizes) == 13


def test_host_generators_are_seeded_and_shaped():
    wl = wls.scaled(wls.WORKLOADS["bert_large_bucket"], 4096)
    a, b = wls.np_grads(wl, 1, 3), wls.np_grads(wl, 1, 3)
    assert a.dtype == np.uint16 and a.shape == (wl.W, 4096) and np.array_equal(a, b)
    assert not np.array_equal(a, wls.np_grads(wl, 1, 4))
    f = wls.bf16_bits_to_f32(a)
    assert np.isfinite(f).all() and 1e-4 < float(np.std(f)) < 1e-1


def test_ncu_traffic_follows_the_kernel_source(tmp_path, monkeypatch):
    sha = bench.kernel_source_sha()
    p = tmp_path / "traffic.json"
    doc = {"workload": "bert_large_bucket", "kernel_source_sha256": sha,
           "kernels": {"worker": {"dram_bytes_per_launch_full": 123456},
                       "server": {"dram_bytes_per_launch_full": 789.0},
                       "apply": {"note": "no figure"}}}
    p.write_text(json.dumps(doc))
    monkeypatch.setattr(bench, "TRAFFIC_JSON", str(p))
    assert bench.ncu_traffic("bert_large_bucket") == {"worker": 123456.0, "server": 789.0}
    assert bench.ncu_traffic("smoke_1m") == {}                # other workload
    doc["kernel_source_sha256"] = "0" * 64
    p.write_text(json.dumps(doc))
    assert bench.ncu_traffic("bert_large_bucket") == {}       # stale: kernels changed since
    monkeypatch.setattr(bench, "TRAFFIC_JSON", str(tmp_path / "missing.json"))
    assert bench.ncu_traffic("bert_large_bucket") == {}


def test_traffic_summary_is_written_from_an_ncu_csv(tmp_path, monkeypatch):
    hdr = ('"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream",'
           '"Block Size","Grid Size","Device","CC","Section Name","Metric Name","Metric Unit",'
           '"Metric Value"')
    names = {"worker": "void k_worker<unsigned short, 1, 1, 8, 0>(WorkerArgs)",
             "server": "void k_server<1, 1, 0>(ServerArgs)", "apply": "k_apply(ApplyArgs)"}
    lines = ["==PROF== Connected to process 1", hdr]
    figures = {}
    for i, (launch, k) in enumerate([(0, "worker"), (0, "server"), (0, "apply"),
                                     (1, "worker"), (1, "server"), (1, "apply")]):
        rd, wr, ns = 1000 * (i + 1), 500 * (i + 1), 10 * (i + 1)
        figures[k] = (rd, wr, ns)      # the later launch of each kernel is the one kept
        for m, v in (("dram__bytes_read.sum", rd), ("dram__bytes_write.sum", wr),
                     ("gpu__time_duration.sum", ns)):
            lines.append('"%d","1","p","h","%s","1","7","(256, 1, 1)","(8, 1, 1)","0","10.0",'
                         '"Command line profiler metrics","%s","byte","%s"'
                         % (i, names[k], m, format(v, ",")))
    csv_path = tmp_path / "t.csv"
    csv_path.write_text("\n".join(lines) + "\n")
    out = tmp_path / "traffic.json"
    cap = 1 << 20
    j = bench.write_traffic_json(str(csv_path), "bert_large_bucket", cap, "cmd", out=str(out))
    wl = wls.WORKLOADS["bert_large_bucket"]
    kb = wl.kernel_bytes_per_param()
    for k, (rd, wr, ns) in figures.items():
        got = j["kernels"][k]
        assert (got["dram_bytes_read"], got["dram_bytes_write"], got["duration_ns"]) == (rd, wr, ns)
        assert got["dram_over_algorithmic"] == round((rd + wr) / (kb[k] * cap), 4)
        assert got["dram_bytes_per_launch_full"] == round((rd + wr) * wl.d / cap)
    monkeypatch.setattr(bench, "TRAFFIC_JSON", str(out))
    assert bench.ncu_traffic("bert_large_bucket") == {
        k: float(round((rd + wr) * wl.d / cap)) for k, (rd, wr, _) in figures.items()}


def test_committed_traffic_summary_parses():
    if not os.path.exists(bench.TRAFFIC_JSON):
        pytest.skip("no ncu traffic summary committed for the current kernels")
    with open(bench.TRAFFIC_JSON) as f:
        doc = json.load(f)
    assert doc["workload"] == "bert_large_bucket" and len(doc["kernel_source_sha256"]) == 64
    for name in ("worker", "server", "apply"):
        assert doc["kernels"][name]["dram_bytes_per_launch_full"] > 0


def test_warmup_phase_figures():
    wl = wls.WORKLOADS["bert_large_bucket"]
    r = bench.warmup_phase(wl, [9.0, 4.0, 4.0])
    assert r["ms_per_step"] == 4.0 and r["bytes_per_step"] == (16 * 2 + 24) * wl.d
    assert r["achieved_gbs"] == pytest.approx(r["bytes_per_step"] / 4e-3 / 1e9)
    assert bench.warmup_phase(wl, [1.0]) is None


def test_clock_sampler_parses_nvidia_smi_lines():
    s = bench.ClockSampler(0)
    s.proc = type("P", (), {"terminate": lambda self: None, "wait": lambda self, timeout: 0})()
    s.t0, s.t1 = 100.0, 101.0
    s.lines = [(100.1, "2026/12/02 17:00:00.000, 0, 1650, 1965, 980.5, 0x4, Not Active, "
                       "Not Active, Not Active, Active"),
               (100.5, "2026/12/02 17:00:00.200, 0, 1700, 1965, 990.0, 0x0, Not Active, "
                       "Not Active, Not Active, Not Active"),
               (150.0, "2026/12/02 17:00:50.000, 0, 120, 1965, 90.0, 0x0, Not Active, "
                       "Not Active, Not Active, Not Active")]
    c = s.stop()
    assert c["samples"] == 2 and c["in_timed_region"]
    assert c["sm_mhz"] in (1650.0, 1700.0) and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"]


def test_step_distribution():
    assert bench.step_distribution([]) is None
    d = bench.step_distribution([5.0, 1.0, 3.0, 2.0, 4.0])
    assert (d["p10"], d["p50"], d["p90"], d["steps"]) == (1.0, 3.0, 5.0, 5)
    d = bench.step_distribution([float(i) for i in range(11)])
    assert (d["p10"], d["p50"], d["p90"]) == (1.0, 5.0, 9.0)


def test_whole_job_rate():
    assert bench.whole_job_rate(1000, 4, 2.0) == pytest.approx(4000 / 0.002)


def test_scaled_sweep_workloads_for_profiling():
    """--scale-d shrinks the sweep points too (ncu captures must stay a few GB)."""
    wl = bench.get_workload("sweep_W64_C0", 1 << 24)
    assert (wl.d, wl.W, wl.C) == (1 << 24, 64, (1 << 24) // 64)
    wl = bench.get_workload("sweep_W64_C4096", 1 << 24)
    assert (wl.d, wl.C) == (1 << 24, 4096)
    assert bench.get_workload("sweep_W2_C0").d == 1 << 28


class _FakeHandle:
    """Stands in for a OneBitAdam handle's state export (host tensors, no GPU)."""

    def __init__(self, d, W, C, seed=3):
        import torch
        gen = torch.Generator().manual_seed(seed)
        self.C = C
        self.st = {"m": torch.randn(d, generator=gen) * 1e-3,
                   "v": torch.rand(d, generator=gen) * 1e-4 + 1e-6,
                   "e_w": torch.zeros(W, d), "e_s": torch.zeros(d)}

    def get_state(self, name):
        return self.st[name]

    def get_chunk_state(self, name, k):
        lo, hi = k * self.C, (k + 1) * self.C
        t = self.st[name]
        return t[..., lo:hi]


@pytest.mark.parametrize("d,W,C,full", [(1 << 20, 4, 1 << 18, True), (1 << 24, 4, 1 << 16, False)])
def test_cpu_baseline_whole_step_or_chunk(d, W, C, full):
    """Small workloads time the oracle's whole step; large ones chunk 0, with the whole step's
    time extrapolated from that rate."""
    import dataclasses
    import torch
    wl = dataclasses.replace(wls.WORKLOADS["smoke_1m"], d=d, W=W, C=C, layer_sizes=())
    x = torch.rand(d) * 0.1 - 0.05
    g = torch.randn(W, d) * 1e-2
    out = bench.cpu_baseline(wl, _FakeHandle(d, W, C), x, g, 0.01)
    assert out["kind"] == "oracle" and out["cores"] == 1 and out["value"] > 0
    n = d if full else C
    assert ("%d params x %d workers" % (n, W)) in out["sample"]
    key = "s_per_step" if full else "extrapolated_s_per_step"
    assert out[key] == pytest.approx(d * W / out["value"])
    assert ("whole workload" in out["sample"]) == full
