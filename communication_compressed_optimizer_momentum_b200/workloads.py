"""Synthetic workloads: the parameter-bucket shapes and seeded input generators.

This module holds the shapes, sizes and value distributions of the workloads the method is
measured on (BERT-Base, BERT-Large and GPT-2 1.5B pre-training buckets, a flat 2^28 sweep and a
1M smoke case) and the seeded generators for their parameters and per-worker gradients. It
contains none of the method's arithmetic: the CUDA path and the CPU oracle both take what these
generators produce as plain input arrays. The pages train on real datasets; seeded synthetic
buckets of the same shapes stand in for them here ("1-bit Adam" index page, Abstract: BERT-Large
pre-training and SQuAD fine-tuning; 0/1 Adam page, abstract: BERT-Base, BERT-Large, GPT-2).

Device generation uses ``torch`` random generators on whatever device the output tensor lives
on; host generation (for CPU-only tests) uses numpy. The two streams are different by design:
parity always hands the oracle the exact bytes the device consumed.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Tuple

import numpy as np

BETA1, BETA2, EPS, LR = 0.9, 0.999, 1e-8, 1e-4


def transformer_layer_params(hidden: int, ffn: int) -> int:
    """Elements of one transformer block: q, k, v, o projections, the two FFN matrices, their
    biases and two LayerNorms (scale + shift each)."""
    return 4 * hidden * hidden + 2 * hidden * ffn + (4 * hidden + ffn + hidden) + 2 * 2 * hidden


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    d: int
    W: int
    C: int
    grad_dtype: str            # "f32" or "bf16"
    grad_kind: str             # "normal", "layer_normal", "outlier_normal", "student_t", "edge_normal"
    sigma: float               # base standard deviation of the gradient distribution
    warmup_steps: int
    compressed_steps: int
    seed: int
    layer_sizes: Tuple[int, ...] = ()   # segment lengths whose sigma is drawn per segment
    lr: float = LR
    last_worker_sigma: float = 1.0   # sigma multiplier of the last worker (scale-spread cases)
    beta1: float = BETA1
    beta2: float = BETA2
    eps: float = EPS
    description: str = ""

    @property
    def nch(self) -> int:
        return (self.d + self.C - 1) // self.C

    @property
    def grad_bytes(self) -> int:
        return 4 if self.grad_dtype == "f32" else 2

    def algorithmic_bytes_per_param(self) -> float:
        """Minimum HBM bytes per parameter of one compressed step when every state element is
        read and written once and each message is written and read once. Per worker: the
        gradient (G), the residual read and written (4 + 4), its sign plane written and read
        (1/8 + 1/8). Shared: the server residual read and written (8), the server plane written,
        read by the apply and read again by the next step's worker pass, which rebuilds the
        momentum m = +-S from it (3/8), v read (4), x read and written (8). Per-chunk scales
        are negligible and left out: W*(G + 8.25) + 20.375."""
        return self.W * (self.grad_bytes + 8.25) + 20.375

    def dp_algorithmic_bytes_per_param(self, R: int) -> float:
        """The same minimum for R data-parallel ranks together (W / R workers each; rank q
        serves a 1/R share of the chunks; x, v and the server plane replicated): every rank's
        worker pass reads the server plane to rebuild m (1/8 each), the server broadcasts its
        plane to every rank (R/8 written) and every rank applies the step to its own x
        (12.125 each). W*(G + 8.25) + 8 + 12.375*R, equal to the single-GPU figure at R = 1."""
        return self.W * (self.grad_bytes + 8.25) + 8.0 + 12.375 * R

    def dp_nvlink_bytes_per_rank(self, R: int) -> float:
        """Bytes one of R data-parallel ranks stores into other ranks' memory per compressed
        step, on average over the ranks: the sign words of its W / R workers for the chunks the
        other ranks serve, and its share of the server plane for every other rank (per-chunk
        scales are negligible). (W / R + 1) * d * (R - 1) / (8 R)."""
        return (self.W / R + 1) * self.d * (R - 1) / (8.0 * R)

    def zero_one_bytes_per_param(self, H: int, K: int) -> float:
        """The 0/1 Adam variant's minimum HBM bytes per parameter per step, averaged over one
        interval of H steps (a synchronisation every H steps, a variance refresh at every K-th
        one). The first step after a synchronisation rebuilds the shared momentum estimate from
        the server plane (1/8) and writes every worker's momentum (W*(G + 4)); its accumulated
        update lr * m_w is not stored but rebuilt by the next step, which reads the momentum and
        writes both (W*(G + 12)); the steps after that read and write both (W*(G + 16)). The
        synchronising step reads them (only the momentum when it is the interval's second
        step), compresses u_w + e_w (residual read and written, sign plane written: W*(G +
        16.125), or W*(G + 12.125)), then the server stage (W/8 + 8.125) and the synchronised
        step (server plane, v, x: 12.125, plus 4 when v is refreshed). With H = 1 every step is
        the 1-bit Adam step's bytes."""
        G, W = self.grad_bytes, self.W
        server = W / 8.0 + 8.125
        apply = 12.125 + (4.0 / K if K > 0 else 0.0)
        if H == 1:
            return W * (G + 8.125) + 0.125 + server + apply
        first = W * (G + 4.0) + 0.125
        if H == 2:
            return (first + W * (G + 12.125) + server + apply) / 2
        second = W * (G + 12.0)
        middle = (H - 3) * W * (G + 16.0)
        sync = W * (G + 16.125) + server + apply
        return (first + second + middle + sync) / H

    def kernel_bytes_per_param(self) -> dict:
        """The same minimum, split by the three streaming kernels of the step."""
        G, W = self.grad_bytes, self.W
        return {"worker": W * (G + 8.125) + 0.125, "server": W / 8.0 + 8.125, "apply": 12.125}


def _ceil_to(x: int, a: int) -> int:
    return (x + a - 1) // a * a


def _bert_like(hidden: int, ffn: int, layers: int, vocab: int) -> Tuple[int, Tuple[int, ...]]:
    per = transformer_layer_params(hidden, ffn)
    sizes = tuple([per] * layers + [vocab * hidden])
    return sum(sizes), sizes


_BB_D, _BB_SIZES = _bert_like(768, 3072, 12, 30522)     # 108,495,360
_BL_D, _BL_SIZES = _bert_like(1024, 4096, 24, 30522)    # 333,563,904
_G2_D, _G2_SIZES = _bert_like(1600, 6400, 48, 50257)    # 1,555,969,600

WORKLOADS = {
    "smoke_1m": Workload(
        "smoke_1m", d=1_048_576, W=4, C=262_144, grad_dtype="f32", grad_kind="normal",
        sigma=1e-2, warmup_steps=20, compressed_steps=10, seed=2102,
        description="1,048,576 fp32 params, W=4, C=d/W, grads N(0, 0.01^2)"),
    "bert_base_bucket": Workload(
        "bert_base_bucket", d=_BB_D, W=8, C=1_048_576, grad_dtype="f32",
        grad_kind="layer_normal", sigma=0.0, warmup_steps=50, compressed_steps=100, seed=2103,
        layer_sizes=_BB_SIZES,
        description="BERT-Base-shaped bucket (12 x [768^2 x4, 768x3072 x2, biases, LN] + "
                    "30522x768 embedding), W=8, C=2^20, fp32 grads N(0, sigma_L^2), "
                    "sigma_L log-uniform in [1e-4, 1e-2] per layer"),
    "bert_large_bucket": Workload(
        "bert_large_bucket", d=_BL_D, W=16, C=_BL_D // 16, grad_dtype="bf16",
        grad_kind="outlier_normal", sigma=1e-3, warmup_steps=20, compressed_steps=100,
        seed=2104, layer_sizes=_BL_SIZES,
        description="BERT-Large-shaped bucket (24 x hidden 1024 / FFN 4096 + 30522x1024 "
                    "embedding), W=16, C=d/W, bf16 grads N(0, 1e-3^2) with 1% x100 outliers"),
    "gpt2_xl_bucket": Workload(
        "gpt2_xl_bucket", d=_G2_D, W=8, C=4_194_304, grad_dtype="bf16", grad_kind="student_t",
        sigma=1e-3, warmup_steps=20, compressed_steps=20, seed=2105, layer_sizes=_G2_SIZES,
        description="GPT-2 1.5B-shaped bucket (48 x hidden 1600 / FFN 6400 + 50257x1600 "
                    "embedding), W=8, C=2^22, bf16 grads Student-t(3) x 1e-3"),
}

SWEEP_D = 1 << 28
SWEEP_W = (2, 4, 8, 16, 32, 64)
SWEEP_C = (4096, 65536, 1 << 20, None)   # None stands for C = d/W


def sweep_workload(W: int, C: Optional[int], d: int = SWEEP_D) -> Workload:
    """One point of the flat-vector sweep: fp32 grads N(0, 1e-2^2) with 0.1% exact zeros and
    0.1% values within 1e-9 of zero."""
    if C is None:
        C = _ceil_to((d + W - 1) // W, 32)
    return Workload("sweep_W%d_C%d" % (W, C), d=d, W=W, C=C, grad_dtype="f32",
                    grad_kind="edge_normal", sigma=1e-2, warmup_steps=20, compressed_steps=10,
                    seed=2106 + 97 * W + (C % 1009),
                    description="2^28 fp32 vector, W=%d, C=%d, grads N(0, 1e-2^2) with 0.1%% "
                                "zeros and 0.1%% near-zeros" % (W, C))


def sweep_points() -> List[Tuple[int, Optional[int]]]:
    return [(W, C) for W in SWEEP_W for C in SWEEP_C]


def scaled(wl: Workload, d: int, W: Optional[int] = None, C: Optional[int] = None) -> Workload:
    """The same distributions on a smaller vector (for tests the oracle finishes in seconds).
    Layer segments are scaled proportionally so every segment keeps its own sigma."""
    W = wl.W if W is None else W
    if C is None:
        C = min(wl.C, _ceil_to((d + W - 1) // W, 32)) if wl.C * wl.W >= wl.d else wl.C
    sizes = ()
    if wl.layer_sizes:
        tot = sum(wl.layer_sizes)
        raw = [max(1, s * d // tot) for s in wl.layer_sizes]
        raw[-1] += d - sum(raw)
        sizes = tuple(raw)
    return dataclasses.replace(wl, name=wl.name + "_d%d" % d, d=d, W=W, C=C, layer_sizes=sizes)


# ----------------------------------------------------------------------------------------------
# seeds

def step_seed(wl: Workload, phase: int, step: int, worker: int) -> int:
    """Seed of one worker's gradient at one step; phase 0 = warm-up, 1 = compressed."""
    return (wl.seed * 1_000_003 + phase * 7_919_311 + step * 104_729 + worker * 1_299_709) % (2**62)


def layer_sigmas(wl: Workload) -> np.ndarray:
    """Per-segment standard deviation, fixed for the whole run (log-uniform in [1e-4, 1e-2]
    for the layer-normal kind; the base sigma for every other kind)."""
    n = max(1, len(wl.layer_sizes))
    if wl.grad_kind != "layer_normal":
        return np.full(n, wl.sigma, dtype=np.float64)
    rng = np.random.default_rng(wl.seed)
    return 10.0 ** rng.uniform(-4.0, -2.0, size=n)


# ----------------------------------------------------------------------------------------------
# host (numpy) generators, for CPU-only tests

def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (round to nearest even), returned as uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    nan = (u & 0x7F800000) == 0x7F800000
    nan &= (u & 0x007FFFFF) != 0
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    r = np.where(nan, (u >> 16) | 0x40, r)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def np_params(wl: Workload) -> np.ndarray:
    rng = np.random.default_rng(wl.seed + 17)
    return rng.uniform(-0.05, 0.05, size=wl.d).astype(np.float32)


def _np_worker_grad(wl: Workload, rng: np.random.Generator, sig: np.ndarray) -> np.ndarray:
    d = wl.d
    if wl.grad_kind == "student_t":
        z = rng.standard_normal(d)
        chi = (rng.standard_normal((3, d)) ** 2).sum(axis=0)
        g = wl.sigma * z / np.sqrt(chi / 3.0)
    else:
        g = rng.standard_normal(d) * _expand_sigma(wl, sig)
        if wl.grad_kind == "outlier_normal":
            g = np.where(rng.random(d) < 0.01, g * 100.0, g)
        if wl.grad_kind == "edge_normal":
            u = rng.random(d)
            g = np.where(u < 0.001, 0.0, g)
            g = np.where((u >= 0.001) & (u < 0.002), rng.uniform(-1e-9, 1e-9, size=d), g)
    return g.astype(np.float32)


def _expand_sigma(wl: Workload, sig: np.ndarray) -> np.ndarray:
    if not wl.layer_sizes:
        return np.full(wl.d, sig[0])
    return np.repeat(sig, wl.layer_sizes)


def np_grads(wl: Workload, phase: int, step: int) -> np.ndarray:
    """[W][d] gradients of one step on the host: float32, or uint16 bf16 bit patterns."""
    sig = layer_sigmas(wl)
    rows = []
    for w in range(wl.W):
        rng = np.random.default_rng(step_seed(wl, phase, step, w))
        mult = wl.last_worker_sigma if w == wl.W - 1 else 1.0
        rows.append((_np_worker_grad(wl, rng, sig) * np.float32(mult)).astype(np.float32))
    g = np.stack(rows)
    return f32_to_bf16_bits(g) if wl.grad_dtype == "bf16" else g


# ----------------------------------------------------------------------------------------------
# device (torch) generators

def torch_dtype(wl: Workload):
    import torch
    return torch.float32 if wl.grad_dtype == "f32" else torch.bfloat16


def torch_params(wl: Workload, device) -> "torch.Tensor":
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(wl.seed + 17)
    x = torch.empty(wl.d, dtype=torch.float32, device=device)
    x.uniform_(-0.05, 0.05, generator=gen)
    return x


def torch_fill_grads(wl: Workload, out, phase: int, step: int, piece: int = 1 << 26) -> None:
    """Fill ``out`` ([W][d], float32 or bfloat16, any device) with one step's gradients.
    Generated in pieces of ``piece`` elements so the temporaries stay small."""
    import torch
    assert tuple(out.shape) == (wl.W, wl.d) and out.dtype == torch_dtype(wl)
    dev = out.device
    sig = layer_sigmas(wl)
    bounds = np.cumsum((0,) + tuple(wl.layer_sizes)) if wl.layer_sizes else None
    gen = torch.Generator(device=dev)
    for w in range(wl.W):
        gen.manual_seed(step_seed(wl, phase, step, w))
        for lo in range(0, wl.d, piece):
            hi = min(wl.d, lo + piece)
            n = hi - lo
            if wl.grad_kind == "student_t":
                z = torch.randn(n, device=dev, generator=gen)
                c = torch.randn(3, n, device=dev, generator=gen).square_().sum(0)
                g = z.mul_(wl.sigma).div_(c.div_(3.0).sqrt_())
            else:
                g = torch.randn(n, device=dev, generator=gen)
                if bounds is not None and wl.grad_kind == "layer_normal":
                    sv = torch.empty(n, device=dev)
                    for li in range(len(sig)):
                        a, b = max(lo, int(bounds[li])), min(hi, int(bounds[li + 1]))
                        if a < b:
                            sv[a - lo:b - lo] = float(sig[li])
                    g.mul_(sv)
                else:
                    g.mul_(float(sig[0]))
                if wl.grad_kind == "outlier_normal":
                    mask = torch.rand(n, device=dev, generator=gen) < 0.01
                    g = torch.where(mask, g * 100.0, g)
                if wl.grad_kind == "edge_normal":
                    u = torch.rand(n, device=dev, generator=gen)
                    near = torch.rand(n, device=dev, generator=gen).mul_(2e-9).sub_(1e-9)
                    g = torch.where(u < 0.001, torch.zeros_like(g), g)
                    g = torch.where((u >= 0.001) & (u < 0.002), near, g)
            if w == wl.W - 1 and wl.last_worker_sigma != 1.0:
                g = g * wl.last_worker_sigma
            out[w, lo:hi].copy_(g)   # float32 -> bfloat16 rounds to nearest even


def chunk_bounds(wl: Workload, k: int) -> Tuple[int, int]:
    lo = k * wl.C
    return lo, min(wl.d, lo + wl.C)


def sample_chunks(wl: Workload, n_random: int = 1) -> List[int]:
    """Chunks checked against the oracle at full size: the first, the second, the last (which
    holds any ragged tail) and seeded random ones. Chunks are independent, so a sample of
    whole chunks checks every output that depends on them."""
    nch = wl.nch
    ks = {0, nch - 1}
    if nch > 1:
        ks.add(1)
    rng = np.random.default_rng(wl.seed + 5)
    for _ in range(n_random):
        ks.add(int(rng.integers(0, nch)))
    return sorted(ks)


def describe(wl: Workload) -> dict:
    return {"workload": wl.name, "d": wl.d, "W": wl.W, "C": wl.C, "nch": wl.nch,
            "grads": wl.grad_dtype, "grad_dist": wl.grad_kind,
            "warmup_steps": wl.warmup_steps, "compressed_steps": wl.compressed_steps}
