"""CPU oracle for the compression phase of 1-bit Adam (arXiv 2102.02888) and of its 0/1 Adam
variant.

TEST INFRASTRUCTURE ONLY. This package wraps ``onebit_oracle.c`` and ``zero_one_oracle.c``,
plain single-threaded C restatements of the methods, with ctypes and numpy. Only the test suite,
the package's smoke check and the benchmark's CPU-baseline leg (and its ``--impl reference`` arm)
may import it; the product path (the CUDA library and its binding) never does, and the two share
no code.

All arrays are numpy, C-contiguous. Grads are float32 ``[W][d]`` or bf16 bit patterns stored as
uint16 ``[W][d]``. Every function follows the conventions R1-R11 (and, for the ``zo_*``
functions of the 0/1 Adam variant, Z1-Z7) stated at the top of the C files; each cites the page
and section it restates.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "onebit_oracle.c")
_SRC01 = os.path.join(_HERE, "zero_one_oracle.c")
_SRCBC = os.path.join(_HERE, "bias_corrected_oracle.c")
SOURCES = (_SRC, _SRC01, _SRCBC)
_LIB = os.path.join(_HERE, "libonebit_oracle.so")

# Flags that keep every fp32 operation a single IEEE operation (R7): no contraction to FMA, no
# fast-math reassociation; SSE arithmetic on x86-64 has no excess precision.
CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
          "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile the oracle to ``oracle/libonebit_oracle.so`` (gcc) if missing or stale."""
    if force or not os.path.exists(_LIB) or any(
            os.path.getmtime(_LIB) < os.path.getmtime(src) for src in SOURCES):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, *SOURCES, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = _load(build())
    return _lib


def _load(path: str):
    L = ctypes.CDLL(path)
    P = ctypes.c_void_p
    i64, i32, f32, c_int = ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_int
    L.oracle_pack.argtypes = [P, i64, P]
    L.oracle_pack.restype = None
    L.oracle_unpack.argtypes = [P, P, i64, i64, P]
    L.oracle_unpack.restype = None
    L.oracle_warmup_step.argtypes = [i64, i32, f32, f32, f32, f32, P, P, P, P, c_int]
    L.oracle_warmup_step.restype = None
    L.oracle_worker.argtypes = [i64, i32, i64, f32, P, P, c_int, P, P, P]
    L.oracle_worker.restype = None
    L.oracle_server.argtypes = [i64, i32, i64, P, P, P, P, P, P]
    L.oracle_server.restype = i64
    L.oracle_apply.argtypes = [i64, i64, f32, f32, P, P, P, P, P]
    L.oracle_apply.restype = None
    L.oracle_compressed_step.argtypes = [i64, i32, i64, f32, f32, f32, P, P, P, P, P, P,
                                         c_int, P, P, P, P, P]
    L.oracle_compressed_step.restype = i64
    L.oracle01_local.argtypes = [i64, i32, f32, f32, P, P, P, c_int]
    L.oracle01_local.restype = None
    L.oracle01_compress.argtypes = [i64, i32, i64, P, P, P, P]
    L.oracle01_compress.restype = None
    L.oracle01_apply.argtypes = [i64, i64, f32, f32, f32, c_int, P, P, P, P, P]
    L.oracle01_apply.restype = None
    L.oracle01_step.argtypes = [i64, i32, i64, f32, f32, f32, f32, f32, c_int, c_int, P, P, P,
                                P, P, P, P, c_int, P, P, P, P, P, P]
    L.oracle01_step.restype = i64
    L.oracle01_local_model.argtypes = [i64, f32, P, P, P, P]
    L.oracle01_local_model.restype = None
    L.oracle_warmup_step_bc.argtypes = [i64, i32, f32, f32, f32, f32, f32, f32, P, P, P, P, c_int]
    L.oracle_warmup_step_bc.restype = None
    L.oracle_freeze_bc.argtypes = [i64, f32, f32, P, P]
    L.oracle_freeze_bc.restype = None
    return L


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return ctypes.c_void_p(a.ctypes.data)


def _f32(a, shape=None):
    a = np.ascontiguousarray(a, dtype=np.float32)
    if shape is not None:
        assert a.shape == shape, (a.shape, shape)
    return a


def _grads(g: np.ndarray):
    """Returns (array, gtype): float32 -> 0, uint16 (bf16 bit patterns) -> 1."""
    if g.dtype == np.float32:
        return np.ascontiguousarray(g), 0
    if g.dtype == np.uint16:
        return np.ascontiguousarray(g), 1
    raise TypeError("grads must be float32 or uint16 bf16 bit patterns, got %s" % g.dtype)


def nchunks(d: int, C: int) -> int:
    return (d + C - 1) // C


def nwords(n: int) -> int:
    return (n + 31) // 32


def pack(x: np.ndarray) -> np.ndarray:
    """Sign bits of x (bit = x >= 0), LSB-first into uint32 words; padding bits are 0 (R3, R4)."""
    x = _f32(x).ravel()
    words = np.zeros(nwords(x.size), dtype=np.uint32)
    lib().oracle_pack(_p(x), x.size, _p(words))
    return words


def unpack(words: np.ndarray, scales: np.ndarray, n: int, C: int) -> np.ndarray:
    """Decompression: +-scales[i // C] by the sign bit of element i."""
    words = np.ascontiguousarray(words, dtype=np.uint32)
    scales = _f32(scales)
    assert words.size >= nwords(n) and scales.size >= nchunks(n, C)
    out = np.empty(n, dtype=np.float32)
    lib().oracle_unpack(_p(words), _p(scales), n, C, _p(out))
    return out


def warmup_step(x, m, v, g, beta1, beta2, eps, lr):
    """Full-precision Adam warm-up step, in place on x, m, v (no bias correction, R6)."""
    g, gt = _grads(g)
    W, d = g.shape
    for a in (x, m, v):
        assert a.dtype == np.float32 and a.shape == (d,) and a.flags["C_CONTIGUOUS"]
    lib().oracle_warmup_step(d, W, beta1, beta2, eps, lr, _p(x), _p(m), _p(v), _p(g), gt)


def bias_corrections(beta1, beta2, t):
    """(c1_t, c2_t) = (1 - beta1^t, 1 - beta2^t): beta^t the fp64 product of t factors beta (the
    fp32 value) in order, 1 - beta^t in fp64, rounded once to fp32 (reading B1 of
    bias_corrected_oracle.c; fp32 arithmetic would lose most digits of 1 - beta2^t to
    cancellation)."""
    p1 = p2 = 1.0
    b1, b2 = float(np.float32(beta1)), float(np.float32(beta2))
    for _ in range(t):
        p1 *= b1
        p2 *= b2
    return float(np.float32(1.0 - p1)), float(np.float32(1.0 - p2))


def warmup_step_bc(x, m, v, g, beta1, beta2, eps, lr, t):
    """Bias-corrected warm-up step t (1-based), in place on x, m, v (m and v stay
    uncorrected; reading B1)."""
    g, gt = _grads(g)
    W, d = g.shape
    for a in (x, m, v):
        assert a.dtype == np.float32 and a.shape == (d,) and a.flags["C_CONTIGUOUS"]
    c1, c2 = bias_corrections(beta1, beta2, t)
    lib().oracle_warmup_step_bc(d, W, beta1, beta2, eps, lr, c1, c2, _p(x), _p(m), _p(v),
                                _p(g), gt)


def freeze_bc(m, v, beta1, beta2, T):
    """The freeze after T bias-corrected warm-up steps: m = m / c1_T, v = v / c2_T (B1)."""
    assert m.dtype == np.float32 and v.dtype == np.float32 and m.shape == v.shape
    c1, c2 = bias_corrections(beta1, beta2, T)
    lib().oracle_freeze_bc(m.size, c1, c2, _p(m), _p(v))


def worker(m, g, e_w, C, beta1):
    """Worker compression for all W workers; e_w ([W][d], explicit) is updated in place.

    Returns (s [W][nch] float32, bits_w [W][ceil(d/32)] uint32)."""
    g, gt = _grads(g)
    W, d = g.shape
    assert e_w.dtype == np.float32 and e_w.shape == (W, d) and e_w.flags["C_CONTIGUOUS"]
    m = _f32(m, (d,))
    s = np.zeros((W, nchunks(d, C)), dtype=np.float32)
    bits = np.zeros((W, nwords(d)), dtype=np.uint32)
    lib().oracle_worker(d, W, C, beta1, _p(m), _p(g), gt, _p(e_w), _p(s), _p(bits))
    return s, bits


def server(s, bits_w, e_s, C):
    """Server stage of the compressed allreduce; e_s ([d], explicit) is updated in place.

    Returns (S [nch] float32, bits_s [ceil(d/32)] uint32, z [d] float32, inexact_chunks)."""
    s = _f32(s)
    W, nch = s.shape
    d = e_s.size
    assert e_s.dtype == np.float32 and e_s.flags["C_CONTIGUOUS"]
    bits_w = np.ascontiguousarray(bits_w, dtype=np.uint32)
    assert bits_w.shape == (W, nwords(d)) and nch == nchunks(d, C)
    S = np.zeros(nch, dtype=np.float32)
    bits_s = np.zeros(nwords(d), dtype=np.uint32)
    z = np.zeros(d, dtype=np.float32)
    inexact = lib().oracle_server(d, W, C, _p(s), _p(bits_w), _p(e_s), _p(z), _p(S), _p(bits_s))
    return S, bits_s, z, int(inexact)


def apply(bits_s, S, v, m, x, C, eps, lr):
    """m = +-S by the server bits; x -= lr * (m / (sqrt(v) + eps)); in place on m and x."""
    d = x.size
    bits_s = np.ascontiguousarray(bits_s, dtype=np.uint32)
    S = _f32(S)
    v = _f32(v, (d,))
    for a in (m, x):
        assert a.dtype == np.float32 and a.shape == (d,) and a.flags["C_CONTIGUOUS"]
    lib().oracle_apply(d, C, eps, lr, _p(bits_s), _p(S), _p(v), _p(m), _p(x))


def compressed_step(x, m, v, e_w, e_s, g, C, beta1, eps, lr):
    """One whole compressed step, in place on x, m, e_w, e_s (v is read only).

    Returns a dict with the step's messages: s, S, bits_w, bits_s, inexact."""
    g, gt = _grads(g)
    W, d = g.shape
    for a in (x, m, e_s):
        assert a.dtype == np.float32 and a.shape == (d,) and a.flags["C_CONTIGUOUS"]
    assert e_w.dtype == np.float32 and e_w.shape == (W, d) and e_w.flags["C_CONTIGUOUS"]
    v = _f32(v, (d,))
    nch = nchunks(d, C)
    s = np.zeros((W, nch), dtype=np.float32)
    S = np.zeros(nch, dtype=np.float32)
    bits_w = np.zeros((W, nwords(d)), dtype=np.uint32)
    bits_s = np.zeros(nwords(d), dtype=np.uint32)
    z = np.zeros(d, dtype=np.float32)
    inexact = lib().oracle_compressed_step(d, W, C, beta1, eps, lr, _p(x), _p(m), _p(v), _p(e_w),
                                           _p(e_s), _p(g), gt, _p(s), _p(S), _p(bits_w),
                                           _p(bits_s), _p(z))
    return {"s": s, "S": S, "bits_w": bits_w, "bits_s": bits_s, "inexact": int(inexact)}


class OracleState:
    """The optimizer state of the method, held on the host: x, m, v and, after the freeze, the
    explicit worker and server residuals. Mirrors the phases of the method: warm-up steps, the
    variance freeze, compressed steps."""

    def __init__(self, x, W, C, beta1=0.9, beta2=0.999, eps=1e-8, bias_correction=False):
        self.x = _f32(x).copy()
        d = self.x.size
        self.d, self.W, self.C = d, W, C
        self.beta1, self.beta2, self.eps = beta1, beta2, eps
        self.bias_correction = bias_correction
        self.t = 0
        self.m = np.zeros(d, dtype=np.float32)
        self.v = np.zeros(d, dtype=np.float32)
        self.e_w = None
        self.e_s = None
        self.frozen = False

    def warmup_step(self, g, lr):
        assert not self.frozen
        self.t += 1
        if self.bias_correction:
            warmup_step_bc(self.x, self.m, self.v, g, self.beta1, self.beta2, self.eps, lr,
                           self.t)
        else:
            warmup_step(self.x, self.m, self.v, g, self.beta1, self.beta2, self.eps, lr)

    def freeze(self):
        """Freeze v as the preconditioner; residuals start at zero (R11). After a
        bias-corrected warm-up, m and v continue corrected (B1)."""
        if self.bias_correction and self.t > 0:
            freeze_bc(self.m, self.v, self.beta1, self.beta2, self.t)
        self.frozen = True
        self.e_w = np.zeros((self.W, self.d), dtype=np.float32)
        self.e_s = np.zeros(self.d, dtype=np.float32)

    def compressed_step(self, g, lr):
        assert self.frozen
        return compressed_step(self.x, self.m, self.v, self.e_w, self.e_s, g, self.C,
                               self.beta1, self.eps, lr)


# ----------------------------------------------------------------------------------------------
# the 0/1 Adam variant (zero_one_oracle.c, readings Z1-Z7)

def _wd(a, W, d, name):
    assert a.dtype == np.float32 and a.shape == (W, d) and a.flags["C_CONTIGUOUS"], name


def zo_local(m_w, u_w, g, beta1, lr):
    """Z3: every worker's local step, in place on m_w and u_w ([W][d])."""
    g, gt = _grads(g)
    W, d = g.shape
    _wd(m_w, W, d, "m_w")
    _wd(u_w, W, d, "u_w")
    lib().oracle01_local(d, W, beta1, lr, _p(m_w), _p(u_w), _p(g), gt)


def zo_compress(u_w, e_w, C):
    """Z4, worker side: 1-bit messages of the accumulated updates; e_w updated in place.

    Returns (s [W][nch] float32, bits_w [W][ceil(d/32)] uint32)."""
    u_w = _f32(u_w)
    W, d = u_w.shape
    _wd(e_w, W, d, "e_w")
    s = np.zeros((W, nchunks(d, C)), dtype=np.float32)
    bits = np.zeros((W, nwords(d)), dtype=np.uint32)
    lib().oracle01_compress(d, W, C, _p(u_w), _p(e_w), _p(s), _p(bits))
    return s, bits


def zo_apply(bits_s, S, v, x, C, eps, gamma, beta2, refresh):
    """Z5-Z6: the synchronised step from the server message, in place on x (and on v when
    `refresh`). Returns mbar [d]."""
    d = x.size
    bits_s = np.ascontiguousarray(bits_s, dtype=np.uint32)
    S = _f32(S)
    for a in (v, x):
        assert a.dtype == np.float32 and a.shape == (d,) and a.flags["C_CONTIGUOUS"]
    mbar = np.zeros(d, dtype=np.float32)
    lib().oracle01_apply(d, C, eps, gamma, beta2, 1 if refresh else 0, _p(bits_s), _p(S),
                         _p(v), _p(x), _p(mbar))
    return mbar


def zo_step(x, m_w, u_w, v, e_w, e_s, g, C, beta1, beta2, eps, lr, gamma, sync, refresh):
    """One step of the variant's compression phase (Z3, and Z4-Z6 when `sync`), in place on
    x, m_w, u_w, v, e_w, e_s. Returns the synchronisation's messages (s, S, bits_w, bits_s,
    mbar, inexact), or None without one."""
    g, gt = _grads(g)
    W, d = g.shape
    for a, nm in ((m_w, "m_w"), (u_w, "u_w"), (e_w, "e_w")):
        _wd(a, W, d, nm)
    for a in (x, v, e_s):
        assert a.dtype == np.float32 and a.shape == (d,) and a.flags["C_CONTIGUOUS"]
    nch = nchunks(d, C)
    s = np.zeros((W, nch), dtype=np.float32)
    S = np.zeros(nch, dtype=np.float32)
    bits_w = np.zeros((W, nwords(d)), dtype=np.uint32)
    bits_s = np.zeros(nwords(d), dtype=np.uint32)
    mbar = np.zeros(d, dtype=np.float32)
    z = np.zeros(d, dtype=np.float32)
    inexact = lib().oracle01_step(d, W, C, beta1, beta2, eps, lr, gamma, 1 if sync else 0,
                                  1 if refresh else 0, _p(x), _p(m_w), _p(u_w), _p(v), _p(e_w),
                                  _p(e_s), _p(g), gt, _p(s), _p(S), _p(bits_w), _p(bits_s),
                                  _p(mbar), _p(z))
    if not sync:
        return None
    return {"s": s, "S": S, "bits_w": bits_w, "bits_s": bits_s, "mbar": mbar,
            "inexact": int(inexact)}


def zo_local_model(x, u, v, eps):
    """Z7: a worker's local model x - u / (sqrt(v) + eps)."""
    x, u, v = _f32(x), _f32(u), _f32(v)
    out = np.zeros(x.size, dtype=np.float32)
    lib().oracle01_local_model(x.size, eps, _p(x), _p(u), _p(v), _p(out))
    return out


class ZeroOneState:
    """The 0/1 Adam variant's state on the host: x, m, v through the warm-up (shared with
    1-bit Adam, Z1); after the freeze every worker's momentum and accumulated update, the
    explicit residuals, and the schedule: a synchronisation every H steps, a variance refresh
    at every K-th synchronisation (K = 0: never), Gamma the fp32 sum of the learning rates since
    the last synchronisation (Z2-Z6)."""

    def __init__(self, x, W, C, H, K, beta1=0.9, beta2=0.999, eps=1e-8):
        assert H >= 1 and K >= 0
        self.x = _f32(x).copy()
        d = self.x.size
        self.d, self.W, self.C, self.H, self.K = d, W, C, H, K
        self.beta1, self.beta2, self.eps = beta1, beta2, eps
        self.m = np.zeros(d, dtype=np.float32)
        self.v = np.zeros(d, dtype=np.float32)
        self.frozen = False
        self.t = 0
        self.syncs = 0
        self.gamma = np.float32(0.0)

    def warmup_step(self, g, lr):
        assert not self.frozen
        warmup_step(self.x, self.m, self.v, g, self.beta1, self.beta2, self.eps, lr)

    def freeze(self):
        """Z2: every worker starts from the warm-up momentum, with u_w = e_w = e_s = 0."""
        self.frozen = True
        self.m_w = np.ascontiguousarray(np.broadcast_to(self.m, (self.W, self.d)),
                                        dtype=np.float32)
        self.u_w = np.zeros((self.W, self.d), dtype=np.float32)
        self.e_w = np.zeros((self.W, self.d), dtype=np.float32)
        self.e_s = np.zeros(self.d, dtype=np.float32)

    def step(self, g, lr):
        assert self.frozen
        self.t += 1
        self.gamma = np.float32(self.gamma + np.float32(lr))
        sync = self.t % self.H == 0
        refresh = sync and self.K > 0 and (self.syncs + 1) % self.K == 0
        out = zo_step(self.x, self.m_w, self.u_w, self.v, self.e_w, self.e_s, g, self.C,
                      self.beta1, self.beta2, self.eps, lr, float(self.gamma), sync, refresh)
        if sync:
            self.syncs += 1
            self.gamma = np.float32(0.0)
            out["refresh"] = refresh
        return out

    def local_model(self, w):
        return zo_local_model(self.x, self.u_w[w], self.v, self.eps)


class use_library:
    """Context manager that routes every oracle call through another build of the C file (the
    test suite uses it to plant mistakes in a copy of the oracle and check its pins catch them)."""

    def __init__(self, path: str):
        self.path = path
        self.saved = None

    def __enter__(self):
        global _lib
        self.saved = _lib
        _lib = _load(self.path)
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False
