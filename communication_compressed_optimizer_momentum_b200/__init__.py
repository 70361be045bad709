"""1-bit Adam compression phase on B200: Python binding of the C ABI (``include/onebit_adam.h``).

Every function below has the name of the C entry point it wraps and does argument marshalling
only (tensor -> device pointer, stream -> cudaStream_t, status code -> exception). All the
arithmetic of the method runs in the library's CUDA kernels; torch provides device memory and
streams. There is no CPU fallback: if the library is missing or the call fails, an exception is
raised.

``OneBitAdam`` is a small convenience owner of one handle and its torch-allocated workspace.
"""
from __future__ import annotations

import ctypes
from typing import Tuple

from . import _abi

ONEBIT_F32, ONEBIT_BF16 = 0, 1
STATE = {"m": 0, "v": 1, "e_w": 2, "e_s": 3, "s": 4, "S": 5, "bits_w": 6, "bits_s": 7}
FLAG_NAN_WORKER, FLAG_NAN_SERVER = 1, 2
KERNELS = ("worker", "worker_scales", "server", "server_scales", "apply")


class OneBitError(RuntimeError):
    def __init__(self, code: int, where: str):
        L = _abi.lib()
        msg = L.onebit_strerror(code).decode()
        extra = L.onebit_last_error().decode() if code == -4 else ""
        super().__init__("%s failed: %s (%d)%s" % (where, msg, code, (": " + extra) if extra else ""))
        self.code = code


def _check(rc: int, where: str) -> None:
    if rc != 0:
        raise OneBitError(rc, where)


def _ptr(t) -> ctypes.c_void_p:
    if t is None:
        return ctypes.c_void_p(None)
    if isinstance(t, int):
        return ctypes.c_void_p(t)
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    import torch
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def dtype_code(dtype) -> int:
    import torch
    if dtype == torch.float32:
        return ONEBIT_F32
    if dtype == torch.bfloat16:
        return ONEBIT_BF16
    raise TypeError("gradients must be float32 or bfloat16, got %s" % dtype)


def _handle(h) -> ctypes.c_void_p:
    return h if isinstance(h, ctypes.c_void_p) else ctypes.c_void_p(h)


# ----------------------------------------------------------------------------------------------
# the C entry points

def onebit_adam_init(d: int, W: int, C: int, beta1: float = 0.9, beta2: float = 0.999,
                     eps: float = 1e-8) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    _check(_abi.lib().onebit_adam_init(ctypes.byref(h), d, W, C, beta1, beta2, eps),
           "onebit_adam_init")
    return h


def onebit_adam_workspace_bytes(h, grad_dtype: int) -> int:
    n = ctypes.c_uint64()
    _check(_abi.lib().onebit_adam_workspace_bytes(_handle(h), grad_dtype, ctypes.byref(n)),
           "onebit_adam_workspace_bytes")
    return n.value


def onebit_adam_bind(h, workspace, nbytes: int, grad_dtype: int, stream=None) -> None:
    _check(_abi.lib().onebit_adam_bind(_handle(h), _ptr(workspace), nbytes, grad_dtype,
                                       _stream(stream)), "onebit_adam_bind")


def onebit_adam_warmup_step(h, x, grads, lr: float, stream=None) -> None:
    _check(_abi.lib().onebit_adam_warmup_step(_handle(h), _ptr(x), _ptr(grads), lr,
                                              _stream(stream)), "onebit_adam_warmup_step")


def onebit_adam_set_bias_correction(h, on: bool) -> None:
    _check(_abi.lib().onebit_adam_set_bias_correction(_handle(h), 1 if on else 0),
           "onebit_adam_set_bias_correction")


def onebit_adam_freeze_variance(h, stream=None) -> None:
    _check(_abi.lib().onebit_adam_freeze_variance(_handle(h), _stream(stream)),
           "onebit_adam_freeze_variance")


def onebit_adam_compressed_step(h, x, grads, lr: float, stream=None) -> None:
    _check(_abi.lib().onebit_adam_compressed_step(_handle(h), _ptr(x), _ptr(grads), lr,
                                                  _stream(stream)),
           "onebit_adam_compressed_step")


def onebit_adam_compressed_step_host(h, x_dev, grads_dev, grads_host, x_host, lr: float,
                                     stream=None) -> None:
    _check(_abi.lib().onebit_adam_compressed_step_host(
        _handle(h), _ptr(x_dev), _ptr(grads_dev), _ptr(grads_host), _ptr(x_host), lr,
        _stream(stream)), "onebit_adam_compressed_step_host")


def onebit_adam_host_wait(h, stream=None) -> None:
    _check(_abi.lib().onebit_adam_host_wait(_handle(h), _stream(stream)), "onebit_adam_host_wait")


def onebit_adam_state_bytes(h, which: int) -> int:
    n = ctypes.c_uint64()
    _check(_abi.lib().onebit_adam_state_bytes(_handle(h), which, ctypes.byref(n)),
           "onebit_adam_state_bytes")
    return n.value


def onebit_adam_get_state(h, which: int, dst, stream=None) -> None:
    _check(_abi.lib().onebit_adam_get_state(_handle(h), which, _ptr(dst), _stream(stream)),
           "onebit_adam_get_state")


def onebit_adam_get_chunk_state(h, which: int, k: int, dst, stream=None) -> None:
    _check(_abi.lib().onebit_adam_get_chunk_state(_handle(h), which, k, _ptr(dst),
                                                  _stream(stream)),
           "onebit_adam_get_chunk_state")


def onebit_adam_set_state(h, which: int, src, stream=None) -> None:
    _check(_abi.lib().onebit_adam_set_state(_handle(h), which, _ptr(src), _stream(stream)),
           "onebit_adam_set_state")


def onebit_adam_status(h, stream=None) -> int:
    f = ctypes.c_uint32()
    _check(_abi.lib().onebit_adam_status(_handle(h), _stream(stream), ctypes.byref(f)),
           "onebit_adam_status")
    return f.value


def onebit_adam_info(h) -> dict:
    out = (ctypes.c_int64 * 8)()
    _check(_abi.lib().onebit_adam_info(_handle(h), out), "onebit_adam_info")
    keys = ("d", "W", "C", "nch", "phase", "steps", "grad_dtype", "launches_per_step")
    return dict(zip(keys, list(out)))


def onebit_adam_timing(h, max_steps: int) -> None:
    _check(_abi.lib().onebit_adam_timing(_handle(h), max_steps), "onebit_adam_timing")


def onebit_adam_timing_read(h) -> Tuple[dict, int]:
    ms = (ctypes.c_double * 5)()
    n = ctypes.c_int32()
    _check(_abi.lib().onebit_adam_timing_read(_handle(h), ms, ctypes.byref(n)),
           "onebit_adam_timing_read")
    return dict(zip(KERNELS, list(ms))), n.value


def onebit_adam_timing_steps(h, cap: int) -> list:
    """The device time (ms) of each step of the current recording window, at most cap."""
    if cap < 0:
        raise ValueError("cap must be >= 0")
    ms = (ctypes.c_double * max(cap, 1))()
    n = ctypes.c_int32()
    _check(_abi.lib().onebit_adam_timing_steps(_handle(h), ms, cap, ctypes.byref(n)),
           "onebit_adam_timing_steps")
    return list(ms)[:min(cap, n.value)]


def onebit_adam_destroy(h) -> None:
    _abi.lib().onebit_adam_destroy(_handle(h))


def onebit_server_layout(d: int, W: int, C: int) -> dict:
    """The server kernel's layout for a handle of shape (d, W, C) (host only)."""
    out = (ctypes.c_int64 * 5)()
    _check(_abi.lib().onebit_server_layout(d, W, C, out), "onebit_server_layout")
    keys = ("bank_private", "segs_per_block", "smem_bytes", "smem_bytes_dp", "blocks")
    return dict(zip(keys, list(out)))


def onebit_dp_chunk_range(nch: int, R: int, q: int) -> Tuple[int, int]:
    k0, k1 = ctypes.c_int64(), ctypes.c_int64()
    _check(_abi.lib().onebit_dp_chunk_range(nch, R, q, ctypes.byref(k0), ctypes.byref(k1)),
           "onebit_dp_chunk_range")
    return k0.value, k1.value


def onebit_dp_init(d: int, W: int, C: int, beta1: float, beta2: float, eps: float, R: int,
                   rank: int) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    _check(_abi.lib().onebit_dp_init(ctypes.byref(h), d, W, C, beta1, beta2, eps, R, rank),
           "onebit_dp_init")
    return h


def onebit_dp_info(h) -> dict:
    out = (ctypes.c_int64 * 8)()
    _check(_abi.lib().onebit_dp_info(_handle(h), out), "onebit_dp_info")
    keys = ("R", "rank", "W", "k0", "k1", "e0", "d_own", "exchange_bytes")
    return dict(zip(keys, list(out)))


def onebit_dp_exchange(h) -> Tuple[int, int]:
    base, n = ctypes.c_void_p(), ctypes.c_uint64()
    _check(_abi.lib().onebit_dp_exchange(_handle(h), ctypes.byref(base), ctypes.byref(n)),
           "onebit_dp_exchange")
    return base.value, n.value


def onebit_dp_ipc_handle(h) -> bytes:
    buf = ctypes.create_string_buffer(64)
    _check(_abi.lib().onebit_dp_ipc_handle(_handle(h), buf), "onebit_dp_ipc_handle")
    return buf.raw


def onebit_dp_open_peer(h, q: int, handle: bytes) -> None:
    buf = ctypes.create_string_buffer(bytes(handle), 64)
    _check(_abi.lib().onebit_dp_open_peer(_handle(h), q, buf), "onebit_dp_open_peer")


def onebit_dp_set_peer(h, q: int, base: int) -> None:
    _check(_abi.lib().onebit_dp_set_peer(_handle(h), q, ctypes.c_void_p(base)),
           "onebit_dp_set_peer")


def onebit_dp_connect(h, stream=None) -> None:
    _check(_abi.lib().onebit_dp_connect(_handle(h), _stream(stream)), "onebit_dp_connect")


def onebit_dp_set_timeout(h, timeout_us: int) -> None:
    _check(_abi.lib().onebit_dp_set_timeout(_handle(h), timeout_us), "onebit_dp_set_timeout")


def onebit_dp_warmup_phase(h, phase: int, x, grads, lr: float, stream=None) -> None:
    _check(_abi.lib().onebit_dp_warmup_phase(_handle(h), phase, _ptr(x), _ptr(grads), lr,
                                             _stream(stream)), "onebit_dp_warmup_phase")


def onebit_dp_compressed_phase(h, phase: int, x, grads, lr: float, stream=None) -> None:
    _check(_abi.lib().onebit_dp_compressed_phase(_handle(h), phase, _ptr(x), _ptr(grads), lr,
                                                 _stream(stream)), "onebit_dp_compressed_phase")


def onebit01_init(d: int, W: int, C: int, beta1: float, beta2: float, eps: float, H: int,
                  K: int) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    _check(_abi.lib().onebit01_init(ctypes.byref(h), d, W, C, beta1, beta2, eps, H, K),
           "onebit01_init")
    return h


def onebit01_step(h, x, grads, lr: float, stream=None) -> None:
    _check(_abi.lib().onebit01_step(_handle(h), _ptr(x), _ptr(grads), lr, _stream(stream)),
           "onebit01_step")


def onebit01_info(h) -> dict:
    out = (ctypes.c_int64 * 6)()
    _check(_abi.lib().onebit01_info(_handle(h), out), "onebit01_info")
    keys = ("H", "K", "steps_since_sync", "syncs", "momentum_source", "launches_next_step")
    return dict(zip(keys, list(out)))


def onebit01_get_worker_state(h, which: int, k: int, dst, stream=None) -> None:
    _check(_abi.lib().onebit01_get_worker_state(_handle(h), which, k, _ptr(dst),
                                                _stream(stream)), "onebit01_get_worker_state")


def onebit01_local_model(h, w: int, x, out, stream=None) -> None:
    _check(_abi.lib().onebit01_local_model(_handle(h), w, _ptr(x), _ptr(out), _stream(stream)),
           "onebit01_local_model")


def onebit01_set_worker_state(h, which: int, src, stream=None) -> None:
    _check(_abi.lib().onebit01_set_worker_state(_handle(h), which, _ptr(src), _stream(stream)),
           "onebit01_set_worker_state")


def onebit01_get_schedule(h) -> dict:
    ints = (ctypes.c_int64 * 2)()
    floats = (ctypes.c_float * 2)()
    _check(_abi.lib().onebit01_get_schedule(_handle(h), ints, floats), "onebit01_get_schedule")
    return {"steps_since_sync": ints[0], "syncs": ints[1], "gamma": floats[0],
            "gamma_prev": floats[1]}


def onebit01_set_schedule(h, sched: dict) -> None:
    ints = (ctypes.c_int64 * 2)(sched["steps_since_sync"], sched["syncs"])
    floats = (ctypes.c_float * 2)(sched["gamma"], sched["gamma_prev"])
    _check(_abi.lib().onebit01_set_schedule(_handle(h), ints, floats), "onebit01_set_schedule")


def onebit01_dp_init(d: int, W: int, C: int, beta1: float, beta2: float, eps: float, H: int,
                     K: int, R: int, rank: int) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    _check(_abi.lib().onebit01_dp_init(ctypes.byref(h), d, W, C, beta1, beta2, eps, H, K, R,
                                       rank), "onebit01_dp_init")
    return h


def onebit01_dp_phase(h, phase: int, x, grads, lr: float, stream=None) -> None:
    _check(_abi.lib().onebit01_dp_phase(_handle(h), phase, _ptr(x), _ptr(grads), lr,
                                        _stream(stream)), "onebit01_dp_phase")


def onebit_strerror(code: int) -> str:
    return _abi.lib().onebit_strerror(code).decode()


def onebit_last_error() -> str:
    return _abi.lib().onebit_last_error().decode()


def onebit_selftest_bounded_wait(polls: int, stream=None) -> bool:
    """Run the bounded-wait self-test; True when the wait gave up as it should."""
    import torch
    flag = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    _check(_abi.lib().onebit_selftest_bounded_wait(polls, _ptr(flag), _stream(stream)),
           "onebit_selftest_bounded_wait")
    return int(flag.item()) == 1


def _device_vector(t, dtype, min_numel: int, name: str, device=None):
    """Check that ``t`` is a contiguous CUDA tensor of ``dtype`` with at least ``min_numel``
    elements (on ``device`` when given) before its pointer goes to the library, which trusts
    the sizes it is given."""
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if t.device.type != "cuda":
        raise ValueError("%s must be a CUDA tensor, got device %s" % (name, t.device))
    if device is not None and t.device != device:
        raise ValueError("%s is on %s, expected %s" % (name, t.device, device))
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if t.numel() < min_numel:
        raise ValueError("%s holds %d elements, needs at least %d" % (name, t.numel(), min_numel))


def _chunk_length(C: int) -> int:
    C = int(C)
    if C <= 0 or C % 32 != 0:
        raise ValueError("chunk length C must be a positive multiple of 32, got %d" % C)
    return C


def onebit_pack(x, words=None, stream=None):
    """Sign-pack a contiguous float32 CUDA tensor into int32 words (LSB-first)."""
    import torch
    _device_vector(x, torch.float32, 0, "x")
    n = x.numel()
    if words is None:
        words = torch.empty((n + 31) // 32, dtype=torch.int32, device=x.device)
    _device_vector(words, torch.int32, (n + 31) // 32, "words", x.device)
    with torch.cuda.device(x.device):
        st = _stream(stream if stream is not None else torch.cuda.current_stream(x.device))
        _check(_abi.lib().onebit_pack(_ptr(x), n, _ptr(words), st), "onebit_pack")
    return words


def onebit_unpack(words, scales, n: int, C: int, out=None, stream=None):
    """Decompress packed words with per-chunk scales into a float32 CUDA tensor (C >= 1)."""
    import torch
    n, C = int(n), int(C)
    if n < 0 or C < 1:
        raise ValueError("need n >= 0 and C >= 1, got n=%d C=%d" % (n, C))
    _device_vector(words, torch.int32, (n + 31) // 32, "words")
    _device_vector(scales, torch.float32, (n + C - 1) // C, "scales", words.device)
    if out is None:
        out = torch.empty(n, dtype=torch.float32, device=words.device)
    _device_vector(out, torch.float32, n, "out", words.device)
    with torch.cuda.device(words.device):
        st = _stream(stream if stream is not None else torch.cuda.current_stream(words.device))
        _check(_abi.lib().onebit_unpack(_ptr(words), _ptr(scales), n, C, _ptr(out), st),
               "onebit_unpack")
    return out


def onebit_compress_static(x, C: int, words=None, scales=None, stream=None):
    """Sign words and per-chunk scales of a float32 CUDA tensor, computed without any device
    allocation inside the library (its scratch is a fixed array in the library). For callers
    that cannot allocate, pass preallocated ``words`` (int32, ceil(n/32)) and ``scales``
    (float32, ceil(n/C)); the defaults here allocate them with torch for convenience."""
    import torch
    C = _chunk_length(C)
    _device_vector(x, torch.float32, 0, "x")
    n = x.numel()
    if words is None:
        words = torch.empty((n + 31) // 32, dtype=torch.int32, device=x.device)
    if scales is None:
        scales = torch.empty((n + C - 1) // C, dtype=torch.float32, device=x.device)
    _device_vector(words, torch.int32, (n + 31) // 32, "words", x.device)
    _device_vector(scales, torch.float32, (n + C - 1) // C, "scales", x.device)
    with torch.cuda.device(x.device):
        st = _stream(stream if stream is not None else torch.cuda.current_stream(x.device))
        _check(_abi.lib().onebit_compress_static(_ptr(x), n, C, _ptr(words), _ptr(scales), st),
               "onebit_compress_static")
    return words, scales


# ----------------------------------------------------------------------------------------------
# convenience owner of one handle + workspace

class OneBitAdam:
    """One optimizer instance: the handle plus its device workspace (allocated with torch).

    Phases follow the method: ``warmup_step`` (full-precision Adam) any number of times, then
    ``freeze()`` (the variance becomes the fixed preconditioner), then ``step`` (compressed)."""

    def __init__(self, d: int, W: int, C: int, beta1: float = 0.9, beta2: float = 0.999,
                 eps: float = 1e-8, grad_dtype=None, device="cuda", stream=None,
                 bias_correction: bool = False):
        h = onebit_adam_init(d, W, C, beta1, beta2, eps)
        if bias_correction:
            onebit_adam_set_bias_correction(h, True)
        self._setup(h, d, W, C, grad_dtype, device, stream)

    def _setup(self, h, d, W, C, grad_dtype, device, stream):
        import torch
        grad_dtype = torch.float32 if grad_dtype is None else grad_dtype
        self.d, self.W, self.C = d, W, C
        self.grad_dtype = grad_dtype
        self.h = h
        code = dtype_code(grad_dtype)
        nbytes = onebit_adam_workspace_bytes(self.h, code)
        raw = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
        shift = (-raw.data_ptr()) % 256
        self._raw = raw
        self.workspace = raw[shift:shift + nbytes]
        self.workspace_bytes = nbytes
        onebit_adam_bind(self.h, self.workspace, nbytes, code, stream)
        self.nch = (d + C - 1) // C

    def warmup_step(self, x, grads, lr: float, stream=None) -> None:
        onebit_adam_warmup_step(self.h, x, grads, lr, stream)

    def freeze(self, stream=None) -> None:
        onebit_adam_freeze_variance(self.h, stream)

    def step(self, x, grads, lr: float, stream=None) -> None:
        onebit_adam_compressed_step(self.h, x, grads, lr, stream)

    def step_host(self, x_dev, grads_dev, grads_host, x_host, lr: float, stream=None) -> None:
        onebit_adam_compressed_step_host(self.h, x_dev, grads_dev, grads_host, x_host, lr, stream)

    def host_wait(self, stream=None) -> None:
        onebit_adam_host_wait(self.h, stream)

    def state_shape(self, which: str):
        d, W, nch, nw = self.d, self.W, self.nch, (self.d + 31) // 32
        return {"m": (d,), "v": (d,), "e_w": (W, d), "e_s": (d,), "s": (W, nch), "S": (nch,),
                "bits_w": (W, nw), "bits_s": (nw,)}[which]

    def get_state(self, which: str, stream=None):
        import torch
        dt = torch.int32 if which.startswith("bits") else torch.float32
        out = torch.empty(self.state_shape(which), dtype=dt, device=self.workspace.device)
        onebit_adam_get_state(self.h, STATE[which], out, stream)
        return out

    def chunk_shape(self, which: str, k: int):
        n = min(self.C, self.d - k * self.C)
        nwk = (n + 31) // 32
        return {"m": (n,), "v": (n,), "e_w": (self.W, n), "e_s": (n,), "s": (self.W,),
                "S": (1,), "bits_w": (self.W, nwk), "bits_s": (nwk,)}[which]

    def get_chunk_state(self, which: str, k: int, stream=None):
        import torch
        dt = torch.int32 if which.startswith("bits") else torch.float32
        out = torch.empty(self.chunk_shape(which, k), dtype=dt, device=self.workspace.device)
        onebit_adam_get_chunk_state(self.h, STATE[which], k, out, stream)
        return out

    def set_state(self, which: str, src, stream=None) -> None:
        assert tuple(src.shape) == self.state_shape(which) and src.is_contiguous()
        onebit_adam_set_state(self.h, STATE[which], src, stream)

    def status(self, stream=None) -> int:
        return onebit_adam_status(self.h, stream)

    def info(self) -> dict:
        return onebit_adam_info(self.h)

    def timing(self, max_steps: int) -> None:
        onebit_adam_timing(self.h, max_steps)

    def timing_read(self):
        return onebit_adam_timing_read(self.h)

    def timing_steps(self, cap: int = 1 << 16):
        """Device time (ms) of each step recorded in the current window (before timing_read)."""
        return onebit_adam_timing_steps(self.h, cap)

    def close(self) -> None:
        if getattr(self, "h", None) is not None:
            onebit_adam_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class ZeroOneAdam(OneBitAdam):
    """One optimizer instance of the 0/1 Adam variant: the warm-up and the freeze of 1-bit Adam,
    then ``step`` runs the variant's compression phase -- a local step on every worker, and
    every H-th step a synchronisation through the compressed allreduce of the workers'
    accumulated updates, with a variance refresh at every K-th synchronisation (K = 0: never)."""

    WORKER_STATE = {"m_w": 0, "u_w": 1}

    def __init__(self, d: int, W: int, C: int, H: int, K: int, beta1: float = 0.9,
                 beta2: float = 0.999, eps: float = 1e-8, grad_dtype=None, device="cuda",
                 stream=None):
        self.H, self.K = H, K
        self._setup(onebit01_init(d, W, C, beta1, beta2, eps, H, K), d, W, C, grad_dtype,
                    device, stream)

    def step(self, x, grads, lr: float, stream=None) -> None:
        onebit01_step(self.h, x, grads, lr, stream)

    def zo_info(self) -> dict:
        return onebit01_info(self.h)

    def get_worker_state(self, which: str, k: int = -1, stream=None):
        """Every worker's momentum ("m_w") or accumulated update ("u_w"): [W][d], or [W][C_k]
        for chunk k."""
        import torch
        n = self.d if k < 0 else min(self.C, self.d - k * self.C)
        out = torch.empty((self.W, n), dtype=torch.float32, device=self.workspace.device)
        onebit01_get_worker_state(self.h, self.WORKER_STATE[which], k, out, stream)
        return out

    def set_worker_state(self, which: str, src, stream=None) -> None:
        """Every worker's momentum ("m_w") or accumulated update ("u_w") from src ([W][d]); the
        next step starts from them (set both)."""
        assert tuple(src.shape) == (self.W, self.d) and src.is_contiguous()
        onebit01_set_worker_state(self.h, self.WORKER_STATE[which], src, stream)

    def schedule(self) -> dict:
        return onebit01_get_schedule(self.h)

    def set_schedule(self, sched: dict) -> None:
        onebit01_set_schedule(self.h, sched)

    def checkpoint(self, stream=None) -> dict:
        """Everything a handle restored after its freeze needs to continue bit for bit (the
        parameters x are the caller's)."""
        st = {nm: self.get_state(nm, stream) for nm in ("v", "e_w", "e_s")}
        st.update({nm: self.get_worker_state(nm, -1, stream) for nm in ("m_w", "u_w")})
        st["schedule"] = self.schedule()
        return st

    def restore(self, st: dict, stream=None) -> None:
        """Load a checkpoint into a frozen handle of the same shape and schedule."""
        for nm in ("v", "e_w", "e_s"):
            self.set_state(nm, st[nm], stream)
        for nm in ("m_w", "u_w"):
            self.set_worker_state(nm, st[nm], stream)
        self.set_schedule(st["schedule"])

    def local_model(self, w: int, x, stream=None):
        import torch
        out = torch.empty(self.d, dtype=torch.float32, device=self.workspace.device)
        onebit01_local_model(self.h, w, x, out, stream)
        return out
