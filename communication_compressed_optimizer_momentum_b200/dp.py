"""Data-parallel ranks of the compressed allreduce (the ``onebit_dp_*`` entry points).

``OneBitAdamRank`` owns one rank's handle and workspace (``ZeroOneAdamRank`` the same for the
0/1 Adam variant, whose synchronising steps use the same exchange). Rank q holds W / R of the W workers and
serves the chunks ``onebit_dp_chunk_range(nch, R, q)``; its kernels store plane slices and scales
straight into the serving rank's exchange region and the server plane into every rank's, with a
device-side barrier after each half of the exchange (see ``include/onebit_adam.h``).

Two ways to connect the ranks:

* ``connect_process_group(rank_opt)``: one process per GPU under ``torch.distributed``; the
  exchange regions are mapped between the processes through CUDA IPC handles that the ranks
  all-gather over the process group (host plumbing only; no tensor of the method crosses it).
* ``EmulatedRanks``: R ranks as R handles in one process on one GPU, their exchange regions
  addressed directly, each step driven phase by phase across the ranks (phase p of every rank
  before phase p + 1 of any), so that no rank's barrier ever waits for a rank that has not been
  launched. The arithmetic and the data movement are those of R real ranks; only the transport
  is this GPU's own memory instead of NVLink.
"""
from __future__ import annotations

from typing import List, Sequence

from . import (OneBitAdam, ZeroOneAdam, onebit01_dp_init, onebit01_dp_phase,
               onebit_dp_chunk_range, onebit_dp_compressed_phase, onebit_dp_connect,
               onebit_dp_exchange, onebit_dp_info, onebit_dp_init, onebit_dp_ipc_handle,
               onebit_dp_open_peer, onebit_dp_set_peer, onebit_dp_set_timeout,
               onebit_dp_warmup_phase)

MAX_RANKS = 8


class OneBitAdamRank(OneBitAdam):
    """Rank ``rank`` of ``R``: W counts the workers of all ranks (W % R == 0); this rank's
    gradients are [W / R][d]. Bind happens here; connect the ranks before the first step."""

    def __init__(self, d: int, W: int, C: int, R: int, rank: int, beta1: float = 0.9,
                 beta2: float = 0.999, eps: float = 1e-8, grad_dtype=None, device="cuda",
                 stream=None):
        self._rank_setup(onebit_dp_init(d, W, C, beta1, beta2, eps, R, rank), d, W, C, R, rank,
                         grad_dtype, device, stream)

    def _rank_setup(self, h, d, W, C, R, rank, grad_dtype, device, stream):
        self.R, self.rank, self.W_all = R, rank, W
        self._setup(h, d, W // R, C, grad_dtype, device, stream)
        info = onebit_dp_info(self.h)
        self.k0, self.k1 = info["k0"], info["k1"]
        self.e0, self.d_own = info["e0"], info["d_own"]
        self.exchange_bytes = info["exchange_bytes"]

    def dp_info(self) -> dict:
        return onebit_dp_info(self.h)

    def exchange(self):
        return onebit_dp_exchange(self.h)

    def ipc_handle(self) -> bytes:
        return onebit_dp_ipc_handle(self.h)

    def open_peer(self, q: int, handle: bytes) -> None:
        onebit_dp_open_peer(self.h, q, handle)

    def set_peer(self, q: int, base: int) -> None:
        onebit_dp_set_peer(self.h, q, base)

    def connect(self, stream=None) -> None:
        onebit_dp_connect(self.h, stream)

    def set_timeout_us(self, timeout_us: int) -> None:
        onebit_dp_set_timeout(self.h, timeout_us)

    def warmup_phase(self, phase: int, x, grads, lr: float, stream=None) -> None:
        onebit_dp_warmup_phase(self.h, phase, x, grads, lr, stream)

    def compressed_phase(self, phase: int, x, grads, lr: float, stream=None) -> None:
        onebit_dp_compressed_phase(self.h, phase, x, grads, lr, stream)

    def state_shape(self, which: str):
        if which == "e_s":
            return (self.d_own,)
        return super().state_shape(which)


class ZeroOneAdamRank(OneBitAdamRank):
    """Rank ``rank`` of ``R`` of the 0/1 Adam variant: a ``OneBitAdamRank`` whose compression
    phase is the variant's (``ZeroOneAdam``): local steps exchange nothing, and every H-th step
    synchronises through the same exchange as 1-bit Adam's data-parallel step. ``step`` is the
    whole step (separate processes); ``zo_phase`` drives emulated ranks phase by phase."""

    WORKER_STATE = ZeroOneAdam.WORKER_STATE

    def __init__(self, d: int, W: int, C: int, R: int, rank: int, H: int, K: int,
                 beta1: float = 0.9, beta2: float = 0.999, eps: float = 1e-8, grad_dtype=None,
                 device="cuda", stream=None):
        self.H, self.K = H, K
        self._rank_setup(onebit01_dp_init(d, W, C, beta1, beta2, eps, H, K, R, rank), d, W, C,
                         R, rank, grad_dtype, device, stream)

    step = ZeroOneAdam.step
    zo_info = ZeroOneAdam.zo_info
    get_worker_state = ZeroOneAdam.get_worker_state
    set_worker_state = ZeroOneAdam.set_worker_state
    schedule = ZeroOneAdam.schedule
    set_schedule = ZeroOneAdam.set_schedule
    checkpoint = ZeroOneAdam.checkpoint
    restore = ZeroOneAdam.restore
    local_model = ZeroOneAdam.local_model

    def zo_phase(self, phase: int, x, grads, lr: float, stream=None) -> None:
        onebit01_dp_phase(self.h, phase, x, grads, lr, stream)


def connect_process_group(opt: OneBitAdamRank, group=None) -> None:
    """Connect this process's rank to the others of a ``torch.distributed`` group (one process
    per GPU, rank order = the group's): all-gather the exchange regions' IPC handles, map the
    peers', build the route, and wait until every rank has done so."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    me = dist.get_rank(group)
    if world != opt.R or me != opt.rank:
        raise ValueError("handle is rank %d of %d, process group rank %d of %d"
                         % (opt.rank, opt.R, me, world))
    handles: List[bytes] = [b""] * world
    dist.all_gather_object(handles, opt.ipc_handle(), group=group)
    for q in range(world):
        if q != me:
            opt.open_peer(q, handles[q])
    opt.connect()
    torch.cuda.synchronize()
    dist.barrier(group=group)


class EmulatedRanks:
    """R ranks of one data-parallel job as R handles on this process's GPU.

    ``xs[r]`` is rank r's copy of the parameters and ``grads[r]`` its [W / R][d] gradients; all
    ranks are stepped together, phase by phase, on one stream."""

    def __init__(self, d: int, W: int, C: int, R: int, beta1: float = 0.9, beta2: float = 0.999,
                 eps: float = 1e-8, grad_dtype=None, device="cuda", stream=None,
                 zero_one=None):
        """zero_one = (H, K): ranks of the 0/1 Adam variant (ZeroOneAdamRank) instead of 1-bit
        Adam's."""
        if not 1 <= R <= MAX_RANKS:
            raise ValueError("1 <= R <= %d" % MAX_RANKS)
        self.d, self.W, self.C, self.R = d, W, C, R
        self.zero_one = zero_one
        if zero_one is None:
            self.ranks = [OneBitAdamRank(d, W, C, R, r, beta1, beta2, eps, grad_dtype, device,
                                         stream) for r in range(R)]
        else:
            H, K = zero_one
            self.ranks = [ZeroOneAdamRank(d, W, C, R, r, H, K, beta1, beta2, eps, grad_dtype,
                                          device, stream) for r in range(R)]
        bases = [opt.exchange()[0] for opt in self.ranks]
        for r, opt in enumerate(self.ranks):
            for q in range(R):
                if q != r:
                    opt.set_peer(q, bases[q])
            opt.connect(stream)

    def warmup_step(self, xs: Sequence, grads: Sequence, lr: float, stream=None) -> None:
        for p in range(3):
            for r, opt in enumerate(self.ranks):
                opt.warmup_phase(p, xs[r], grads[r], lr, stream)

    def freeze(self, stream=None) -> None:
        for opt in self.ranks:
            opt.freeze(stream)

    def step(self, xs: Sequence, grads: Sequence, lr: float, stream=None) -> None:
        for p in range(3):
            for r, opt in enumerate(self.ranks):
                if self.zero_one is None:
                    opt.compressed_phase(p, xs[r], grads[r], lr, stream)
                else:
                    opt.zo_phase(p, xs[r], grads[r], lr, stream)

    def status(self, stream=None) -> int:
        flags = 0
        for opt in self.ranks:
            flags |= opt.status(stream)
        return flags

    def owner(self, k: int) -> int:
        """The rank that serves chunk k."""
        nch = (self.d + self.C - 1) // self.C
        for q in range(self.R):
            k0, k1 = onebit_dp_chunk_range(nch, self.R, q)
            if k0 <= k < k1:
                return q
        raise IndexError(k)

    def close(self) -> None:
        """Release every rank together (a rank must not step once a peer's exchange region is
        freed); waits for the device first."""
        import torch
        if self.ranks:
            torch.cuda.synchronize()
        for opt in self.ranks:
            opt.close()
        self.ranks = []
