"""The no-allocation compression entry point, onebit_compress_static.

Some callers cannot allocate device memory: code embedded in a host application or plugin that
receives only its input and output buffers while the application owns the whole device pool,
or latency-critical paths that cannot afford the synchronisation cudaMalloc/cudaFree imply.
onebit_compress_static gives them the worker compression (sign words plus per-chunk scales)
with its scratch held in a fixed array inside the library. These tests call it through the C
ABI and check its output on two calls in a row -- so that anything the first call leaves in the
shared scratch cannot leak into the second -- against the CPU oracle's worker compression (the
words bit for bit, the scales within the relative 1e-5 of the parity tests) and against the
existing entry points (the words and, since the fp64 partial sums run in the worker kernel's
order, the scales bit for bit).

This file is collected last on purpose: a run that stops at its first failure has already run
every other test before it gets here.
"""
import ctypes

import numpy as np
import pytest
import torch

import communication_compressed_optimizer_momentum_b200 as ob
import oracle
from communication_compressed_optimizer_momentum_b200 import _abi

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
RTOL = 1e-5


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _message_no_alloc(x, C):
    n = x.numel()
    words = torch.empty((n + 31) // 32, dtype=torch.int32, device=DEV)
    scales = torch.empty((n + C - 1) // C, dtype=torch.float32, device=DEV)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = _abi.lib().onebit_compress_static(_ptr(x), n, C, _ptr(words), _ptr(scales), stream)
    assert rc == 0, _abi.lib().onebit_last_error().decode()
    torch.cuda.synchronize()
    return words, scales


def _message_existing(x, C):
    """The same message from the existing entry points: onebit_pack gives the words; a fresh
    W = 1 handle with beta1 = 0 and zero residuals compresses exactly x in its first compressed
    step, which gives the scales (and the words once more)."""
    n = x.numel()
    words = ob.onebit_pack(x)
    opt = ob.OneBitAdam(n, 1, C, beta1=0.0, device=DEV)
    opt.freeze()
    params = torch.zeros(n, device=DEV)
    opt.step(params, x.view(1, n), 1e-3)
    scales = opt.get_state("s").view(-1)
    words_step = opt.get_state("bits_w").view(-1)
    torch.cuda.synchronize()
    opt.close()
    return words, words_step, scales


def _message_oracle(x, C):
    """The oracle's worker compression of x itself: one worker, beta1 = 0 (so the worker's
    momentum is its gradient, here x), zero momentum and zero residuals, so x_w = x exactly."""
    xh = x.detach().cpu().numpy().astype(np.float32)
    n = xh.size
    e_w = np.zeros((1, n), np.float32)
    s, bits = oracle.worker(np.zeros(n, np.float32), xh.reshape(1, n), e_w, C, 0.0)
    return bits.reshape(-1), s.reshape(-1)


def _check_against_oracle(words, scales, x, C):
    ref_words, ref_scales = _message_oracle(x, C)
    np.testing.assert_array_equal(words.cpu().numpy().view(np.uint32), ref_words)
    got = scales.cpu().numpy()
    assert np.all(np.abs(got - ref_scales) <= RTOL * np.abs(ref_scales)), \
        "scales differ from the oracle beyond relative 1e-5"
    return int((got == ref_scales).sum()), got.size


def _vector(n, seed):
    gen = torch.Generator(device=DEV)
    gen.manual_seed(seed)
    x = torch.randn(n, device=DEV, generator=gen) * 1e-2
    x[torch.rand(n, device=DEV, generator=gen) < 0.01] = 0.0
    return x


def test_two_calls_in_a_row_match_existing_entry_points():
    # the second call is smaller and uses another chunk length, so stale partials of the first
    # call would show up in its scales
    for n, C, seed in ((1_000_003, 65_536, 1), (300_001, 8192, 2)):
        x = _vector(n, seed)
        words, scales = _message_no_alloc(x, C)
        _check_against_oracle(words, scales, x, C)
        ref_words, ref_words_step, ref_scales = _message_existing(x, C)
        assert torch.equal(words, ref_words)
        assert torch.equal(words, ref_words_step)
        assert torch.equal(scales, ref_scales)


def test_small_chunks_and_ragged_tail():
    # the last case is shorter than one chunk and not a whole number of words (n < C,
    # n % 32 != 0): one chunk of the true length n
    for n, C, seed in ((777, 32, 3), (4096 * 3 + 100, 4096, 4), (1000, 65_536, 5)):
        x = _vector(n, seed)
        words, scales = _message_no_alloc(x, C)
        _check_against_oracle(words, scales, x, C)
        ref_words, _, ref_scales = _message_existing(x, C)
        assert torch.equal(words, ref_words)
        assert torch.equal(scales, ref_scales)


def test_rejects_inputs_beyond_the_fixed_scratch():
    n, C = 65_537 * 32, 32                      # 65,537 one-segment chunks: one too many
    x = torch.zeros(n, device=DEV)
    words = torch.empty((n + 31) // 32, dtype=torch.int32, device=DEV)
    scales = torch.empty(n // C, dtype=torch.float32, device=DEV)
    rc = _abi.lib().onebit_compress_static(_ptr(x), n, C, _ptr(words), _ptr(scales), None)
    assert rc == -5                              # ONEBIT_ERR_SPACE, before any device work
    assert "fixed scratch" in _abi.lib().onebit_last_error().decode()
