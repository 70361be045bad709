"""The C ABI without a GPU: the library loads, exports every function the public header
declares, and rejects bad arguments on the host before any device work."""
import ctypes
import os
import re

import pytest

import communication_compressed_optimizer_momentum_b200 as ob
from communication_compressed_optimizer_momentum_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "onebit_adam.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(onebit\w*)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from communication_compressed_optimizer_momentum_b200 import build
    build.build()
    return _abi.lib()


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("onebit_adam_init", "onebit_adam_warmup_step", "onebit_adam_freeze_variance",
              "onebit_adam_compressed_step", "onebit_pack", "onebit_unpack"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    # the binding wraps each of them with the same name
    assert set(names) <= set(_abi.SIGNATURES)
    for n in names:
        assert hasattr(ob, n), n


def test_init_validates_arguments(lib):
    h = ctypes.c_void_p()
    ok = lib.onebit_adam_init(ctypes.byref(h), 1000, 4, 256, 0.9, 0.999, 1e-8)
    assert ok == 0 and h.value
    lib.onebit_adam_destroy(h)
    bad = [
        ((-1, 4, 256, 0.9, 0.999, 1e-8), -1),     # negative d
        ((1000, 0, 256, 0.9, 0.999, 1e-8), -1),   # no workers
        ((1000, 257, 256, 0.9, 0.999, 1e-8), -1), # too many workers
        ((1000, 4, 0, 0.9, 0.999, 1e-8), -1),     # empty chunk
        ((1000, 4, 100, 0.9, 0.999, 1e-8), -2),   # chunk not a multiple of 32
        ((1000, 4, 256, 1.0, 0.999, 1e-8), -1),   # beta1 out of [0, 1)
        ((1000, 4, 256, 0.9, -0.1, 1e-8), -1),    # beta2 out of [0, 1)
        ((1000, 4, 256, 0.9, 0.999, -1.0), -1),   # negative eps
        ((1000, 4, 256, float("nan"), 0.999, 1e-8), -1),
    ]
    for args, code in bad:
        h = ctypes.c_void_p()
        assert lib.onebit_adam_init(ctypes.byref(h), *args) == code, args
        assert not h.value
    assert lib.onebit_adam_init(None, 10, 1, 32, 0.9, 0.999, 1e-8) == -1


def test_empty_vector_is_a_valid_problem(lib):
    h = ob.onebit_adam_init(0, 3, 64)
    info = ob.onebit_adam_info(h)
    assert info["d"] == 0 and info["nch"] == 0 and info["phase"] == 0
    assert ob.onebit_adam_state_bytes(h, ob.STATE["e_w"]) == 0
    ob.onebit_adam_destroy(h)


def test_phase_rules_before_bind(lib):
    """Unbound handles refuse every step with ONEBIT_ERR_PHASE, before touching the device."""
    h = ob.onebit_adam_init(4096, 2, 1024)
    for fn in (lambda: lib.onebit_adam_compressed_step(h, None, None, ctypes.c_float(1e-3), None),
               lambda: lib.onebit_adam_warmup_step(h, None, None, ctypes.c_float(1e-3), None),
               lambda: lib.onebit_adam_freeze_variance(h, None)):
        assert fn() == -3
    flags = ctypes.c_uint32()
    assert lib.onebit_adam_status(h, None, ctypes.byref(flags)) == -3
    ob.onebit_adam_destroy(h)


def test_workspace_size_and_bind_checks(lib):
    h = ob.onebit_adam_init(100_003, 5, 4096)
    n32 = ob.onebit_adam_workspace_bytes(h, ob.ONEBIT_F32)
    # m, v, e_s, e_w (W+3 fp32 vectors) plus planes, scales and partials
    assert n32 >= (5 + 3) * 100_003 * 4
    with pytest.raises(ob.OneBitError):
        ob.onebit_adam_workspace_bytes(h, 7)
    # misaligned or short workspaces are rejected on the host
    assert lib.onebit_adam_bind(h, ctypes.c_void_p(0x1001), n32, 0, None) == -2
    assert lib.onebit_adam_bind(h, ctypes.c_void_p(0x100000), n32 - 1, 0, None) == -5
    assert lib.onebit_adam_bind(h, ctypes.c_void_p(0x100000), n32, 3, None) == -1
    assert lib.onebit_adam_bind(h, None, n32, 0, None) == -1
    ob.onebit_adam_destroy(h)


def test_state_sizes(lib):
    d, W, C = 1000, 3, 256
    h = ob.onebit_adam_init(d, W, C)
    nch, nw = 4, 32
    exp = {"m": d * 4, "v": d * 4, "e_w": W * d * 4, "e_s": d * 4, "s": W * nch * 4,
           "S": nch * 4, "bits_w": W * nw * 4, "bits_s": nw * 4}
    for k, v in exp.items():
        assert ob.onebit_adam_state_bytes(h, ob.STATE[k]) == v, k
    with pytest.raises(ob.OneBitError):
        ob.onebit_adam_state_bytes(h, 99)
    ob.onebit_adam_destroy(h)


def test_pack_unpack_host_checks(lib):
    assert lib.onebit_pack(None, -1, None, None) == -1
    assert lib.onebit_pack(None, 0, None, None) == 0          # empty input: nothing to do
    assert lib.onebit_pack(ctypes.c_void_p(0x1004), 10, ctypes.c_void_p(0x2000), None) == -2
    assert lib.onebit_unpack(None, None, 0, 32, None, None) == 0
    assert lib.onebit_unpack(None, None, 10, 0, None, None) == -1


def test_timing_arguments(lib):
    h = ob.onebit_adam_init(1000, 2, 256)
    with pytest.raises(ob.OneBitError):
        ob.onebit_adam_timing(h, -1)
    ob.onebit_adam_timing(h, 0)
    ms, n = ob.onebit_adam_timing_read(h)
    assert n == 0 and all(v == 0.0 for v in ms.values())
    ob.onebit_adam_destroy(h)


def test_strerror_covers_codes(lib):
    for c in (0, -1, -2, -3, -4, -5):
        assert lib.onebit_strerror(c).decode() != "unknown status"
    assert lib.onebit_strerror(12345).decode() == "unknown status"


def test_zero_one_entry_points_validate_on_the_host(lib):
    """The 0/1 Adam variant's entry points reject bad arguments and wrong handles before any
    device work."""
    h = ctypes.c_void_p()
    assert lib.onebit01_init(ctypes.byref(h), 1000, 4, 256, 0.9, 0.999, 1e-8, 0, 1) == -1
    assert h.value is None
    assert lib.onebit01_init(ctypes.byref(h), 1000, 4, 256, 0.9, 0.999, 1e-8, 4, -1) == -1
    assert lib.onebit01_init(ctypes.byref(h), 1000, 4, 100, 0.9, 0.999, 1e-8, 4, 1) == -2
    assert lib.onebit01_init(ctypes.byref(h), 1000, 4, 256, 0.9, 0.999, 1e-8, 4, 2) == 0
    info = (ctypes.c_int64 * 6)()
    assert lib.onebit01_info(h, info) == 0
    assert list(info)[:4] == [4, 2, 0, 0]
    # unbound: no step, no state
    assert lib.onebit01_step(h, None, None, ctypes.c_float(1e-3), None) == -3
    assert lib.onebit01_get_worker_state(h, 0, -1, ctypes.c_void_p(0x1000), None) == -3
    assert lib.onebit01_get_worker_state(h, 2, -1, ctypes.c_void_p(0x1000), None) == -1
    assert lib.onebit01_local_model(h, 4, ctypes.c_void_p(0x1000), ctypes.c_void_p(0x2000),
                                    None) == -1
    lib.onebit_adam_destroy(h)
    # a 1-bit Adam handle is not a 0/1 handle
    one = ctypes.c_void_p()
    assert lib.onebit_adam_init(ctypes.byref(one), 1000, 4, 256, 0.9, 0.999, 1e-8) == 0
    assert lib.onebit01_info(one, info) == -1
    assert lib.onebit01_step(one, None, None, ctypes.c_float(1e-3), None) == -3
    lib.onebit_adam_destroy(one)


def test_zero_one_ranks_validate_on_the_host(lib):
    """The 0/1 variant's data-parallel entry points check their arguments, the handle kind and
    the phase before any device work, and a rank's workspace holds its own workers' state."""
    h = ctypes.c_void_p()
    args = (1000, 4, 256, 0.9, 0.999, 1e-8)
    assert lib.onebit01_dp_init(ctypes.byref(h), *args, 0, 1, 2, 0) == -1        # H = 0
    assert h.value is None
    assert lib.onebit01_dp_init(ctypes.byref(h), *args, 3, -1, 2, 0) == -1       # K < 0
    assert lib.onebit01_dp_init(ctypes.byref(h), 1000, 6, 256, 0.9, 0.999, 1e-8, 3, 1, 4, 0) == -1
    assert lib.onebit01_dp_init(ctypes.byref(h), *args, 3, 1, 2, 2) == -1        # rank >= R
    assert lib.onebit01_dp_init(ctypes.byref(h), 1000, 4, 100, 0.9, 0.999, 1e-8, 3, 1, 2, 0) == -2
    assert lib.onebit01_dp_init(ctypes.byref(h), *args, 3, 1, 2, 1) == 0
    info = (ctypes.c_int64 * 6)()
    assert lib.onebit01_info(h, info) == 0 and list(info)[:4] == [3, 1, 0, 0]
    lr = ctypes.c_float(1e-3)
    assert lib.onebit01_dp_phase(h, 0, None, None, lr, None) == -3              # before freeze
    assert lib.onebit01_dp_phase(h, 3, None, None, lr, None) == -1
    assert lib.onebit01_dp_phase(h, 0, None, None, ctypes.c_float(float("nan")), None) == -1
    # a 1-bit rank's phases and a 0/1 rank's are not interchangeable; single-GPU handles have
    # no phases
    one = ctypes.c_void_p()
    assert lib.onebit_dp_init(ctypes.byref(one), *args, 2, 1) == 0
    single = ctypes.c_void_p()
    assert lib.onebit01_init(ctypes.byref(single), *args, 3, 1) == 0
    assert lib.onebit01_dp_phase(single, 0, None, None, lr, None) == -1
    na, nb = ctypes.c_uint64(), ctypes.c_uint64()
    assert lib.onebit_adam_workspace_bytes(one, 0, ctypes.byref(na)) == 0
    assert lib.onebit_adam_workspace_bytes(h, 0, ctypes.byref(nb)) == 0
    assert nb.value - na.value >= 2 * 2 * 1024 * 4      # m_w and u_w of this rank's 2 workers
    for x in (h, one, single):
        lib.onebit_adam_destroy(x)


def test_zero_one_checkpoint_entry_points_validate_on_the_host(lib):
    h = ctypes.c_void_p()
    assert lib.onebit01_init(ctypes.byref(h), 1000, 4, 256, 0.9, 0.999, 1e-8, 3, 1) == 0
    ints, floats = (ctypes.c_int64 * 2)(), (ctypes.c_float * 2)()
    assert lib.onebit01_get_schedule(h, ints, floats) == 0
    assert list(ints) == [0, 0] and list(floats) == [0.0, 0.0]
    assert lib.onebit01_get_schedule(h, None, floats) == -1
    src = ctypes.c_void_p(0x1000)
    assert lib.onebit01_set_worker_state(h, 2, src, None) == -1           # which
    assert lib.onebit01_set_worker_state(h, 0, src, None) == -3           # before the freeze
    assert lib.onebit01_set_schedule(h, ints, floats) == -3
    assert lib.onebit01_set_schedule(h, None, floats) == -1
    lib.onebit_adam_destroy(h)
    one = ctypes.c_void_p()
    assert lib.onebit_adam_init(ctypes.byref(one), 1000, 4, 256, 0.9, 0.999, 1e-8) == 0
    assert lib.onebit01_get_schedule(one, ints, floats) == -1             # not a 0/1 handle
    assert lib.onebit01_set_worker_state(one, 0, src, None) == -1
    lib.onebit_adam_destroy(one)


def test_zero_one_workspace_holds_per_worker_state(lib):
    a, b = ctypes.c_void_p(), ctypes.c_void_p()
    d, W = 100_000, 4
    assert lib.onebit_adam_init(ctypes.byref(a), d, W, 4096, 0.9, 0.999, 1e-8) == 0
    assert lib.onebit01_init(ctypes.byref(b), d, W, 4096, 0.9, 0.999, 1e-8, 4, 0) == 0
    na, nb = ctypes.c_uint64(), ctypes.c_uint64()
    assert lib.onebit_adam_workspace_bytes(a, 0, ctypes.byref(na)) == 0
    assert lib.onebit_adam_workspace_bytes(b, 0, ctypes.byref(nb)) == 0
    ld = (d + 63) // 64 * 64
    assert nb.value - na.value >= 2 * W * ld * 4        # m_w and u_w, fp32[W][d] each
    lib.onebit_adam_destroy(a)
    lib.onebit_adam_destroy(b)


def test_bias_correction_switch_validates_on_the_host(lib):
    h = ctypes.c_void_p()
    assert lib.onebit_adam_init(ctypes.byref(h), 1000, 4, 256, 0.9, 0.999, 1e-8) == 0
    assert lib.onebit_adam_set_bias_correction(h, 2) == -1
    assert lib.onebit_adam_set_bias_correction(h, 1) == 0
    assert lib.onebit_adam_set_bias_correction(h, 0) == 0
    lib.onebit_adam_destroy(h)
    r = ctypes.c_void_p()
    assert lib.onebit_dp_init(ctypes.byref(r), 1000, 4, 256, 0.9, 0.999, 1e-8, 2, 0) == 0
    assert lib.onebit_adam_set_bias_correction(r, 1) == -1      # single-GPU handles only
    lib.onebit_adam_destroy(r)


def test_server_layout_fits_shared_memory_for_every_shape(lib):
    """For every W (1-256) and a spread of chunk lengths and sizes, the server kernel's dynamic
    shared memory fits a B200 block (227 KB opt-in), bank-private tables are chosen only for 2,
    4 or 8 groups of workers with at least 8 segments per chunk (2 groups: at least 2048 x 8
    segments in all), and 16 segments per block only with them. The same numbers the library
    uses at init; no GPU needed."""
    from communication_compressed_optimizer_momentum_b200 import onebit_server_layout
    max_smem = 232448
    seg = 4096
    for W in range(1, 257):
        groups = (W + 7) // 8
        for C in (32, 2048, 4096, 28672, 32768, 65536, 1 << 20, 20847744):
            for d in (C, 17 * C + 96, 333563904):
                lay = onebit_server_layout(d, W, C)
                assert 0 < lay["smem_bytes"] <= max_smem, (W, C, d, lay)
                assert 0 < lay["smem_bytes_dp"] <= max_smem, (W, C, d, lay)
                nseg = -(-min(C, d) // seg)
                nch = -(-d // C)
                if lay["bank_private"]:
                    assert groups in (2, 4, 8) and nseg >= 8, (W, C, d)
                    if groups == 2:
                        assert nch * -(-nseg // 8) >= 2048, (W, C, d)
                else:
                    assert lay["segs_per_block"] == 8
                assert lay["segs_per_block"] in (8, 16)
                assert lay["blocks"] == nch * -(-nseg // lay["segs_per_block"])
    with pytest.raises(ob.OneBitError):
        onebit_server_layout(1000, 0, 256)
    with pytest.raises(ob.OneBitError):
        onebit_server_layout(1000, 4, 100)
