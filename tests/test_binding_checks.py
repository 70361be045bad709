"""The binding checks tensors before their pointers reach the library, which trusts the sizes
it is given: a CPU tensor, a wrong dtype, a non-contiguous view, a too-short output or an
invalid chunk length raises in Python, before any device work (no GPU needed)."""
import pytest
import torch

import communication_compressed_optimizer_momentum_b200 as ob


def test_pack_rejects_host_and_wrong_dtype():
    with pytest.raises(ValueError, match="CUDA tensor"):
        ob.onebit_pack(torch.zeros(10))
    with pytest.raises(TypeError):
        ob.onebit_pack([0.0] * 10)


def test_unpack_rejects_bad_sizes_before_the_library():
    with pytest.raises(ValueError):
        ob.onebit_unpack(torch.zeros(1, dtype=torch.int32), torch.zeros(1), 10, 0)
    with pytest.raises(ValueError):
        ob.onebit_unpack(torch.zeros(1, dtype=torch.int32), torch.zeros(1), -1, 32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        ob.onebit_unpack(torch.zeros(1, dtype=torch.int32), torch.zeros(1), 10, 32)


@pytest.mark.parametrize("C", [0, -32, 48, 1])
def test_compress_static_rejects_bad_chunk_length(C):
    with pytest.raises(ValueError, match="multiple of 32"):
        ob.onebit_compress_static(torch.zeros(64), C)


def test_compress_static_rejects_host_tensor():
    with pytest.raises(ValueError, match="CUDA tensor"):
        ob.onebit_compress_static(torch.zeros(64), 32)
