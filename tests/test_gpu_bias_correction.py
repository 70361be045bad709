"""The optional bias-corrected warm-up on the GPU against the oracle (reading B1): every
warm-up step's x, m and v bit for bit (elementwise, same operation order and the same
corrections 1 - beta^t on both sides), the freeze's corrected moments bit for bit, and the first
compressed step after it within the parity tolerances."""
import numpy as np
import pytest
import torch

import communication_compressed_optimizer_momentum_b200 as ob
import oracle
from gpu_helpers import DEV, check_compressed_step, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_bias_corrected_warmup_matches_the_oracle(dt):
    d, W, C, T = 50_000, 4, 8192, 6
    b1, b2, eps, lr = 0.9, 0.999, 1e-8, 1e-3
    gen = torch.Generator(device=DEV)
    gen.manual_seed(11)
    x = (torch.rand(d, device=DEV, generator=gen) - 0.5) * 0.1
    opt = ob.OneBitAdam(d, W, C, b1, b2, eps, grad_dtype=dt, device=DEV, bias_correction=True)
    st = oracle.OracleState(to_np(x), W, C, b1, b2, eps, bias_correction=True)
    for _ in range(T):
        g = (torch.randn(W, d, device=DEV, generator=gen) * 1e-2).to(dt)
        opt.warmup_step(x, g, lr)
        st.warmup_step(to_np(g), lr)
        torch.cuda.synchronize()
        assert np.array_equal(to_np(x).view(np.uint32), st.x.view(np.uint32))
        assert np.array_equal(to_np(opt.get_state("m")).view(np.uint32), st.m.view(np.uint32))
        assert np.array_equal(to_np(opt.get_state("v")).view(np.uint32), st.v.view(np.uint32))
    pre = {"x": to_np(x)}
    opt.freeze()
    st.freeze()
    torch.cuda.synchronize()
    assert np.array_equal(to_np(opt.get_state("m")).view(np.uint32), st.m.view(np.uint32))
    assert np.array_equal(to_np(opt.get_state("v")).view(np.uint32), st.v.view(np.uint32))
    pre.update(m=st.m.copy(), v=st.v.copy(), e_w=np.zeros((W, d), np.float32),
               e_s=np.zeros(d, np.float32))
    g = (torch.randn(W, d, device=DEV, generator=gen) * 1e-2).to(dt)
    opt.step(x, g, lr)
    post = {"x": to_np(x)}
    for nm in ("m", "e_w", "e_s", "s", "S", "bits_w", "bits_s"):
        post[nm] = to_np(opt.get_state(nm))
    check_compressed_step(pre, to_np(g), post, C, b1, eps, lr)
    assert opt.status() == 0
    opt.close()


def test_bias_correction_cannot_change_mid_warmup():
    opt = ob.OneBitAdam(4096, 2, 1024, device=DEV)
    x = torch.zeros(4096, device=DEV)
    opt.warmup_step(x, torch.ones(2, 4096, device=DEV), 1e-3)
    with pytest.raises(ob.OneBitError) as e:
        ob.onebit_adam_set_bias_correction(opt.h, True)
    assert e.value.code == -3
    opt.close()
