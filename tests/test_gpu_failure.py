"""Failure detection without a GPU fault: a pipeline stage that never fills
makes a tcgen05 kernel's bounded waits run out under a short limit; the call
returns, the device status reports LCSA_DEV_TIMEOUT, and the next call on
the same stream is correct (the kernel drained its copies and freed its
tensor memory)."""
import numpy as np
import pytest
import torch

from oracle import lcsa_oracle as O

pytestmark = pytest.mark.gpu

DEV = "cuda"
LCSA_DEV_TIMEOUT = 1


@pytest.fixture(scope="module")
def lcsa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from conftest import build_library
    return build_library()


def _case(seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    T, n_h, c, gr, d_g, d = 300, 64, 512, 8, 1024, 1024
    K = n_h // gr * c
    o = torch.randn(T, n_h, c, device=DEV, generator=g).to(torch.bfloat16)
    w1 = (torch.randn(gr, d_g, K, device=DEV, generator=g) / K ** 0.5).to(torch.bfloat16)
    w2 = (torch.randn(d, gr * d_g, device=DEV, generator=g) / (gr * d_g) ** 0.5).to(torch.bfloat16)
    return o, w1, w2


def _check(lcsa, y, o, w1, w2):
    ref = O.grouped_out_proj(o.double().cpu().numpy(), w1.double().cpu().numpy(), w2.double().cpu().numpy())
    got = y.double().cpu().numpy()
    scale = np.sqrt(np.mean(ref * ref))
    assert np.abs(got - ref).max() <= 2e-2 * scale + 8e-3 * np.abs(ref).max()


def test_withheld_stage_times_out_and_the_next_call_is_clean(lcsa):
    o, w1, w2 = _case(501)
    assert lcsa.get_device_status() == 0
    lcsa.set_wait_limit_ns(20_000_000)                # 20 ms instead of 2 s
    try:
        lcsa.lib.lcsa_test_withhold_stage(1)          # k-chunk 1 of CTA 0 never arrives
        lcsa.grouped_out_proj(o, w1, w2)              # returns: the launch itself is valid
        torch.cuda.synchronize()
        assert lcsa.get_device_status() == LCSA_DEV_TIMEOUT
        assert lcsa.get_device_status() == 0          # read and cleared
        # the hook was one-shot: the same call on the same stream is correct
        y = lcsa.grouped_out_proj(o, w1, w2)
        torch.cuda.synchronize()
        assert lcsa.get_device_status() == 0
        _check(lcsa, y, o, w1, w2)
    finally:
        lcsa.lib.lcsa_test_withhold_stage(-1)
        lcsa.set_wait_limit_ns(0)                     # back to the default


def test_short_limit_does_not_disturb_normal_calls(lcsa):
    """A 20 ms limit is far above any stage hand-off of a normal call."""
    o, w1, w2 = _case(502)
    lcsa.set_wait_limit_ns(20_000_000)
    try:
        y = lcsa.grouped_out_proj(o, w1, w2)
        torch.cuda.synchronize()
        assert lcsa.get_device_status() == 0
        _check(lcsa, y, o, w1, w2)
    finally:
        lcsa.set_wait_limit_ns(0)
