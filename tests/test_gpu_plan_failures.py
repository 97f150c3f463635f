"""Every failure path of plan creation: the test hook makes the n-th resource
the plan would create (device buffer, stream, host object) fail, and the
call must return HYENA_ERR_NOMEM (HYENA_ERR_CUDA for a stream) having
released everything it had created, leaving the library usable."""
import pytest
import torch

from long_convolution_sequence_hyena_b200 import capi

pytestmark = pytest.mark.gpu

# shape, channels, order, dtype, resources a plan holds: twiddles, error word,
# then (staged paths) three lane streams, the spectrum scratch and its lock;
# the plan object last
CASES = [
    ((2048,), 4, 2, capi.HYENA_BF16, 3),
    ((65536,), 4, 3, capi.HYENA_BF16, 8),
    ((32, 32), 3, 1, capi.HYENA_F32, 3),
    ((256, 256), 2, 1, capi.HYENA_BF16, 8),
    ((16, 16, 16), 2, 1, capi.HYENA_F32, 3),
]


def _create(shape, D, N, dt):
    return capi.hyena_plan_create(len(shape), list(shape), D, N, dt, 1 if len(shape) == 1 else 0)


@pytest.mark.parametrize("shape,D,N,dt,count", CASES)
def test_every_creation_failure_unwinds(shape, D, N, dt, count):
    torch.cuda.synchronize()
    base = capi.hyena_debug_plan_resources()
    st, h = _create(shape, D, N, dt)
    assert st == capi.HYENA_OK
    assert capi.hyena_debug_plan_resources() - base == count
    assert capi.hyena_plan_destroy(h) == capi.HYENA_OK
    assert capi.hyena_debug_plan_resources() == base
    stream_steps = {3, 4, 5} if count == 8 else set()
    try:
        for k in range(1, count + 1):
            assert capi.lib.hyena_debug_fail_allocation(k) == capi.HYENA_OK
            st, h = _create(shape, D, N, dt)
            assert h is None, k
            assert st == (capi.HYENA_ERR_CUDA if k in stream_steps else capi.HYENA_ERR_NOMEM), (k, st)
            assert capi.hyena_debug_plan_resources() == base, k
    finally:
        capi.lib.hyena_debug_fail_allocation(0)
    # armed past the last resource: creation succeeds
    assert capi.lib.hyena_debug_fail_allocation(count + 1) == capi.HYENA_OK
    st, h = _create(shape, D, N, dt)
    capi.lib.hyena_debug_fail_allocation(0)
    assert st == capi.HYENA_OK
    assert capi.hyena_plan_destroy(h) == capi.HYENA_OK
    assert capi.hyena_debug_plan_resources() == base


def test_library_usable_after_failures():
    from long_convolution_sequence_hyena_b200 import api
    try:
        capi.lib.hyena_debug_fail_allocation(1)
        st, h = _create((4096,), 8, 2, capi.HYENA_F32)
        assert st == capi.HYENA_ERR_NOMEM and h is None
    finally:
        capi.lib.hyena_debug_fail_allocation(0)
    plan = api.Plan((4096,), 8, 2, torch.float32)
    g = torch.Generator(device="cuda").manual_seed(5)
    v = torch.randn(2, 8, 4096, device="cuda", generator=g)
    gates = [torch.ones_like(v) for _ in range(2)]
    h = torch.zeros(2, 8, 4096, device="cuda")
    h[:, :, 0] = 1.0   # delta filters: y = v
    H = plan.filter_spectrum(h=h)
    y = plan.forward(v, gates, H, None)
    torch.cuda.synchronize()
    assert torch.allclose(y, v, atol=1e-5)
    plan.close()
