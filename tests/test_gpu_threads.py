"""Calls on one plan from several host threads, each on a stream of its own.

A staged plan owns two streams (and, for the spectra, a scratch buffer);
every call forks those streams off its own stream with events of its own, and
the plan orders the spectrum scratch on them, so concurrent calls must give
exactly the results of the same calls made one after another. ctypes releases
the GIL during each C call, so the two threads' launch sequences interleave."""
import threading

import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("own_ws", [False, True])
@pytest.mark.parametrize("shape,B,D,N", [((32768,), 2, 80, 2), ((256, 256), 1, 70, 1)])
def test_concurrent_calls_on_one_plan(shape, B, D, N, own_ws):
    """own_ws: each thread's spectrum calls bring their own scratch
    (hyena_filter_spectrum_ws), so they need not wait for each other."""
    from long_convolution_sequence_hyena_b200 import api

    plan = api.Plan(shape, D, N, torch.bfloat16)
    sets = []
    for seed in (11, 12):
        g = torch.Generator(device="cuda")
        g.manual_seed(seed)
        v = torch.randn(B, D, *shape, device="cuda", generator=g).bfloat16()
        gates = [torch.randn(B, D, *shape, device="cuda", generator=g).bfloat16() for _ in range(N)]
        dskip = torch.randn(N, D, device="cuda", generator=g)
        if len(shape) == 1:
            t = torch.arange(shape[0], device="cuda", dtype=torch.float32)
            h = torch.randn(N, D, shape[0], device="cuda", generator=g) * torch.exp(-1e-3 * t)
        else:
            h = torch.randn(N, D, 2 * shape[0], 2 * shape[1], device="cuda", generator=g) * 0.01
        H_ref = plan.filter_spectrum(h=h)
        y_ref = plan.forward(v, gates, H_ref, dskip)
        torch.cuda.synchronize()
        sets.append(dict(v=v, gates=gates, dskip=dskip, h=h, H_ref=H_ref, y_ref=y_ref,
                         H=torch.empty_like(H_ref), y=torch.empty_like(y_ref),
                         ws=torch.empty(max(1, plan.workspace_bytes(B)), dtype=torch.uint8, device="cuda"),
                         sws=(torch.empty(max(1, plan.spectrum_workspace_bytes()), dtype=torch.uint8, device="cuda")
                              if own_ws else None),
                         stream=torch.cuda.Stream()))
    torch.cuda.synchronize()
    errors = []

    def worker(s):
        try:
            torch.cuda.set_device(0)
            for it in range(12):
                plan.filter_spectrum(h=s["h"], out=s["H"], stream=s["stream"], workspace=s["sws"])
                plan.forward(s["v"], s["gates"], s["H"], s["dskip"], out=s["y"], workspace=s["ws"],
                             stream=s["stream"])
                s["stream"].synchronize()
                if not (torch.equal(s["H"], s["H_ref"]) and torch.equal(s["y"], s["y_ref"])):
                    errors.append(it)
                    return
        except Exception as e:  # reported below
            errors.append(repr(e))

    threads = [threading.Thread(target=worker, args=(s,)) for s in sets]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not any(t.is_alive() for t in threads)
    assert not errors, errors
    plan.close()


def test_spectrum_workspace_checks():
    from long_convolution_sequence_hyena_b200 import api, capi
    plan = api.Plan((65536,), 4, 1, torch.float32)
    need = plan.spectrum_workspace_bytes()
    assert need > 0
    h = torch.randn(1, 4, 65536, device="cuda")
    H = torch.empty(plan.spectrum_shape, dtype=torch.complex64, device="cuda")
    small = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    assert capi.hyena_filter_spectrum_ws(plan.handle, h.data_ptr(), None, H.data_ptr(), small.data_ptr(),
                                         small.numel(), 0) == capi.HYENA_ERR_WORKSPACE
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    H1 = plan.filter_spectrum(h=h, workspace=ws)
    H2 = plan.filter_spectrum(h=h)
    torch.cuda.synchronize()
    assert torch.equal(H1, H2)
    plan2 = api.Plan((2048,), 4, 1, torch.float32)   # spectra without scratch
    assert plan2.spectrum_workspace_bytes() == 0
    plan.close()
    plan2.close()
