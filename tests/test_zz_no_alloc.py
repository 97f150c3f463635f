"""hyena_forward_no_alloc: the forward for callers that cannot allocate device
memory where they run the operator (a plain C host program without an
allocator of its own, a process whose device memory belongs to a framework's
allocator, a loop that must not call cudaMalloc). Its scratch is a fixed
device array inside the library, so it takes no workspace. It runs the same
kernels as hyena_forward over smaller chunks, so its output must equal
hyena_forward's, call after call, because every call reuses the same array;
sampled rows are also checked against the fp64 oracle directly.

This file is collected last, so that a failure here stops a run only after
every other test has run."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _rel_l2(a, b):
    a, b = a.double(), b.double()
    return float(torch.linalg.vector_norm(a - b) / torch.linalg.vector_norm(b))


@pytest.mark.parametrize("L,B,D,N,dtype,tol", [
    (32768, 1, 70, 2, torch.float32, 1e-5),    # 70 rows: two chunks of the 64 rows the array holds
    (65536, 2, 20, 3, torch.bfloat16, 2e-2),   # 40 rows: two chunks of 32
    (16385, 3, 1, 2, torch.float32, 1e-5),     # odd length, odd row count (the last pair has one row)
    (40001, 1, 35, 1, torch.bfloat16, 2e-2),   # odd length at M = 131072, two chunks, odd rows
])
def test_no_alloc_matches_forward_twice(L, B, D, N, dtype, tol):
    import oracle
    from long_convolution_sequence_hyena_b200 import api, capi

    plan = api.Plan((L,), D, N, dtype)
    assert plan.path == capi.HYENA_PATH_STAGED
    g = torch.Generator(device="cuda")
    g.manual_seed(L + D)
    v = torch.randn(B, D, L, device="cuda", generator=g).to(dtype)
    gates = [torch.randn(B, D, L, device="cuda", generator=g).to(dtype) for _ in range(N)]
    t = torch.arange(L, device="cuda", dtype=torch.float32)
    h = torch.randn(N, D, L, device="cuda", generator=g) * torch.exp(-1e-3 * t)
    dskip = torch.randn(N, D, device="cuda", generator=g)
    H = plan.filter_spectrum(h=h)
    y_ref = plan.forward(v, gates, H, dskip)    # the entry point with a caller-provided workspace
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):                       # the array keeps the last call's contents
        y = torch.full_like(v, float("nan"))
        st = capi.hyena_forward_no_alloc(plan.handle, B, v.data_ptr(), [x.data_ptr() for x in gates],
                                         H.data_ptr(), dskip.data_ptr(), y.data_ptr(), stream)
        assert st == capi.HYENA_OK, capi.hyena_status_string(st)
        torch.cuda.synchronize()
        assert torch.isfinite(y.float()).all()
        err = _rel_l2(y, y_ref)
        assert err <= tol, (call, err)
        assert torch.equal(y, y_ref), call      # same kernels, same per-row arithmetic
    # a few rows against the fp64 oracle (first, last, and one in the second chunk)
    R = B * D
    rows = sorted({0, R - 1, min(R - 1, 33)})
    v64 = v.double().cpu().reshape(R, L).numpy()[rows]
    g64 = np.stack([x.double().cpu().reshape(R, L).numpy()[rows] for x in gates])
    ref = oracle.hyena_1d(v64, g64, h.double().cpu().numpy(), dskip.double().cpu().numpy(),
                          fidx=np.array(rows) % D)
    got = y.double().cpu().reshape(R, L).numpy()[rows]
    err = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert err <= tol, err
    plan.close()


def test_no_alloc_rejects_other_paths():
    from long_convolution_sequence_hyena_b200 import api, capi

    plan = api.Plan((4096,), 2, 1, torch.float32)     # single-CTA path: needs no workspace at all
    v = torch.zeros(1, 2, 4096, device="cuda")
    H = torch.zeros(plan.spectrum_shape, dtype=torch.complex64, device="cuda")
    st = capi.hyena_forward_no_alloc(plan.handle, 1, v.data_ptr(), [v.data_ptr()], H.data_ptr(), None,
                                     v.data_ptr(), 0)
    assert st == capi.HYENA_ERR_UNSUPPORTED
    assert capi.hyena_forward_no_alloc(None, 1, 0, None, 0, None, 0, 0) == capi.HYENA_ERR_INVALID_ARG
    plan.close()
