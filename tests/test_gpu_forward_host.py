"""hyena_forward_host: the forward on page-locked host activations, pipelined
over the batch (copies in, forward, copy out). Each stage runs hyena_forward
on its batch elements, and every row (plane) is computed independently of the
others, so the result must equal hyena_forward's on device copies of the same
inputs bit for bit; sampled rows are also checked against the fp64 oracle."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _inputs(plan, shape, B, D, N, dtype, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    v = torch.randn(B, D, *shape, device="cuda", generator=g).to(dtype)
    gates = [torch.randn(B, D, *shape, device="cuda", generator=g).to(dtype) for _ in range(N)]
    dskip = torch.randn(N, D, device="cuda", generator=g)
    if len(shape) == 1:
        t = torch.arange(shape[0], device="cuda", dtype=torch.float32)
        h = torch.randn(N, D, shape[0], device="cuda", generator=g) * torch.exp(-1e-3 * t)
    else:
        h = torch.randn(N, D, 2 * shape[0], 2 * shape[1], device="cuda", generator=g) * 0.01
    return v, gates, h, dskip


@pytest.mark.parametrize("shape,B,D,N,dtype,stages", [
    ((8192,), 6, 256, 2, torch.bfloat16, 3),    # two-row kernel, three stages of 2
    ((16384,), 5, 64, 2, torch.float32, 3),     # single-CTA kernel, stages of 2, 2 and 1
    ((32768,), 3, 2, 2, torch.bfloat16, 1),     # staged long rows, one stage
    ((32, 32), 3, 4, 2, torch.float32, 1),      # 2D
    ((256, 256), 3, 16, 1, torch.bfloat16, 2),  # staged 2D, stages of 2 and 1
    ((256, 256), 2, 64, 1, torch.bfloat16, 2),  # staged 2D, one batch element per stage
])
def test_forward_host_matches_device_forward(shape, B, D, N, dtype, stages):
    from long_convolution_sequence_hyena_b200 import api

    plan = api.Plan(shape, D, N, dtype)
    v, gates, h, dskip = _inputs(plan, shape, B, D, N, dtype, seed=B * 1000 + D)
    H = plan.filter_spectrum(h=h)
    y_dev = plan.forward(v, gates, H, dskip)
    io = 4 if dtype == torch.float32 else 2
    per_b_in = (N + 1) * D * int(np.prod(shape)) * io
    bc = -(-(8 << 20) // per_b_in)
    bc = min(bc + (bc & 1) if len(shape) == 1 else bc, B)
    assert -(-B // bc) == stages
    vh = v.cpu().pin_memory()
    gh = [x.cpu().pin_memory() for x in gates]
    for call in range(2):
        yh = torch.full_like(vh, float("nan")).pin_memory()
        out = plan.forward_host(vh, gh, H, dskip, out=yh)
        torch.cuda.synchronize()
        assert out.data_ptr() == yh.data_ptr()
        assert torch.equal(yh, y_dev.cpu()), call
    plan.close()


@pytest.mark.parametrize("L,B,D,N,dtype,chunk", [
    (65536, 1, 72, 3, torch.bfloat16, 32),   # channel stages of 32, 32 and 8 rows
    (65536, 2, 40, 2, torch.float32, 32),    # two batch elements of stages of 32 and 8
    (100000, 1, 48, 1, torch.bfloat16, 16),  # M = 262144: chunks of 16 rows, stages of 32 and 16
])
def test_forward_host_channel_stages(L, B, D, N, dtype, chunk):
    """Long 1D rows: a batch element over 16 MiB of input is cut into channel
    ranges of whole staged chunks, each an independent forward; the result
    still equals hyena_forward's bit for bit."""
    from long_convolution_sequence_hyena_b200 import api

    plan = api.Plan((L,), D, N, dtype)
    io = 4 if dtype == torch.float32 else 2
    per_ch = (N + 1) * L * io
    assert per_ch * D > 16 << 20
    dc = max(chunk, (16 << 20) // per_ch // chunk * chunk)
    assert dc < D
    v, gates, h, dskip = _inputs(plan, (L,), B, D, N, dtype, seed=L + D)
    H = plan.filter_spectrum(h=h)
    y_dev = plan.forward(v, gates, H, dskip)
    vh = v.cpu().pin_memory()
    gh = [x.cpu().pin_memory() for x in gates]
    yh = torch.full_like(vh, float("nan")).pin_memory()
    plan.forward_host(vh, gh, H, dskip, out=yh)
    torch.cuda.synchronize()
    assert torch.equal(yh, y_dev.cpu())
    # no Dskip: the channel ranges index the spectrum only
    y0 = plan.forward(v, gates, H, None)
    yh0 = torch.full_like(vh, float("nan")).pin_memory()
    plan.forward_host(vh, gh, H, None, out=yh0)
    torch.cuda.synchronize()
    assert torch.equal(yh0, y0.cpu())
    plan.close()


def test_forward_host_sampled_rows_match_oracle():
    import oracle
    from long_convolution_sequence_hyena_b200 import api

    shape, B, D, N = (8192,), 4, 64, 2
    plan = api.Plan(shape, D, N, torch.bfloat16)
    v, gates, h, dskip = _inputs(plan, shape, B, D, N, torch.bfloat16, seed=17)
    H = plan.filter_spectrum(h=h)
    vh = v.cpu().pin_memory()
    gh = [x.cpu().pin_memory() for x in gates]
    y = plan.forward_host(vh, gh, H, dskip)
    torch.cuda.synchronize()
    L = shape[0]
    rows = np.array([0, 1, 63, 64, 130, 255])
    ref = oracle.hyena_1d(vh.double().reshape(B * D, L).numpy()[rows],
                          torch.stack([x.double() for x in gh]).reshape(N, B * D, L).numpy()[:, rows],
                          h.double().cpu().numpy(), dskip.double().cpu().numpy(), fidx=rows % D)
    got = y.double().reshape(B * D, L).numpy()[rows]
    err = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert err <= 2e-2, err
    plan.close()


def test_forward_host_rejects():
    from long_convolution_sequence_hyena_b200 import api, capi

    shape, B, D, N = (2048,), 2, 4, 1
    plan = api.Plan(shape, D, N, torch.float32)
    v, gates, h, dskip = _inputs(plan, shape, B, D, N, torch.float32, seed=3)
    H = plan.filter_spectrum(h=h)
    vh = v.cpu().pin_memory()
    gh = [x.cpu().pin_memory() for x in gates]
    yh = torch.empty_like(vh).pin_memory()
    need = plan.host_workspace_bytes(B)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream

    def call(v_ptr, g_ptrs, y_ptr, ws_bytes=need, batch=B):
        return capi.hyena_forward_host(plan.handle, batch, v_ptr, g_ptrs, H.data_ptr(), dskip.data_ptr(), y_ptr,
                                       ws.data_ptr(), ws_bytes, s)

    gp = [x.data_ptr() for x in gh]
    assert call(vh.data_ptr(), gp, yh.data_ptr()) == capi.HYENA_OK
    pageable = v.cpu()
    assert not pageable.is_pinned()
    assert call(pageable.data_ptr(), gp, yh.data_ptr()) == capi.HYENA_ERR_INVALID_ARG
    assert call(vh.data_ptr(), gp, pageable.data_ptr()) == capi.HYENA_ERR_INVALID_ARG
    assert call(vh.data_ptr(), gp, vh.data_ptr()) == capi.HYENA_ERR_INVALID_ARG     # y overlaps v
    assert call(vh.data_ptr(), gp, gp[0]) == capi.HYENA_ERR_INVALID_ARG             # y overlaps a gate
    assert call(vh.data_ptr(), gp, yh.data_ptr(), ws_bytes=need - 1) == capi.HYENA_ERR_WORKSPACE
    assert call(0, None, 0, batch=0) == capi.HYENA_OK
    torch.cuda.synchronize()
    plan.close()
