"""The library's launch counter (hyena_launch_count) against the launch
sequence each path is built from: one fused launch per forward on the
single-launch 1D paths, and 2N + 1 launches (a column kernel, then a row and a
column kernel per order) per chunk of rows on the staged long-row path."""
import pytest
import torch

from long_convolution_sequence_hyena_b200 import api, capi

pytestmark = pytest.mark.gpu


def _forward_launches(L, B, D, N):
    plan = api.Plan((L,), D, N, torch.bfloat16)
    g = torch.Generator(device="cuda").manual_seed(L + B + D + N)
    v = torch.randn(B, D, L, device="cuda", generator=g).to(torch.bfloat16)
    gates = [torch.randn(B, D, L, device="cuda", generator=g).to(torch.bfloat16) for _ in range(N)]
    h = torch.randn(N, D, L, device="cuda", generator=g) * 0.01
    H = plan.filter_spectrum(h=h)
    dsk = torch.randn(N, D, device="cuda", generator=g)
    ws = torch.empty(max(1, plan.workspace_bytes(B)), dtype=torch.uint8, device="cuda")
    y = torch.empty_like(v)
    torch.cuda.synchronize()
    n0 = capi.hyena_launch_count()
    plan.forward(v, gates, H, dsk, out=y, workspace=ws)
    n1 = capi.hyena_launch_count()
    torch.cuda.synchronize()
    assert torch.isfinite(y.float()).all()
    return plan, n1 - n0


@pytest.mark.parametrize("L,B,D,N", [(2048, 8, 16, 2), (2048, 3, 5, 3), (16384, 2, 4, 1)])
def test_single_launch_paths(L, B, D, N):
    plan, n = _forward_launches(L, B, D, N)
    assert plan.path == capi.HYENA_PATH_CTA
    assert n == 1


@pytest.mark.parametrize("B,D,N", [(1, 8, 3), (1, 70, 3), (2, 33, 2)])
def test_staged_path_counts_every_chunk(B, D, N):
    # L = 65536 pads to M = 131072: 512 KB transforms, chunks of 32 rows (16 MB)
    plan, n = _forward_launches(65536, B, D, N)
    assert plan.path == capi.HYENA_PATH_STAGED
    chunks = -(-(B * D) // 32)
    assert n == chunks * (2 * N + 1)
