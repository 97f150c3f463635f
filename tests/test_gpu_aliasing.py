"""y may alias v or a gate on every path (each row or plane is read completely
before it is written): the staged paths, where a row is split over many CTAs
and chunks run on two streams, the cluster path and the 2D paths included.
An aliased call must give exactly the output of the same call into a fresh
buffer (same kernels, same arithmetic)."""
import pytest
import torch

from hyena_cases import explicit_case, explicit_case_2d, to_gpu
from long_convolution_sequence_hyena_b200.workloads import make_inputs

pytestmark = pytest.mark.gpu

CASES = [
    # (workload, expected path)
    (explicit_case(2, 3, 1000, 2, "bf16", seed=31), 0),                   # two rows in lockstep
    (explicit_case(3, 2, 9000, 3, "f32", seed=32), 0),                    # single-CTA rows (odd batch)
    (explicit_case(1, 130, 32768, 2, "bf16", seed=33, alpha=(1e-4, 1e-2)), 3),   # staged, three chunks of 64 rows
    (explicit_case(1, 3, 40001, 2, "f32", seed=34, alpha=(1e-4, 1e-2)), 3),      # staged, odd length
    (explicit_case(1, 2, 100000, 2, "f32", seed=35, alpha=(1e-4, 1e-2)), 1),     # cluster (forced)
    (explicit_case_2d(1, 3, 64, 2, "f32", seed=36), 2),                   # 2D cluster
    (explicit_case_2d(2, 35, 256, 1, "bf16", seed=37), 2),                # 2D staged, two chunks of 64 planes
]


@pytest.mark.parametrize("case", range(len(CASES)))
@pytest.mark.parametrize("alias", ["v", "first_gate", "last_gate"])
def test_output_aliases_an_input(case, alias, monkeypatch):
    from long_convolution_sequence_hyena_b200 import api
    w, path = CASES[case]
    if path == 1:   # the thread-block-cluster kernel runs only when forced (the staged path is faster)
        monkeypatch.setenv("HYENA_FORCE_PATH", "cluster")
    inp = make_inputs(w)
    g = to_gpu(inp)
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    plan = api.Plan(w.shape, w.D, w.order, dt)
    assert plan.path == path
    H = plan.filter_spectrum(h=g["h"])
    ref = plan.forward(g["v"], g["gates"], H, g["dskip"])
    v = g["v"].clone()
    gates = [x.clone() for x in g["gates"]]
    out = {"v": v, "first_gate": gates[0], "last_gate": gates[-1]}[alias]
    plan.forward(v, gates, H, g["dskip"], out=out)
    torch.cuda.synchronize()
    assert torch.equal(out, ref), (w.name, alias)
    plan.close()
