"""bench.py on a host without a GPU: the reference arm (the fp64 oracle) prints
its JSON line with the contract's keys, and our arm fails loudly instead of
falling back to anything that runs on the CPU."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(*args, timeout=300):
    return subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, capture_output=True, text=True,
                          timeout=timeout)


def test_reference_arm_prints_its_line():
    out = _bench("--impl", "reference", "--steps", "2", "--warmup", "1", "--ref-seconds", "3")
    assert out.returncode == 0, out.stderr[-2000:]
    d = json.loads(out.stdout.strip().splitlines()[-1])
    assert d["impl"] == "reference"
    assert d["unit"] == "elems/s" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["steps"] == 2 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["config"]["workload"] == "order3_bf16_b1_d768_l65536"   # the headline: longest single-GPU case
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "elems/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


@pytest.mark.skipif(os.path.exists("/dev/nvidia0"), reason="checks the behaviour on a host without a GPU")
def test_our_arm_fails_without_a_gpu():
    out = _bench("--steps", "1", "--warmup", "1", "--no-cpu-baseline", timeout=120)
    assert out.returncode != 0
    assert not out.stdout.strip()


def test_reference_arm_under_torchrun_prints_once():
    """Launched as the multi-GPU run is (torchrun, two ranks), the reference arm runs on rank 0 only:
    exactly one JSON line, and every rank exits 0."""
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "1", "--ref-seconds", "2"]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0


def test_cost_model_of_the_default_workload():
    """The roofline convention, worked by hand for order 3, bf16, B 1, D 768, L 65536
    (M = 131072): v, three gates and y at 2 bytes per element, every spectrum row
    (M/2 + 1 complex64 bins) and Dskip once; two 5 M log2 M transforms per row and order."""
    sys.path.insert(0, ROOT)
    import bench
    from long_convolution_sequence_hyena_b200.workloads import WORKLOADS
    c = bench.cost_model(WORKLOADS["order3_bf16_b1_d768_l65536"])
    assert c["M"] == 131072
    act = 5 * 768 * 65536 * 2
    spec = 3 * 768 * 65537 * 8
    assert c["bytes"] == act + spec + 3 * 768 * 4 == 1711303680
    assert c["flops"] == 2 * 3 * 768 * 5.0 * 131072 * 17
    g = bench.cost_model(WORKLOADS["gated_order1_bf16_2d_b2_c256_256x256"])
    # q, k, one gate and y over B C H W, the kernel spectra [C, W + 1, 2H], Dskip
    assert g["bytes"] == 4 * 2 * 256 * 256 * 256 * 2 + 256 * 257 * 512 * 8 + 256 * 4


def test_traffic_record_is_tied_to_the_sources(monkeypatch):
    """A committed DRAM-traffic record is reported only for the source version it was
    taken at."""
    sys.path.insert(0, ROOT)
    import bench
    from long_convolution_sequence_hyena_b200 import build
    from long_convolution_sequence_hyena_b200.workloads import WORKLOADS
    w = WORKLOADS["order3_bf16_b1_d768_l65536"]
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic_%s.json" % w.name)))
    monkeypatch.setattr(build, "source_hash", lambda: rec["source_hash"])
    assert bench.traffic_record(w) == rec["dram_bytes_per_launch"]
    monkeypatch.setattr(build, "source_hash", lambda: "0" * 16)
    assert bench.traffic_record(w) is None
