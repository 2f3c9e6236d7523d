"""bench.py's host-side logic on CPU: work models, the traffic table, the reference arm."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from seeded_inputs import Workload  # noqa: E402


@pytest.mark.parametrize("Nq,Nkv,causal", [(7, 7, True), (5, 9, True), (9, 4, True), (6, 3, False)])
def test_prefill_pairs_counts_visible_pairs(Nq, Nkv, causal):
    w = Workload("t", 2, 3, Nq, Nkv, 64, causal, 0)
    i = np.arange(Nq)[:, None]
    j = np.arange(Nkv)[None, :]
    vis = (j <= i + (Nkv - Nq)) if causal else np.ones((Nq, Nkv), bool)
    assert bench.prefill_pairs(w) == int(vis.sum())
    assert bench.prefill_flops(w) == 4.0 * 64 * 2 * 3 * int(vis.sum())
    assert bench.bwd_flops(w) == 2.5 * bench.prefill_flops(w)


def test_decode_bytes_model():
    w = Workload("d", 2, 4, 1, 1000, 128, False, 0, num_splits=8)
    kv = 2 * 2 * 4 * 1000 * 128 * 2
    assert bench.decode_kv_bytes(w) == kv
    assert bench.decode_partial_bytes(w) == kv + 2 * 4 * (128 * 2 + 8 * 129 * 4)


def test_recorded_traffic_needs_matching_source_hash(monkeypatch):
    good = bench.recorded_traffic()
    for (name, workload), nbytes in good.items():
        assert name in bench.KERNEL_SOURCES and workload and nbytes > 0
    monkeypatch.setattr(bench, "kernel_source_hash", lambda kernel: "0000000000000000")
    assert bench.recorded_traffic() == {}


def test_reference_arm_prints_the_contract_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0"], capture_output=True, text=True,
                         timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads([l for l in out.stdout.splitlines() if l.startswith("{")][-1])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == "TFLOP/s"
    assert line["value"] > 0 and line["higher_is_better"] is True
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_l2_flush_plan():
    """Inputs that fit in L2 are flushed before every timed step; larger ones are not."""
    import bench
    l2 = 126 << 20
    on, note = bench.l2_flush_plan(50_700_000, l2, False)       # gpt2_1k forward
    assert on and "fit in L2" in note and "flush" in note
    on, note = bench.l2_flush_plan(192 << 20, l2, False)        # prefill_8k forward
    assert not on and "larger than L2" in note
    on, note = bench.l2_flush_plan(1 << 10, l2, True)           # reduced batch for profiling
    assert not on and note == "reduced batch for profiling"


def test_reference_arm_never_loads_the_cuda_library():
    """The oracle arm shares no process image with the product: after a full
    reference run neither the package nor its shared library is loaded."""
    code = (
        "import runpy, sys\n"
        f"sys.argv = ['bench.py', '--impl', 'reference', '--steps', '1', '--warmup', '0']\n"
        "try:\n"
        f"    runpy.run_path({os.path.join(ROOT, 'bench.py')!r}, run_name='__main__')\n"
        "except SystemExit as e:\n"
        "    assert not e.code, e.code\n"
        "maps = open('/proc/self/maps').read()\n"
        "assert 'libexact_attn_b200' not in maps, 'CUDA library mapped'\n"
        "assert not any(m.startswith('exact_io_aware_70_b200') for m in sys.modules)\n"
        "assert 'liboracle' in maps\n"
        "print('CLEAN')\n")
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                         timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    assert "CLEAN" in out.stdout


def test_oracle_sample_counts_flops_of_the_workload_it_samples():
    """The per-workload CPU baseline counts causal and non-causal rows right."""
    from seeded_inputs import WORKLOADS
    tiny = bench.oracle_prefill_sample(0.05, max_heads=1, w=WORKLOADS["tiny"])
    w = WORKLOADS["tiny"]                        # non-causal: every row sees all keys
    assert tiny["flops"] == tiny["heads"] * tiny["rows"] * 4.0 * w.d * w.Nkv
    g = WORKLOADS["gpt2_1k"]
    s = bench.oracle_prefill_sample(0.05, max_rows=64, max_heads=1, w=g)
    rows = np.linspace(0, g.Nq - 1, s["rows"]).astype(np.int64)
    assert s["flops"] == s["heads"] * sum(4.0 * g.d * (int(r) + 1) for r in rows)
    cb = bench.prefill_cpu_baseline(g, 0.05)
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] > 0 and "gpt2_1k" in cb["sample"]
