"""The debug build of the library on the B200.

The library can be compiled with -DATTN_DEBUG; its kernels then check every
global-memory index they compute against the tensor it addresses, skip an
access that fails and report ATTN_ERR_INDEX_CHECK through attn_status() -- a
bounds check that stands in for the memory checker, without trapping the GPU.
This runs a set of the parity tests (ragged tails, causal alignments, several
persistent rounds, the split and paged decodes, the merge, the backward pass)
in a child process against the debug build: each of those tests requires
attn_status() == ATTN_OK after every call, so a failed index check fails it.
"""
import importlib.util
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_parity_suite_under_the_index_checking_build():
    spec = importlib.util.spec_from_file_location(
        "exact_attn_cuda_build", os.path.join(ROOT, "exact_io_aware_70_b200", "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    lib = build.build(debug=True)
    env = dict(os.environ, EXACT_ATTN_LIB=lib)
    tests = ["tests/test_gpu_fwd.py::test_fwd_sweep", "tests/test_gpu_fwd.py::test_tiny_workload",
             "tests/test_gpu_fwd.py::test_gpt2_1k_workload_full",
             "tests/test_gpu_decode.py::test_decode_splitkv_full",
             "tests/test_gpu_decode.py::test_lse_merge_matches_oracle",
             "tests/test_gpu_kvsplit.py", "tests/test_gpu_paged.py",
             "tests/test_gpu_fp8.py::test_fp8_matches_oracle",
             "tests/test_gpu_bwd.py::test_bwd_matches_oracle"]
    out = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                          "-m", "gpu", *tests], cwd=ROOT, env=env, capture_output=True,
                         text=True, timeout=1800)
    assert out.returncode == 0, out.stdout[-4000:] + out.stderr[-2000:]
    assert " passed" in out.stdout
