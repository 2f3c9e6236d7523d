"""Failure detection without a GPU fault: a kernel wait that can never complete
gives up after its time limit, the host reads ATTN_ERR_TIMEOUT from
attn_status(), the status clears, and the context keeps working."""
import ctypes
import time

import numpy as np
import pytest
import torch

from tests import gpu_util

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_context_survives():
    m = gpu_util.ea()
    f = m.lib.attn_selftest_wait_timeout
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_uint, ctypes.c_void_p]
    stream = torch.cuda.current_stream().cuda_stream
    assert m.attn_status() == m.ATTN_OK
    assert f(0, stream) == m.ATTN_ERR_INVALID_ARG          # limits are range-checked
    t0 = time.perf_counter()
    assert f(20_000, stream) == m.ATTN_OK                   # 20 ms limit
    assert m.attn_status() == m.ATTN_ERR_TIMEOUT
    dt = time.perf_counter() - t0
    assert 0.015 < dt < 2.0, dt
    assert m.attn_status() == m.ATTN_OK                     # read-and-clear
    # the context is still usable: an ordinary call passes parity
    gpu_util.fwd_full_parity(1, 1, 200, 200, 128, True, seed=9)
