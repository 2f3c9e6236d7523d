"""attn_decode_splitkv_noalloc: split-KV decode for callers that cannot allocate.

Some callers may not call cudaMalloc or hand over a device buffer (code inside
an allocator's callbacks, plugins whose host framework owns all device
memory). The no-allocation entry point keeps its partials in a fixed array
owned by the library instead of a caller workspace. These tests call it through
the C ABI and check that two calls in a row give bit for bit what the
workspace entry point (attn_decode_splitkv) gives on the same inputs -- both
run the same deterministic kernels on the same arguments, so any difference
would mean stale or misplaced partials in the shared array -- that the second
call also matches the fp64 oracle within the parity tolerance, and that sizes
beyond the fixed array are refused without launching.

This file is collected last on purpose, and must pass both alone in a fresh
process and after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from seeded_inputs import bf16_bits, make_qkv
from tests.parity import compare

pytestmark = pytest.mark.gpu


def _lib():
    import exact_io_aware_70_b200 as ea
    L = ea.lib
    f = L.attn_decode_splitkv_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 4 + [ctypes.c_float, ctypes.c_int,
                                                               ctypes.c_void_p]
    return ea, f


def _run_both(ea, noalloc, B, H, Nkv, d, S, seed, check_oracle=False):
    q_h, k_h, v_h = make_qkv(B, H, 1, Nkv, d, seed)
    q, k, v = q_h.cuda(), k_h.cuda(), v_h.cuda()
    scale = float(np.float32(1.0 / np.sqrt(d)))
    stream = torch.cuda.current_stream().cuda_stream
    o_ref = torch.empty((B, H, 1, d), dtype=torch.bfloat16, device="cuda")
    l_ref = torch.empty((B, H, 1), dtype=torch.float32, device="cuda")
    ws = torch.empty(ea.attn_decode_workspace_bytes(B, H, d, S), dtype=torch.uint8, device="cuda")
    ea.attn_decode_splitkv(q, k, v, o_ref, l_ref, scale, S, ws)
    o = torch.full((B, H, 1, d), 7.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, H, 1), 7.0, dtype=torch.float32, device="cuda")
    rc = noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, Nkv,
                 d, scale, S, stream)
    assert rc == 0, ea.attn_strerror(rc)
    assert ea.attn_status() == 0
    assert torch.equal(o, o_ref), "no-alloc O differs from the workspace entry point"
    assert torch.equal(lse, l_ref), "no-alloc LSE differs from the workspace entry point"
    if check_oracle:
        o_or, l_or = oracle.get().attn_fwd_bf16(bf16_bits(q_h), bf16_bits(k_h), bf16_bits(v_h),
                                                False, scale)
        compare(o.float().cpu().numpy(), lse.cpu().numpy(), o_or, l_or,
                f"no-alloc decode B{B} H{H} Nkv{Nkv} d{d} S{S}")


def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row():
    ea, noalloc = _lib()
    # the second call has other sizes and inputs, so stale contents left in the
    # shared array by the first call would show up as a mismatch
    _run_both(ea, noalloc, B=4, H=8, Nkv=5000, d=128, S=16, seed=21)
    _run_both(ea, noalloc, B=2, H=3, Nkv=777, d=64, S=7, seed=22, check_oracle=True)


def test_noalloc_refuses_sizes_beyond_its_array():
    ea, noalloc = _lib()
    # decode_32k's own partials (16.9 MB) fit; 4x the heads would need 67.6 MB
    assert ea.attn_decode_workspace_bytes(16, 128, 128, 64) > 32 << 20
    p = 0x10000   # never dereferenced: the call must return before launching
    rc = noalloc(p, p, p, p, p, 16, 128, 32768, 128, 0.088, 64, None)
    assert rc == 6, ea.attn_strerror(rc)        # ATTN_ERR_SCRATCH_LIMIT
    assert "32 MiB" in ea.attn_strerror(rc)
