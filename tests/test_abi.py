"""The C-ABI library loads, exports every declared entry point, and rejects bad
arguments before touching the GPU (so these run on a CPU-only host)."""
import ctypes
import importlib.util
import os
import re
import shutil
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "exact_attn.h")


@pytest.fixture(scope="module")
def ea():
    # the build script is loaded by path: importing the package first would
    # refuse to load without the library this builds
    spec = importlib.util.spec_from_file_location(
        "exact_attn_cuda_build", os.path.join(ROOT, "exact_io_aware_70_b200", "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    build.build()
    import exact_io_aware_70_b200 as m
    return m


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("attn_fwd", "attn_decode_partials", "attn_lse_merge", "attn_decode_splitkv",
                 "attn_decode_workspace_bytes", "attn_status", "attn_strerror",
                 "attn_abi_version", "attn_bwd", "attn_bwd_workspace_bytes", "attn_fwd_fp8"):
        assert want in names


def test_library_exports_every_declared_symbol(ea):
    lib = ctypes.CDLL(ea.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in exact_attn.h but not exported"


def test_version_and_strerror(ea):
    assert ea.abi_version() == 1
    for code in range(9):
        assert ea.attn_strerror(code)
    assert "unknown" in ea.attn_strerror(99)


def test_fwd_rejects_bad_arguments_without_launching(ea):
    L = ea.lib
    p = 0x10000  # never dereferenced: every case below fails validation first
    ok = dict(q=p, k=p, v=p, o=p, lse=p, B=1, H=1, Nq=128, Nkv=128, d=64, causal=0, scale=0.125)

    def call(**kw):
        a = dict(ok, **kw)
        return L.attn_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["Nq"],
                          a["Nkv"], a["d"], a["causal"], a["scale"], None)

    assert call(q=None) == ea.ATTN_ERR_INVALID_ARG
    assert call(lse=None) == ea.ATTN_ERR_INVALID_ARG
    assert call(B=0) == ea.ATTN_ERR_INVALID_ARG
    assert call(Nq=0) == ea.ATTN_ERR_INVALID_ARG
    assert call(Nkv=-5) == ea.ATTN_ERR_INVALID_ARG
    assert call(causal=2) == ea.ATTN_ERR_INVALID_ARG
    assert call(scale=0.0) == ea.ATTN_ERR_INVALID_ARG
    assert call(scale=float("nan")) == ea.ATTN_ERR_INVALID_ARG
    assert call(d=96) == ea.ATTN_ERR_UNSUPPORTED
    assert call(d=256) == ea.ATTN_ERR_UNSUPPORTED
    assert call(q=p + 8) == ea.ATTN_ERR_ALIGNMENT
    assert call(o=p + 2) == ea.ATTN_ERR_ALIGNMENT
    assert call(lse=p + 2) == ea.ATTN_ERR_ALIGNMENT


def test_decode_and_merge_reject_bad_arguments(ea):
    L = ea.lib
    p = 0x10000
    assert L.attn_decode_partials(None, p, p, p, p, 1, 1, 64, 128, 0.1, 4, None) == 1
    assert L.attn_decode_partials(p, p, p, p, p, 1, 1, 64, 128, 0.1, 0, None) == 1
    assert L.attn_decode_partials(p, p, p, p, p, 1, 1, 64, 80, 0.1, 4, None) == 2
    assert L.attn_decode_partials(p, p + 4, p, p, p, 1, 1, 64, 128, 0.1, 4, None) == 3
    assert L.attn_lse_merge(p, p, p, p, 1, 1, 0, 128, None) == 1
    assert L.attn_lse_merge(p, p, p, p, 1, 1, 4, 32, None) == 2
    assert L.attn_lse_merge(p, p + 1, p, p, 1, 1, 4, 128, None) == 3
    need = ea.attn_decode_workspace_bytes(2, 3, 128, 8)
    assert need == ((2 * 3 * 8 * 128 * 4 + 255) // 256 + (2 * 3 * 8 * 4 + 255) // 256) * 256
    assert ea.attn_decode_workspace_bytes(2, 3, 96, 8) == 0
    assert L.attn_decode_splitkv(p, p, p, p, p, 2, 3, 64, 128, 0.1, 8, p, need - 1, None) == 1
    assert L.attn_decode_splitkv(p, p, p, p, p, 2, 3, 64, 128, 0.1, 8, p + 16, need, None) == 3
    assert L.attn_decode_splitkv(p, p, p, p, p, 2, 3, 64, 96, 0.1, 8, p, need, None) == 2


def test_noalloc_decode_rejects_bad_arguments_before_launching(ea):
    """Every argument error of the allocation-free decode is returned before its
    partial kernel is enqueued into the shared scratch array (the pointers are
    never dereferenced; no GPU is needed)."""
    f = ea.lib.attn_decode_splitkv_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 4 + [ctypes.c_float, ctypes.c_int,
                                                               ctypes.c_void_p]
    p = 0x10000

    def call(**kw):
        a = dict(dict(q=p, k=p, v=p, o=p, lse=p, B=2, H=3, Nkv=64, d=128, scale=0.088, S=8),
                 **kw)
        return f(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["Nkv"], a["d"],
                 a["scale"], a["S"], None)

    assert call(o=None) == ea.ATTN_ERR_INVALID_ARG
    assert call(lse=None) == ea.ATTN_ERR_INVALID_ARG
    assert call(q=None) == ea.ATTN_ERR_INVALID_ARG
    assert call(Nkv=0) == ea.ATTN_ERR_INVALID_ARG
    assert call(S=0) == ea.ATTN_ERR_INVALID_ARG
    assert call(S=65536) == ea.ATTN_ERR_INVALID_ARG
    assert call(B=256, H=256) == ea.ATTN_ERR_INVALID_ARG      # B*H beyond the grid's y limit
    assert call(scale=float("inf")) == ea.ATTN_ERR_INVALID_ARG
    assert call(d=96) == ea.ATTN_ERR_UNSUPPORTED
    assert call(o=p + 1) == ea.ATTN_ERR_ALIGNMENT
    assert call(lse=p + 2) == ea.ATTN_ERR_ALIGNMENT
    assert call(k=p + 8) == ea.ATTN_ERR_ALIGNMENT
    # partials of 16 x 128 heads x 64 chunks (67.6 MB) exceed the fixed array
    assert call(B=16, H=128, Nkv=32768, S=64) == ea.ATTN_ERR_SCRATCH_LIMIT


def test_bwd_rejects_bad_arguments_without_launching(ea):
    L = ea.lib
    p = 0x10000
    ws_need = ea.attn_bwd_workspace_bytes(1, 2, 300, 128)
    # D and LSE * log2(e) rows padded to 64 and to 256 bytes, 256 bytes of maxima,
    # then the dQ accumulator in its int64 form
    assert ws_need == 2 * ((2 * 320 * 4 + 255) // 256 * 256) + 256 + 2 * 300 * 128 * 8
    assert ea.attn_bwd_workspace_bytes(1, 2, 300, 96) == 0
    assert ea.attn_bwd_workspace_bytes(1, 2, 0, 128) == 0
    for fn in (L.attn_bwd, L.attn_bwd_deterministic):
        _bwd_bad_arguments(ea, fn, p, ws_need)


def _bwd_bad_arguments(ea, fn, p, ws_need):
    def call(ws_bytes=ws_need, **kw):
        a = dict(dict(q=p, k=p, v=p, o=p, do=p, lse=p, dq=p, dk=p, dv=p, ws=p, B=1, H=2, Nq=300,
                      Nkv=300, d=128, causal=1, scale=0.088), **kw)
        return fn(a["q"], a["k"], a["v"], a["o"], a["do"], a["lse"], a["dq"], a["dk"],
                  a["dv"], a["B"], a["H"], a["Nq"], a["Nkv"], a["d"], a["causal"],
                  a["scale"], a["ws"], ws_bytes, None)

    assert call(do=None) == ea.ATTN_ERR_INVALID_ARG
    assert call(ws=None) == ea.ATTN_ERR_INVALID_ARG
    assert call(ws_bytes=ws_need - 1) == ea.ATTN_ERR_INVALID_ARG
    assert call(causal=2) == ea.ATTN_ERR_INVALID_ARG
    assert call(scale=float("nan")) == ea.ATTN_ERR_INVALID_ARG
    assert call(Nkv=0) == ea.ATTN_ERR_INVALID_ARG
    assert call(B=70000) == ea.ATTN_ERR_INVALID_ARG
    assert call(d=80) == ea.ATTN_ERR_UNSUPPORTED
    assert call(dk=p + 8) == ea.ATTN_ERR_ALIGNMENT
    assert call(ws=p + 16) == ea.ATTN_ERR_ALIGNMENT


def test_fwd_fp8_rejects_bad_arguments_without_launching(ea):
    L = ea.lib
    p = 0x10000

    def call(**kw):
        a = dict(dict(q=p, k=p, v=p, qd=p, kd=p, vd=p, o=p, lse=p, B=1, H=2, Nq=300, Nkv=300,
                      d=128, causal=1, scale=0.088), **kw)
        return L.attn_fwd_fp8(a["q"], a["k"], a["v"], a["qd"], a["kd"], a["vd"], a["o"],
                              a["lse"], a["B"], a["H"], a["Nq"], a["Nkv"], a["d"], a["causal"],
                              a["scale"], None)

    assert call(vd=None) == ea.ATTN_ERR_INVALID_ARG
    assert call(Nq=0) == ea.ATTN_ERR_INVALID_ARG
    assert call(causal=3) == ea.ATTN_ERR_INVALID_ARG
    assert call(scale=-1.0) == ea.ATTN_ERR_INVALID_ARG
    assert call(d=96) == ea.ATTN_ERR_UNSUPPORTED
    assert call(k=p + 8) == ea.ATTN_ERR_ALIGNMENT
    assert call(qd=p + 2) == ea.ATTN_ERR_ALIGNMENT


def test_package_fails_loudly_without_the_library(tmp_path):
    """No silent fallback: the binding refuses to import when the .so is absent."""
    src = os.path.join(ROOT, "exact_io_aware_70_b200", "__init__.py")
    pkg = tmp_path / "fake_pkg"
    pkg.mkdir()
    shutil.copy(src, pkg / "__init__.py")
    spec = importlib.util.spec_from_file_location("fake_pkg", pkg / "__init__.py")
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError, match="missing"):
        spec.loader.exec_module(mod)
    sys.modules.pop("fake_pkg", None)


def test_debug_build_compiles_and_exports_every_symbol():
    """The index-checking debug build (-DATTN_DEBUG) of the same sources builds
    for sm_100a and exports the same entry points."""
    spec = importlib.util.spec_from_file_location(
        "exact_attn_cuda_build", os.path.join(ROOT, "exact_io_aware_70_b200", "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    path = build.build(debug=True)
    assert path.endswith("libexact_attn_b200_debug.so")
    lib = ctypes.CDLL(path)
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} missing from the debug build"
    lib.attn_strerror.restype = ctypes.c_char_p
    assert b"debug build" in lib.attn_strerror(8)
