"""exact_io_aware_70_b200 -- exact IO-aware attention for B200 (sm_100a).

Python binding of the C ABI declared in include/exact_attn.h. Argument
marshalling only: every step of the computation runs in the CUDA kernels of
``libexact_attn_b200.so``. Importing this package fails loudly if that library
has not been built; there is no fallback implementation.

Entry points (same names as the C ABI):
  attn_fwd(q, k, v, o, lse, causal, scale)            prefill forward, O and LSE
  attn_fwd_fp8(q, k, v, q_descale, k_descale, v_descale, o, lse, causal, scale)
  attn_bwd(q, k, v, o, dout, lse, dq, dk, dv, causal, scale, workspace[, deterministic])
  attn_bwd_workspace_bytes(B, H, Nq, d)
  attn_decode_partials(q, k, v, o_part, lse_part, scale, num_splits)
  attn_lse_merge(o_part, lse_part, o, lse)
  attn_lse_merge_gathered(o_part, lse_part, o, lse)  merge of partials gathered from R GPUs
  attn_decode_splitkv(q, k, v, o, lse, scale, num_splits, workspace)
  attn_decode_workspace_bytes(B, H, d, num_splits)
  attn_decode_paged(q, k_cache, v_cache, block_table, seq_lens, o, lse, scale, num_splits,
                    workspace)                        paged-KV split-KV decode
  attn_status(stream) / attn_strerror(code)
Tensor arguments are torch tensors on the current CUDA device (bf16 for
q/k/v/o, fp32 for lse and partials, contiguous); ``stream`` defaults to torch's
current stream. ``lib`` is the raw ctypes handle for pointer-level calls.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# EXACT_ATTN_LIB may name another build of the same library (e.g. the debug
# build, libexact_attn_b200_debug.so, whose kernels check their indices); it
# must exist, there is no fallback either way.
LIB_PATH = os.environ.get("EXACT_ATTN_LIB") or os.path.join(_HERE, "libexact_attn_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python exact_io_aware_70_b200/build.py` "
        "(this package has no CPU or fallback path)")

lib = ctypes.CDLL(LIB_PATH)

_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float
_sz = ctypes.c_size_t

lib.attn_abi_version.restype = _i
lib.attn_abi_version.argtypes = []
lib.attn_strerror.restype = ctypes.c_char_p
lib.attn_strerror.argtypes = [_i]
lib.attn_fwd.restype = _i
lib.attn_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp]
lib.attn_fwd_fp8.restype = _i
lib.attn_fwd_fp8.argtypes = [_vp] * 8 + [_i] * 6 + [_f, _vp]
lib.attn_decode_partials.restype = _i
lib.attn_decode_partials.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp]
lib.attn_lse_merge.restype = _i
lib.attn_lse_merge.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp]
lib.attn_lse_merge_gathered.restype = _i
lib.attn_lse_merge_gathered.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]
lib.attn_decode_workspace_bytes.restype = _sz
lib.attn_decode_workspace_bytes.argtypes = [_i, _i, _i, _i]
lib.attn_decode_splitkv.restype = _i
lib.attn_decode_splitkv.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp, _sz,
                                    _vp]
lib.attn_decode_paged_partials.restype = _i
lib.attn_decode_paged_partials.argtypes = [_vp] * 7 + [_i] * 6 + [_f, _i, _vp]
lib.attn_decode_paged.restype = _i
lib.attn_decode_paged.argtypes = [_vp] * 7 + [_i] * 6 + [_f, _i, _vp, _sz, _vp]
lib.attn_bwd_workspace_bytes.restype = _sz
lib.attn_bwd_workspace_bytes.argtypes = [_i, _i, _i, _i]
lib.attn_bwd.restype = _i
lib.attn_bwd.argtypes = [_vp] * 9 + [_i] * 6 + [_f, _vp, _sz, _vp]
lib.attn_bwd_deterministic.restype = _i
lib.attn_bwd_deterministic.argtypes = lib.attn_bwd.argtypes
lib.attn_status.restype = _i
lib.attn_status.argtypes = [_vp]

ATTN_OK = 0
ATTN_ERR_INVALID_ARG = 1
ATTN_ERR_UNSUPPORTED = 2
ATTN_ERR_ALIGNMENT = 3
ATTN_ERR_CUDA = 4
ATTN_ERR_TIMEOUT = 5
ATTN_ERR_SCRATCH_LIMIT = 6
ATTN_ERR_BAD_INDEX = 7
ATTN_ERR_INDEX_CHECK = 8   # debug build only: a kernel index check failed


class AttnError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {attn_strerror(code)} (status {code})")
        self.code = code


def attn_strerror(code: int) -> str:
    return lib.attn_strerror(int(code)).decode()


def _check(code: int, what: str) -> None:
    if code != ATTN_OK:
        raise AttnError(code, what)


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return int(stream)


def _tensor(t, dtype, name):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor")
    if t.dtype != dtype or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor of {dtype}")
    return t.data_ptr()


def attn_fwd(q, k, v, o, lse, causal: bool, scale: float, stream=None) -> None:
    """O and LSE of exact attention. q/o [B,H,Nq,d], k/v [B,H,Nkv,d] bf16; lse [B,H,Nq] fp32."""
    import torch
    B, H, Nq, d = q.shape
    Nkv = k.shape[2]
    if tuple(k.shape) != (B, H, Nkv, d) or tuple(v.shape) != (B, H, Nkv, d) \
            or tuple(o.shape) != (B, H, Nq, d) or tuple(lse.shape) != (B, H, Nq):
        raise ValueError("attn_fwd: inconsistent shapes")
    _check(lib.attn_fwd(_tensor(q, torch.bfloat16, "q"), _tensor(k, torch.bfloat16, "k"),
                        _tensor(v, torch.bfloat16, "v"), _tensor(o, torch.bfloat16, "o"),
                        _tensor(lse, torch.float32, "lse"), B, H, Nq, Nkv, d, int(bool(causal)),
                        float(scale), _stream(stream)), "attn_fwd")


def attn_fwd_fp8(q, k, v, q_descale, k_descale, v_descale, o, lse, causal: bool, scale: float,
                 stream=None) -> None:
    """O and LSE from e4m3 inputs. q [B,H,Nq,d], k/v [B,H,Nkv,d] torch.float8_e4m3fn (d 64
    or 128); *_descale [B,H] fp32; o [B,H,Nq,d] bf16; lse [B,H,Nq] fp32."""
    import torch
    B, H, Nq, d = q.shape
    Nkv = k.shape[2]
    if tuple(k.shape) != (B, H, Nkv, d) or tuple(v.shape) != (B, H, Nkv, d) \
            or tuple(o.shape) != (B, H, Nq, d) or tuple(lse.shape) != (B, H, Nq) \
            or any(tuple(t.shape) != (B, H) for t in (q_descale, k_descale, v_descale)):
        raise ValueError("attn_fwd_fp8: inconsistent shapes")
    f8 = torch.float8_e4m3fn
    _check(lib.attn_fwd_fp8(_tensor(q, f8, "q"), _tensor(k, f8, "k"), _tensor(v, f8, "v"),
                            _tensor(q_descale, torch.float32, "q_descale"),
                            _tensor(k_descale, torch.float32, "k_descale"),
                            _tensor(v_descale, torch.float32, "v_descale"),
                            _tensor(o, torch.bfloat16, "o"), _tensor(lse, torch.float32, "lse"),
                            B, H, Nq, Nkv, d, int(bool(causal)), float(scale), _stream(stream)),
           "attn_fwd_fp8")


def attn_decode_partials(q, k, v, o_part, lse_part, scale: float, num_splits: int,
                         stream=None) -> None:
    """Per-chunk partials. q [B,H,1,d], k/v [B,H,Nkv,d] bf16; o_part [B,H,S,d], lse_part [B,H,S] fp32."""
    import torch
    B, H, one, d = q.shape
    Nkv = k.shape[2]
    if one != 1 or tuple(o_part.shape) != (B, H, num_splits, d) \
            or tuple(lse_part.shape) != (B, H, num_splits):
        raise ValueError("attn_decode_partials: inconsistent shapes")
    _check(lib.attn_decode_partials(_tensor(q, torch.bfloat16, "q"),
                                    _tensor(k, torch.bfloat16, "k"),
                                    _tensor(v, torch.bfloat16, "v"),
                                    _tensor(o_part, torch.float32, "o_part"),
                                    _tensor(lse_part, torch.float32, "lse_part"), B, H, Nkv, d,
                                    float(scale), int(num_splits), _stream(stream)),
           "attn_decode_partials")


def attn_lse_merge(o_part, lse_part, o, lse, stream=None) -> None:
    """Max-and-sum merge. o_part [B,H,S,d], lse_part [B,H,S] fp32 -> o [B,H,1,d] bf16, lse [B,H,1] fp32."""
    import torch
    B, H, S, d = o_part.shape
    if tuple(o.shape) != (B, H, 1, d) or tuple(lse.shape) != (B, H, 1):
        raise ValueError("attn_lse_merge: inconsistent shapes")
    _check(lib.attn_lse_merge(_tensor(o_part, torch.float32, "o_part"),
                              _tensor(lse_part, torch.float32, "lse_part"),
                              _tensor(o, torch.bfloat16, "o"), _tensor(lse, torch.float32, "lse"),
                              B, H, S, d, _stream(stream)), "attn_lse_merge")


def attn_lse_merge_gathered(o_part, lse_part, o, lse, stream=None) -> None:
    """Max-and-sum merge of partials gathered from R ranks' KV shards.
    o_part [R,B,H,S,d], lse_part [R,B,H,S] fp32 -> o [B,H,1,d] bf16, lse [B,H,1] fp32."""
    import torch
    R, B, H, S, d = o_part.shape
    if (tuple(lse_part.shape) != (R, B, H, S) or tuple(o.shape) != (B, H, 1, d)
            or tuple(lse.shape) != (B, H, 1)):
        raise ValueError("attn_lse_merge_gathered: inconsistent shapes")
    _check(lib.attn_lse_merge_gathered(_tensor(o_part, torch.float32, "o_part"),
                                       _tensor(lse_part, torch.float32, "lse_part"),
                                       _tensor(o, torch.bfloat16, "o"),
                                       _tensor(lse, torch.float32, "lse"),
                                       R, B, H, S, d, _stream(stream)), "attn_lse_merge_gathered")


def attn_decode_workspace_bytes(B: int, H: int, d: int, num_splits: int) -> int:
    return int(lib.attn_decode_workspace_bytes(B, H, d, num_splits))


def attn_decode_splitkv(q, k, v, o, lse, scale: float, num_splits: int, workspace,
                        stream=None) -> None:
    """Split-KV decode (partials + merge). workspace: uint8 CUDA tensor of the required size."""
    import torch
    B, H, one, d = q.shape
    Nkv = k.shape[2]
    if one != 1 or tuple(o.shape) != (B, H, 1, d) or tuple(lse.shape) != (B, H, 1):
        raise ValueError("attn_decode_splitkv: inconsistent shapes")
    _check(lib.attn_decode_splitkv(_tensor(q, torch.bfloat16, "q"), _tensor(k, torch.bfloat16, "k"),
                                   _tensor(v, torch.bfloat16, "v"),
                                   _tensor(o, torch.bfloat16, "o"),
                                   _tensor(lse, torch.float32, "lse"), B, H, Nkv, d, float(scale),
                                   int(num_splits), _tensor(workspace, torch.uint8, "workspace"),
                                   workspace.numel(), _stream(stream)), "attn_decode_splitkv")


def attn_decode_paged(q, k_cache, v_cache, block_table, seq_lens, o, lse, scale: float,
                      num_splits: int, workspace, num_pages: int | None = None,
                      stream=None) -> None:
    """Paged-KV split-KV decode. q [B,H,1,d]; caches [num_pages,H,page_size,d] bf16;
    block_table [B,max_pages] int32; seq_lens [B] int32; o [B,H,1,d]; lse [B,H,1]."""
    import torch
    B, H, one, d = q.shape
    P, H2, page_size, d2 = k_cache.shape
    if one != 1 or H2 != H or d2 != d or tuple(v_cache.shape) != tuple(k_cache.shape) \
            or block_table.shape[0] != B or tuple(seq_lens.shape) != (B,):
        raise ValueError("attn_decode_paged: inconsistent shapes")
    _check(lib.attn_decode_paged(_tensor(q, torch.bfloat16, "q"),
                                 _tensor(k_cache, torch.bfloat16, "k_cache"),
                                 _tensor(v_cache, torch.bfloat16, "v_cache"),
                                 _tensor(block_table, torch.int32, "block_table"),
                                 _tensor(seq_lens, torch.int32, "seq_lens"),
                                 _tensor(o, torch.bfloat16, "o"), _tensor(lse, torch.float32, "lse"),
                                 B, H, d, page_size, block_table.shape[1],
                                 P if num_pages is None else int(num_pages), float(scale),
                                 int(num_splits), _tensor(workspace, torch.uint8, "workspace"),
                                 workspace.numel(), _stream(stream)), "attn_decode_paged")


def attn_bwd_workspace_bytes(B: int, H: int, Nq: int, d: int) -> int:
    return int(lib.attn_bwd_workspace_bytes(B, H, Nq, d))


def attn_bwd(q, k, v, o, dout, lse, dq, dk, dv, causal: bool, scale: float, workspace,
             stream=None, deterministic: bool = False) -> None:
    """dQ, dK, dV of sum(dO*O). q/o/dout/dq [B,H,Nq,d], k/v/dk/dv [B,H,Nkv,d] bf16; lse [B,H,Nq] fp32;
    workspace: a device buffer of at least attn_bwd_workspace_bytes(B, H, Nq, d) bytes.
    deterministic: call attn_bwd_deterministic (dQ bit-identical from run to run)."""
    import torch
    B, H, Nq, d = q.shape
    Nkv = k.shape[2]
    qs, ks = (B, H, Nq, d), (B, H, Nkv, d)
    if any(tuple(t.shape) != qs for t in (o, dout, dq)) \
            or any(tuple(t.shape) != ks for t in (k, v, dk, dv)) or tuple(lse.shape) != (B, H, Nq):
        raise ValueError("attn_bwd: inconsistent shapes")
    if not workspace.is_contiguous():
        raise ValueError("attn_bwd: workspace must be contiguous")
    fn = lib.attn_bwd_deterministic if deterministic else lib.attn_bwd
    _check(fn(_tensor(q, torch.bfloat16, "q"), _tensor(k, torch.bfloat16, "k"),
              _tensor(v, torch.bfloat16, "v"), _tensor(o, torch.bfloat16, "o"),
              _tensor(dout, torch.bfloat16, "dout"), _tensor(lse, torch.float32, "lse"),
              _tensor(dq, torch.bfloat16, "dq"), _tensor(dk, torch.bfloat16, "dk"),
              _tensor(dv, torch.bfloat16, "dv"), B, H, Nq, Nkv, d, int(bool(causal)),
              float(scale), ctypes.c_void_p(workspace.data_ptr()),
              workspace.numel() * workspace.element_size(), _stream(stream)),
           "attn_bwd_deterministic" if deterministic else "attn_bwd")


def attn_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status (0 = ok)."""
    return int(lib.attn_status(_stream(stream)))


def abi_version() -> int:
    return int(lib.attn_abi_version())
