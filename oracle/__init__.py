"""fp64 CPU oracle for exact attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and bench.py's CPU-baseline leg may
import this package. It wraps ``attn_oracle.c`` (plain C, double precision),
which evaluates the naive definition S = scale*Q K^T (masked), P = softmax(S),
O = P V, LSE = ln sum exp(S), plus per-chunk split-KV partials and their
max-and-sum merge. It shares no code with the CUDA library.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_c_long = ctypes.c_long
_dp = ctypes.POINTER(ctypes.c_double)
_fp = ctypes.POINTER(ctypes.c_float)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_i64p = ctypes.POINTER(ctypes.c_int64)


def _ptr(a: np.ndarray, t):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(t)


class Oracle:
    """ctypes handle on one build of the oracle library (normal or a mutant)."""

    def __init__(self, path: str | None = None):
        path = path or _build.build()
        self.path = path
        lib = ctypes.CDLL(path)
        lib.oracle_attn_head_f64.argtypes = [_dp, _dp, _dp, _c_long, _c_long, _c_long,
                                             ctypes.c_int, ctypes.c_double, _dp, _dp, _dp]
        lib.oracle_attn_fwd_bf16.argtypes = [_u16p, _u16p, _u16p, _c_long, _c_long, _c_long,
                                             _c_long, _c_long, ctypes.c_int, ctypes.c_double,
                                             _dp, _dp]
        lib.oracle_attn_rows_bf16.argtypes = [_u16p, _u16p, _u16p, _c_long, _c_long, _c_long,
                                              ctypes.c_int, ctypes.c_double, _i64p, _c_long,
                                              _dp, _dp]
        lib.oracle_decode_partials_bf16.argtypes = [_u16p, _u16p, _u16p, _c_long, _c_long,
                                                    ctypes.c_double, _c_long, _dp, _dp]
        lib.oracle_lse_merge_f64.argtypes = [_dp, _dp, _c_long, _c_long, _dp, _dp]
        lib.oracle_lse_merge_f32in.argtypes = [_fp, _fp, _c_long, _c_long, _c_long, _dp, _dp]
        _i32p = ctypes.POINTER(ctypes.c_int32)
        lib.oracle_decode_paged_bf16.argtypes = [_u16p, _u16p, _u16p, _i32p, _i32p, _c_long,
                                                 _c_long, _c_long, _c_long, _c_long, _c_long,
                                                 ctypes.c_double, _dp, _dp]
        lib.oracle_attn_bwd_head_f64.argtypes = [_dp, _dp, _dp, _dp, _c_long, _c_long, _c_long,
                                                 ctypes.c_int, ctypes.c_double, _dp, _dp, _dp]
        lib.oracle_attn_bwd_bf16.argtypes = [_u16p, _u16p, _u16p, _u16p, _c_long, _c_long,
                                             _c_long, _c_long, _c_long, ctypes.c_int,
                                             ctypes.c_double, _dp, _dp, _dp]
        lib.oracle_e4m3_decode.argtypes = [_u8p, _c_long, _dp]
        lib.oracle_attn_fwd_fp8.argtypes = [_u8p, _u8p, _u8p, _fp, _fp, _fp, _c_long, _c_long,
                                            _c_long, _c_long, _c_long, ctypes.c_int,
                                            ctypes.c_double, _dp, _dp]
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        self.lib = lib

    # -- double-precision entry (one head) ---------------------------------
    def attn_head_f64(self, q, k, v, causal: bool, scale: float, want_p: bool = False):
        q = np.ascontiguousarray(q, dtype=np.float64)
        k = np.ascontiguousarray(k, dtype=np.float64)
        v = np.ascontiguousarray(v, dtype=np.float64)
        Nq, d = q.shape
        Nkv = k.shape[0]
        assert k.shape == (Nkv, d) and v.shape == (Nkv, d)
        o = np.zeros((Nq, d))
        lse = np.zeros(Nq)
        p = np.zeros((Nq, Nkv)) if want_p else None
        rc = self.lib.oracle_attn_head_f64(_ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), Nq, Nkv,
                                           d, int(causal), float(scale), _ptr(o, _dp),
                                           _ptr(lse, _dp), _ptr(p, _dp) if want_p else None)
        if rc:
            raise RuntimeError("oracle_attn_head_f64 failed")
        return (o, lse, p) if want_p else (o, lse)

    # -- bf16 entries ---------------------------------------------------------
    def attn_fwd_bf16(self, q_bits, k_bits, v_bits, causal: bool, scale: float):
        """q_bits [B,H,Nq,d], k_bits/v_bits [B,H,Nkv,d] uint16 -> (O f64, LSE f64)."""
        B, H, Nq, d = q_bits.shape
        Nkv = k_bits.shape[2]
        q, k, v = (np.ascontiguousarray(x, dtype=np.uint16) for x in (q_bits, k_bits, v_bits))
        o = np.zeros((B, H, Nq, d))
        lse = np.zeros((B, H, Nq))
        rc = self.lib.oracle_attn_fwd_bf16(_ptr(q, _u16p), _ptr(k, _u16p), _ptr(v, _u16p), B, H,
                                           Nq, Nkv, d, int(causal), float(scale),
                                           _ptr(o, _dp), _ptr(lse, _dp))
        if rc:
            raise RuntimeError("oracle_attn_fwd_bf16 failed")
        return o, lse

    def attn_rows_bf16(self, q_head, k_head, v_head, rows, causal: bool, scale: float):
        """One head: q_head [Nq,d], k_head/v_head [Nkv,d] uint16; rows: query indices."""
        Nq, d = q_head.shape
        Nkv = k_head.shape[0]
        q, k, v = (np.ascontiguousarray(x, dtype=np.uint16) for x in (q_head, k_head, v_head))
        r = np.ascontiguousarray(rows, dtype=np.int64)
        o = np.zeros((len(r), d))
        lse = np.zeros(len(r))
        rc = self.lib.oracle_attn_rows_bf16(_ptr(q, _u16p), _ptr(k, _u16p), _ptr(v, _u16p), Nq,
                                            Nkv, d, int(causal), float(scale), _ptr(r, _i64p),
                                            len(r), _ptr(o, _dp), _ptr(lse, _dp))
        if rc:
            raise RuntimeError("oracle_attn_rows_bf16 failed")
        return o, lse

    def decode_partials_bf16(self, q_row, k_head, v_head, scale: float, num_splits: int):
        d = q_row.shape[-1]
        Nkv = k_head.shape[0]
        q, k, v = (np.ascontiguousarray(x, dtype=np.uint16) for x in (q_row, k_head, v_head))
        o = np.zeros((num_splits, d))
        lse = np.zeros(num_splits)
        rc = self.lib.oracle_decode_partials_bf16(_ptr(q, _u16p), _ptr(k, _u16p), _ptr(v, _u16p),
                                                  Nkv, d, float(scale), num_splits,
                                                  _ptr(o, _dp), _ptr(lse, _dp))
        if rc:
            raise RuntimeError("oracle_decode_partials_bf16 failed")
        return o, lse

    def attn_bwd_head_f64(self, q, k, v, dout, causal: bool, scale: float):
        """Gradients of sum(dout * O) for one head -> (dq, dk, dv) in double."""
        q, k, v, dout = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v, dout))
        Nq, d = q.shape
        Nkv = k.shape[0]
        dq, dk, dv = np.zeros((Nq, d)), np.zeros((Nkv, d)), np.zeros((Nkv, d))
        rc = self.lib.oracle_attn_bwd_head_f64(_ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp),
                                               _ptr(dout, _dp), Nq, Nkv, d, int(causal),
                                               float(scale), _ptr(dq, _dp), _ptr(dk, _dp),
                                               _ptr(dv, _dp))
        if rc:
            raise RuntimeError("oracle_attn_bwd_head_f64 failed")
        return dq, dk, dv

    def attn_bwd_bf16(self, q_bits, k_bits, v_bits, dout_bits, causal: bool, scale: float):
        """[B,H,N,d] uint16 inputs -> (dq, dk, dv) double arrays of the same shapes."""
        B, H, Nq, d = q_bits.shape
        Nkv = k_bits.shape[2]
        q, k, v, do = (np.ascontiguousarray(x, dtype=np.uint16)
                       for x in (q_bits, k_bits, v_bits, dout_bits))
        dq, dk, dv = np.zeros((B, H, Nq, d)), np.zeros((B, H, Nkv, d)), np.zeros((B, H, Nkv, d))
        rc = self.lib.oracle_attn_bwd_bf16(_ptr(q, _u16p), _ptr(k, _u16p), _ptr(v, _u16p),
                                           _ptr(do, _u16p), B, H, Nq, Nkv, d, int(causal),
                                           float(scale), _ptr(dq, _dp), _ptr(dk, _dp),
                                           _ptr(dv, _dp))
        if rc:
            raise RuntimeError("oracle_attn_bwd_bf16 failed")
        return dq, dk, dv

    def e4m3_decode(self, codes):
        """Values of e4m3 codes (uint8 array) as doubles, from the format's definition."""
        c = np.ascontiguousarray(codes, dtype=np.uint8)
        out = np.zeros(c.shape)
        self.lib.oracle_e4m3_decode(_ptr(c, _u8p), c.size, _ptr(out, _dp))
        return out

    def attn_fwd_fp8(self, q_codes, k_codes, v_codes, q_descale, k_descale, v_descale,
                     causal: bool, scale: float):
        """e4m3 codes [B,H,N,d] (uint8) and fp32 descales [B,H] -> (O f64, LSE f64)."""
        B, H, Nq, d = q_codes.shape
        Nkv = k_codes.shape[2]
        q, k, v = (np.ascontiguousarray(x, dtype=np.uint8) for x in (q_codes, k_codes, v_codes))
        qd, kd, vd = (np.ascontiguousarray(x, dtype=np.float32).reshape(B * H)
                      for x in (q_descale, k_descale, v_descale))
        o, lse = np.zeros((B, H, Nq, d)), np.zeros((B, H, Nq))
        rc = self.lib.oracle_attn_fwd_fp8(_ptr(q, _u8p), _ptr(k, _u8p), _ptr(v, _u8p),
                                          _ptr(qd, _fp), _ptr(kd, _fp), _ptr(vd, _fp), B, H, Nq,
                                          Nkv, d, int(causal), float(scale), _ptr(o, _dp),
                                          _ptr(lse, _dp))
        if rc:
            raise RuntimeError("oracle_attn_fwd_fp8 failed")
        return o, lse

    def decode_paged_bf16(self, q_bits, k_cache_bits, v_cache_bits, block_table, seq_lens,
                          scale: float):
        """q [B,H,d]; caches [num_pages,H,page_size,d] uint16; block_table [B,max_pages] int32;
        seq_lens [B] int32 -> (O [B,H,d] f64, LSE [B,H] f64)."""
        q = np.ascontiguousarray(q_bits, dtype=np.uint16)
        kc = np.ascontiguousarray(k_cache_bits, dtype=np.uint16)
        vc = np.ascontiguousarray(v_cache_bits, dtype=np.uint16)
        bt = np.ascontiguousarray(block_table, dtype=np.int32)
        sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
        B, H, d = q.shape
        num_pages, H2, page_size, d2 = kc.shape
        assert H2 == H and d2 == d and vc.shape == kc.shape and bt.shape[0] == B
        o = np.zeros((B, H, d))
        lse = np.zeros((B, H))
        i32 = ctypes.POINTER(ctypes.c_int32)
        rc = self.lib.oracle_decode_paged_bf16(_ptr(q, _u16p), _ptr(kc, _u16p), _ptr(vc, _u16p),
                                               _ptr(bt, i32), _ptr(sl, i32), B, H, d, page_size,
                                               bt.shape[1], num_pages, float(scale),
                                               _ptr(o, _dp), _ptr(lse, _dp))
        if rc:
            raise RuntimeError("oracle_decode_paged_bf16 failed")
        return o, lse

    def lse_merge_f64(self, o_part, lse_part):
        o_part = np.ascontiguousarray(o_part, dtype=np.float64)
        lse_part = np.ascontiguousarray(lse_part, dtype=np.float64)
        S, d = o_part.shape
        o = np.zeros(d)
        lse = np.zeros(1)
        rc = self.lib.oracle_lse_merge_f64(_ptr(o_part, _dp), _ptr(lse_part, _dp), S, d,
                                           _ptr(o, _dp), _ptr(lse, _dp))
        if rc:
            raise RuntimeError("oracle_lse_merge_f64 failed")
        return o, float(lse[0])

    def lse_merge_f32in(self, o_part, lse_part):
        """o_part [B,H,S,d] f32, lse_part [B,H,S] f32 -> (O [B,H,d] f64, LSE [B,H] f64)."""
        o_part = np.ascontiguousarray(o_part, dtype=np.float32)
        lse_part = np.ascontiguousarray(lse_part, dtype=np.float32)
        B, H, S, d = o_part.shape
        o = np.zeros((B, H, d))
        lse = np.zeros((B, H))
        rc = self.lib.oracle_lse_merge_f32in(_ptr(o_part, _fp), _ptr(lse_part, _fp), B * H, S, d,
                                             _ptr(o, _dp), _ptr(lse, _dp))
        if rc:
            raise RuntimeError("oracle_lse_merge_f32in failed")
        return o, lse

    def num_threads(self) -> int:
        return int(self.lib.oracle_num_threads())

    def set_num_threads(self, n: int) -> None:
        self.lib.oracle_set_num_threads(int(n))


_default: Oracle | None = None


def get() -> Oracle:
    """The oracle built from the unmodified source (built on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def build_mutant(n: int, out_dir: str) -> Oracle:
    """A copy of the oracle with planted mistake ``n`` (1..13), for the pin tests."""
    out = os.path.join(out_dir, f"liboracle_mutant{n}.so")
    _build.build(out=out, mutant=n, force=True)
    return Oracle(out)
