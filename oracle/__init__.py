"""fp64 CPU oracle for exact attention, its paged forms (decode and varlen
prefill), its FP8-input form and its gradients.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
benchmark's CPU-baseline leg import this package; the library under
`tiled_attention_17_b200` never does, and this package never imports it.

The arithmetic lives in oracle.c (plain C, fp64, OpenMP over rows); this file
only marshals numpy arrays through ctypes.  See oracle.c's header for the
definition followed and the readings taken where the pages are silent.
"""
from __future__ import annotations

import ctypes
import math

import numpy as np

from . import build as _build

def _bind(path):
    L = ctypes.CDLL(path)
    c_u16p = ctypes.POINTER(ctypes.c_uint16)
    c_i32p = ctypes.POINTER(ctypes.c_int32)
    c_i64p = ctypes.POINTER(ctypes.c_int64)
    c_dp = ctypes.POINTER(ctypes.c_double)
    L.oracle_attn.argtypes = [c_u16p, c_u16p, c_u16p] + [ctypes.c_int] * 6 + [
        ctypes.c_double, ctypes.c_int, c_i64p, ctypes.c_int64, c_dp, c_dp]
    L.oracle_attn.restype = ctypes.c_int
    L.oracle_paged_gather.argtypes = [c_u16p, c_u16p, c_i32p, c_i32p] + [ctypes.c_int] * 6 + [
        ctypes.c_int64, c_u16p, c_u16p]
    L.oracle_paged_gather.restype = ctypes.c_int
    L.oracle_paged_decode.argtypes = [c_u16p, c_u16p, c_u16p, c_i32p, c_i32p] + [ctypes.c_int] * 6 + [
        ctypes.c_int64, ctypes.c_double, c_i32p, ctypes.c_int, c_dp, c_dp]
    L.oracle_paged_decode.restype = ctypes.c_int
    L.oracle_paged_prefill.argtypes = [c_u16p, c_u16p, c_u16p, c_i32p, c_i32p, c_i32p, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int64, ctypes.c_double, ctypes.c_int, c_i32p, ctypes.c_int, c_dp, c_dp]
    L.oracle_paged_prefill.restype = ctypes.c_int
    L.oracle_attn_bwd.argtypes = [c_u16p, c_u16p, c_u16p, c_u16p] + [ctypes.c_int] * 6 + [
        ctypes.c_double, ctypes.c_int, c_i64p, ctypes.c_int64, c_dp, c_dp, c_dp]
    L.oracle_attn_bwd.restype = ctypes.c_int
    c_u8p = ctypes.POINTER(ctypes.c_uint8)
    L.oracle_e4m3_decode.argtypes = [c_u8p, ctypes.c_int64, c_dp]
    L.oracle_e4m3_decode.restype = None
    L.oracle_attn_fp8.argtypes = [c_u8p, c_u8p, c_u8p] + [ctypes.c_double] * 3 + [ctypes.c_int] * 6 + [
        ctypes.c_double, ctypes.c_int, c_i64p, ctypes.c_int64, c_dp, c_dp]
    L.oracle_attn_fp8.restype = ctypes.c_int
    L.oracle_num_threads.restype = ctypes.c_int
    L.oracle_set_num_threads.argtypes = [ctypes.c_int]
    return L


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = _bind(_build.build())
    return _lib


class OracleError(RuntimeError):
    pass


def _p(a, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def num_threads() -> int:
    return lib().oracle_num_threads()


def set_num_threads(n: int) -> None:
    lib().oracle_set_num_threads(int(n))


def attn(q, k, v, causal: bool, scale: float | None = None, rows=None, _L=None):
    """Exact attention in fp64.

    q [B,Hq,Nq,d], k/v [B,Hkv,Nkv,d] as uint16 bf16 bit arrays.
    rows: optional flat row ids (b*Hq + hq)*Nq + i; default all rows.
    Returns (o [nrows, d] float64, lse [nrows] float64); with rows=None o is
    reshaped to [B,Hq,Nq,d] and lse to [B,Hq,Nq].
    """
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    v = np.ascontiguousarray(v, dtype=np.uint16)
    B, Hq, Nq, d = q.shape
    _, Hkv, Nkv, _ = k.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if rows is None:
        n = B * Hq * Nq
        rp = None
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        n = rows.size
        rp = _p(rows, ctypes.c_int64)
    o = np.zeros((max(n, 1), d), dtype=np.float64)
    lse = np.zeros(max(n, 1), dtype=np.float64)
    err = (_L or lib()).oracle_attn(_p(q, ctypes.c_uint16), _p(k, ctypes.c_uint16), _p(v, ctypes.c_uint16),
                            B, Hq, Hkv, Nq, Nkv, d, float(scale), int(bool(causal)), rp, n,
                            _p(o, ctypes.c_double), _p(lse, ctypes.c_double))
    if err:
        raise OracleError(f"oracle_attn failed with code {err}")
    o, lse = o[:n], lse[:n]
    if rows is None:
        return o.reshape(B, Hq, Nq, d), lse.reshape(B, Hq, Nq)
    return o, lse


def e4m3_decode(codes, _L=None):
    """Values (float64) of OCP E4M3 ("e4m3fn") codes; NaN for S.1111.111."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(codes.shape, dtype=np.float64)
    (_L or lib()).oracle_e4m3_decode(_p(codes, ctypes.c_uint8), codes.size, _p(out, ctypes.c_double))
    return out


def attn_fp8(q, k, v, descale, causal: bool, scale: float | None = None, rows=None, _L=None):
    """Exact attention in fp64 of FP8 inputs.

    q [B,Hq,Nq,d], k/v [B,Hkv,Nkv,d] as uint8 E4M3 codes; descale =
    (q_descale, k_descale, v_descale), the real inputs being q_descale * e4m3(q)
    and so on.  rows and the returned shapes as attn().
    """
    q = np.ascontiguousarray(q, dtype=np.uint8)
    k = np.ascontiguousarray(k, dtype=np.uint8)
    v = np.ascontiguousarray(v, dtype=np.uint8)
    B, Hq, Nq, d = q.shape
    _, Hkv, Nkv, _ = k.shape
    dq, dk, dv = (float(x) for x in descale)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if rows is None:
        n = B * Hq * Nq
        rp = None
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        n = rows.size
        rp = _p(rows, ctypes.c_int64)
    o = np.zeros((max(n, 1), d), dtype=np.float64)
    lse = np.zeros(max(n, 1), dtype=np.float64)
    err = (_L or lib()).oracle_attn_fp8(_p(q, ctypes.c_uint8), _p(k, ctypes.c_uint8), _p(v, ctypes.c_uint8),
                                        dq, dk, dv, B, Hq, Hkv, Nq, Nkv, d, float(scale), int(bool(causal)), rp, n,
                                        _p(o, ctypes.c_double), _p(lse, ctypes.c_double))
    if err:
        raise OracleError(f"oracle_attn_fp8 failed with code {err}")
    o, lse = o[:n], lse[:n]
    if rows is None:
        return o.reshape(B, Hq, Nq, d), lse.reshape(B, Hq, Nq)
    return o, lse


def paged_gather(k_cache, v_cache, block_table, seq_lens, seq: int, hkv: int, _L=None):
    """Explicitly gathered logical K and V rows of (seq, hkv): two [len, d] uint16 arrays."""
    k_cache = np.ascontiguousarray(k_cache, dtype=np.uint16)
    v_cache = np.ascontiguousarray(v_cache, dtype=np.uint16)
    block_table = np.ascontiguousarray(block_table, dtype=np.int32)
    seq_lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    P, Hkv, ps, d = k_cache.shape
    L = int(max(seq_lens[seq], 0))
    ko = np.zeros((max(L, 1), d), dtype=np.uint16)
    vo = np.zeros((max(L, 1), d), dtype=np.uint16)
    err = (_L or lib()).oracle_paged_gather(_p(k_cache, ctypes.c_uint16), _p(v_cache, ctypes.c_uint16),
                                    _p(block_table, ctypes.c_int32), _p(seq_lens, ctypes.c_int32),
                                    int(seq), int(hkv), ps, Hkv, d, block_table.shape[1], P,
                                    _p(ko, ctypes.c_uint16), _p(vo, ctypes.c_uint16))
    if err:
        raise OracleError(f"oracle_paged_gather failed with code {err}")
    return ko[:L], vo[:L]


def paged_decode(q, k_cache, v_cache, block_table, seq_lens, scale: float | None = None, seqs=None,
                 _L=None):
    """Paged decode in fp64: q [S,Hq,d]; caches [P,Hkv,page,d]; returns (o, lse).

    seqs: optional subset of sequence ids; outputs follow that order
    (o [len(seqs),Hq,d], lse [len(seqs),Hq]).
    """
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k_cache = np.ascontiguousarray(k_cache, dtype=np.uint16)
    v_cache = np.ascontiguousarray(v_cache, dtype=np.uint16)
    block_table = np.ascontiguousarray(block_table, dtype=np.int32)
    seq_lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    S, Hq, d = q.shape
    P, Hkv, ps, _ = k_cache.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if seqs is None:
        n, sp = S, None
    else:
        seqs = np.ascontiguousarray(seqs, dtype=np.int32)
        n, sp = seqs.size, _p(seqs, ctypes.c_int32)
    o = np.zeros((max(n, 1), Hq, d), dtype=np.float64)
    lse = np.zeros((max(n, 1), Hq), dtype=np.float64)
    err = (_L or lib()).oracle_paged_decode(_p(q, ctypes.c_uint16), _p(k_cache, ctypes.c_uint16),
                                    _p(v_cache, ctypes.c_uint16), _p(block_table, ctypes.c_int32),
                                    _p(seq_lens, ctypes.c_int32), ps, S, Hq, Hkv, d,
                                    block_table.shape[1], P, float(scale), sp, n,
                                    _p(o, ctypes.c_double), _p(lse, ctypes.c_double))
    if err:
        raise OracleError(f"oracle_paged_decode failed with code {err}")
    return o[:n], lse[:n]


def paged_prefill(q, k_cache, v_cache, block_table, cu_seqlens, seq_lens, causal: bool, scale: float | None = None,
                  seqs=None, _L=None):
    """Varlen prefill against the paged cache in fp64.

    q [total_q, Hq, d] (bf16 bits, sequences packed by cu_seqlens [S+1]);
    caches [P, Hkv, page, d]; block_table [S, max_pages]; seq_lens [S] keys per
    sequence.  Returns o [total_q, Hq, d] and lse [total_q, Hq] (rows of
    sequences outside `seqs` are zero).
    """
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k_cache = np.ascontiguousarray(k_cache, dtype=np.uint16)
    v_cache = np.ascontiguousarray(v_cache, dtype=np.uint16)
    block_table = np.ascontiguousarray(block_table, dtype=np.int32)
    cu_seqlens = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    seq_lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    T, Hq, d = q.shape
    P, Hkv, ps, _ = k_cache.shape
    S = seq_lens.size
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if seqs is None:
        n, sp = S, None
    else:
        seqs = np.ascontiguousarray(seqs, dtype=np.int32)
        n, sp = seqs.size, _p(seqs, ctypes.c_int32)
    o = np.zeros((max(T, 1), Hq, d), dtype=np.float64)
    lse = np.zeros((max(T, 1), Hq), dtype=np.float64)
    err = (_L or lib()).oracle_paged_prefill(_p(q, ctypes.c_uint16), _p(k_cache, ctypes.c_uint16),
                                             _p(v_cache, ctypes.c_uint16), _p(block_table, ctypes.c_int32),
                                             _p(cu_seqlens, ctypes.c_int32), _p(seq_lens, ctypes.c_int32), ps, S, T,
                                             Hq, Hkv, d, block_table.shape[1], P, float(scale), int(bool(causal)), sp,
                                             n, _p(o, ctypes.c_double), _p(lse, ctypes.c_double))
    if err:
        raise OracleError(f"oracle_paged_prefill failed with code {err}")
    return o[:T], lse[:T]


def attn_bwd(q, k, v, dout, causal: bool, scale: float | None = None, groups=None, _L=None):
    """Gradients (dq, dk, dv) of attention in fp64 for the loss gradient dout.

    q, dout [B,Hq,Nq,d]; k, v [B,Hkv,Nkv,d] as uint16 bf16 bit arrays.
    groups: optional flat KV-head ids b*Hkv + hkv to evaluate (with all rows of
    their query heads); gradients of other heads are returned as zeros.
    Returns dq [B,Hq,Nq,d], dk [B,Hkv,Nkv,d], dv [B,Hkv,Nkv,d] as float64.
    """
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    v = np.ascontiguousarray(v, dtype=np.uint16)
    dout = np.ascontiguousarray(dout, dtype=np.uint16)
    B, Hq, Nq, d = q.shape
    _, Hkv, Nkv, _ = k.shape
    if dout.shape != q.shape:
        raise OracleError("dout must have the shape of q")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if groups is None:
        n, gp = B * Hkv, None
    else:
        groups = np.ascontiguousarray(groups, dtype=np.int64)
        n, gp = groups.size, _p(groups, ctypes.c_int64)
    dq = np.zeros((B, Hq, Nq, d), dtype=np.float64)
    dk = np.zeros((B, Hkv, Nkv, d), dtype=np.float64)
    dv = np.zeros((B, Hkv, Nkv, d), dtype=np.float64)
    err = (_L or lib()).oracle_attn_bwd(_p(q, ctypes.c_uint16), _p(k, ctypes.c_uint16), _p(v, ctypes.c_uint16),
                                        _p(dout, ctypes.c_uint16), B, Hq, Hkv, Nq, Nkv, d, float(scale),
                                        int(bool(causal)), gp, n, _p(dq, ctypes.c_double),
                                        _p(dk, ctypes.c_double), _p(dv, ctypes.c_double))
    if err:
        raise OracleError(f"oracle_attn_bwd failed with code {err}")
    return dq, dk, dv


class Variant:
    """The same wrappers bound to another build of oracle.c (used by the
    tests that check the pins catch planted mistakes)."""

    def __init__(self, path):
        self._L = _bind(path)

    def attn(self, *a, **kw):
        return attn(*a, _L=self._L, **kw)

    def paged_gather(self, *a, **kw):
        return paged_gather(*a, _L=self._L, **kw)

    def paged_decode(self, *a, **kw):
        return paged_decode(*a, _L=self._L, **kw)

    def attn_bwd(self, *a, **kw):
        return attn_bwd(*a, _L=self._L, **kw)

    def paged_prefill(self, *a, **kw):
        return paged_prefill(*a, _L=self._L, **kw)

    def e4m3_decode(self, *a, **kw):
        return e4m3_decode(*a, _L=self._L, **kw)

    def attn_fp8(self, *a, **kw):
        return attn_fp8(*a, _L=self._L, **kw)
