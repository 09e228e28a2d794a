"""fp64 CPU oracle for exact attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never loads it and
shares no code with it.

Each function takes CPU tensors (torch bf16, or numpy uint16 bf16 bit
patterns) and returns float64 numpy arrays.  The C source ``oracle.c`` states
the definition it follows ("What attention costs", samanvya.dev: softmax of
scaled scores times V, two-pass; "Flash-Decoding" for the log-sum-exp merge).
"""
from __future__ import annotations

import ctypes
import math

import numpy as np

from .build import build_oracle

_lib = None

_u16p = np.ctypeslib.ndpointer(dtype=np.uint16, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_i64p = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_u8p = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build_oracle())
        L.oracle_set_num_threads.argtypes = [ctypes.c_int]
        L.oracle_max_threads.restype = ctypes.c_int
        L.oracle_attn.argtypes = [_u16p, _u16p, _u16p] + [ctypes.c_int] * 7 + [
            ctypes.c_double, _f64p, _f64p]
        L.oracle_attn.restype = ctypes.c_int
        L.oracle_attn_varlen_rows.argtypes = [
            _u16p, _u16p, _u16p, _i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
            ctypes.c_void_p, ctypes.c_int64, _f64p, _f64p]
        L.oracle_attn_varlen_rows.restype = ctypes.c_int
        L.oracle_probs.argtypes = [
            _u16p, _u16p, _u16p, _i32p] + [ctypes.c_int] * 8 + [ctypes.c_double, _f64p]
        L.oracle_probs.restype = ctypes.c_int
        L.oracle_decode_paged.argtypes = [
            _u16p, _u16p, _u16p, _i32p, _i32p] + [ctypes.c_int] * 6 + [
            ctypes.c_int64, ctypes.c_double, _f64p, _f64p]
        L.oracle_decode_paged.restype = ctypes.c_int
        L.oracle_lse_combine.argtypes = [_f64p, _f64p, ctypes.c_int, ctypes.c_int64,
                                         ctypes.c_int, _f64p, _f64p]
        L.oracle_lse_combine.restype = ctypes.c_int
        L.oracle_attn_varlen_rows_sinks.argtypes = [
            _u16p, _u16p, _u16p, _i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double, _f64p,
            ctypes.c_void_p, ctypes.c_int64, _f64p, _f64p]
        L.oracle_attn_varlen_rows_sinks.restype = ctypes.c_int
        L.oracle_attn_varlen_rows_doc.argtypes = [
            _u16p, _u16p, _u16p, _i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double, _i32p,
            ctypes.c_void_p, ctypes.c_int64, _f64p, _f64p]
        L.oracle_attn_varlen_rows_doc.restype = ctypes.c_int
        L.oracle_decode_paged_sinks.argtypes = [
            _u16p, _u16p, _u16p, _i32p, _i32p] + [ctypes.c_int] * 6 + [
            ctypes.c_int64, ctypes.c_double, _f64p, _f64p, _f64p]
        L.oracle_decode_paged_sinks.restype = ctypes.c_int
        L.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_value.restype = ctypes.c_double
        L.oracle_decode_paged_fp8.argtypes = [
            _u16p, _u8p, _u8p, _f32p, _f32p, _i32p, _i32p] + [ctypes.c_int] * 6 + [
            ctypes.c_int64, ctypes.c_double, ctypes.c_void_p, _f64p, _f64p]
        L.oracle_decode_paged_fp8.restype = ctypes.c_int
        L.oracle_prefill_paged.argtypes = [
            _u16p, _u16p, _u16p, _i32p, _i32p, _i32p] + [ctypes.c_int] * 6 + [
            ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_void_p,
            _f64p, _f64p]
        L.oracle_prefill_paged.restype = ctypes.c_int
        L.oracle_attn_bwd_varlen.argtypes = [
            _u16p, _u16p, _u16p, _u16p, _i32p] + [ctypes.c_int] * 6 + [
            ctypes.c_double, _f64p, _f64p, _f64p]
        L.oracle_attn_bwd_varlen.restype = ctypes.c_int
        L.oracle_attn_bwd_varlen_sinks.argtypes = [
            _u16p, _u16p, _u16p, _u16p, _i32p] + [ctypes.c_int] * 6 + [
            ctypes.c_double, _f64p, _f64p, _f64p, _f64p, _f64p]
        L.oracle_attn_bwd_varlen_sinks.restype = ctypes.c_int
        L.oracle_attn_bwd_dq_rows.argtypes = [
            _u16p, _u16p, _u16p, _u16p, _i32p] + [ctypes.c_int] * 6 + [
            ctypes.c_double, _i64p, ctypes.c_int64, _f64p]
        L.oracle_attn_bwd_dq_rows.restype = ctypes.c_int
        L.oracle_attn_bwd_dkv_rows.argtypes = [
            _u16p, _u16p, _u16p, _u16p, _i32p] + [ctypes.c_int] * 6 + [
            ctypes.c_double, _i64p, ctypes.c_int64, _f64p, _f64p]
        L.oracle_attn_bwd_dkv_rows.restype = ctypes.c_int
        L.oracle_attn_varlen_rows_sink_tokens.argtypes = [
            _u16p, _u16p, _u16p, _i32p] + [ctypes.c_int] * 6 + [
            ctypes.c_double, ctypes.c_void_p, ctypes.c_int64, _f64p, _f64p]
        L.oracle_attn_varlen_rows_sink_tokens.restype = ctypes.c_int
        L.oracle_hadamard_rotate.argtypes = [_u16p, ctypes.c_int64, ctypes.c_int,
                                             ctypes.c_void_p, _f64p]
        L.oracle_hadamard_rotate.restype = ctypes.c_int
        L.oracle_e4m3_encode.argtypes = [ctypes.c_double]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_block_scale.argtypes = [ctypes.c_double]
        L.oracle_e4m3_block_scale.restype = ctypes.c_float
        L.oracle_quantize_e4m3_blocks.argtypes = [_f64p] + [ctypes.c_int] * 5 + [_u8p, _f32p]
        L.oracle_quantize_e4m3_blocks.restype = ctypes.c_int
        L.oracle_attn_fp8.argtypes = [_u8p, _f32p, ctypes.c_int, _u8p, _f32p, ctypes.c_int,
                                      _u8p, _f32p] + [ctypes.c_int] * 7 + [
            ctypes.c_double, ctypes.c_void_p, ctypes.c_int64, _f64p, _f64p]
        L.oracle_attn_fp8.restype = ctypes.c_int
        _lib = L
    return _lib


def _bits(x) -> np.ndarray:
    """bf16 bit patterns (uint16, C-contiguous) of a torch bf16 tensor or array."""
    if isinstance(x, np.ndarray):
        if x.dtype != np.uint16:
            raise TypeError("numpy inputs must be uint16 bf16 bit patterns")
        return np.ascontiguousarray(x)
    import torch
    if x.dtype != torch.bfloat16:
        raise TypeError("torch inputs must be bfloat16")
    return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _i32(x) -> np.ndarray:
    if not isinstance(x, np.ndarray):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(x, dtype=np.int32)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what}: bad arguments (rc={rc})")


def set_num_threads(n: int) -> None:
    lib().oracle_set_num_threads(int(n))


def max_threads() -> int:
    return int(lib().oracle_max_threads())


def attn(q, k, v, causal=False, window=0, scale=None):
    """Dense batch.  q [B,N,Hq,d], k/v [B,N,Hkv,d] -> O [B,N,Hq,d], LSE [B,Hq,N]."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, N, Hq, d = qb.shape
    Hkv = kb.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = np.empty((B, N, Hq, d), np.float64)
    lse = np.empty((B, Hq, N), np.float64)
    _check(lib().oracle_attn(qb, kb, vb, B, Hq, Hkv, N, d, int(causal), int(window),
                             float(scale), o, lse), "attn")
    return o, lse


def attn_varlen(q, k, v, cu_seqlens, causal=False, window=0, scale=None, rows=None):
    """Packed sequences.  q [T,Hq,d], k/v [T,Hkv,d], cu_seqlens [S+1].

    Returns O [T,Hq,d] and LSE [Hq,T]; with ``rows`` (global token indices)
    only those rows: O [R,Hq,d], LSE [R,Hq].
    """
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    T, Hq, d = qb.shape
    Hkv = kb.shape[1]
    cu = _i32(cu_seqlens)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if rows is None:
        nrows, rp = T, None
    else:
        r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        nrows, rp = r.size, r.ctypes.data_as(ctypes.c_void_p)
    o = np.empty((nrows, Hq, d), np.float64)
    lse = np.empty((nrows, Hq), np.float64)
    _check(lib().oracle_attn_varlen_rows(qb, kb, vb, cu, len(cu) - 1, Hq, Hkv, d,
                                         int(causal), int(window), float(scale),
                                         rp, nrows, o, lse), "attn_varlen")
    if rows is None:
        return o, np.ascontiguousarray(lse.T)
    return o, lse


def attn_rows(q, k, v, rows, causal=False, window=0, scale=None):
    """Dense batch, only query tokens ``rows`` = list of (b, i).

    Returns O [R,Hq,d] and LSE [R,Hq].
    """
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, N, Hq, d = qb.shape
    cu = np.arange(B + 1, dtype=np.int32) * N
    flat = [int(b) * N + int(i) for b, i in rows]
    return attn_varlen(qb.reshape(B * N, Hq, d), kb.reshape(B * N, -1, d),
                       vb.reshape(B * N, -1, d), cu, causal, window, scale, rows=flat)


def probs(q, k, v, cu_seqlens, seq, h, causal=False, window=0, scale=None):
    """Softmax probability matrix [L, L] of one (sequence, head)."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    T, Hq, d = qb.shape
    Hkv = kb.shape[1]
    cu = _i32(cu_seqlens)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    L = int(cu[seq + 1] - cu[seq])
    p = np.empty((L, L), np.float64)
    _check(lib().oracle_probs(qb, kb, vb, cu, len(cu) - 1, int(seq), int(h), Hq, Hkv, d,
                              int(causal), int(window), float(scale), p), "probs")
    return p


def decode_paged(q, k_cache, v_cache, block_table, seq_lens, scale=None):
    """q [S,Hq,d], caches [P,ps,Hkv,d] -> O [S,Hq,d], LSE [S,Hq]."""
    qb, kb, vb = _bits(q), _bits(k_cache), _bits(v_cache)
    S, Hq, d = qb.shape
    P, ps, Hkv, _ = kb.shape
    bt = _i32(block_table)
    sl = _i32(seq_lens)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = np.empty((S, Hq, d), np.float64)
    lse = np.empty((S, Hq), np.float64)
    _check(lib().oracle_decode_paged(qb, kb, vb, bt, sl, S, Hq, Hkv, d, ps,
                                     bt.shape[1], P, float(scale), o, lse),
           "decode_paged")
    return o, lse


def lse_combine(o_parts, lse_parts):
    """Merge partials: o_parts [P,R,d], lse_parts [P,R] -> O [R,d], LSE [R]."""
    op = np.ascontiguousarray(o_parts, dtype=np.float64)
    lp = np.ascontiguousarray(lse_parts, dtype=np.float64)
    P, R, d = op.shape
    o = np.empty((R, d), np.float64)
    lse = np.empty((R,), np.float64)
    _check(lib().oracle_lse_combine(op, lp, P, R, d, o, lse), "lse_combine")
    return o, lse


def attn_bwd_varlen(q, k, v, dout, cu_seqlens, causal=False, window=0, scale=None):
    """Gradients of packed attention for upstream dO.  q/dout [T,Hq,d],
    k/v [T,Hkv,d], cu_seqlens [S+1] -> dQ [T,Hq,d], dK [T,Hkv,d], dV [T,Hkv,d]."""
    qb, kb, vb, db = _bits(q), _bits(k), _bits(v), _bits(dout)
    T, Hq, d = qb.shape
    Hkv = kb.shape[1]
    cu = _i32(cu_seqlens)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = np.empty((T, Hq, d), np.float64)
    dk = np.empty((T, Hkv, d), np.float64)
    dv = np.empty((T, Hkv, d), np.float64)
    _check(lib().oracle_attn_bwd_varlen(qb, kb, vb, db, cu, len(cu) - 1, Hq, Hkv, d,
                                        int(causal), int(window), float(scale), dq, dk, dv),
           "attn_bwd_varlen")
    return dq, dk, dv


def attn_bwd(q, k, v, dout, causal=False, window=0, scale=None):
    """Dense batch gradients.  q/dout [B,N,Hq,d], k/v [B,N,Hkv,d]
    -> dQ [B,N,Hq,d], dK [B,N,Hkv,d], dV [B,N,Hkv,d]."""
    qb, kb, vb, db = _bits(q), _bits(k), _bits(v), _bits(dout)
    B, N, Hq, d = qb.shape
    Hkv = kb.shape[2]
    cu = np.arange(B + 1, dtype=np.int32) * N
    dq, dk, dv = attn_bwd_varlen(qb.reshape(B * N, Hq, d), kb.reshape(B * N, Hkv, d),
                                 vb.reshape(B * N, Hkv, d), db.reshape(B * N, Hq, d), cu,
                                 causal, window, scale)
    return (dq.reshape(B, N, Hq, d), dk.reshape(B, N, Hkv, d), dv.reshape(B, N, Hkv, d))


def attn_bwd_dq_rows(q, k, v, dout, cu_seqlens, rows, causal=False, window=0, scale=None):
    """dQ of the packed tokens ``rows`` only (all query heads) -> [R, Hq, d]."""
    qb, kb, vb, db = _bits(q), _bits(k), _bits(v), _bits(dout)
    T, Hq, d = qb.shape
    Hkv = kb.shape[1]
    cu = _i32(cu_seqlens)
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = np.empty((r.size, Hq, d), np.float64)
    _check(lib().oracle_attn_bwd_dq_rows(qb, kb, vb, db, cu, len(cu) - 1, Hq, Hkv, d,
                                         int(causal), int(window), float(scale), r, r.size, dq),
           "attn_bwd_dq_rows")
    return dq


def attn_bwd_dkv_rows(q, k, v, dout, cu_seqlens, rows, causal=False, window=0, scale=None):
    """dK and dV of the packed key tokens ``rows`` only (all KV heads)
    -> ([R, Hkv, d], [R, Hkv, d]): the sums over the query rows that see each
    key, from every row's LSE and D = rowsum(P * dP) taken first."""
    qb, kb, vb, db = _bits(q), _bits(k), _bits(v), _bits(dout)
    T, Hq, d = qb.shape
    Hkv = kb.shape[1]
    cu = _i32(cu_seqlens)
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dk = np.empty((r.size, Hkv, d), np.float64)
    dv = np.empty((r.size, Hkv, d), np.float64)
    _check(lib().oracle_attn_bwd_dkv_rows(qb, kb, vb, db, cu, len(cu) - 1, Hq, Hkv, d,
                                          int(causal), int(window), float(scale), r, r.size,
                                          dk, dv), "attn_bwd_dkv_rows")
    return dk, dv


def attn_varlen_sinks(q, k, v, cu_seqlens, sinks, causal=False, window=0, scale=None, rows=None):
    """attn_varlen with a learned sink logit per query head (``sinks`` [Hq],
    in units of scaled scores): the sink joins each row's softmax denominator
    as one extra key with a zero value.  Returns O and LSE as attn_varlen."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    T, Hq, d = qb.shape
    Hkv = kb.shape[1]
    cu = _i32(cu_seqlens)
    sk = np.ascontiguousarray(np.asarray(sinks, dtype=np.float64).reshape(Hq))
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if rows is None:
        nrows, rp = T, None
    else:
        r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        nrows, rp = r.size, r.ctypes.data_as(ctypes.c_void_p)
    o = np.empty((nrows, Hq, d), np.float64)
    lse = np.empty((nrows, Hq), np.float64)
    _check(lib().oracle_attn_varlen_rows_sinks(qb, kb, vb, cu, len(cu) - 1, Hq, Hkv, d,
                                               int(causal), int(window), float(scale), sk,
                                               rp, nrows, o, lse), "attn_varlen_sinks")
    if rows is None:
        return o, np.ascontiguousarray(lse.T)
    return o, lse


def attn_sinks(q, k, v, sinks, causal=False, window=0, scale=None):
    """Dense batch with sinks -> O [B,N,Hq,d], LSE [B,Hq,N]."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, N, Hq, d = qb.shape
    Hkv = kb.shape[2]
    cu = np.arange(B + 1, dtype=np.int32) * N
    o, lse = attn_varlen_sinks(qb.reshape(B * N, Hq, d), kb.reshape(B * N, Hkv, d),
                               vb.reshape(B * N, Hkv, d), cu, sinks, causal, window, scale)
    return o.reshape(B, N, Hq, d), np.ascontiguousarray(lse.reshape(Hq, B, N).transpose(1, 0, 2))


def decode_paged_sinks(q, k_cache, v_cache, block_table, seq_lens, sinks, scale=None):
    """decode_paged with a learned sink logit per query head."""
    qb, kb, vb = _bits(q), _bits(k_cache), _bits(v_cache)
    S, Hq, d = qb.shape
    P, ps, Hkv, _ = kb.shape
    bt = _i32(block_table)
    sl = _i32(seq_lens)
    sk = np.ascontiguousarray(np.asarray(sinks, dtype=np.float64).reshape(Hq))
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = np.empty((S, Hq, d), np.float64)
    lse = np.empty((S, Hq), np.float64)
    _check(lib().oracle_decode_paged_sinks(qb, kb, vb, bt, sl, S, Hq, Hkv, d, ps,
                                           bt.shape[1], P, float(scale), sk, o, lse),
           "decode_paged_sinks")
    return o, lse


def e4m3_value(code: int) -> float:
    """The real value of one FP8 E4M3 ("fn") code."""
    return float(lib().oracle_e4m3_value(int(code) & 0xFF))


def _u8(x) -> np.ndarray:
    if not isinstance(x, np.ndarray):
        import torch
        x = x.detach().cpu().contiguous()
        if x.dtype != torch.uint8:
            x = x.view(torch.uint8)
        x = x.numpy()
    return np.ascontiguousarray(x, dtype=np.uint8)


def decode_paged_fp8(q, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens, scale=None,
                     sinks=None):
    """Paged decode over an FP8 (E4M3) cache.  k_codes/v_codes [P,ps,Hkv,d] uint8 codes
    (or torch float8_e4m3fn), k_scale/v_scale [P,Hkv] fp32 -> O [S,Hq,d], LSE [S,Hq]."""
    qb = _bits(q)
    kc, vc = _u8(k_codes), _u8(v_codes)
    S, Hq, d = qb.shape
    P, ps, Hkv, _ = kc.shape
    ks = np.ascontiguousarray(np.asarray(k_scale, dtype=np.float32).reshape(P, Hkv))
    vs = np.ascontiguousarray(np.asarray(v_scale, dtype=np.float32).reshape(P, Hkv))
    bt = _i32(block_table)
    sl = _i32(seq_lens)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    sp = None
    if sinks is not None:
        sk = np.ascontiguousarray(np.asarray(sinks, dtype=np.float64).reshape(Hq))
        sp = sk.ctypes.data_as(ctypes.c_void_p)
    o = np.empty((S, Hq, d), np.float64)
    lse = np.empty((S, Hq), np.float64)
    _check(lib().oracle_decode_paged_fp8(qb, kc, vc, ks, vs, bt, sl, S, Hq, Hkv, d, ps,
                                         bt.shape[1], P, float(scale), sp, o, lse),
           "decode_paged_fp8")
    return o, lse


def prefill_paged(q, k_cache, v_cache, block_table, cu_seqlens_q, seq_lens_k, causal=True,
                  window=0, scale=None, sinks=None):
    """Chunked prefill over a paged cache: q [Tq,Hq,d] holds each sequence's
    last L_q tokens; caches [P,ps,Hkv,d]; -> O [Tq,Hq,d], LSE [Hq,Tq]."""
    qb, kb, vb = _bits(q), _bits(k_cache), _bits(v_cache)
    Tq, Hq, d = qb.shape
    P, ps, Hkv, _ = kb.shape
    bt = _i32(block_table)
    cu = _i32(cu_seqlens_q)
    sl = _i32(seq_lens_k)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    sp = None
    if sinks is not None:
        sk = np.ascontiguousarray(np.asarray(sinks, dtype=np.float64).reshape(Hq))
        sp = sk.ctypes.data_as(ctypes.c_void_p)
    o = np.empty((Tq, Hq, d), np.float64)
    lse = np.empty((Tq, Hq), np.float64)
    _check(lib().oracle_prefill_paged(qb, kb, vb, bt, cu, sl, len(cu) - 1, Hq, Hkv, d, ps,
                                      bt.shape[1], P, int(causal), int(window), float(scale),
                                      sp, o, lse), "prefill_paged")
    return o, np.ascontiguousarray(lse.T)


def attn_bwd_sinks(q, k, v, dout, sinks, causal=False, window=0, scale=None):
    """Dense-batch gradients with learned sinks: -> dQ, dK, dV, dsinks [Hq]."""
    qb, kb, vb, db = _bits(q), _bits(k), _bits(v), _bits(dout)
    B, N, Hq, d = qb.shape
    Hkv = kb.shape[2]
    cu = np.arange(B + 1, dtype=np.int32) * N
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    sk = np.ascontiguousarray(np.asarray(sinks, dtype=np.float64).reshape(Hq))
    dq = np.empty((B * N, Hq, d), np.float64)
    dk = np.empty((B * N, Hkv, d), np.float64)
    dv = np.empty((B * N, Hkv, d), np.float64)
    ds = np.empty((Hq,), np.float64)
    _check(lib().oracle_attn_bwd_varlen_sinks(
        qb.reshape(B * N, Hq, d), kb.reshape(B * N, Hkv, d), vb.reshape(B * N, Hkv, d),
        db.reshape(B * N, Hq, d), cu, B, Hq, Hkv, d, int(causal), int(window), float(scale),
        sk, dq, dk, dv, ds), "attn_bwd_sinks")
    return (dq.reshape(B, N, Hq, d), dk.reshape(B, N, Hkv, d), dv.reshape(B, N, Hkv, d), ds)


def attn_doc(q, k, v, doc_ids, causal=False, window=0, scale=None, rows=None):
    """Dense batch with a document mask: doc_ids [B,N] int32; key j is visible
    from query i only if doc_ids[b,i] == doc_ids[b,j].  -> O [B,N,Hq,d], LSE
    [B,Hq,N]; with ``rows`` (list of (b, i)) only those: O [R,Hq,d], LSE [R,Hq]."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, N, Hq, d = qb.shape
    Hkv = kb.shape[2]
    doc = _i32(doc_ids).reshape(B * N)
    cu = np.arange(B + 1, dtype=np.int32) * N
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if rows is None:
        nrows, rp = B * N, None
    else:
        r = np.ascontiguousarray(np.asarray([int(b) * N + int(i) for b, i in rows], dtype=np.int64))
        nrows, rp = r.size, r.ctypes.data_as(ctypes.c_void_p)
    o = np.empty((nrows, Hq, d), np.float64)
    lse = np.empty((nrows, Hq), np.float64)
    _check(lib().oracle_attn_varlen_rows_doc(qb.reshape(B * N, Hq, d), kb.reshape(B * N, Hkv, d),
                                             vb.reshape(B * N, Hkv, d), cu, B, Hq, Hkv, d,
                                             int(causal), int(window), float(scale), doc, rp,
                                             nrows, o, lse), "attn_doc")
    if rows is not None:
        return o, lse
    return o.reshape(B, N, Hq, d), np.ascontiguousarray(lse.reshape(B, N, Hq).transpose(0, 2, 1))


def attn_sink_tokens(q, k, v, window, n_sink, scale=None, rows=None):
    """Dense causal batch with a sliding window of W keys that also keeps the
    first n_sink tokens visible (StreamingLLM's sink tokens).  -> O [B,N,Hq,d],
    LSE [B,Hq,N]; with ``rows`` (list of (b, i)) only those: O [R,Hq,d], LSE [R,Hq]."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, N, Hq, d = qb.shape
    Hkv = kb.shape[2]
    cu = np.arange(B + 1, dtype=np.int32) * N
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if rows is None:
        nrows, rp = B * N, None
    else:
        r = np.ascontiguousarray(np.asarray([int(b) * N + int(i) for b, i in rows], dtype=np.int64))
        nrows, rp = r.size, r.ctypes.data_as(ctypes.c_void_p)
    o = np.empty((nrows, Hq, d), np.float64)
    lse = np.empty((nrows, Hq), np.float64)
    _check(lib().oracle_attn_varlen_rows_sink_tokens(
        qb.reshape(B * N, Hq, d), kb.reshape(B * N, Hkv, d), vb.reshape(B * N, Hkv, d), cu, B,
        Hq, Hkv, d, int(window), int(n_sink), float(scale), rp, nrows, o, lse),
        "attn_sink_tokens")
    if rows is not None:
        return o, lse
    return o.reshape(B, N, Hq, d), np.ascontiguousarray(lse.reshape(B, N, Hq).transpose(0, 2, 1))


def attn_varlen_sink_tokens(q, k, v, cu_seqlens, window, n_sink, scale=None):
    """Packed sequences with a causal window that keeps each sequence's first
    n_sink tokens visible: q [T,Hq,d], k/v [T,Hkv,d] -> O [T,Hq,d], LSE [Hq,T]."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    T, Hq, d = qb.shape
    Hkv = kb.shape[1]
    cu = _i32(cu_seqlens)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = np.empty((T, Hq, d), np.float64)
    lse = np.empty((T, Hq), np.float64)
    _check(lib().oracle_attn_varlen_rows_sink_tokens(qb, kb, vb, cu, cu.size - 1, Hq, Hkv, d,
                                                     int(window), int(n_sink), float(scale),
                                                     None, T, o, lse),
           "attn_varlen_sink_tokens")
    return o, np.ascontiguousarray(lse.T)


# ---------------------------------------------------------------- FP8 prefill
# Incoherent processing ("FlashAttention-3", samanvya.dev "Attention Is the
# Bottleneck"): Q and K rotated by diag(signs) H / sqrt(d) (H Sylvester
# Hadamard), then E4M3 with a power-of-two scale per (batch, head, 128-token
# block); V unrotated with one scale per (batch, KV head).  oracle.c states the
# readings.
FP8_BLOCK = 128


def hadamard_rotate(x, signs=None) -> np.ndarray:
    """x [..., d] bf16 -> fp64 x diag(signs) H / sqrt(d) (signs None: x widened)."""
    xb = _bits(x)
    d = xb.shape[-1]
    rows = xb.size // d
    y = np.empty(xb.shape, np.float64)
    sp = None
    if signs is not None:
        sg = np.ascontiguousarray(np.asarray(signs, dtype=np.float64).reshape(d))
        sp = sg.ctypes.data_as(ctypes.c_void_p)
    _check(lib().oracle_hadamard_rotate(xb, rows, d, sp, y), "hadamard_rotate")
    return y


def e4m3_encode(y: float) -> int:
    """The E4M3 code nearest to y (ties to even, saturating at 448)."""
    return int(lib().oracle_e4m3_encode(float(y)))


def e4m3_block_scale(amax: float) -> float:
    """The scale of a block with largest magnitude amax: the smallest power of
    two 2^k (k >= -126) with amax / 2^k <= 448; 1 for amax = 0."""
    return float(lib().oracle_e4m3_block_scale(float(amax)))


def quantize_e4m3_blocks(x, block):
    """x [B, N, H, d] fp64 -> (codes uint8 [B, N, H, d], scales fp32 [B, H, nblk])."""
    xd = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    B, N, H, d = xd.shape
    nblk = (N + block - 1) // block
    codes = np.empty(xd.shape, np.uint8)
    scales = np.empty((B, H, nblk), np.float32)
    _check(lib().oracle_quantize_e4m3_blocks(xd, B, N, H, d, int(block), codes, scales),
           "quantize_e4m3_blocks")
    return codes, scales


def fp8_prepare(q, k, v, signs=None):
    """The quantised operands of the FP8 prefill: q, k, v [B, N, H, d] bf16 ->
    dict(q8, q_scale [B,Hq,nblk], k8, k_scale [B,Hkv,nblk], v8, v_scale [B,Hkv])."""
    q8, qs = quantize_e4m3_blocks(hadamard_rotate(q, signs), FP8_BLOCK)
    k8, ks = quantize_e4m3_blocks(hadamard_rotate(k, signs), FP8_BLOCK)
    vd = hadamard_rotate(v, None)
    N = vd.shape[1]
    v8, vs = quantize_e4m3_blocks(vd, max(N, 1))
    return {"q8": q8, "q_scale": qs, "k8": k8, "k_scale": ks, "v8": v8,
            "v_scale": np.ascontiguousarray(vs.reshape(vs.shape[0], vs.shape[1]))}


def attn_fp8(q8, q_scale, k8, k_scale, v8, v_scale, causal=False, window=0, scale=None,
             qblock=FP8_BLOCK, kblock=FP8_BLOCK, rows=None):
    """Attention over E4M3 codes [B, N, H, d] and their scales -> O [B,R,Hq,d], LSE [B,Hq,R]
    for the query positions ``rows`` of every batch (default: all N)."""
    q8, k8, v8 = _u8(q8), _u8(k8), _u8(v8)
    B, N, Hq, d = q8.shape
    Hkv = k8.shape[2]
    qs = np.ascontiguousarray(np.asarray(q_scale, dtype=np.float32))
    ks = np.ascontiguousarray(np.asarray(k_scale, dtype=np.float32))
    vs = np.ascontiguousarray(np.asarray(v_scale, dtype=np.float32))
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    rp, R = None, N
    if rows is not None:
        ra = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))
        rp, R = ra.ctypes.data_as(ctypes.c_void_p), ra.size
    o = np.empty((B, R, Hq, d), np.float64)
    lse = np.empty((B, Hq, R), np.float64)
    _check(lib().oracle_attn_fp8(q8, qs, int(qblock), k8, ks, int(kblock), v8, vs, B, N, Hq,
                                 Hkv, d, int(causal), int(window), float(scale), rp, R, o, lse),
           "attn_fp8")
    return o, lse


def fp8_prefill(q, k, v, signs=None, causal=False, window=0, scale=None):
    """The whole FP8 prefill: rotate, quantise, attend.  -> (O, LSE, prepared operands)."""
    prep = fp8_prepare(q, k, v, signs)
    o, lse = attn_fp8(prep["q8"], prep["q_scale"], prep["k8"], prep["k_scale"], prep["v8"],
                      prep["v_scale"], causal, window, scale)
    return o, lse, prep
