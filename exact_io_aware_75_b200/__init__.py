"""Exact IO-aware attention for B200 (sm_100a): Python binding of libfa_sm100.so.

The binding only marshals arguments: it takes torch CUDA tensors, passes their
device pointers, sizes and the current CUDA stream to the C ABI declared in
``include/fa.h``, and raises :class:`FAError` on a non-zero status.  All
arithmetic runs in the library's kernels.  There is no fallback: if the
shared library is missing or fails to load, importing this package raises.

Functions mirror the C entry points:
    fwd            -> fa_fwd            (dense prefill)
    fwd_varlen     -> fa_fwd_varlen     (packed sequences, cu_seqlens)
    bwd            -> fa_bwd            (dense backward: dQ, dK, dV)
    bwd_varlen     -> fa_bwd_varlen     (packed-sequence backward)
    decode_paged   -> fa_decode_paged   (paged split-KV decode)
    fp8_prepare    -> fa_fp8_prepare    (Hadamard rotation + E4M3 operands)
    fwd_fp8        -> fa_fwd_fp8        (FP8 prefill on those operands)
    decode_paged_noalloc, decode_workspace_bytes, bwd_workspace_bytes,
    check_device_error, selftest_watchdog, status_string, version
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa_sm100.so")

FA_OK = 0
FA_ERR_INVALID_ARG = -1
FA_ERR_UNSUPPORTED = -2
FA_ERR_ALIGNMENT = -3
FA_ERR_WORKSPACE = -4
FA_ERR_CUDA = -5
FA_ERR_TIMEOUT = -6
FA_OUT_BF16 = 0
FA_OUT_FP32 = 1

EXPORTS = ("fa_fwd", "fa_fwd_varlen", "fa_fwd_sinks", "fa_fwd_varlen_sinks", "fa_fwd_paged",
           "fa_fwd_doc", "fa_fwd_sink_tokens", "fa_fwd_varlen_sink_tokens",
           "fa_bwd_workspace_bytes", "fa_bwd", "fa_bwd_varlen", "fa_bwd_sinks",
           "fa_bwd_varlen_sinks",
           "fa_decode_workspace_bytes", "fa_decode_paged", "fa_decode_paged_sinks",
           "fa_decode_paged_fp8", "fa_fp8_workspace_bytes", "fa_fp8_prepare", "fa_fwd_fp8",
           "fa_decode_paged_noalloc", "fa_status_string", "fa_check_device_error",
           "fa_selftest_watchdog", "fa_version")


class FAError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} (status {status})")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing; build it with `python exact_io_aware_75_b200/build.py` "
            "(or __graft_entry__.build()).  There is no fallback path.")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp] + [i] * 7 + [f, i, vp]
    lib.fa_fwd.restype = i
    lib.fa_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp] + [i] * 8 + [f, i, vp]
    lib.fa_fwd_varlen.restype = i
    lib.fa_fwd_sinks.argtypes = [vp] * 6 + [i] * 7 + [f, i, vp]
    lib.fa_fwd_sinks.restype = i
    lib.fa_fwd_varlen_sinks.argtypes = [vp] * 7 + [i] * 8 + [f, i, vp]
    lib.fa_fwd_varlen_sinks.restype = i
    lib.fa_decode_paged_sinks.argtypes = [vp] * 8 + [i] * 7 + [f, vp, sz, vp]
    lib.fa_decode_paged_sinks.restype = i
    lib.fa_fwd_sink_tokens.argtypes = [vp] * 5 + [i] * 7 + [f, i, vp]
    lib.fa_fwd_sink_tokens.restype = i
    lib.fa_fwd_varlen_sink_tokens.argtypes = [vp] * 6 + [i] * 8 + [f, i, vp]
    lib.fa_fwd_varlen_sink_tokens.restype = i
    lib.fa_fwd_doc.argtypes = [vp] * 6 + [i] * 7 + [f, i, vp]
    lib.fa_fwd_doc.restype = i
    lib.fa_fwd_paged.argtypes = [vp] * 9 + [i] * 11 + [f, i, vp]
    lib.fa_fwd_paged.restype = i
    lib.fa_decode_paged_fp8.argtypes = [vp] * 10 + [i] * 7 + [f, vp, sz, vp]
    lib.fa_decode_paged_fp8.restype = i
    lib.fa_fp8_workspace_bytes.argtypes = [i] * 3
    lib.fa_fp8_workspace_bytes.restype = sz
    lib.fa_fp8_prepare.argtypes = [vp] * 10 + [i] * 5 + [vp, sz, vp]
    lib.fa_fp8_prepare.restype = i
    lib.fa_fwd_fp8.argtypes = [vp] * 8 + [i] * 7 + [f, i, vp]
    lib.fa_fwd_fp8.restype = i
    lib.fa_bwd_workspace_bytes.argtypes = [i] * 3
    lib.fa_bwd_workspace_bytes.restype = sz
    lib.fa_bwd.argtypes = [vp] * 9 + [i] * 7 + [f, vp, sz, vp]
    lib.fa_bwd.restype = i
    lib.fa_bwd_varlen.argtypes = [vp] * 10 + [i] * 8 + [f, vp, sz, vp]
    lib.fa_bwd_varlen.restype = i
    lib.fa_bwd_sinks.argtypes = [vp] * 11 + [i] * 7 + [f, vp, sz, vp]
    lib.fa_bwd_sinks.restype = i
    lib.fa_bwd_varlen_sinks.argtypes = [vp] * 12 + [i] * 8 + [f, vp, sz, vp]
    lib.fa_bwd_varlen_sinks.restype = i
    lib.fa_decode_workspace_bytes.argtypes = [i] * 5
    lib.fa_decode_workspace_bytes.restype = sz
    lib.fa_decode_paged.argtypes = [vp] * 7 + [i] * 7 + [f, vp, sz, vp]
    lib.fa_decode_paged.restype = i
    lib.fa_decode_paged_noalloc.argtypes = [vp] * 7 + [i] * 7 + [f, vp]
    lib.fa_decode_paged_noalloc.restype = i
    lib.fa_status_string.argtypes = [i]
    lib.fa_status_string.restype = ctypes.c_char_p
    lib.fa_check_device_error.argtypes = [vp]
    lib.fa_check_device_error.restype = i
    lib.fa_selftest_watchdog.argtypes = [vp]
    lib.fa_selftest_watchdog.restype = i
    lib.fa_version.argtypes = []
    lib.fa_version.restype = i
    return lib


_lib = _load()


def library():
    """The loaded ctypes handle (for tests that call the C ABI directly)."""
    return _lib


def status_string(status: int) -> str:
    return _lib.fa_status_string(int(status)).decode()


def version() -> int:
    return int(_lib.fa_version())


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(rc: int, where: str):
    if rc != FA_OK:
        raise FAError(rc, where)


def _need(t, dtype, ndim, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise FAError(FA_ERR_INVALID_ARG, f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise FAError(FA_ERR_INVALID_ARG, f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise FAError(FA_ERR_INVALID_ARG, f"{name} must have {ndim} dims, got {t.dim()}")
    if not t.is_contiguous():
        raise FAError(FA_ERR_INVALID_ARG, f"{name} must be contiguous")


def fwd(q, k, v, causal=False, window=0, scale=None, out_dtype=torch.bfloat16,
        out=None, lse=None, return_lse=True, stream=None, sinks=None, doc_ids=None,
        sink_tokens=None):
    """Dense prefill.  q [B,N,Hq,d], k/v [B,N,Hkv,d] bf16 -> (O [B,N,Hq,d], LSE [B,Hq,N]).
    ``sinks`` (fp32 [Hq], device) selects fa_fwd_sinks; ``doc_ids`` (int32 [B,N],
    device) selects fa_fwd_doc; ``sink_tokens`` (an int, with causal and a window)
    selects fa_fwd_sink_tokens."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, 4, n)
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    if tuple(k.shape) != (B, N, Hkv, d) or tuple(v.shape) != (B, N, Hkv, d):
        raise FAError(FA_ERR_INVALID_ARG, "k/v shape")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, N, Hq, d), dtype=out_dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    od = FA_OUT_FP32 if out.dtype == torch.float32 else FA_OUT_BF16
    if sink_tokens is not None:
        if sinks is not None or doc_ids is not None or not causal:
            raise FAError(FA_ERR_UNSUPPORTED, "sink_tokens with sinks, doc_ids or non-causal")
        _check(_lib.fa_fwd_sink_tokens(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq,
                                       Hkv, N, d, int(window), int(sink_tokens), float(scale),
                                       od, _stream(stream)), "fa_fwd_sink_tokens")
        return out, lse
    if doc_ids is not None:
        if sinks is not None:
            raise FAError(FA_ERR_UNSUPPORTED, "sinks with doc_ids")
        _need(doc_ids, torch.int32, 2, "doc_ids")
        if tuple(doc_ids.shape) != (B, N):
            raise FAError(FA_ERR_INVALID_ARG, "doc_ids shape")
        _check(_lib.fa_fwd_doc(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(doc_ids),
                               B, Hq, Hkv, N, d, int(causal), int(window), float(scale), od,
                               _stream(stream)), "fa_fwd_doc")
        return out, lse
    if sinks is not None:
        _need(sinks, torch.float32, 1, "sinks")
        _check(_lib.fa_fwd_sinks(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(sinks),
                                 B, Hq, Hkv, N, d, int(causal), int(window), float(scale), od,
                                 _stream(stream)), "fa_fwd_sinks")
        return out, lse
    _check(_lib.fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, N, d,
                       int(causal), int(window), float(scale), od, _stream(stream)), "fa_fwd")
    return out, lse


FP8_BLOCK = 128   # tokens per Q / K scale block


def fp8_workspace_bytes(B, N, Hkv) -> int:
    return int(_lib.fa_fp8_workspace_bytes(int(B), int(N), int(Hkv)))


def fp8_prepare(q, k, v, signs=None, out=None, workspace=None, stream=None):
    """E4M3 operands of the FP8 prefill.  q [B,N,Hq,128], k/v [B,N,Hkv,128] bf16;
    signs fp32 [128] of +-1 (device) or None (no rotation).  Returns a dict with
    q8 [B,N,Hq,128], k8 [B,N,Hkv,128] uint8 codes, vt8 [B,Hkv,128,vt_stride]
    uint8 (V transposed), q_scale [B,Hq,nblk], k_scale [B,Hkv,nblk], v_scale
    [B,Hkv] fp32.  ``out`` may be such a dict to fill in place."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, 4, n)
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    if tuple(k.shape) != (B, N, Hkv, d) or tuple(v.shape) != (B, N, Hkv, d):
        raise FAError(FA_ERR_INVALID_ARG, "k/v shape")
    if signs is not None:
        _need(signs, torch.float32, 1, "signs")
        if signs.numel() != d:
            raise FAError(FA_ERR_INVALID_ARG, "signs shape")
    nblk = (N + FP8_BLOCK - 1) // FP8_BLOCK
    vts = (N + 15) // 16 * 16
    dev = q.device
    if out is None:
        out = {"q8": torch.empty((B, N, Hq, d), dtype=torch.uint8, device=dev),
               "k8": torch.empty((B, N, Hkv, d), dtype=torch.uint8, device=dev),
               "vt8": torch.empty((B, Hkv, d, vts), dtype=torch.uint8, device=dev),
               "q_scale": torch.empty((B, Hq, nblk), dtype=torch.float32, device=dev),
               "k_scale": torch.empty((B, Hkv, nblk), dtype=torch.float32, device=dev),
               "v_scale": torch.empty((B, Hkv), dtype=torch.float32, device=dev)}
    ws_need = fp8_workspace_bytes(B, N, Hkv)
    if workspace is None:
        workspace = torch.empty(max(ws_need, 4), dtype=torch.uint8, device=dev)
    _check(_lib.fa_fp8_prepare(_ptr(q), _ptr(k), _ptr(v), _ptr(signs), _ptr(out["q8"]),
                               _ptr(out["k8"]), _ptr(out["vt8"]), _ptr(out["q_scale"]),
                               _ptr(out["k_scale"]), _ptr(out["v_scale"]), B, N, Hq, Hkv, d,
                               _ptr(workspace), workspace.numel() * workspace.element_size(),
                               _stream(stream)), "fa_fp8_prepare")
    return out


def fwd_fp8(prep, causal=False, window=0, scale=None, out_dtype=torch.bfloat16, out=None,
            lse=None, return_lse=True, stream=None):
    """FP8 prefill on fp8_prepare's operands -> (O [B,N,Hq,128], LSE [B,Hq,N])."""
    q8, k8, vt8 = prep["q8"], prep["k8"], prep["vt8"]
    _need(q8, torch.uint8, 4, "q8")
    _need(k8, torch.uint8, 4, "k8")
    _need(vt8, torch.uint8, 4, "vt8")
    B, N, Hq, d = q8.shape
    Hkv = k8.shape[2]
    if tuple(k8.shape) != (B, N, Hkv, d) or tuple(vt8.shape) != (B, Hkv, d, (N + 15) // 16 * 16):
        raise FAError(FA_ERR_INVALID_ARG, "k8/vt8 shape")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, N, Hq, d), dtype=out_dtype, device=q8.device)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q8.device)
    od = FA_OUT_FP32 if out.dtype == torch.float32 else FA_OUT_BF16
    _check(_lib.fa_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(vt8), _ptr(prep["q_scale"]),
                           _ptr(prep["k_scale"]), _ptr(prep["v_scale"]), _ptr(out), _ptr(lse),
                           B, Hq, Hkv, N, d, int(causal), int(window), float(scale), od,
                           _stream(stream)), "fa_fwd_fp8")
    return out, lse


def fwd_varlen(q, k, v, cu_seqlens, max_seqlen, causal=False, window=0, scale=None,
               out_dtype=torch.bfloat16, out=None, lse=None, return_lse=True, stream=None,
               sinks=None, sink_tokens=None):
    """Packed prefill.  q [T,Hq,d], k/v [T,Hkv,d], cu_seqlens [S+1] int32 (device)
    -> (O [T,Hq,d], LSE [Hq,T]).  ``sinks`` selects fa_fwd_varlen_sinks;
    ``sink_tokens`` (an int, with causal and a window) fa_fwd_varlen_sink_tokens."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, 3, n)
    _need(cu_seqlens, torch.int32, 1, "cu_seqlens")
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((T, Hq, d), dtype=out_dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((Hq, T), dtype=torch.float32, device=q.device)
    od = FA_OUT_FP32 if out.dtype == torch.float32 else FA_OUT_BF16
    if sink_tokens is not None:
        if sinks is not None or not causal:
            raise FAError(FA_ERR_UNSUPPORTED, "sink_tokens with sinks or non-causal")
        _check(_lib.fa_fwd_varlen_sink_tokens(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                              _ptr(cu_seqlens), cu_seqlens.numel() - 1, T,
                                              int(max_seqlen), Hq, Hkv, d, int(window),
                                              int(sink_tokens), float(scale), od,
                                              _stream(stream)), "fa_fwd_varlen_sink_tokens")
        return out, lse
    if sinks is not None:
        _need(sinks, torch.float32, 1, "sinks")
        _check(_lib.fa_fwd_varlen_sinks(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                        _ptr(sinks), _ptr(cu_seqlens), cu_seqlens.numel() - 1,
                                        T, int(max_seqlen), Hq, Hkv, d, int(causal),
                                        int(window), float(scale), od, _stream(stream)),
               "fa_fwd_varlen_sinks")
        return out, lse
    _check(_lib.fa_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                              _ptr(cu_seqlens), cu_seqlens.numel() - 1, T, int(max_seqlen),
                              Hq, Hkv, d, int(causal), int(window), float(scale), od,
                              _stream(stream)), "fa_fwd_varlen")
    return out, lse


def fwd_paged(q, k_cache, v_cache, block_table, cu_seqlens_q, seq_lens_k, max_seqlen_q,
              causal=True, window=0, scale=None, sinks=None, out_dtype=torch.bfloat16, out=None,
              lse=None, return_lse=True, stream=None):
    """Chunked prefill over a paged cache.  q [Tq,Hq,d] (each sequence's last L_q
    tokens), caches [P,16,Hkv,d], block_table [S,maxp], cu_seqlens_q [S+1],
    seq_lens_k [S] -> (O [Tq,Hq,d], LSE [Hq,Tq])."""
    _need(q, torch.bfloat16, 3, "q")
    _need(k_cache, torch.bfloat16, 4, "k_cache")
    _need(v_cache, torch.bfloat16, 4, "v_cache")
    _need(block_table, torch.int32, 2, "block_table")
    _need(cu_seqlens_q, torch.int32, 1, "cu_seqlens_q")
    _need(seq_lens_k, torch.int32, 1, "seq_lens_k")
    T, Hq, d = q.shape
    P, ps, Hkv, _ = k_cache.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((T, Hq, d), dtype=out_dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((Hq, T), dtype=torch.float32, device=q.device)
    if sinks is not None:
        _need(sinks, torch.float32, 1, "sinks")
    od = FA_OUT_FP32 if out.dtype == torch.float32 else FA_OUT_BF16
    _check(_lib.fa_fwd_paged(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                             _ptr(cu_seqlens_q), _ptr(seq_lens_k), _ptr(out), _ptr(lse),
                             _ptr(sinks), cu_seqlens_q.numel() - 1, T, int(max_seqlen_q), P,
                             Hq, Hkv, d, ps, block_table.shape[1], int(causal), int(window),
                             float(scale), od, _stream(stream)), "fa_fwd_paged")
    return out, lse


def bwd_workspace_bytes(total_tokens, Hq, d) -> int:
    return int(_lib.fa_bwd_workspace_bytes(int(total_tokens), int(Hq), int(d)))


def bwd(q, k, v, o, dout, lse, causal=False, window=0, scale=None, dq=None, dk=None, dv=None,
        workspace=None, stream=None, sinks=None, dsinks=None):
    """Dense backward.  q/o/dout [B,N,Hq,d], k/v [B,N,Hkv,d] bf16, lse [B,Hq,N] fp32
    (from fwd) -> (dQ, dK, dV) bf16; with ``sinks`` (the forward's sink logits,
    fp32 [Hq]) fa_bwd_sinks, returning (dQ, dK, dV, dsinks)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _need(t, torch.bfloat16, 4, n)
    _need(lse, torch.float32, 3, "lse")
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    if (tuple(k.shape) != (B, N, Hkv, d) or tuple(v.shape) != (B, N, Hkv, d)
            or tuple(o.shape) != (B, N, Hq, d) or tuple(dout.shape) != (B, N, Hq, d)
            or tuple(lse.shape) != (B, Hq, N)):
        raise FAError(FA_ERR_INVALID_ARG, "bwd shapes")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if workspace is None:
        workspace = torch.empty(max(bwd_workspace_bytes(B * N, Hq, d), 1), dtype=torch.uint8,
                                device=q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if sinks is not None:
        _need(sinks, torch.float32, 1, "sinks")
        if dsinks is None:
            dsinks = torch.empty((Hq,), dtype=torch.float32, device=q.device)
        _check(_lib.fa_bwd_sinks(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse),
                                 _ptr(sinks), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dsinks), B, Hq,
                                 Hkv, N, d, int(causal), int(window), float(scale),
                                 _ptr(workspace), workspace.numel(), _stream(stream)),
               "fa_bwd_sinks")
        return dq, dk, dv, dsinks
    _check(_lib.fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq),
                       _ptr(dk), _ptr(dv), B, Hq, Hkv, N, d, int(causal), int(window),
                       float(scale), _ptr(workspace), workspace.numel(), _stream(stream)),
           "fa_bwd")
    return dq, dk, dv


def bwd_varlen(q, k, v, o, dout, lse, cu_seqlens, max_seqlen, causal=False, window=0,
               scale=None, dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Packed backward.  q/o/dout [T,Hq,d], k/v [T,Hkv,d], lse [Hq,T], cu_seqlens [S+1]
    -> (dQ, dK, dV) bf16."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _need(t, torch.bfloat16, 3, n)
    _need(lse, torch.float32, 2, "lse")
    _need(cu_seqlens, torch.int32, 1, "cu_seqlens")
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if workspace is None:
        workspace = torch.empty(max(bwd_workspace_bytes(T, Hq, d), 1), dtype=torch.uint8,
                                device=q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check(_lib.fa_bwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse),
                              _ptr(dq), _ptr(dk), _ptr(dv), _ptr(cu_seqlens),
                              cu_seqlens.numel() - 1, T, int(max_seqlen), Hq, Hkv, d,
                              int(causal), int(window), float(scale), _ptr(workspace),
                              workspace.numel(), _stream(stream)), "fa_bwd_varlen")
    return dq, dk, dv


def decode_workspace_bytes(num_seqs, Hq, d, page_size, max_pages_per_seq) -> int:
    return int(_lib.fa_decode_workspace_bytes(int(num_seqs), int(Hq), int(d), int(page_size),
                                              int(max_pages_per_seq)))


def decode_paged(q, k_cache, v_cache, block_table, seq_lens, scale=None, out=None, lse=None,
                 return_lse=True, workspace=None, stream=None, sinks=None):
    """Paged decode.  q [S,Hq,d], caches [P,ps,Hkv,d], block_table [S,maxp] int32,
    seq_lens [S] int32 -> (O [S,Hq,d] bf16, LSE [S,Hq])."""
    _need(q, torch.bfloat16, 3, "q")
    _need(k_cache, torch.bfloat16, 4, "k_cache")
    _need(v_cache, torch.bfloat16, 4, "v_cache")
    _need(block_table, torch.int32, 2, "block_table")
    _need(seq_lens, torch.int32, 1, "seq_lens")
    S, Hq, d = q.shape
    P, ps, Hkv, _ = k_cache.shape
    maxp = block_table.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = decode_workspace_bytes(S, Hq, d, ps, maxp)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty((S, Hq, d), dtype=torch.bfloat16, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((S, Hq), dtype=torch.float32, device=q.device)
    if sinks is not None:
        _need(sinks, torch.float32, 1, "sinks")
        _check(_lib.fa_decode_paged_sinks(_ptr(q), _ptr(k_cache), _ptr(v_cache),
                                          _ptr(block_table), _ptr(seq_lens), _ptr(out),
                                          _ptr(lse), _ptr(sinks), S, P, Hq, Hkv, d, ps, maxp,
                                          float(scale), _ptr(workspace),
                                          workspace.numel() * workspace.element_size(),
                                          _stream(stream)), "fa_decode_paged_sinks")
        return out, lse
    _check(_lib.fa_decode_paged(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                _ptr(seq_lens), _ptr(out), _ptr(lse), S, P, Hq, Hkv, d, ps,
                                maxp, float(scale), _ptr(workspace),
                                workspace.numel() * workspace.element_size(),
                                _stream(stream)), "fa_decode_paged")
    return out, lse


def decode_paged_fp8(q, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens, scale=None,
                     sinks=None, out=None, lse=None, return_lse=True, workspace=None,
                     stream=None):
    """Paged decode over an FP8 E4M3 cache.  k_codes/v_codes [P,ps,Hkv,d] uint8 (or
    float8_e4m3fn), k_scale/v_scale [P,Hkv] fp32 -> (O [S,Hq,d] bf16, LSE [S,Hq])."""
    _need(q, torch.bfloat16, 3, "q")
    if k_codes.dtype == torch.float8_e4m3fn:
        k_codes, v_codes = k_codes.view(torch.uint8), v_codes.view(torch.uint8)
    _need(k_codes, torch.uint8, 4, "k_codes")
    _need(v_codes, torch.uint8, 4, "v_codes")
    _need(k_scale, torch.float32, 2, "k_scale")
    _need(v_scale, torch.float32, 2, "v_scale")
    _need(block_table, torch.int32, 2, "block_table")
    _need(seq_lens, torch.int32, 1, "seq_lens")
    S, Hq, d = q.shape
    P, ps, Hkv, _ = k_codes.shape
    maxp = block_table.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = decode_workspace_bytes(S, Hq, d, ps, maxp)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty((S, Hq, d), dtype=torch.bfloat16, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((S, Hq), dtype=torch.float32, device=q.device)
    if sinks is not None:
        _need(sinks, torch.float32, 1, "sinks")
    _check(_lib.fa_decode_paged_fp8(_ptr(q), _ptr(k_codes), _ptr(v_codes), _ptr(k_scale),
                                    _ptr(v_scale), _ptr(block_table), _ptr(seq_lens), _ptr(out),
                                    _ptr(lse), _ptr(sinks), S, P, Hq, Hkv, d, ps, maxp,
                                    float(scale), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(),
                                    _stream(stream)), "fa_decode_paged_fp8")
    return out, lse


def decode_paged_noalloc(q, k_cache, v_cache, block_table, seq_lens, scale=None, out=None,
                         lse=None, return_lse=True, stream=None):
    """Paged decode with the library's fixed device scratch instead of a
    workspace, for callers that cannot allocate device memory (see
    fa_decode_paged_noalloc in include/fa.h: 32 MiB limit, first call per
    device before any stream capture, overlapping calls race)."""
    _need(q, torch.bfloat16, 3, "q")
    _need(k_cache, torch.bfloat16, 4, "k_cache")
    _need(v_cache, torch.bfloat16, 4, "v_cache")
    _need(block_table, torch.int32, 2, "block_table")
    _need(seq_lens, torch.int32, 1, "seq_lens")
    S, Hq, d = q.shape
    P, ps, Hkv, _ = k_cache.shape
    maxp = block_table.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((S, Hq, d), dtype=torch.bfloat16, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((S, Hq), dtype=torch.float32, device=q.device)
    _check(_lib.fa_decode_paged_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache),
                                        _ptr(block_table), _ptr(seq_lens), _ptr(out),
                                        _ptr(lse), S, P, Hq, Hkv, d, ps, maxp, float(scale),
                                        _stream(stream)), "fa_decode_paged_noalloc")
    return out, lse


def selftest_watchdog(stream=None) -> int:
    """Launch the watchdog diagnostic (a wait that must time out); read the
    result with check_device_error()."""
    return int(_lib.fa_selftest_watchdog(_stream(stream)))


def check_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error status."""
    return int(_lib.fa_check_device_error(_stream(stream)))
