"""ctypes binding of libsas.so (C ABI in include/sas.h).

Argument marshalling only: shapes are read off torch tensors, outputs and
workspaces are allocated with torch on the input's device, and every call
goes straight to the library on torch's current CUDA stream. There is no
fallback: if libsas.so is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsas.so")

SAS_OK, SAS_ERR_INVALID_ARG, SAS_ERR_UNSUPPORTED, SAS_ERR_CUDA, SAS_ERR_TIMEOUT = 0, 1, 2, 3, 4
SAS_F32, SAS_BF16 = 0, 1

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_Z = ctypes.c_size_t

# name -> (restype, argtypes); must match include/sas.h
SIGNATURES = {
    "sas_last_error": (ctypes.c_char_p, []),
    "sas_kernel_launches": (ctypes.c_uint64, []),
    "sas_get_error_flag": (_I, [_P]),
    "sas_select": (_I, [_P, _I, _I, _I, _I, _P, _I, _I, _P, _P, _P, _P, _P]),
    "sas_select_varlen": (_I, [_P, _I, _I, _I, _I, _P, _I, _I, _P, _P, _P, _P, _P]),
    "sas_attn_fwd": (_I, [_I, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _F, _P, _P, _P]),
    "sas_attn_fwd_varlen": (_I, [_I, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _F, _P, _P, _P]),
    "sas_attn_bwd_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I, _I]),
    "sas_attn_bwd_varlen_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I, _I, _I]),
    "sas_attn_bwd": (_I, [_I, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P,
                          _I, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _P, _P, _Z, _P]),
    "sas_attn_bwd_varlen": (_I, [_I, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P,
                                 _I, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _P, _P, _Z, _P]),
    "sas_score_select_workspace_size": (_Z, [_I, _I, _I, _I, _I]),
    "sas_score_select": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _I, _P, _P, _P, _P, _P, _Z, _P]),
    "sas_pool_pages": (_I, [_P, _I, _I, _I, _I, _P, _I, _P, _P]),
    "sas_score_select_decode": (_I, [_P, _P, _I, _P, _I, _P, _I, _I, _I, _I, _I, _P, _I, _I, _P, _I,
                                     _P, _P, _P, _P, _P]),
    "sas_decode_workspace_size": (_Z, [_I, _I, _I, _I, _I]),
    "sas_decode_paged": (_I, [_P, _P, _P, _I, _P, _I, _P, _I, _I, _I, _I, _I, _I,
                              _P, _P, _P, _F, _P, _P, _P, _Z, _P]),
    "sas_decode_paged_noalloc": (_I, [_P, _P, _P, _I, _P, _I, _P, _I, _I, _I, _I, _I, _I,
                                      _P, _P, _P, _F, _P, _P, _P]),
    "sas_selftest_bounded_wait": (_I, [_P]),
}


class SasError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"libsas status {code}: {msg}")
        self.code = code


_lib = None


def lib() -> ctypes.CDLL:
    """Load libsas.so once; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m trainable_gated_block_b200.build`")
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(h, name)
            fn.restype = res
            fn.argtypes = args
        _lib = h
    return _lib


def _check(code: int):
    if code != SAS_OK:
        raise SasError(code, lib().sas_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return SAS_BF16
    if t.dtype == torch.float32:
        return SAS_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def kernel_launches() -> int:
    """Kernels libsas.so has enqueued in this process so far."""
    return int(lib().sas_kernel_launches())


def get_error_flag(stream=None):
    """Synchronise the stream and raise if a kernel flagged bad data or a timeout."""
    _check(lib().sas_get_error_flag(_stream(stream)))


def selftest_bounded_wait(stream=None):
    """Enqueue the library's bounded-wait fault injection: a kernel whose wait can never
    complete gives up after its budget (about 2 s) and the next get_error_flag raises
    SasError with SAS_ERR_TIMEOUT."""
    _check(lib().sas_selftest_bounded_wait(_stream(stream)))


def select(s, K: int, kv_len=None, block_size: int = 64):
    """Top-K + log-gates. Prefill: s [B,Hkv,NQB,ld]. Decode: s [N,Hkv,ld], kv_len [N].

    Returns idx, cnt, log_gate, lse_s shaped [B,Hkv,R,K], [B,Hkv,R], [B,Hkv,R,K],
    [B,Hkv,R] (decode: R dimension dropped).
    """
    decode = kv_len is not None
    s4 = s[:, :, None, :] if decode else s
    _contig(s4, kv_len)
    B, H, R, ld = s4.shape
    dev = s.device
    idx = torch.empty((B, H, R, K), dtype=torch.int32, device=dev)
    cnt = torch.empty((B, H, R), dtype=torch.int32, device=dev)
    lg = torch.empty((B, H, R, K), dtype=torch.float32, device=dev)
    lse_s = torch.empty((B, H, R), dtype=torch.float32, device=dev)
    _check(lib().sas_select(_ptr(s4), B, H, R, ld, _ptr(kv_len), block_size, K,
                            _ptr(idx), _ptr(cnt), _ptr(lg), _ptr(lse_s), _stream()))
    if decode:
        return idx[:, :, 0], cnt[:, :, 0], lg[:, :, 0], lse_s[:, :, 0]
    return idx, cnt, lg, lse_s


def select_varlen(s, K: int, cu_seqlens, block_size: int = 64):
    """Top-K + log-gates for a packed batch: s [B,Hkv,R,ld] (R >= blocks of the longest
    sequence), cu_seqlens int32 [B+1] on the device. Padding rows come back empty."""
    _contig(s, cu_seqlens)
    B, H, R, ld = s.shape
    dev = s.device
    idx = torch.empty((B, H, R, K), dtype=torch.int32, device=dev)
    cnt = torch.empty((B, H, R), dtype=torch.int32, device=dev)
    lg = torch.empty((B, H, R, K), dtype=torch.float32, device=dev)
    lse_s = torch.empty((B, H, R), dtype=torch.float32, device=dev)
    _check(lib().sas_select_varlen(_ptr(s), B, H, R, ld, _ptr(cu_seqlens), block_size, K,
                                   _ptr(idx), _ptr(cnt), _ptr(lg), _ptr(lse_s), _stream()))
    return idx, cnt, lg, lse_s


def score_select(q, k, K: int, noise=None, block_size: int = 64, workspace=None, s_out=None):
    """Stand-in selector scores (block-pooled q . k / sqrt(D) + noise), then Top-K and
    log-gates, in one call. q [B,S,Hq,D], k [B,S,Hkv,D] bf16; noise [B,Hkv,NQB,ld] fp32 or None.
    Returns s [B,Hkv,NQB,NQB] (entries j >= i are whatever s_out held, zero when it is
    allocated here), idx, cnt, log_gate, lse_s."""
    _contig(q, k, noise)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    NQB = S // block_size
    dev = q.device
    if s_out is None:
        s_out = torch.zeros((B, Hkv, NQB, NQB), dtype=torch.float32, device=dev)
    need = int(lib().sas_score_select_workspace_size(B, S, Hq, Hkv, D))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    idx = torch.empty((B, Hkv, NQB, K), dtype=torch.int32, device=dev)
    cnt = torch.empty((B, Hkv, NQB), dtype=torch.int32, device=dev)
    lg = torch.empty((B, Hkv, NQB, K), dtype=torch.float32, device=dev)
    lse_s = torch.empty((B, Hkv, NQB), dtype=torch.float32, device=dev)
    ld_noise = 0 if noise is None else noise.shape[-1]
    _check(lib().sas_score_select(_ptr(q), _ptr(k), _ptr(noise), ld_noise, B, S, Hq, Hkv, D, block_size, K,
                                  _ptr(s_out), s_out.shape[-1], _ptr(idx), _ptr(cnt), _ptr(lg), _ptr(lse_s),
                                  _ptr(workspace), workspace.numel(), _stream()))
    return s_out, idx, cnt, lg, lse_s


def attn_fwd(q, k, v, idx, cnt, log_gate, sm_scale=None, block_size: int = 64):
    """Gated block-sparse causal attention forward. Returns o [B,S,Hq,D], lse [B,Hq,S]."""
    _contig(q, k, v, idx, cnt, log_gate)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    K = idx.shape[-1]
    sm_scale = 1.0 / math.sqrt(D) if sm_scale is None else sm_scale
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, S), dtype=torch.float32, device=q.device)
    _check(lib().sas_attn_fwd(_dtype_code(q), _ptr(q), _ptr(k), _ptr(v), B, S, Hq, Hkv, D, block_size, K,
                              _ptr(idx), _ptr(cnt), _ptr(log_gate), sm_scale, _ptr(o), _ptr(lse), _stream()))
    return o, lse


def attn_fwd_varlen(q, k, v, cu_seqlens, max_seqlen: int, idx, cnt, log_gate, sm_scale=None,
                    block_size: int = 64):
    """Forward for a packed batch: q [T,Hq,D], k/v [T,Hkv,D]. Returns o [T,Hq,D] and
    lse [B,Hq,max_seqlen] (entries past a sequence's end are left unwritten)."""
    _contig(q, k, v, cu_seqlens, idx, cnt, log_gate)
    T, Hq, D = q.shape
    Hkv = k.shape[1]
    B = cu_seqlens.shape[0] - 1
    K = idx.shape[-1]
    sm_scale = 1.0 / math.sqrt(D) if sm_scale is None else sm_scale
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, max_seqlen), dtype=torch.float32, device=q.device)
    _check(lib().sas_attn_fwd_varlen(_dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), B, max_seqlen,
                                     T, Hq, Hkv, D, block_size, K, _ptr(idx), _ptr(cnt), _ptr(log_gate),
                                     sm_scale, _ptr(o), _ptr(lse), _stream()))
    return o, lse


def bwd_workspace_bytes(q, k, K: int) -> int:
    B, S, Hq, D = q.shape
    return int(lib().sas_attn_bwd_workspace_size(_dtype_code(q), B, S, Hq, k.shape[2], D, K))


def attn_bwd(q, k, v, o, do, lse, s, lse_s, idx, cnt, log_gate, sm_scale=None, block_size: int = 64,
             workspace=None):
    """Backward. Returns dq, dk, dv (input dtype) and ds fp32 [B,Hkv,NQB,ld_s]."""
    _contig(q, k, v, o, do, lse, s, lse_s, idx, cnt, log_gate)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    K = idx.shape[-1]
    ld_s = s.shape[-1]
    sm_scale = 1.0 / math.sqrt(D) if sm_scale is None else sm_scale
    need = bwd_workspace_bytes(q, k, K)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    ds = torch.empty(s.shape, dtype=torch.float32, device=q.device)
    _check(lib().sas_attn_bwd(_dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse),
                              _ptr(s), ld_s, _ptr(lse_s), _ptr(idx), _ptr(cnt), _ptr(log_gate),
                              B, S, Hq, Hkv, D, block_size, K, sm_scale,
                              _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ds), _ptr(workspace), workspace.numel(),
                              _stream()))
    return dq, dk, dv, ds


def attn_bwd_varlen(q, k, v, o, do, lse, s, lse_s, idx, cnt, log_gate, cu_seqlens, max_seqlen: int,
                    sm_scale=None, block_size: int = 64, workspace=None):
    """Backward for a packed batch. Returns dq [T,Hq,D], dk, dv [T,Hkv,D] (rows of no
    sequence left unwritten) and ds fp32 shaped like s (padding rows zero)."""
    _contig(q, k, v, o, do, lse, s, lse_s, idx, cnt, log_gate, cu_seqlens)
    T, Hq, D = q.shape
    Hkv = k.shape[1]
    B = cu_seqlens.shape[0] - 1
    K = idx.shape[-1]
    ld_s = s.shape[-1]
    sm_scale = 1.0 / math.sqrt(D) if sm_scale is None else sm_scale
    need = int(lib().sas_attn_bwd_varlen_workspace_size(_dtype_code(q), B, max_seqlen, T, Hq, Hkv, D, K))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    ds = torch.empty(s.shape, dtype=torch.float32, device=q.device)
    _check(lib().sas_attn_bwd_varlen(_dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse),
                                     _ptr(s), ld_s, _ptr(lse_s), _ptr(idx), _ptr(cnt), _ptr(log_gate),
                                     _ptr(cu_seqlens), B, max_seqlen, T, Hq, Hkv, D, block_size, K, sm_scale,
                                     _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ds), _ptr(workspace), workspace.numel(),
                                     _stream()))
    return dq, dk, dv, ds


def pool_pages(k_cache, pages=None, kpool=None, page_size: int = 64):
    """Pooled-key cache kpool [P,Hkv,D] fp32: the mean key of each (page, KV head) of
    k_cache [P,Hkv,64,D]; only `pages` (int32 ids) when given."""
    _contig(k_cache, pages, kpool)
    P, Hkv, _, D = k_cache.shape
    if kpool is None:
        kpool = torch.zeros((P, Hkv, D), dtype=torch.float32, device=k_cache.device)
    n = 0 if pages is None else pages.numel()
    _check(lib().sas_pool_pages(_ptr(k_cache), P, Hkv, D, page_size, _ptr(pages), n, _ptr(kpool), _stream()))
    return kpool


def score_select_decode(q, kpool, page_table, kv_len, K: int, ld_s: int, noise=None, page_size: int = 64):
    """Decode stand-in scores from the pooled-key cache, then Top-K + log-gates.
    Returns s [N,Hkv,ld_s], idx [N,Hkv,K], cnt [N,Hkv], log_gate [N,Hkv,K], lse_s [N,Hkv]."""
    _contig(q, kpool, page_table, kv_len, noise)
    N, Hq, D = q.shape
    P, Hkv = kpool.shape[0], kpool.shape[1]
    dev = q.device
    s = torch.zeros((N, Hkv, ld_s), dtype=torch.float32, device=dev)
    idx = torch.empty((N, Hkv, K), dtype=torch.int32, device=dev)
    cnt = torch.empty((N, Hkv), dtype=torch.int32, device=dev)
    lg = torch.empty((N, Hkv, K), dtype=torch.float32, device=dev)
    lse_s = torch.empty((N, Hkv), dtype=torch.float32, device=dev)
    ld_noise = 0 if noise is None else noise.shape[-1]
    _check(lib().sas_score_select_decode(_ptr(q), _ptr(kpool), P, _ptr(page_table), page_table.shape[1],
                                         _ptr(kv_len), N, Hq, Hkv, D, page_size, _ptr(noise), ld_noise, K,
                                         _ptr(s), ld_s, _ptr(idx), _ptr(cnt), _ptr(lg), _ptr(lse_s), _stream()))
    return s, idx, cnt, lg, lse_s


def decode_workspace_bytes(N: int, Hq: int, Hkv: int, D: int, K: int) -> int:
    return int(lib().sas_decode_workspace_size(N, Hq, Hkv, D, K))


def decode_paged(q, k_cache, v_cache, page_table, kv_len, idx, cnt, log_gate, sm_scale=None,
                 page_size: int = 64, workspace=None, with_lse: bool = True):
    """Paged decode. q [N,Hq,D]; caches [P,Hkv,64,D]. Returns o [N,Hq,D] and lse [N,Hq] (or None)."""
    _contig(q, k_cache, v_cache, page_table, kv_len, idx, cnt, log_gate)
    N, Hq, D = q.shape
    P, Hkv = k_cache.shape[0], k_cache.shape[1]
    K = idx.shape[-1]
    sm_scale = 1.0 / math.sqrt(D) if sm_scale is None else sm_scale
    need = decode_workspace_bytes(N, Hq, Hkv, D, K)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    o = torch.empty_like(q)
    lse = torch.empty((N, Hq), dtype=torch.float32, device=q.device) if with_lse else None
    _check(lib().sas_decode_paged(_ptr(q), _ptr(k_cache), _ptr(v_cache), P, _ptr(page_table),
                                  page_table.shape[1], _ptr(kv_len), N, Hq, Hkv, D, page_size, K,
                                  _ptr(idx), _ptr(cnt), _ptr(log_gate), sm_scale, _ptr(o), _ptr(lse),
                                  _ptr(workspace), workspace.numel(), _stream()))
    return o, lse
