"""Grouped-query flash attention for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI in ``include/attn.h`` (libgqa_attn.so):
argument marshalling and output allocation with torch, nothing else.  Every
step of the computation runs in the library's CUDA kernels; there is no CPU or
library fallback, and every call raises if the library is missing or reports
an error.

Layouts: q/out [B, Sq, Hq, D], k/v [B, Skv, Hkv, D] (bf16, contiguous),
lse [B, Hq, Sq] fp32, partials [S, B, Sq, Hq, D] and [S, B, Hq, Sq] fp32.

Calls (each returns torch tensors it allocated unless out/lse are given):
  prefill(q, k, v)                      one launch; D 64, 128, 256, 512
  decode_split / merge / decode         split-KV partials, their LSE merge,
                                        or both (two launches)
  decode_fused(q, k, v, num_splits)     split and merge in one launch
  decode_split_kv / decode_kv / prefill_kv
                                        over strided or paged K/V (block_table),
                                        lengths per sequence (seq_lens), fp8
                                        e4m3 K/V (k_scale, v_scale) and V
                                        narrower than K (576/512, 320/256,
                                        192/128)
  decode_noalloc                        decode + merge with no workspace
Optional logit terms: softcap, alibi_max_bias, window, mask (bf16 [B or 1,
Sq, Skv]) on every attention call; sinks (fp32 [Hq]) on the calls that
produce the final O (prefill*, merge, decode*, decode_fused).
"""
from __future__ import annotations

import ctypes
import math
import os
import re
import threading

import torch

__all__ = [
    "AttnError", "library", "library_path", "declared_functions", "prefill", "decode_split",
    "merge", "decode", "decode_workspace_bytes", "last_status", "status_string",
    "watchdog_selftest", "version", "ATTN_OK", "ATTN_ERR_INVALID_ARG", "ATTN_ERR_UNSUPPORTED",
    "ATTN_ERR_ALIGNMENT", "ATTN_ERR_CUDA", "ATTN_ERR_TIMEOUT", "ATTN_ERR_TOO_LARGE", "decode_noalloc",
    "AttnOptions", "AttnKVView", "decode_split_kv", "decode_kv", "ATTN_FP8_E4M3", "prefill_kv",
    "decode_fused",
]

ATTN_OK = 0
ATTN_ERR_INVALID_ARG = -1
ATTN_ERR_UNSUPPORTED = -2
ATTN_ERR_ALIGNMENT = -3
ATTN_ERR_CUDA = -4
ATTN_ERR_TIMEOUT = -5
ATTN_ERR_TOO_LARGE = -6

_PKG = os.path.dirname(os.path.abspath(__file__))
_HEADER = os.path.join(os.path.dirname(_PKG), "include", "attn.h")
_lock = threading.Lock()
_lib = None

_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float

_SIGNATURES = {
    "attn_prefill": (_i, [_vp, _vp, _vp, _vp, _vp] + [_i] * 8 + [_f, _i, _vp]),
    "attn_decode_split": (_i, [_vp, _vp, _vp, _vp, _vp] + [_i] * 8 + [_f, _i, _vp]),
    "attn_merge": (_i, [_vp, _vp, _vp, _vp] + [_i] * 6 + [_vp]),
    "attn_decode_workspace_bytes": (ctypes.c_size_t, [_i] * 5),
    "attn_last_status": (_i, [_vp]),
    "attn_status_string": (ctypes.c_char_p, [_i]),
    "attn_watchdog_selftest": (_i, [ctypes.c_ulonglong, _vp]),
    "attn_version": (_i, []),
    "attn_decode_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp] + [_i] * 8 + [_f, _i, _i, _vp]),
    "attn_prefill_ex": (_i, [_vp, _vp, _vp, _vp, _vp] + [_i] * 8 + [_f, _i, _vp, _vp]),
    "attn_decode_split_ex": (_i, [_vp, _vp, _vp, _vp, _vp] + [_i] * 8 + [_f, _i, _vp, _vp]),
    "attn_merge_ex": (_i, [_vp, _vp, _vp, _vp] + [_i] * 6 + [_vp, _vp]),
    "attn_decode_split_kv": (_i, [_vp, _vp, _vp, _vp] + [_i] * 8 + [_f, _i, _vp, _vp]),
    "attn_prefill_kv": (_i, [_vp, _vp, _vp, _vp] + [_i] * 8 + [_f, _i, _vp, _vp]),
    "attn_decode_fused": (_i, [_vp, _vp, _vp, _vp] + [_i] * 8 + [_f, _i, _i, _vp, _vp]),
}


class AttnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {status_string(status)} ({status})")


def library_path() -> str:
    return os.path.join(_PKG, "libgqa_attn.so")


def library():
    """The loaded C library; raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            path = library_path()
            if not os.path.exists(path):
                raise RuntimeError(
                    f"{path} is missing: build it with `python -m gqa_flash_attention_attn_b200.build`")
            lib = ctypes.CDLL(path)
            for name, (res, args) in _SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def declared_functions() -> list[str]:
    """Names of the functions include/attn.h declares."""
    text = open(_HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z0-9_]+)\s*\(", text)))


def status_string(status: int) -> str:
    return library().attn_status_string(int(status)).decode()


def version() -> int:
    return library().attn_version()


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(fn: str, status: int):
    if status != ATTN_OK:
        raise AttnError(fn, status)


def _need(t, name, dtype, ndim):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


_OUT_CODES = {torch.bfloat16: 0, torch.float32: 1}


class AttnOptions(ctypes.Structure):
    """The C ``attn_options`` struct: optional logit terms (zero / NULL = off)."""
    _fields_ = [("softcap", ctypes.c_float), ("alibi_max_bias", ctypes.c_float),
                ("sinks", ctypes.c_void_p), ("window", ctypes.c_int), ("mask", ctypes.c_void_p),
                ("mask_stride_seq", ctypes.c_longlong), ("mask_stride_row", ctypes.c_longlong)]


class AttnKVView(ctypes.Structure):
    """The C ``attn_kv_view`` struct: a strided, optionally paged K/V cache."""
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("stride_seq", ctypes.c_longlong),
                ("stride_token", ctypes.c_longlong), ("stride_head", ctypes.c_longlong),
                ("block_table", ctypes.c_void_p), ("max_pages", ctypes.c_int), ("page_size", ctypes.c_int),
                ("num_pages", ctypes.c_int), ("seq_lens", ctypes.c_void_p), ("kv_dtype", ctypes.c_int),
                ("k_scale", ctypes.c_void_p), ("v_scale", ctypes.c_void_p), ("head_dim_v", ctypes.c_int),
                ("v_stride_seq", ctypes.c_longlong), ("v_stride_token", ctypes.c_longlong),
                ("v_stride_head", ctypes.c_longlong)]


ATTN_FP8_E4M3 = 2
_FP8_DTYPES = (torch.uint8, torch.float8_e4m3fn)


def _kv_view(k, v, block_table, seq_lens, k_scale=None, v_scale=None):
    """AttnKVView of k/v (4-D views with a contiguous last dim) and Skv.

    Unpaged: k, v are [B, Skv, Hkv, D] views.  Paged: k, v are
    [num_pages, page_size, Hkv, D] views and block_table is int32 [B, max_pages].
    bf16 K/V, or fp8 e4m3 codes (uint8 or float8_e4m3fn) with fp32 per-head
    k_scale and v_scale [Hkv].  v may have fewer columns than k (Dv < D: the
    head sizes (576, 512), (320, 256), (192, 128)), e.g. v = k[..., :Dv] for
    a cache whose V is the front of K; v's strides may differ from k's."""
    fp8 = isinstance(k, torch.Tensor) and k.dtype in _FP8_DTYPES
    for t, n in ((k, "k"), (v, "v")):
        ok_dtype = t.dtype in _FP8_DTYPES if fp8 else t.dtype == torch.bfloat16
        if not isinstance(t, torch.Tensor) or t.device.type != "cuda" or not ok_dtype or t.dim() != 4:
            raise ValueError(f"{n} must be a 4-D CUDA tensor, bf16 or fp8 e4m3 like the other")
        if t.stride(3) != 1:
            raise ValueError(f"{n} must be contiguous in its last dimension")
    if k.shape[:3] != v.shape[:3]:
        raise ValueError("k and v must have the same leading shape")
    view = AttnKVView(k.data_ptr(), v.data_ptr(), k.stride(0), k.stride(1), k.stride(2), None, 0, 0, 0, None,
                      0, None, None, 0 if v.shape[3] == k.shape[3] else v.shape[3])
    if v.stride()[:3] != k.stride()[:3]:
        view.v_stride_seq, view.v_stride_token, view.v_stride_head = v.stride(0), v.stride(1), v.stride(2)
    if fp8:
        for sc, n in ((k_scale, "k_scale"), (v_scale, "v_scale")):
            _need(sc, n, torch.float32, 1)
            if sc.shape[0] != k.shape[2]:
                raise ValueError(f"{n} must have one entry per K/V head")
        view.kv_dtype = ATTN_FP8_E4M3
        view.k_scale = k_scale.data_ptr()
        view.v_scale = v_scale.data_ptr()
    if block_table is not None:
        _need(block_table, "block_table", torch.int32, 2)
        view.block_table = block_table.data_ptr()
        view.max_pages = block_table.shape[1]
        view.page_size = k.shape[1]
        view.num_pages = k.shape[0]
        skv = block_table.shape[1] * k.shape[1]
    else:
        skv = k.shape[1]
    if seq_lens is not None:
        _need(seq_lens, "seq_lens", torch.int32, 1)
        view.seq_lens = seq_lens.data_ptr()
    return view, skv


def _options(softcap, alibi_max_bias, sinks, window, Hq, mask=None, B=None, Sq=None, Skv=None):
    """An AttnOptions for the given terms, or None when every term is off.

    mask: bf16 [B or 1, Sq, Skv] (or [Sq, Skv]), last dim contiguous; added to
    the logits (-inf removes a key)."""
    if not softcap and not alibi_max_bias and sinks is None and not window and mask is None:
        return None
    if sinks is not None:
        _need(sinks, "sinks", torch.float32, 1)
        if sinks.shape[0] != Hq:
            raise ValueError(f"sinks must have Hq = {Hq} entries")
    opt = AttnOptions(float(softcap), float(alibi_max_bias), None if sinks is None else sinks.data_ptr(),
                      int(window), None, 0, 0)
    if mask is not None:
        if not isinstance(mask, torch.Tensor) or mask.device.type != "cuda" or mask.dtype != torch.bfloat16:
            raise ValueError("mask must be a bf16 CUDA tensor")
        if mask.dim() == 2:
            mask = mask.unsqueeze(0)
        if mask.dim() != 3 or mask.shape[1:] != (Sq, Skv) or mask.shape[0] not in (1, B) or mask.stride(2) != 1:
            raise ValueError(f"mask must be [B or 1, {Sq}, {Skv}] with a contiguous last dim")
        opt.mask = mask.data_ptr()
        opt.mask_stride_seq = 0 if mask.shape[0] == 1 else mask.stride(0)
        opt.mask_stride_row = mask.stride(1)
    return opt


def prefill(q, k, v, *, causal=True, q_offset=0, scale=None, out_dtype=torch.bfloat16,
            out=None, lse=None, return_lse=True, stream=None, softcap=0.0, alibi_max_bias=0.0,
            sinks=None, window=0, mask=None):
    """O = softmax(scale * Q K^T + causal mask) V and its LSE, in one launch.

    Optional logit terms (off by default): softcap (z = c tanh(z / c)),
    alibi_max_bias (per-head geometric slope times (t - pos)), sinks (fp32 [Hq]
    logits that join only the softmax denominator) and window (key t visible
    only when pos - window < t; needs causal and q_offset + Sq <= Skv) and
    mask (bf16 [B or 1, Sq, Skv] added to the logits; -inf removes a key)."""
    _need(q, "q", torch.bfloat16, 4)
    _need(k, "k", torch.bfloat16, 4)
    _need(v, "v", torch.bfloat16, 4)
    B, Sq, Hq, D = q.shape
    _, Skv, Hkv, _ = k.shape
    if v.shape != k.shape or k.shape[0] != B or k.shape[3] != D:
        raise ValueError("k/v shapes do not match q")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty((B, Sq, Hq, D), dtype=out_dtype, device=q.device)
    else:
        _need(out, "out", out.dtype, 4)
    if out.dtype not in _OUT_CODES:
        raise ValueError("out must be bf16 or fp32")
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    opt = _options(softcap, alibi_max_bias, sinks, window, Hq, mask, B, Sq, Skv)
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Sq, Skv, D, int(q_offset),
            int(bool(causal)), float(scale), _OUT_CODES[out.dtype])
    if opt is None:
        _check("attn_prefill", library().attn_prefill(*args, _stream_ptr(stream)))
    else:
        _check("attn_prefill_ex", library().attn_prefill_ex(*args, ctypes.byref(opt), _stream_ptr(stream)))
    return out, lse


def decode_workspace_bytes(B, Hq, Sq, D, num_splits) -> int:
    return library().attn_decode_workspace_bytes(B, Hq, Sq, D, num_splits)


def decode_split(q, k, v, num_splits, *, causal=True, q_offset=0, scale=None,
                 partial_out=None, partial_lse=None, stream=None, softcap=0.0, alibi_max_bias=0.0,
                 window=0, mask=None):
    """Per-split normalised partial outputs [S,B,Sq,Hq,D] and LSEs [S,B,Hq,Sq].

    softcap, alibi_max_bias, window and mask as in prefill(); sinks belong to merge()."""
    _need(q, "q", torch.bfloat16, 4)
    _need(k, "k", torch.bfloat16, 4)
    _need(v, "v", torch.bfloat16, 4)
    B, Sq, Hq, D = q.shape
    _, Skv, Hkv, _ = k.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if partial_out is None:
        partial_out = torch.empty((num_splits, B, Sq, Hq, D), dtype=torch.float32, device=q.device)
    if partial_lse is None:
        partial_lse = torch.empty((num_splits, B, Hq, Sq), dtype=torch.float32, device=q.device)
    opt = _options(softcap, alibi_max_bias, None, window, Hq, mask, B, Sq, Skv)
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(partial_out), _ptr(partial_lse), B, Hq, Hkv, Sq, Skv, D,
            int(q_offset), int(bool(causal)), float(scale), int(num_splits))
    if opt is None:
        _check("attn_decode_split", library().attn_decode_split(*args, _stream_ptr(stream)))
    else:
        _check("attn_decode_split_ex",
               library().attn_decode_split_ex(*args, ctypes.byref(opt), _stream_ptr(stream)))
    return partial_out, partial_lse


def merge(partial_out, partial_lse, *, out_dtype=torch.bfloat16, out=None, lse=None, return_lse=True,
          stream=None, sinks=None):
    """Combine split partials by their LSE into out [B,Sq,Hq,D] and lse [B,Hq,Sq].

    sinks: optional fp32 [Hq] logits that join the denominator and the LSE."""
    _need(partial_out, "partial_out", torch.float32, 5)
    _need(partial_lse, "partial_lse", torch.float32, 4)
    S, B, Sq, Hq, D = partial_out.shape
    if out is None:
        out = torch.empty((B, Sq, Hq, D), dtype=out_dtype, device=partial_out.device)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=partial_out.device)
    args = (_ptr(partial_out), _ptr(partial_lse), _ptr(out), _ptr(lse), B, Hq, Sq, D, S, _OUT_CODES[out.dtype])
    if sinks is None:
        _check("attn_merge", library().attn_merge(*args, _stream_ptr(stream)))
    else:
        _need(sinks, "sinks", torch.float32, 1)
        if sinks.shape[0] != Hq:
            raise ValueError(f"sinks must have Hq = {Hq} entries")
        _check("attn_merge_ex", library().attn_merge_ex(*args, _ptr(sinks), _stream_ptr(stream)))
    return out, lse


def decode(q, k, v, num_splits, *, causal=True, q_offset=0, scale=None, out_dtype=torch.bfloat16,
           workspace=None, out=None, lse=None, stream=None, softcap=0.0, alibi_max_bias=0.0, sinks=None,
           window=0, mask=None):
    """Split-KV decode followed by the LSE merge (two launches on one stream)."""
    B, Sq, Hq, D = q.shape
    po = pl = None
    if workspace is not None:
        po, pl = workspace
    po, pl = decode_split(q, k, v, num_splits, causal=causal, q_offset=q_offset, scale=scale,
                          partial_out=po, partial_lse=pl, stream=stream, softcap=softcap,
                          alibi_max_bias=alibi_max_bias, window=window, mask=mask)
    return merge(po, pl, out_dtype=out_dtype, out=out, lse=lse, stream=stream, sinks=sinks)


def decode_split_kv(q, k, v, num_splits, *, block_table=None, seq_lens=None, causal=True, q_offset=0,
                    scale=None, partial_out=None, partial_lse=None, stream=None, softcap=0.0,
                    alibi_max_bias=0.0, window=0, mask=None, k_scale=None, v_scale=None):
    """decode_split over a strided or paged K/V cache (see attn_kv_view).

    Unpaged: k, v are [B, Skv, Hkv, D] views (any strides, last dim
    contiguous).  Paged: k, v are [num_pages, page_size, Hkv, D] and
    block_table int32 [B, max_pages] maps logical to physical pages.
    fp8 e4m3 K/V: k, v as uint8 codes (or float8_e4m3fn) with fp32 k_scale,
    v_scale [Hkv]: K = code * k_scale[kvh], V = code * v_scale[kvh].
    v may be Dv < D columns wide (see _kv_view); the partials are then Dv wide.
    seq_lens (int32 [B], optional): keys per sequence; the query rows then sit
    at the last Sq positions of each sequence and q_offset is ignored."""
    _need(q, "q", torch.bfloat16, 4)
    B, Sq, Hq, D = q.shape
    view, Skv = _kv_view(k, v, block_table, seq_lens, k_scale, v_scale)
    Hkv = k.shape[2]
    if k.shape[3] != D:
        raise ValueError("k/v head size does not match q")
    if block_table is None and k.shape[0] != B:
        raise ValueError("unpaged k/v must have B sequences")
    if block_table is not None and block_table.shape[0] != B:
        raise ValueError("block_table must have B rows")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    Dv = v.shape[3]
    if partial_out is None:
        partial_out = torch.empty((num_splits, B, Sq, Hq, Dv), dtype=torch.float32, device=q.device)
    if partial_lse is None:
        partial_lse = torch.empty((num_splits, B, Hq, Sq), dtype=torch.float32, device=q.device)
    opt = _options(softcap, alibi_max_bias, None, window, Hq, mask, B, Sq, Skv)
    st = library().attn_decode_split_kv(_ptr(q), ctypes.byref(view), _ptr(partial_out), _ptr(partial_lse), B, Hq,
                                        Hkv, Sq, Skv, D, int(q_offset), int(bool(causal)), float(scale),
                                        int(num_splits), None if opt is None else ctypes.byref(opt),
                                        _stream_ptr(stream))
    _check("attn_decode_split_kv", st)
    return partial_out, partial_lse


def decode_kv(q, k, v, num_splits, *, block_table=None, seq_lens=None, causal=True, q_offset=0, scale=None,
              out_dtype=torch.bfloat16, workspace=None, out=None, lse=None, stream=None, softcap=0.0,
              alibi_max_bias=0.0, sinks=None, window=0, mask=None, k_scale=None, v_scale=None):
    """decode_split_kv followed by the LSE merge (two launches on one stream)."""
    po = pl = None
    if workspace is not None:
        po, pl = workspace
    po, pl = decode_split_kv(q, k, v, num_splits, block_table=block_table, seq_lens=seq_lens, causal=causal,
                             q_offset=q_offset, scale=scale, partial_out=po, partial_lse=pl, stream=stream,
                             softcap=softcap, alibi_max_bias=alibi_max_bias, window=window, mask=mask,
                             k_scale=k_scale, v_scale=v_scale)
    return merge(po, pl, out_dtype=out_dtype, out=out, lse=lse, stream=stream, sinks=sinks)


def decode_fused(q, k, v, num_splits, *, block_table=None, seq_lens=None, causal=True, q_offset=0, scale=None,
                 out_dtype=torch.bfloat16, out=None, lse=None, return_lse=True, stream=None, softcap=0.0,
                 alibi_max_bias=0.0, sinks=None, window=0, mask=None, k_scale=None, v_scale=None):
    """decode_kv in one launch: the key ranges of each (sequence, K/V head)
    form a thread-block cluster that merges them in shared memory (n = the
    largest power of two <= min(num_splits, 8) ranges).  Arguments as in
    decode_kv; returns out [B, Sq, Hq, Dv] and lse [B, Hq, Sq]."""
    _need(q, "q", torch.bfloat16, 4)
    B, Sq, Hq, D = q.shape
    view, Skv = _kv_view(k, v, block_table, seq_lens, k_scale, v_scale)
    Hkv = k.shape[2]
    if k.shape[3] != D:
        raise ValueError("k head size does not match q")
    if block_table is None and k.shape[0] != B:
        raise ValueError("unpaged k/v must have B sequences")
    if block_table is not None and block_table.shape[0] != B:
        raise ValueError("block_table must have B rows")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    Dv = v.shape[3]
    if out is None:
        out = torch.empty((B, Sq, Hq, Dv), dtype=out_dtype, device=q.device)
    else:
        _need(out, "out", out.dtype, 4)
    if out.dtype not in _OUT_CODES:
        raise ValueError("out must be bf16 or fp32")
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    opt = _options(softcap, alibi_max_bias, sinks, window, Hq, mask, B, Sq, Skv)
    st = library().attn_decode_fused(_ptr(q), ctypes.byref(view), _ptr(out), _ptr(lse), B, Hq, Hkv, Sq, Skv, D,
                                     int(q_offset), int(bool(causal)), float(scale), int(num_splits),
                                     _OUT_CODES[out.dtype], None if opt is None else ctypes.byref(opt),
                                     _stream_ptr(stream))
    _check("attn_decode_fused", st)
    return out, lse


def prefill_kv(q, k, v, *, block_table=None, seq_lens=None, causal=True, q_offset=0, scale=None,
               out_dtype=torch.bfloat16, out=None, lse=None, return_lse=True, stream=None, softcap=0.0,
               alibi_max_bias=0.0, sinks=None, window=0, mask=None, k_scale=None, v_scale=None):
    """prefill() over a strided or paged K/V cache, fp8 codes, lengths per
    sequence or Dv < D (k, v, block_table, seq_lens, k_scale, v_scale as in
    decode_split_kv).  One launch; out is [B, Sq, Hq, Dv]."""
    _need(q, "q", torch.bfloat16, 4)
    B, Sq, Hq, D = q.shape
    view, Skv = _kv_view(k, v, block_table, seq_lens, k_scale, v_scale)
    Hkv = k.shape[2]
    if k.shape[3] != D:
        raise ValueError("k head size does not match q")
    if block_table is None and k.shape[0] != B:
        raise ValueError("unpaged k/v must have B sequences")
    if block_table is not None and block_table.shape[0] != B:
        raise ValueError("block_table must have B rows")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    Dv = v.shape[3]
    if out is None:
        out = torch.empty((B, Sq, Hq, Dv), dtype=out_dtype, device=q.device)
    else:
        _need(out, "out", out.dtype, 4)
    if out.dtype not in _OUT_CODES:
        raise ValueError("out must be bf16 or fp32")
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    opt = _options(softcap, alibi_max_bias, sinks, window, Hq, mask, B, Sq, Skv)
    st = library().attn_prefill_kv(_ptr(q), ctypes.byref(view), _ptr(out), _ptr(lse), B, Hq, Hkv, Sq, Skv, D,
                                   int(q_offset), int(bool(causal)), float(scale), _OUT_CODES[out.dtype],
                                   None if opt is None else ctypes.byref(opt), _stream_ptr(stream))
    _check("attn_prefill_kv", st)
    return out, lse


def last_status(stream=None) -> int:
    """Synchronise, then read and clear the device status word."""
    return library().attn_last_status(_stream_ptr(stream))


def watchdog_selftest(limit_ns: int, stream=None):
    _check("attn_watchdog_selftest", library().attn_watchdog_selftest(int(limit_ns), _stream_ptr(stream)))


def decode_noalloc(q, k, v, num_splits, *, causal=True, q_offset=0, scale=None, out_dtype=torch.bfloat16,
                   out=None, lse=None, return_lse=True, stream=None):
    """Split-KV decode + merge with the partials in the library's fixed device
    array instead of a caller workspace, for callers that cannot allocate
    device memory.  Same result as decode(); calls must not overlap on the GPU."""
    _need(q, "q", torch.bfloat16, 4)
    _need(k, "k", torch.bfloat16, 4)
    _need(v, "v", torch.bfloat16, 4)
    B, Sq, Hq, D = q.shape
    _, Skv, Hkv, _ = k.shape
    if v.shape != k.shape or k.shape[0] != B or k.shape[3] != D:
        raise ValueError("k/v shapes do not match q")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty((B, Sq, Hq, D), dtype=out_dtype, device=q.device)
    else:
        if out.dtype not in _OUT_CODES:
            raise ValueError("out must be bf16 or fp32")
        _need(out, "out", out.dtype, 4)
        if tuple(out.shape) != (B, Sq, Hq, D):
            raise ValueError(f"out must be [{B}, {Sq}, {Hq}, {D}]")
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    elif lse is not None:
        _need(lse, "lse", torch.float32, 3)
        if tuple(lse.shape) != (B, Hq, Sq):
            raise ValueError(f"lse must be [{B}, {Hq}, {Sq}]")
    for t, n in ((k, "k"), (v, "v"), (out, "out"), (lse, "lse")):
        if t is not None and t.device != q.device:
            raise ValueError(f"{n} must be on {q.device}, like q")
    # the library looks up its scratch array on the current device: make it q's
    with torch.cuda.device(q.device):
        st = library().attn_decode_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Sq, Skv,
                                           D, int(q_offset), int(bool(causal)), float(scale), int(num_splits),
                                           _OUT_CODES[out.dtype], _stream_ptr(stream))
    _check("attn_decode_noalloc", st)
    return out, lse
