"""Float64 CPU oracle for grouped-query attention.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package.  The CUDA library never
imports, links or calls it, and it imports nothing from the CUDA library.

The arithmetic lives in ``oracle.c`` (plain C, fp64, OpenMP over rows); this
module compiles it with gcc on first use and marshals numpy arrays.  Every
function takes arrays that are widened EXACTLY from the values the GPU sees
(bf16 -> float64 is exact), and the scale as the same float32 value the GPU
receives, widened.

Functions and the passage each follows (all pinned by tests/test_oracle_pins.py):
  attention       the definition of softmax attention with grouped-query heads
                  ("ggml-org/llama.cpp PR #28507", Setup: GQA 8; FLASH_ATTN_EXT
                  case list: nr23, mask=1)
  attention_rows  the same definition on selected (b, h, s) rows
  probs           the normalised attention weights of one row
  split           per-split partials with their LSE metadata
                  ("Anbeeld/beellama.cpp PR #149", Overview: every block
                  publishes its (max, rowsum))
  merge           the LSE combine of split partials (same page, review of the
                  combine kernel for parallel_blocks > 1)
  attention_fp8   attention over an fp8 e4m3 K/V cache with per-head scales
                  (decodes each code from the format's definition)
  *_ex            the same with the optional logit terms of the FLASH_ATTN_EXT
                  operator ("ggml-org/llama.cpp PR #28507", Crash 1: sinks,
                  max_bias, logit_softcap, mask) and a sliding window (see oracle.c)

V narrower than K (attention_ex, attention_rows_ex: v with Dv < D columns, the
hsk != hsv cases of the FLASH_ATTN_EXT list, e.g. hsk=320, hsv=256): column j
of O = P V reads only column j of V, so V is zero-padded to D columns, the
fp64 kernel runs unchanged and the first Dv columns of O are returned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_i64 = ctypes.c_int64
_dp = ctypes.POINTER(ctypes.c_double)
_lp = ctypes.POINTER(ctypes.c_int64)


def build(src: str = _SRC, out: str = _LIB_PATH, extra_flags=()) -> str:
    """Compile oracle.c into a shared library (gcc -O2, OpenMP, no fast-math)."""
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", *extra_flags,
           "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _needs_build(src: str, out: str) -> bool:
    return (not os.path.exists(out)) or os.path.getmtime(out) < os.path.getmtime(src)


def load(path: str | None = None):
    """Load (building if stale) the oracle library; returns a ctypes handle."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            if _needs_build(_SRC, _LIB_PATH):
                build()
            _lib = _bind(ctypes.CDLL(_LIB_PATH))
    return _lib


def _bind(lib):
    lib.oracle_attention.argtypes = [_dp, _dp, _dp, _dp, _dp] + [_i64] * 7 + [ctypes.c_int, ctypes.c_double]
    lib.oracle_attention.restype = None
    lib.oracle_attention_rows.argtypes = [_dp, _dp, _dp, _lp, _i64, _dp, _dp] + [_i64] * 7 + [ctypes.c_int, ctypes.c_double]
    lib.oracle_attention_rows.restype = None
    lib.oracle_probs.argtypes = [_dp, _dp, _i64, _i64, _i64, _dp] + [_i64] * 6 + [ctypes.c_int, ctypes.c_double]
    lib.oracle_probs.restype = None
    lib.oracle_split.argtypes = [_dp, _dp, _dp, _dp, _dp] + [_i64] * 7 + [ctypes.c_int, ctypes.c_double, _i64]
    lib.oracle_split.restype = None
    lib.oracle_merge.argtypes = [_dp, _dp, _dp, _dp] + [_i64] * 5
    lib.oracle_merge.restype = None
    lib.oracle_num_threads.argtypes = []
    lib.oracle_num_threads.restype = ctypes.c_int
    msk = [_dp, _i64, _i64]
    ext = [ctypes.c_double, ctypes.c_double, _dp, _i64] + msk
    lib.oracle_attention_ex.argtypes = [_dp, _dp, _dp, _dp, _dp] + [_i64] * 7 + [ctypes.c_int, ctypes.c_double] + ext
    lib.oracle_attention_ex.restype = None
    lib.oracle_attention_rows_ex.argtypes = ([_dp, _dp, _dp, _lp, _i64, _dp, _dp] + [_i64] * 7 +
                                             [ctypes.c_int, ctypes.c_double] + ext)
    lib.oracle_attention_rows_ex.restype = None
    lib.oracle_split_ex.argtypes = ([_dp, _dp, _dp, _dp, _dp] + [_i64] * 7 + [ctypes.c_int, ctypes.c_double, _i64] +
                                    [ctypes.c_double, ctypes.c_double, _i64] + msk)
    lib.oracle_split_ex.restype = None
    lib.oracle_merge_ex.argtypes = [_dp, _dp, _dp, _dp] + [_i64] * 5 + [_dp]
    lib.oracle_merge_ex.restype = None
    lib.oracle_e4m3_value.argtypes = [ctypes.c_int]
    lib.oracle_e4m3_value.restype = ctypes.c_double
    _bp = ctypes.POINTER(ctypes.c_ubyte)
    lib.oracle_attention_fp8.argtypes = ([_dp, _bp, _bp, _dp, _dp, _dp, _dp] + [_i64] * 7 +
                                         [ctypes.c_int, ctypes.c_double] + ext)
    lib.oracle_attention_fp8.restype = None
    lib.oracle_alibi_slope.argtypes = [_i64, _i64, ctypes.c_double]
    lib.oracle_alibi_slope.restype = ctypes.c_double
    return lib


def _f64(x) -> np.ndarray:
    """Widen to a contiguous float64 numpy array (exact for bf16/fp32 inputs)."""
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu")
        x = x.double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(_dp)


def _dims(q, k):
    B, Sq, Hq, D = q.shape
    Bk, Skv, Hkv, Dk = k.shape
    if Bk != B or Dk != D:
        raise ValueError("q and k disagree on batch or head dim")
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    return B, Hq, Hkv, Sq, Skv, D


def num_threads(lib=None) -> int:
    return (lib or load()).oracle_num_threads()


def attention(q, k, v, *, scale, causal=True, q_offset=0, lib=None):
    """O [B,Sq,Hq,D] and LSE [B,Hq,Sq] in float64 for the whole problem."""
    lib = lib or load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Hkv, Sq, Skv, D = _dims(q, k)
    out = np.zeros((B, Sq, Hq, D), dtype=np.float64)
    lse = np.zeros((B, Hq, Sq), dtype=np.float64)
    lib.oracle_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                         B, Hq, Hkv, Sq, Skv, D, int(q_offset), int(bool(causal)), float(scale))
    return out, lse


def attention_rows(q, k, v, rows, *, scale, causal=True, q_offset=0, lib=None):
    """O rows [n,D] and LSE [n] for the (b, h, s) triples in ``rows``."""
    lib = lib or load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Hkv, Sq, Skv, D = _dims(q, k)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    n = rows.shape[0]
    out = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    lib.oracle_attention_rows(_ptr(q), _ptr(k), _ptr(v), rows.ctypes.data_as(_lp), n,
                              _ptr(out), _ptr(lse), B, Hq, Hkv, Sq, Skv, D,
                              int(q_offset), int(bool(causal)), float(scale))
    return out, lse


def probs(q, k, b, h, s, *, scale, causal=True, q_offset=0, lib=None):
    """Normalised attention weights of row (b, h, s) over all Skv keys."""
    lib = lib or load()
    q, k = _f64(q), _f64(k)
    B, Hq, Hkv, Sq, Skv, D = _dims(q, k)
    p = np.zeros((Skv,), dtype=np.float64)
    lib.oracle_probs(_ptr(q), _ptr(k), int(b), int(h), int(s), _ptr(p),
                     Hq, Hkv, Sq, Skv, D, int(q_offset), int(bool(causal)), float(scale))
    return p


def split(q, k, v, num_splits, *, scale, causal=True, q_offset=0, lib=None):
    """Per-split partial O [S,B,Sq,Hq,D] and LSE [S,B,Hq,Sq]."""
    lib = lib or load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Hkv, Sq, Skv, D = _dims(q, k)
    pout = np.zeros((num_splits, B, Sq, Hq, D), dtype=np.float64)
    plse = np.zeros((num_splits, B, Hq, Sq), dtype=np.float64)
    lib.oracle_split(_ptr(q), _ptr(k), _ptr(v), _ptr(pout), _ptr(plse),
                     B, Hq, Hkv, Sq, Skv, D, int(q_offset), int(bool(causal)), float(scale),
                     int(num_splits))
    return pout, plse


def merge(pout, plse, lib=None):
    """Combine split partials: returns O [B,Sq,Hq,D] and LSE [B,Hq,Sq]."""
    lib = lib or load()
    pout, plse = _f64(pout), _f64(plse)
    S, B, Sq, Hq, D = pout.shape
    out = np.zeros((B, Sq, Hq, D), dtype=np.float64)
    lse = np.zeros((B, Hq, Sq), dtype=np.float64)
    lib.oracle_merge(_ptr(pout), _ptr(plse), _ptr(out), _ptr(lse), B, Hq, Sq, D, S)
    return out, lse


def _sinks_arg(sinks):
    if sinks is None:
        return None, None
    arr = _f64(sinks).reshape(-1)
    return arr, _ptr(arr)


def _mask_arg(mask, B, Sq, Skv):
    """An additive mask [Sq, Skv], [1, Sq, Skv] or [B, Sq, Skv] as a float64
    array with its batch and row strides (batch stride 0: shared)."""
    if mask is None:
        return None, None, 0, 0
    arr = _f64(mask)
    if arr.ndim == 2:
        arr = arr[None]
    if arr.shape[1:] != (Sq, Skv) or arr.shape[0] not in (1, B):
        raise ValueError(f"mask must be [B or 1, {Sq}, {Skv}]")
    arr = np.ascontiguousarray(arr)
    return arr, _ptr(arr), (Sq * Skv if arr.shape[0] == B and B > 1 else 0), Skv


def e4m3_value(code, lib=None):
    """The value of one fp8 e4m3 code (0..255)."""
    return (lib or load()).oracle_e4m3_value(int(code))


def attention_fp8(q, k_codes, v_codes, k_scale, v_scale, *, scale, causal=True, q_offset=0, softcap=0.0,
                  alibi_max_bias=0.0, sinks=None, window=0, mask=None, lib=None):
    """attention_ex() over an fp8 e4m3 K/V cache: codes uint8 [B, Skv, Hkv, D]
    (or torch float8_e4m3fn), one fp32 scale per K/V head for K and for V."""
    lib = lib or load()
    q = _f64(q)
    kc, vc = _codes(k_codes), _codes(v_codes)
    B, Sq, Hq, D = q.shape
    _, Skv, Hkv, _ = kc.shape
    ks, vs = _f64(k_scale).reshape(-1), _f64(v_scale).reshape(-1)
    if ks.shape[0] != Hkv or vs.shape[0] != Hkv:
        raise ValueError("one K and one V scale per K/V head")
    sk, skp = _sinks_arg(sinks)
    mk, mkp, msb, mss = _mask_arg(mask, B, Sq, Skv)
    out = np.zeros((B, Sq, Hq, D), dtype=np.float64)
    lse = np.zeros((B, Hq, Sq), dtype=np.float64)
    _bp = ctypes.POINTER(ctypes.c_ubyte)
    lib.oracle_attention_fp8(_ptr(q), kc.ctypes.data_as(_bp), vc.ctypes.data_as(_bp), _ptr(ks), _ptr(vs),
                             _ptr(out), _ptr(lse), B, Hq, Hkv, Sq, Skv, D, int(q_offset), int(bool(causal)),
                             float(scale), float(softcap), float(alibi_max_bias), skp, int(window), mkp, msb, mss)
    return out, lse


def _codes(x):
    """uint8 codes of an fp8 array (numpy uint8, or a torch uint8 / float8 tensor)."""
    if hasattr(x, "detach"):  # torch tensor: reinterpret float8 storage as bytes
        import torch
        x = x.detach().to("cpu")
        if x.dtype != torch.uint8:
            x = x.view(torch.uint8)
        x = x.numpy()
    x = np.ascontiguousarray(x)
    if x.dtype != np.uint8:
        raise ValueError("fp8 codes must be uint8")
    return x


def _pad_v(k, v):
    """v widened to k's head size with zero columns, and the original Dv."""
    D, Dv = k.shape[-1], v.shape[-1]
    if Dv == D:
        return v, Dv
    if Dv > D or v.shape[:-1] != k.shape[:-1]:
        raise ValueError("v must have k's leading shape and at most D columns")
    pad = np.zeros(v.shape[:-1] + (D,), dtype=np.float64)
    pad[..., :Dv] = v
    return pad, Dv


def alibi_slope(h, Hq, max_bias, lib=None):
    return (lib or load()).oracle_alibi_slope(int(h), int(Hq), float(max_bias))


def attention_ex(q, k, v, *, scale, causal=True, q_offset=0, softcap=0.0, alibi_max_bias=0.0, sinks=None,
                 window=0, mask=None, lib=None):
    """attention() with softcap, ALiBi, sink logits [Hq], a sliding window and
    an additive mask [B or 1, Sq, Skv].  v may have Dv < D columns."""
    lib = lib or load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    v, Dv = _pad_v(k, v)
    B, Hq, Hkv, Sq, Skv, D = _dims(q, k)
    sk, skp = _sinks_arg(sinks)
    mk, mkp, msb, mss = _mask_arg(mask, B, Sq, Skv)
    out = np.zeros((B, Sq, Hq, D), dtype=np.float64)
    lse = np.zeros((B, Hq, Sq), dtype=np.float64)
    lib.oracle_attention_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Sq, Skv, D,
                            int(q_offset), int(bool(causal)), float(scale), float(softcap),
                            float(alibi_max_bias), skp, int(window), mkp, msb, mss)
    return np.ascontiguousarray(out[..., :Dv]), lse


def attention_rows_ex(q, k, v, rows, *, scale, causal=True, q_offset=0, softcap=0.0, alibi_max_bias=0.0,
                      sinks=None, window=0, mask=None, lib=None):
    """attention_ex() on selected (b, h, s) rows; v may have Dv < D columns."""
    lib = lib or load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    v, Dv = _pad_v(k, v)
    B, Hq, Hkv, Sq, Skv, D = _dims(q, k)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    n = rows.shape[0]
    sk, skp = _sinks_arg(sinks)
    mk, mkp, msb, mss = _mask_arg(mask, B, Sq, Skv)
    out = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    lib.oracle_attention_rows_ex(_ptr(q), _ptr(k), _ptr(v), rows.ctypes.data_as(_lp), n, _ptr(out), _ptr(lse),
                                 B, Hq, Hkv, Sq, Skv, D, int(q_offset), int(bool(causal)), float(scale),
                                 float(softcap), float(alibi_max_bias), skp, int(window), mkp, msb, mss)
    return np.ascontiguousarray(out[:, :Dv]), lse


def split_ex(q, k, v, num_splits, *, scale, causal=True, q_offset=0, softcap=0.0, alibi_max_bias=0.0,
             window=0, mask=None, lib=None):
    """split() with softcap, ALiBi, a window and an additive mask (sinks belong
    to the merge)."""
    lib = lib or load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Hkv, Sq, Skv, D = _dims(q, k)
    mk, mkp, msb, mss = _mask_arg(mask, B, Sq, Skv)
    pout = np.zeros((num_splits, B, Sq, Hq, D), dtype=np.float64)
    plse = np.zeros((num_splits, B, Hq, Sq), dtype=np.float64)
    lib.oracle_split_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(pout), _ptr(plse), B, Hq, Hkv, Sq, Skv, D,
                        int(q_offset), int(bool(causal)), float(scale), int(num_splits), float(softcap),
                        float(alibi_max_bias), int(window), mkp, msb, mss)
    return pout, plse


def merge_ex(pout, plse, sinks=None, lib=None):
    """merge() with optional sink logits [Hq] in the denominator."""
    lib = lib or load()
    pout, plse = _f64(pout), _f64(plse)
    S, B, Sq, Hq, D = pout.shape
    sk, skp = _sinks_arg(sinks)
    out = np.zeros((B, Sq, Hq, D), dtype=np.float64)
    lse = np.zeros((B, Hq, Sq), dtype=np.float64)
    lib.oracle_merge_ex(_ptr(pout), _ptr(plse), _ptr(out), _ptr(lse), B, Hq, Sq, D, S, skp)
    return out, lse
