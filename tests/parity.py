"""Comparison helpers for GPU-vs-oracle parity tests.

Tolerances for floating-point results (bf16 inputs, fp32 accumulation):
    O    max-abs error <= 2e-2 and RMSE <= 2e-3
    LSE  abs error <= 1e-3 (rows with no visible key must be exactly -inf)
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

O_MAXABS = 2e-2
O_RMSE = 2e-3
LSE_ABS = 1e-3


def to_f64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu").double().numpy()
    return np.asarray(t, dtype=np.float64)


def o_errors(got, want):
    err = to_f64(got) - to_f64(want)
    if err.size == 0:
        return 0.0, 0.0
    return float(np.abs(err).max()), float(np.sqrt(np.mean(err * err)))


def assert_o_close(got, want, what=""):
    g = to_f64(got)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    mx, rmse = o_errors(g, want)
    assert mx <= O_MAXABS and rmse <= O_RMSE, f"{what}: O max-abs {mx:.3e} rmse {rmse:.3e}"


def assert_lse_close(got, want, what=""):
    g, w = to_f64(got), to_f64(want)
    ninf = np.isneginf(w)
    assert np.array_equal(np.isneginf(g), ninf), f"{what}: -inf pattern differs"
    if (~ninf).any():
        err = np.abs(g[~ninf] - w[~ninf]).max()
        assert err <= LSE_ABS, f"{what}: LSE abs error {err:.3e}"


def oracle_rows_by_batch(q, k, v, rows, *, scale, causal, q_offset, **terms):
    """Oracle O rows [n, Dv] and LSE [n] for (b, h, s) triples, slicing per batch so
    only one batch entry is widened to float64 at a time.  terms (softcap,
    sinks, ...) or a V narrower than K go through attention_rows_ex."""
    rows = np.asarray(rows, dtype=np.int64).reshape(-1, 3)
    Dv = v.shape[3]
    fn = oracle.attention_rows_ex if (terms or Dv != k.shape[3]) else oracle.attention_rows
    out = np.zeros((rows.shape[0], Dv))
    lse = np.zeros((rows.shape[0],))
    for b in np.unique(rows[:, 0]):
        sel = np.nonzero(rows[:, 0] == b)[0]
        sub = rows[sel].copy()
        sub[:, 0] = 0
        o, l = fn(q[b:b + 1], k[b:b + 1], v[b:b + 1], sub, scale=scale, causal=causal, q_offset=q_offset, **terms)
        out[sel] = o
        lse[sel] = l
    return out, lse


def oracle_attention_by_batch(q, k, v, *, scale, causal, q_offset):
    """oracle.attention over every row, one batch entry at a time, so only
    one sequence's K/V is widened to float64 at once (a 32K-key decode cache
    is gigabytes in float64)."""
    B, Sq, Hq, _ = q.shape
    Dv = v.shape[3]
    out = np.zeros((B, Sq, Hq, Dv))
    lse = np.zeros((B, Hq, Sq))
    for b in range(B):
        o, l = oracle.attention(q[b:b + 1], k[b:b + 1], v[b:b + 1], scale=scale, causal=causal, q_offset=q_offset)
        out[b] = o[0]
        lse[b] = l[0]
    return out, lse


def gather_rows(out, lse, rows):
    """GPU O [B,Sq,Hq,D] and LSE [B,Hq,Sq] at (b, h, s) triples."""
    rows = torch.as_tensor(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    b, h, s = rows[:, 0], rows[:, 1], rows[:, 2]
    o = out.detach().to("cpu")[b, s, h]
    l = lse.detach().to("cpu")[b, h, s] if lse is not None else None
    return o, l
