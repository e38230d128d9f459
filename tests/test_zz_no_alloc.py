"""attn_decode_noalloc: split-KV decode for callers that cannot allocate a
device workspace (plugin hosts that own the device memory pool; decode loops
that must not call cudaMalloc).  Its partials live in the library's fixed
device array.  These tests call it through the C ABI and compare it with the
workspace-based decode (attn_decode_split + attn_merge) on the same inputs,
and with the float64 oracle.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import gqa_flash_attention_attn_b200 as ga
from gqa_flash_attention_attn_b200.inputs import make_qkv
import oracle
from parity import O_MAXABS, O_RMSE, LSE_ABS, assert_lse_close, assert_o_close

# ATTN_NOALLOC_SCRATCH_BYTES in include/attn.h
SCRATCH_BYTES = 24 * 1024 * 1024


def _call(lib, q, k, v, out, lse, num_splits, causal, q_offset, scale):
    B, Sq, Hq, D = q.shape
    _, Skv, Hkv, _ = k.shape
    odt = 1 if out.dtype == torch.float32 else 0
    return lib.attn_decode_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                   ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                                   ctypes.c_void_p(lse.data_ptr()), B, Hq, Hkv, Sq, Skv, D, q_offset,
                                   int(causal), scale, num_splits, odt,
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _scratch_need(B, Hq, Sq, D, S):
    """Bytes of the scratch array a call uses: partial O, then partial LSE at
    the next 256-byte boundary (as the entry point lays them out)."""
    return ((S * B * Sq * Hq * D * 4 + 255) // 256) * 256 + S * B * Hq * Sq * 4


def _close(got_o, got_l, ref_o, ref_l):
    err = (got_o.double() - ref_o.double()).abs()
    assert err.max().item() <= O_MAXABS
    assert math.sqrt((err * err).mean().item()) <= O_RMSE
    fin = torch.isfinite(ref_l)
    assert torch.equal(torch.isneginf(got_l), torch.isneginf(ref_l))
    assert (got_l[fin] - ref_l[fin]).abs().max().item() <= LSE_ABS


@pytest.mark.gpu
def test_noalloc_matches_workspace_decode_and_oracle_on_calls_in_a_row():
    lib = ga.library()
    # Problems back to back: each call finds the previous call's partials in
    # the shared array and must not be affected by them.  The third leaves
    # empty or wholly masked splits (which publish lse = -inf, O = 0) where
    # the first two left finite partials.
    problems = [
        # (B, Hq, Hkv, Sq, Skv, D, q_offset, num_splits)
        (4, 32, 8, 8, 4096, 128, 4088, 16),   # 8 verify rows per sequence
        (2, 16, 1, 1, 3000, 512, 2999, 7),    # one query row, D = 512, fewer splits
        (2, 16, 2, 8, 1000, 128, 2, 9),       # causal rows see keys <= 9: splits 1-8 wholly masked
        (1, 8, 1, 1, 9, 128, 8, 4),           # 9 keys in chunks of 3: the fourth split is empty
    ]
    for i, (B, Hq, Hkv, Sq, Skv, D, q_offset, S) in enumerate(problems):
        qh, kh, vh = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=20 + i)
        q, k, v = qh.cuda(), kh.cuda(), vh.cuda()
        scale = float(torch.tensor(1.0 / math.sqrt(D), dtype=torch.float32))
        ref_o, ref_l = ga.decode(q, k, v, S, causal=True, q_offset=q_offset, scale=scale,
                                 out_dtype=torch.float32)
        out = torch.full((B, Sq, Hq, D), float("nan"), device="cuda")
        lse = torch.full((B, Hq, Sq), float("nan"), device="cuda")
        assert _call(lib, q, k, v, out, lse, S, True, q_offset, scale) == ga.ATTN_OK
        torch.cuda.synchronize()
        assert ga.last_status() == ga.ATTN_OK
        _close(out, lse, ref_o, ref_l)
        want_o, want_l = oracle.attention(qh, kh, vh, scale=scale, causal=True, q_offset=q_offset)
        assert_o_close(out, want_o, f"noalloc {i}")
        assert_lse_close(lse, want_l, f"noalloc {i}")


@pytest.mark.gpu
def test_noalloc_capacity_boundary():
    lib = ga.library()
    # B1 Hq16 Hkv1 Sq1 D512: 32 832 bytes of partials per split.  The largest
    # split count that fits is accepted (and correct); one split more is
    # rejected on the host before anything is launched.
    B, Hq, Hkv, Sq, Skv, D = 1, 16, 1, 1, 2000, 512
    s_max = max(S for S in range(1, Skv + 1) if _scratch_need(B, Hq, Sq, D, S) <= SCRATCH_BYTES)
    assert _scratch_need(B, Hq, Sq, D, s_max + 1) > SCRATCH_BYTES
    qh, kh, vh = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=30)
    q, k, v = qh.cuda(), kh.cuda(), vh.cuda()
    scale = float(torch.tensor(1.0 / math.sqrt(D), dtype=torch.float32))
    out = torch.full((B, Sq, Hq, D), float("nan"), device="cuda")
    lse = torch.full((B, Hq, Sq), float("nan"), device="cuda")
    assert _call(lib, q, k, v, out, lse, s_max, True, Skv - 1, scale) == ga.ATTN_OK
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    want_o, want_l = oracle.attention(qh, kh, vh, scale=scale, causal=True, q_offset=Skv - 1)
    assert_o_close(out, want_o, "noalloc at capacity")
    assert_lse_close(lse, want_l, "noalloc at capacity")

    out2 = torch.full_like(out, 7.0)
    st = _call(lib, q, k, v, out2, lse, s_max + 1, True, Skv - 1, scale)
    assert st == ga.ATTN_ERR_TOO_LARGE
    assert ga.status_string(st) == "problem exceeds the fixed no-alloc scratch"
    torch.cuda.synchronize()
    assert torch.all(out2 == 7.0)   # nothing ran


@pytest.mark.gpu
def test_noalloc_rejects_problems_far_beyond_its_scratch():
    lib = ga.library()
    out = torch.empty((64, 1, 16, 512), device="cuda")
    lse = torch.empty((64, 16, 1), device="cuda")
    # 256 splits x 64 batch x 16 heads x 512 x 4 bytes = 128 MiB of partials
    big_q = torch.empty((64, 1, 16, 512), dtype=torch.bfloat16, device="cuda")
    big_k = torch.empty((64, 256, 1, 512), dtype=torch.bfloat16, device="cuda")
    st = _call(lib, big_q, big_k, big_k, out, lse, 256, True, 255, 0.04)
    assert st == ga.ATTN_ERR_TOO_LARGE
