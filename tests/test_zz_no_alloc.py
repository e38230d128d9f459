"""attn_decode_noalloc: split-KV decode for callers that cannot allocate a
device workspace (plugin hosts that own the device memory pool; decode loops
that must not call cudaMalloc).  Its partials live in the library's fixed
device array; these tests call it through the C ABI and compare it with the
workspace-based decode (attn_decode_split + attn_merge) on the same inputs.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import gqa_flash_attention_attn_b200 as ga
from gqa_flash_attention_attn_b200 import build as gbuild
from gqa_flash_attention_attn_b200.inputs import make_qkv
from parity import O_MAXABS, O_RMSE, LSE_ABS


def _call(lib, q, k, v, out, lse, num_splits, causal, q_offset, scale):
    B, Sq, Hq, D = q.shape
    _, Skv, Hkv, _ = k.shape
    odt = 1 if out.dtype == torch.float32 else 0
    return lib.attn_decode_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                   ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                                   ctypes.c_void_p(lse.data_ptr()), B, Hq, Hkv, Sq, Skv, D, q_offset,
                                   int(causal), scale, num_splits, odt,
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _close(got_o, got_l, ref_o, ref_l):
    err = (got_o.double() - ref_o.double()).abs()
    assert err.max().item() <= O_MAXABS
    assert math.sqrt((err * err).mean().item()) <= O_RMSE
    assert (got_l - ref_l).abs().max().item() <= LSE_ABS


@pytest.mark.gpu
def test_noalloc_matches_workspace_decode_on_two_calls_in_a_row():
    lib = ga.library()
    # Two different problems back to back: the second call finds the first
    # call's partials in the shared array and must not be affected by them.
    problems = [
        # (B, Hq, Hkv, Sq, Skv, D, q_offset, num_splits)
        (4, 32, 8, 8, 4096, 128, 4088, 16),   # 8 verify rows per sequence
        (2, 16, 1, 1, 3000, 512, 2999, 7),    # one query row, D = 512, fewer splits
    ]
    for i, (B, Hq, Hkv, Sq, Skv, D, q_offset, S) in enumerate(problems):
        q, k, v = (t.cuda() for t in make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=20 + i))
        scale = float(torch.tensor(1.0 / math.sqrt(D), dtype=torch.float32))
        ref_o, ref_l = ga.decode(q, k, v, S, causal=True, q_offset=q_offset, scale=scale,
                                 out_dtype=torch.float32)
        out = torch.full((B, Sq, Hq, D), float("nan"), device="cuda")
        lse = torch.full((B, Hq, Sq), float("nan"), device="cuda")
        assert _call(lib, q, k, v, out, lse, S, True, q_offset, scale) == ga.ATTN_OK
        torch.cuda.synchronize()
        assert ga.last_status() == ga.ATTN_OK
        _close(out, lse, ref_o, ref_l)


@pytest.mark.gpu
def test_noalloc_rejects_problems_beyond_its_scratch():
    gbuild.build()
    lib = ga.library()
    q, k, v = (t.cuda() for t in make_qkv(1, 16, 1, 1, 256, 512, seed=0))
    out = torch.empty((64, 1, 16, 512), device="cuda")
    lse = torch.empty((64, 16, 1), device="cuda")
    # 256 splits x 64 batch x 16 heads x 512 x 4 bytes = 128 MiB of partials
    big_q = torch.empty((64, 1, 16, 512), dtype=torch.bfloat16, device="cuda")
    big_k = torch.empty((64, 256, 1, 512), dtype=torch.bfloat16, device="cuda")
    st = _call(lib, big_q, big_k, big_k, out, lse, 256, True, 255, 0.04)
    assert st == ga.ATTN_ERR_TOO_LARGE
    assert ga.status_string(st) == "problem exceeds the fixed no-alloc scratch"
