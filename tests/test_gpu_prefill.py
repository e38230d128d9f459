"""Prefill kernel vs the float64 oracle, through the C ABI (needs a B200)."""
import math

import numpy as np
import pytest
import torch

import gqa_flash_attention_attn_b200 as ga
from gqa_flash_attention_attn_b200.inputs import WORKLOADS, make_qkv, make_workload_inputs, sample_rows
import oracle
from parity import (assert_lse_close, assert_o_close, gather_rows, oracle_rows_by_batch)

pytestmark = pytest.mark.gpu

# (B, Hq, Hkv, Sq, Skv, D, q_offset, causal, out_dtype)
CASES = [
    (1, 4, 1, 128, 128, 64, 0, True, torch.float32),      # tiny causal GQA prefill workload
    (2, 4, 2, 300, 300, 64, 0, True, torch.bfloat16),      # ragged tail, several tiles
    (1, 8, 2, 257, 257, 128, 0, True, torch.bfloat16),     # group of 4
    (1, 6, 2, 200, 200, 128, 0, True, torch.float32),      # odd group of 3
    (1, 2, 2, 130, 130, 128, 0, True, torch.bfloat16),     # MHA (group of 1)
    (1, 4, 2, 100, 400, 128, 300, True, torch.bfloat16),   # new rows at depth
    (1, 4, 2, 64, 500, 64, 0, False, torch.bfloat16),      # non-causal, Sq < Skv
    (1, 4, 4, 1, 1, 128, 0, True, torch.float32),          # one query, one key
    (1, 2, 1, 5, 1000, 128, 995, True, torch.bfloat16),    # few rows over a long prefix
    (1, 4, 2, 200, 200, 256, 0, True, torch.bfloat16),     # D = 256
    (1, 4, 2, 150, 700, 256, 550, True, torch.bfloat16),   # D = 256 at depth
    (1, 2, 1, 129, 129, 256, 0, False, torch.float32),
    (2, 8, 8, 128, 128, 64, 0, True, torch.bfloat16),
    (1, 4, 1, 300, 200, 128, 0, True, torch.bfloat16),     # Sq > Skv: late rows see every key
    (1, 4, 2, 256, 1100, 128, 0, False, torch.float32),    # non-causal, many tiles
]


def _run(B, Hq, Hkv, Sq, Skv, D, q_offset, causal, out_dtype, seed=0):
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=seed)
    scale = float(torch.tensor(1.0 / math.sqrt(D), dtype=torch.float32))
    out, lse = ga.prefill(q.cuda(), k.cuda(), v.cuda(), causal=causal, q_offset=q_offset, scale=scale,
                          out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    return q, k, v, scale, out, lse


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}H{c[1]}/{c[2]}S{c[3]}x{c[4]}D{c[5]}o{c[6]}{'c' if c[7] else 'n'}"
                                             for c in CASES])
def test_prefill_matches_oracle(case):
    B, Hq, Hkv, Sq, Skv, D, q_offset, causal, out_dtype = case
    q, k, v, scale, out, lse = _run(*case)
    want_o, want_lse = oracle.attention(q, k, v, scale=scale, causal=causal, q_offset=q_offset)
    assert out.dtype == out_dtype
    assert_o_close(out, want_o, str(case))
    assert_lse_close(lse, want_lse, str(case))


def test_single_visible_key_returns_value_row():
    # causal row 0 at q_offset 0 sees key 0 only: O = V[0], LSE = scale * q0.k0
    q, k, v, scale, out, lse = _run(1, 4, 2, 130, 130, 128, 0, True, torch.float32, seed=3)
    o = out.cpu()[0, 0]                       # [Hq, D]
    for h in range(4):
        vr = v[0, 0, h // 2].float()
        assert torch.allclose(o[h], vr, rtol=1e-6, atol=1e-6)
        z = scale * float((q[0, 0, h].double() * k[0, 0, h // 2].double()).sum())
        assert abs(float(lse.cpu()[0, h, 0]) - z) < 1e-3


def test_causal_rows_ignore_future_keys():
    B, Hq, Hkv, S, D = 1, 4, 2, 256, 128
    q, k, v = make_qkv(B, Hq, Hkv, S, S, D, seed=5)
    out1, lse1 = ga.prefill(q.cuda(), k.cuda(), v.cuda(), causal=True)
    k2, v2 = k.clone(), v.clone()
    cut = 150
    k2[:, cut + 1:] = torch.randn_like(k2[:, cut + 1:].float()).bfloat16()
    v2[:, cut + 1:] = torch.randn_like(v2[:, cut + 1:].float()).bfloat16()
    out2, lse2 = ga.prefill(q.cuda(), k2.cuda(), v2.cuda(), causal=True)
    torch.cuda.synchronize()
    assert torch.equal(out1[:, : cut + 1], out2[:, : cut + 1])
    assert torch.equal(lse1[:, :, : cut + 1], lse2[:, :, : cut + 1])


def test_repeated_calls_are_deterministic():
    q, k, v = make_qkv(1, 8, 2, 384, 384, 128, seed=7)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    a, la = ga.prefill(qc, kc, vc)
    b, lb = ga.prefill(qc, kc, vc)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(la, lb)


@pytest.mark.parametrize("name", ["gqa_causal_prefill_4k_d128", "prefill_at_depth_d256"])
def test_full_size_workload_sampled_rows(name):
    w = WORKLOADS[name]
    q, k, v = make_workload_inputs(w)
    out, lse = ga.prefill(q.cuda(), k.cuda(), v.cuda(), causal=w.causal, q_offset=w.q_offset, scale=w.scale,
                          out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    rows = sample_rows(w, 96)
    want_o, want_lse = oracle_rows_by_batch(q, k, v, rows, scale=w.scale, causal=w.causal, q_offset=w.q_offset)
    got_o, got_lse = gather_rows(out, lse, rows)
    assert_o_close(got_o, want_o, name)
    assert_lse_close(got_lse, want_lse, name)
    # every row, not only the sampled ones, is finite
    assert torch.isfinite(out).all()
    assert torch.isfinite(lse).all()
