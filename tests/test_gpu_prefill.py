"""Prefill kernel vs the float64 oracle, through the C ABI (needs a B200)."""
import math

import numpy as np
import pytest
import torch

import gqa_flash_attention_attn_b200 as ga
from gqa_flash_attention_attn_b200.inputs import WORKLOADS, make_qkv, make_workload_inputs, sample_rows
import oracle
from parity import (oracle_attention_by_batch, assert_lse_close, assert_o_close, gather_rows, oracle_rows_by_batch)

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
    (1, 6, 1, 300, 300, 256, 0, True, torch.bfloat16),     # D = 256, group of 6: three CTA pairs per K/V head
    (1, 2, 2, 200, 333, 256, 133, True, torch.float32),    # D = 256, MHA: one CTA per head (no pair)
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


@pytest.mark.parametrize("name", ["tiny_causal_gqa_prefill", "gqa_causal_prefill_4k_d128", "prefill_at_depth_d256"])
def test_full_size_workload_every_row(name):
    """The timed prefill workloads at full size, in the launch configuration
    the benchmark times: every output row against the float64 oracle."""
    w = WORKLOADS[name]
    q, k, v = make_workload_inputs(w)
    odt = torch.float32 if w.out_dtype == "f32" else torch.bfloat16
    out, lse = ga.prefill(q.cuda(), k.cuda(), v.cuda(), causal=w.causal, q_offset=w.q_offset, scale=w.scale,
                          out_dtype=odt)
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    want_o, want_lse = oracle_attention_by_batch(q, k, v, scale=w.scale, causal=w.causal, q_offset=w.q_offset)
    assert_o_close(out, want_o, name)
    assert_lse_close(lse, want_lse, name)


# More work units than twice the persistent grid (148 CTAs on a B200), so
# every CTA runs several units and carries its barrier phases, TMEM buffers
# and K/V ring position from one unit to the next.
# (B, Hq, Hkv, Sq, Skv, D, q_offset, causal, out_dtype)
MULTI_UNIT = [
    (2, 32, 8, 2048, 2048, 128, 0, True, torch.bfloat16),     # 2 x 16 x 16 = 512 units, two head slots
    (2, 16, 8, 2048, 2048, 256, 0, True, torch.bfloat16),     # 2 x 16 x 16 = 512 units, one slot, S double buffered
    (3, 12, 4, 700, 1500, 128, 800, True, torch.float32),     # odd group (3): second slot idle in half the units
    (4, 8, 8, 640, 640, 64, 0, False, torch.bfloat16),        # non-causal D = 64, 160 equal units
]


@pytest.mark.parametrize("case", MULTI_UNIT, ids=[f"B{c[0]}H{c[1]}/{c[2]}S{c[3]}x{c[4]}D{c[5]}" for c in MULTI_UNIT])
def test_prefill_many_units_per_cta(case):
    B, Hq, Hkv, Sq, Skv, D, q_offset, causal, out_dtype = case
    q, k, v, scale, out, lse = _run(*case, seed=11)
    want_o, want_lse = oracle.attention(q, k, v, scale=scale, causal=causal, q_offset=q_offset)
    assert_o_close(out, want_o, str(case))
    assert_lse_close(lse, want_lse, str(case))


# D = 512 (the split-KV kernel in query-chunk mode):
# (B, Hq, Hkv, Sq, Skv, q_offset, causal, out_dtype, options)
WIDE = [
    (1, 4, 1, 300, 300, 0, True, torch.float32, {}),                 # group 4: 8 rows per CTA
    (2, 16, 1, 130, 130, 0, True, torch.bfloat16, {}),               # group 16: 2 rows per CTA
    (1, 8, 8, 77, 500, 423, True, torch.bfloat16, {}),               # MHA at depth, 32 rows per CTA
    (1, 8, 2, 64, 333, 0, False, torch.float32, {}),                 # non-causal, ragged keys
    (1, 8, 1, 100, 400, 300, True, torch.float32,
     dict(softcap=20.0, alibi_max_bias=4.0, window=150, sinks=True, mask=True)),
]


@pytest.mark.parametrize("case", WIDE, ids=[f"w{i}" for i in range(len(WIDE))])
def test_prefill_d512_matches_oracle(case):
    from gqa_flash_attention_attn_b200.inputs import make_mask, make_sinks
    B, Hq, Hkv, Sq, Skv, q_offset, causal, out_dtype, opts = case
    D = 512
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=61)
    scale = float(torch.tensor(1.0 / math.sqrt(D), dtype=torch.float32))
    kw = {kk: vv for kk, vv in opts.items() if kk not in ("sinks", "mask")}
    sinks = make_sinks(Hq, seed=62) if opts.get("sinks") else None
    mask = make_mask(B, Sq, Skv, seed=63) if opts.get("mask") else None
    out, lse = ga.prefill(q.cuda(), k.cuda(), v.cuda(), causal=causal, q_offset=q_offset, scale=scale,
                          out_dtype=out_dtype, sinks=None if sinks is None else sinks.cuda(),
                          mask=None if mask is None else mask.cuda(), **kw)
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    want_o, want_l = oracle.attention_ex(q, k, v, scale=scale, causal=causal, q_offset=q_offset,
                                         sinks=None if sinks is None else sinks.numpy(), mask=mask, **kw)
    assert out.dtype == out_dtype
    assert_o_close(out, want_o, str(case))
    assert_lse_close(lse, want_l, str(case))


def test_prefill_d512_workload_full_size_sampled():
    """The timed D = 512 prefill workload, in its timed launch configuration."""
    w = WORKLOADS["prefill_d512_g16_4k"]
    q, k, v = make_workload_inputs(w, seed=0)
    out, lse = ga.prefill(q.cuda(), k.cuda(), v.cuda(), causal=w.causal, q_offset=w.q_offset, scale=w.scale)
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    rows = sample_rows(w, 40, seed=31)
    got_o, got_l = gather_rows(out, lse, rows)
    want_o, want_l = oracle_rows_by_batch(q, k, v, rows, scale=w.scale, causal=w.causal, q_offset=w.q_offset)
    assert_o_close(got_o, want_o, w.name)
    assert_lse_close(got_l, want_l, w.name)
