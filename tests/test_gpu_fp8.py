"""Split-KV decode over an fp8 e4m3 K/V cache (per-head scales), through
attn_decode_split_kv, vs the float64 oracle's fp8 attention (B200)."""
import math

import numpy as np
import pytest
import torch

import gqa_flash_attention_attn_b200 as ga
from gqa_flash_attention_attn_b200.inputs import (WORKLOADS, make_fp8_kv, make_mask, make_paged, make_qkv,
                                                  make_sinks, make_workload_inputs, sample_rows)
import oracle
from parity import assert_lse_close, assert_o_close, gather_rows

pytestmark = pytest.mark.gpu


def _scale(D):
    return float(torch.tensor(1.0 / math.sqrt(D), dtype=torch.float32))


def _dequant(codes, sc):
    return codes.view(torch.float8_e4m3fn).double() * sc.double().view(1, 1, -1, 1)


# (B, Hq, Hkv, Sq, Skv, D, q_offset, causal, num_splits, q_mult)
CASES = [
    (2, 16, 1, 1, 1000, 512, 999, True, 4, 1.0),       # single-query decode, D = 512
    (1, 32, 8, 8, 700, 128, 692, True, 3, 1.0),        # 8 draft rows per sequence
    (2, 8, 2, 3, 500, 256, 497, True, 5, 1.0),
    (1, 8, 1, 1, 100, 128, 99, True, 30, 1.0),         # empty splits
    (1, 8, 1, 1, 777, 128, 0, False, 6, 1.0),          # non-causal
    (1, 16, 2, 4, 640, 128, 636, True, 2, 20.0),       # large |q|: the power-of-two Q scale
    (1, 16, 2, 4, 640, 256, 636, True, 2, 1e-3),       # small |q|
]


@pytest.mark.parametrize("case", CASES, ids=[f"H{c[1]}/{c[2]}S{c[3]}x{c[4]}D{c[5]}S{c[8]}q{c[9]}" for c in CASES])
def test_fp8_decode_matches_oracle(case):
    B, Hq, Hkv, Sq, Skv, D, q_offset, causal, S, qm = case
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=71)
    q = (q.float() * qm).to(torch.bfloat16)
    kc, vc, ks, vs = make_fp8_kv(k, v)
    scale = _scale(D)
    po, pl = ga.decode_split_kv(q.cuda(), kc.cuda(), vc.cuda(), S, causal=causal, q_offset=q_offset, scale=scale,
                                k_scale=ks.cuda(), v_scale=vs.cuda())
    out, lse = ga.merge(po, pl, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    kd, vd = _dequant(kc, ks), _dequant(vc, vs)
    want_po, want_pl = oracle.split(q, kd, vd, S, scale=scale, causal=causal, q_offset=q_offset)
    assert_lse_close(pl, want_pl, f"partial lse {case}")
    assert_o_close(po, want_po, f"partial out {case}")
    want_o, want_l = oracle.attention_fp8(q, kc, vc, ks, vs, scale=scale, causal=causal, q_offset=q_offset)
    assert_o_close(out, want_o, f"merged {case}")
    assert_lse_close(lse, want_l, f"merged {case}")


def test_fp8_paged_with_every_term():
    B, Hq, Hkv, Sq, Skv, D, S = 2, 16, 2, 4, 1024, 128, 4
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=72)
    kc, vc, ks, vs = make_fp8_kv(k, v)
    kp, vp, bt = make_paged(kc, vc, 64, seed=73)
    mask = make_mask(B, Sq, Skv, seed=74)
    sinks = make_sinks(Hq, seed=75)
    terms = dict(softcap=20.0, alibi_max_bias=4.0, window=600)
    out, lse = ga.decode_kv(q.cuda(), kp.cuda(), vp.cuda(), S, block_table=bt.cuda(), q_offset=Skv - Sq,
                            out_dtype=torch.float32, k_scale=ks.cuda(), v_scale=vs.cuda(), sinks=sinks.cuda(),
                            mask=mask.cuda(), **terms)
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    want_o, want_l = oracle.attention_fp8(q, kc, vc, ks, vs, scale=_scale(D), causal=True, q_offset=Skv - Sq,
                                          sinks=sinks.numpy(), mask=mask, **terms)
    assert_o_close(out, want_o, "fp8 paged, every term")
    assert_lse_close(lse, want_l, "fp8 paged, every term")


@pytest.mark.parametrize("name", [n for n, w in WORKLOADS.items() if w.kv_dtype == "fp8"])
def test_fp8_workload_full_size_sampled(name):
    """Each timed fp8 workload, in its timed launch configuration, on sampled rows."""
    w = WORKLOADS[name]
    q, k, v = make_workload_inputs(w, seed=0)
    kc, vc, ks, vs = make_fp8_kv(k, v)
    out, lse = ga.decode_kv(q.cuda(), kc.cuda(), vc.cuda(), w.num_splits, causal=w.causal, q_offset=w.q_offset,
                            scale=w.scale, k_scale=ks.cuda(), v_scale=vs.cuda())
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    rows = sample_rows(w, 32, seed=29)
    got_o, got_l = gather_rows(out, lse, rows)
    rows_np = np.asarray(rows, dtype=np.int64)
    want_o = np.zeros((len(rows), w.D))
    want_l = np.zeros((len(rows),))
    kd, vd = _dequant(kc, ks), _dequant(vc, vs)
    for b in np.unique(rows_np[:, 0]):
        sel = np.nonzero(rows_np[:, 0] == b)[0]
        sub = rows_np[sel].copy()
        sub[:, 0] = 0
        o, l = oracle.attention_rows(q[b:b + 1], kd[b:b + 1], vd[b:b + 1], sub, scale=w.scale, causal=w.causal,
                                     q_offset=w.q_offset)
        want_o[sel] = o
        want_l[sel] = l
    assert_o_close(got_o, want_o, name)
    assert_lse_close(got_l, want_l, name)
