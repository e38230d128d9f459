"""Split-KV decode and LSE merge vs the float64 oracle, through the C ABI (B200)."""
import math

import numpy as np
import pytest
import torch

import gqa_flash_attention_attn_b200 as ga
from gqa_flash_attention_attn_b200.inputs import WORKLOADS, make_qkv, make_workload_inputs, sample_rows
import oracle
from parity import (oracle_attention_by_batch, assert_lse_close, assert_o_close, gather_rows, oracle_rows_by_batch, to_f64)

pytestmark = pytest.mark.gpu

# (B, Hq, Hkv, Sq, Skv, D, q_offset, causal, num_splits)
CASES = [
    (2, 16, 1, 1, 1000, 512, 999, True, 4),     # single-query decode, D = 512
    (1, 32, 8, 8, 700, 128, 692, True, 3),      # 8 draft rows per sequence
    (2, 8, 2, 3, 500, 256, 497, True, 5),
    (1, 4, 4, 1, 1, 128, 0, True, 1),           # one key
    (1, 8, 1, 1, 100, 128, 99, True, 30),       # splits 25..29 hold no key
    (1, 4, 1, 8, 1000, 128, 0, True, 9),        # causal at q_offset 0: most splits fully masked
    (1, 16, 4, 2, 300, 512, 298, True, 2),      # 8 rows padded to 16
    (1, 8, 1, 1, 777, 128, 0, False, 6),        # non-causal
    (1, 16, 2, 8, 515, 128, 507, True, 1),      # 64 rows, one split, ragged tail
    # D = 64: one 64-column box per K and V tile
    (2, 8, 1, 1, 1000, 64, 999, True, 4),       # single-query decode
    (1, 32, 8, 8, 700, 64, 692, True, 3),       # 8 draft rows per sequence (32 rows per K/V head)
    (1, 8, 1, 1, 100, 64, 99, True, 30),        # splits 25..29 hold no key
    (1, 4, 1, 8, 1000, 64, 0, True, 9),         # causal at q_offset 0: most splits fully masked
    (1, 8, 1, 1, 777, 64, 0, False, 6),         # non-causal
    (1, 80, 8, 8, 333, 64, 325, True, 2),       # 80 rows per K/V head (the D = 64 limit), ragged
]


def _scale(D):
    return float(torch.tensor(1.0 / math.sqrt(D), dtype=torch.float32))


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}H{c[1]}/{c[2]}S{c[3]}x{c[4]}D{c[5]}o{c[6]}S{c[8]}" for c in CASES])
def test_decode_split_and_merge_match_oracle(case):
    B, Hq, Hkv, Sq, Skv, D, q_offset, causal, S = case
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=1)
    scale = _scale(D)
    po, pl = ga.decode_split(q.cuda(), k.cuda(), v.cuda(), S, causal=causal, q_offset=q_offset, scale=scale)
    out, lse = ga.merge(po, pl, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    want_po, want_pl = oracle.split(q, k, v, S, scale=scale, causal=causal, q_offset=q_offset)
    # every split publishes: the -inf pattern of the partial LSE is exact
    assert_lse_close(pl, want_pl, f"partial lse {case}")
    assert_o_close(po, want_po, f"partial out {case}")
    want_o, want_lse = oracle.attention(q, k, v, scale=scale, causal=causal, q_offset=q_offset)
    assert_o_close(out, want_o, f"merged {case}")
    assert_lse_close(lse, want_lse, f"merged {case}")


def test_merge_of_oracle_partials():
    # the merge kernel alone, on partials (including -inf splits) from the oracle
    B, Hq, Hkv, Sq, Skv, D, S = 2, 8, 2, 4, 90, 128, 16
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=2)
    scale = _scale(D)
    po, pl = oracle.split(q, k, v, S, scale=scale, causal=True, q_offset=20)
    assert np.isneginf(pl).any()
    out, lse = ga.merge(torch.from_numpy(po).float().cuda(), torch.from_numpy(pl).float().cuda(),
                        out_dtype=torch.float32)
    want_o, want_lse = oracle.merge(po, pl)
    assert_o_close(out, want_o, "merge")
    assert_lse_close(lse, want_lse, "merge")


def test_merge_all_splits_empty_gives_zero_and_neg_inf():
    po = torch.zeros((3, 1, 2, 4, 128), device="cuda")
    pl = torch.full((3, 1, 4, 2), float("-inf"), device="cuda")
    out, lse = ga.merge(po, pl, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.all(out == 0)
    assert torch.all(torch.isneginf(lse))


def test_split_count_does_not_change_result():
    B, Hq, Hkv, Sq, Skv, D = 1, 16, 2, 4, 2000, 128
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=4)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    ref_o, ref_l = ga.prefill(qc, kc, vc, causal=True, q_offset=Skv - Sq, out_dtype=torch.float32)
    for S in (1, 2, 7, 16, 63):
        o, l = ga.decode(qc, kc, vc, S, causal=True, q_offset=Skv - Sq, out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert (o - ref_o).abs().max().item() < 2e-2
        assert (l - ref_l).abs().max().item() < 1e-3


@pytest.mark.parametrize("name", ["split_kv_decode_d512", "spec_verify_decode_d128"])
def test_full_size_workload_every_row(name):
    """The timed decode workloads at full size, in the launch configuration
    the benchmark times (decode_split with its split count, then merge):
    every output row against the float64 oracle."""
    w = WORKLOADS[name]
    q, k, v = make_workload_inputs(w)
    po, pl = ga.decode_split(q.cuda(), k.cuda(), v.cuda(), w.num_splits, causal=w.causal, q_offset=w.q_offset,
                             scale=w.scale)
    out, lse = ga.merge(po, pl, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    want_o, want_lse = oracle_attention_by_batch(q, k, v, scale=w.scale, causal=w.causal, q_offset=w.q_offset)
    assert_o_close(out, want_o, name)
    assert_lse_close(lse, want_lse, name)


# (B, Hq, Hkv, Sq, Skv, D, q_offset, causal, num_splits): enough CTAs that each
# takes a group of consecutive splits (3, 4 and 8 per CTA on a 148-SM part)
GROUPED = [
    (100, 8, 1, 1, 300, 128, 299, True, 7),      # groups of 3, the last of 1
    (64, 16, 2, 2, 513, 256, 100, True, 9),      # causal: splits past key 101 empty inside groups
    (128, 8, 4, 1, 2048, 128, 2047, True, 8),    # groups of 8
    (40, 16, 1, 1, 1000, 512, 0, False, 30),     # non-causal D512, groups of 3
    (128, 8, 2, 1, 2048, 64, 2047, True, 8),     # D64, groups of 8
    (64, 16, 2, 2, 513, 64, 100, True, 9),       # D64, causal: empty splits inside groups
]


@pytest.mark.parametrize("case", GROUPED, ids=[f"B{c[0]}H{c[1]}/{c[2]}x{c[4]}D{c[5]}S{c[8]}" for c in GROUPED])
def test_grouped_splits_publish_every_partial(case):
    B, Hq, Hkv, Sq, Skv, D, q_offset, causal, S = case
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=81)
    scale = _scale(D)
    po, pl = ga.decode_split(q.cuda(), k.cuda(), v.cuda(), S, causal=causal, q_offset=q_offset, scale=scale)
    out, lse = ga.merge(po, pl, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    want_po, want_pl = oracle.split(q, k, v, S, scale=scale, causal=causal, q_offset=q_offset)
    assert_lse_close(pl, want_pl, f"partial lse {case}")
    assert_o_close(po, want_po, f"partial out {case}")
    want_o, want_lse = oracle.merge(want_po, want_pl)
    assert_o_close(out, want_o, f"merged {case}")
    assert_lse_close(lse, want_lse, f"merged {case}")
