"""Split-KV decode with the merge fused into one launch (attn_decode_fused:
the key ranges of each (sequence, K/V head) merge inside a thread-block
cluster), vs the float64 oracle (B200)."""
import math

import pytest
import torch

import gqa_flash_attention_attn_b200 as ga
from gqa_flash_attention_attn_b200.inputs import (WORKLOADS, make_fp8_kv, make_mask, make_paged, make_qkv,
                                                  make_seq_lens, make_sinks, make_workload_inputs, sample_rows)
import oracle
from parity import assert_lse_close, assert_o_close, gather_rows, oracle_rows_by_batch

pytestmark = pytest.mark.gpu


def _scale(D):
    return float(torch.tensor(1.0 / math.sqrt(D), dtype=torch.float32))


def _ok():
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK


# (B, Hq, Hkv, Sq, Skv, D, q_offset, causal, num_splits)
CASES = [
    (2, 16, 1, 1, 3000, 512, 2999, True, 32),     # 16 ranges
    (1, 32, 8, 8, 2000, 128, 1992, True, 8),      # 8 draft rows, 8 ranges
    (2, 8, 2, 3, 1500, 256, 1497, True, 4),
    (1, 16, 1, 1, 100, 512, 99, True, 16),        # ranges of 7 keys, most of them partial tiles
    (1, 8, 1, 1, 777, 128, 0, False, 3),          # non-causal, 2 ranges
    (2, 16, 2, 4, 640, 128, 636, True, 1),        # a cluster of one
    (1, 64, 8, 2, 5000, 128, 4998, True, 16),     # 16 rows per K/V head
    (2, 32, 4, 4, 1300, 64, 1296, True, 8),       # D = 64: 32 rows per K/V head, 8 ranges
]


@pytest.mark.parametrize("case", CASES, ids=[f"D{c[5]}g{c[1] // c[2]}Sq{c[3]}x{c[4]}S{c[8]}" for c in CASES])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_fused_matches_oracle(case, out_dtype):
    B, Hq, Hkv, Sq, Skv, D, q_offset, causal, S = case
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=101)
    scale = _scale(D)
    out, lse = ga.decode_fused(q.cuda(), k.cuda(), v.cuda(), S, causal=causal, q_offset=q_offset, scale=scale,
                               out_dtype=out_dtype)
    _ok()
    want_o, want_l = oracle.attention(q, k, v, scale=scale, causal=causal, q_offset=q_offset)
    assert_o_close(out, want_o, f"fused {case}")
    assert_lse_close(lse, want_l, f"fused {case}")


def test_fused_is_deterministic():
    B, Hq, Hkv, Sq, Skv, D, S = 2, 16, 1, 1, 4096, 512, 32
    q, k, v = (t.cuda() for t in make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=102))
    o1, l1 = ga.decode_fused(q, k, v, S, q_offset=Skv - Sq)
    o2, l2 = ga.decode_fused(q, k, v, S, q_offset=Skv - Sq)
    _ok()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


TERMS = [dict(softcap=20.0, alibi_max_bias=8.0, window=300), dict(mask=True), dict(window=50)]


@pytest.mark.parametrize("terms", TERMS, ids=["cap_alibi_w300", "mask", "w50"])
def test_fused_with_terms_and_sinks(terms):
    B, Hq, Hkv, Sq, Skv, D, S = 2, 32, 8, 4, 1800, 128, 8
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=103)
    sinks = make_sinks(Hq, seed=104)
    terms = dict(terms)
    if terms.pop("mask", False):
        terms["mask"] = make_mask(B, Sq, Skv, seed=105)
    dev = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in terms.items()}
    out, lse = ga.decode_fused(q.cuda(), k.cuda(), v.cuda(), S, q_offset=Skv - Sq, out_dtype=torch.float32,
                               sinks=sinks.cuda(), **dev)
    _ok()
    want_o, want_l = oracle.attention_ex(q, k, v, scale=_scale(D), causal=True, q_offset=Skv - Sq,
                                         sinks=sinks.numpy(), **terms)
    assert_o_close(out, want_o, f"terms {list(terms)}")
    assert_lse_close(lse, want_l, f"terms {list(terms)}")


@pytest.mark.parametrize("page_size", [16, 64, 256])
def test_fused_paged_seq_lens(page_size):
    B, Hq, Hkv, Sq, Skv, D, S = 3, 16, 1, 1, 2048, 512, 16
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=106)
    kc, vc, bt = make_paged(k, v, page_size, seed=107)
    lens = make_seq_lens(B, Skv, seed=108)
    lens[0] = Skv
    lens[2] = 1                                    # one key: every range but the first is empty
    out, lse = ga.decode_fused(q.cuda(), kc.cuda(), vc.cuda(), S, block_table=bt.cuda(), seq_lens=lens.cuda(),
                               out_dtype=torch.float32)
    _ok()
    for b in range(B):
        n = int(lens[b])
        wo, wl = oracle.attention(q[b:b + 1], k[b:b + 1, :n], v[b:b + 1, :n], scale=_scale(D), causal=True,
                                  q_offset=n - Sq)
        assert_o_close(out[b:b + 1], wo, f"len {n}")
        assert_lse_close(lse[b:b + 1], wl, f"len {n}")


@pytest.mark.parametrize("D,Sq,Hq", [(512, 1, 16), (128, 8, 32)], ids=["D512", "D128_verify"])
def test_fused_fp8(D, Sq, Hq):
    B, Hkv, Skv, S = 2, (1 if D == 512 else 8), 2500, 16
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=109)
    kc, vc, ks, vs = make_fp8_kv(k, v)
    out, lse = ga.decode_fused(q.cuda(), kc.cuda(), vc.cuda(), S, q_offset=Skv - Sq, k_scale=ks.cuda(),
                               v_scale=vs.cuda(), out_dtype=torch.float32)
    _ok()
    want_o, want_l = oracle.attention_fp8(q, kc, vc, ks, vs, scale=_scale(D), causal=True, q_offset=Skv - Sq)
    assert_o_close(out, want_o, f"fp8 D{D}")
    assert_lse_close(lse, want_l, f"fp8 D{D}")


def test_fused_latent_cache():
    """576-wide K with V its first 512 columns."""
    B, Hq, Hkv, Sq, Skv, D, Dv, S = 2, 16, 1, 1, 3000, 576, 512, 16
    q, k, _ = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=110)
    kc = k.cuda()
    out, lse = ga.decode_fused(q.cuda(), kc, kc[..., :Dv], S, q_offset=Skv - Sq, out_dtype=torch.float32)
    _ok()
    want_o, want_l = oracle.attention_ex(q, k, k[..., :Dv], scale=_scale(D), causal=True, q_offset=Skv - Sq)
    assert_o_close(out, want_o, "latent")
    assert_lse_close(lse, want_l, "latent")


@pytest.mark.parametrize("name", ["split_kv_decode_d512", "spec_verify_decode_d128"])
def test_fused_workload_full_size_sampled(name):
    w = WORKLOADS[name]
    q, k, v = make_workload_inputs(w, seed=0)
    out, lse = ga.decode_fused(q.cuda(), k.cuda(), v.cuda(), w.num_splits, causal=w.causal, q_offset=w.q_offset,
                               scale=w.scale)
    _ok()
    rows = sample_rows(w, 40, seed=31)
    got_o, got_l = gather_rows(out, lse, rows)
    want_o, want_l = oracle_rows_by_batch(q, k, v, rows, scale=w.scale, causal=w.causal, q_offset=w.q_offset)
    assert_o_close(got_o, want_o, w.name)
    assert_lse_close(got_l, want_l, w.name)
