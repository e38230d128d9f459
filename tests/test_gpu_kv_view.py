"""Split-KV decode over strided and paged K/V views with per-sequence lengths,
through attn_decode_split_kv, vs the float64 oracle (B200)."""
import math

import numpy as np
import pytest
import torch

import gqa_flash_attention_attn_b200 as ga
from gqa_flash_attention_attn_b200.inputs import make_paged, make_qkv, make_seq_lens, make_sinks
import oracle
from parity import assert_lse_close, assert_o_close

pytestmark = pytest.mark.gpu


def _scale(D):
    return float(torch.tensor(1.0 / math.sqrt(D), dtype=torch.float32))


def _oracle_per_sequence(q, k, v, lens, *, scale, causal=True, **terms):
    """Oracle O [B,Sq,Hq,D] and LSE [B,Hq,Sq]: sequence b attends to its first
    lens[b] keys with its query rows at positions lens[b] - Sq + s."""
    B, Sq, Hq, D = q.shape
    out = np.zeros((B, Sq, Hq, D))
    lse = np.zeros((B, Hq, Sq))
    for b in range(B):
        n = int(lens[b])
        o, l = oracle.attention_ex(q[b:b + 1], k[b:b + 1, :n], v[b:b + 1, :n], scale=scale, causal=causal,
                                   q_offset=n - Sq, **terms)
        out[b] = o[0]
        lse[b] = l[0]
    return out, lse


# (B, Hq, Hkv, Sq, Skv, D, num_splits)
SHAPES = [(2, 16, 1, 1, 1024, 512, 4), (1, 32, 8, 8, 1024, 128, 4), (2, 8, 2, 3, 1024, 256, 2),
          (2, 32, 4, 2, 1024, 64, 4)]


@pytest.mark.parametrize("page_size", [16, 32, 64, 128, 256])
@pytest.mark.parametrize("shape", SHAPES, ids=[f"D{s[5]}g{s[1] // s[2]}Sq{s[3]}" for s in SHAPES])
def test_paged_partials_equal_contiguous(shape, page_size):
    """With 256-key splits (a multiple of 128) the paged and the contiguous
    runs visit the same tiles: their partials are bit-identical."""
    B, Hq, Hkv, Sq, Skv, D, S = shape
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=31)
    kc, vc, bt = make_paged(k, v, page_size, seed=32)
    q = q.cuda()
    po, pl = ga.decode_split(q, k.cuda(), v.cuda(), S, q_offset=Skv - Sq)
    po2, pl2 = ga.decode_split_kv(q, kc.cuda(), vc.cuda(), S, block_table=bt.cuda(), q_offset=Skv - Sq)
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    assert torch.equal(po, po2) and torch.equal(pl, pl2)


TERMS = [dict(), dict(softcap=20.0, alibi_max_bias=8.0, window=300), dict(window=40)]


@pytest.mark.parametrize("terms", TERMS, ids=["plain", "cap_alibi_w300", "w40"])
@pytest.mark.parametrize("page_size", [16, 64, 256])
def test_paged_seq_lens_match_oracle(page_size, terms):
    B, Hq, Hkv, Sq, D, S = 3, 16, 2, 4, 128, 5
    Skv = 700
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=33)
    kc, vc, bt = make_paged(k, v, page_size, seed=34)
    lens = make_seq_lens(B, Skv, seed=35, low=Sq)
    lens[0] = Skv                                   # one full-length sequence
    sinks = make_sinks(Hq, seed=36)
    out, lse = ga.decode_kv(q.cuda(), kc.cuda(), vc.cuda(), S, block_table=bt.cuda(), seq_lens=lens.cuda(),
                            out_dtype=torch.float32, sinks=sinks.cuda(), **terms)
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    want_o, want_l = _oracle_per_sequence(q, k, v, lens.numpy(), scale=_scale(D), sinks=sinks.numpy(), **terms)
    assert_o_close(out, want_o, f"paged {page_size} {terms}")
    assert_lse_close(lse, want_l, f"paged {page_size} {terms}")


def test_unpaged_seq_lens_match_oracle():
    """A padded [B, Skv_max] cache with a length per sequence (ragged batch)."""
    B, Hq, Hkv, Sq, Skv, D, S = 4, 16, 1, 1, 3000, 512, 8
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=37)
    lens = make_seq_lens(B, Skv, seed=38)
    lens[1] = 1                                      # a single key
    out, lse = ga.decode_kv(q.cuda(), k.cuda(), v.cuda(), S, seq_lens=lens.cuda(), out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    want_o, want_l = _oracle_per_sequence(q, k, v, lens.numpy(), scale=_scale(D))
    assert_o_close(out, want_o, "ragged")
    assert_lse_close(lse, want_l, "ragged")


def test_strided_views_equal_contiguous():
    """K and V interleaved in one tensor, and a head-major cache, as views:
    bit-identical to the contiguous run."""
    B, Hq, Hkv, Sq, Skv, D, S = 2, 32, 8, 8, 900, 128, 3
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=39)
    q = q.cuda()
    po, pl = ga.decode_split(q, k.cuda(), v.cuda(), S, q_offset=Skv - Sq)
    kv = torch.stack([k, v], dim=2).cuda()           # [B, Skv, 2, Hkv, D]
    po2, pl2 = ga.decode_split_kv(q, kv[:, :, 0], kv[:, :, 1], S, q_offset=Skv - Sq)
    kh = k.permute(0, 2, 1, 3).contiguous().cuda()   # [B, Hkv, Skv, D]
    vh = v.permute(0, 2, 1, 3).contiguous().cuda()
    po3, pl3 = ga.decode_split_kv(q, kh.permute(0, 2, 1, 3), vh.permute(0, 2, 1, 3), S, q_offset=Skv - Sq)
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    assert torch.equal(po, po2) and torch.equal(pl, pl2)
    assert torch.equal(po, po3) and torch.equal(pl, pl3)


def test_bad_lengths_are_clamped_and_reported():
    B, Hq, Hkv, Sq, Skv, D, S = 3, 16, 1, 1, 512, 512, 2
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=40)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    bad = torch.tensor([Skv + 77, -3, 100], dtype=torch.int32).cuda()
    good = torch.tensor([Skv, 0, 100], dtype=torch.int32).cuda()
    o1, l1 = ga.decode_kv(qc, kc, vc, S, seq_lens=bad, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_ERR_INVALID_ARG
    o2, l2 = ga.decode_kv(qc, kc, vc, S, seq_lens=good, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    # the empty sequence: no visible key
    assert float(o2[1].abs().max()) == 0.0 and bool(torch.isneginf(l2[1]).all())


def test_pages_outside_the_cache_read_as_zeros():
    """A block-table entry outside [0, num_pages) reads zeros (TMA fill), so
    those keys carry logit 0 and value 0."""
    B, Hq, Hkv, Sq, Skv, D, S, ps = 1, 16, 1, 1, 512, 512, 2, 64
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=41)
    kc, vc, bt = make_paged(k, v, ps, seed=42, extra_pages=0)
    bt2 = bt.clone()
    bt2[0, 2] = kc.shape[0]           # one past the last page
    bt2[0, 5] = -1
    out, lse = ga.decode_kv(q.cuda(), kc.cuda(), vc.cuda(), S, block_table=bt2.cuda(), q_offset=Skv - Sq,
                            out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    kz, vz = k.clone(), v.clone()
    for j in (2, 5):
        kz[0, j * ps:(j + 1) * ps] = 0
        vz[0, j * ps:(j + 1) * ps] = 0
    want_o, want_l = oracle.attention(q, kz, vz, scale=_scale(D), causal=True, q_offset=Skv - Sq)
    assert_o_close(out, want_o, "zero pages")
    assert_lse_close(lse, want_l, "zero pages")


def test_paged_workload_full_size_sampled():
    """The timed paged-decode workload, in its timed launch configuration."""
    from gqa_flash_attention_attn_b200.inputs import WORKLOADS, make_workload_inputs, sample_rows
    from parity import gather_rows, oracle_rows_by_batch
    w = WORKLOADS["paged_decode_d512_p64"]
    q, k, v = make_workload_inputs(w, seed=0)
    kc, vc, bt = make_paged(k, v, w.page_size, seed=0)
    out, lse = ga.decode_kv(q.cuda(), kc.cuda(), vc.cuda(), w.num_splits, block_table=bt.cuda(),
                            causal=w.causal, q_offset=w.q_offset, scale=w.scale)
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    rows = sample_rows(w, 40, seed=23)
    got_o, got_l = gather_rows(out, lse, rows)
    want_o, want_l = oracle_rows_by_batch(q, k, v, rows, scale=w.scale, causal=w.causal, q_offset=w.q_offset)
    assert_o_close(got_o, want_o, w.name)
    assert_lse_close(got_l, want_l, w.name)
