"""V narrower than K (Dv < D: 576/512, 320/256, 192/128) in decode and
prefill, and prefill over K/V views (attn_prefill_kv: strided, paged, lengths
per sequence, fp8), vs the float64 oracle (B200)."""
import math

import numpy as np
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


def _qkv(B, Hq, Hkv, Sq, Skv, D, Dv, v_of_k, seed):
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=seed, Dv=Dv)
    if v_of_k:
        v = k[..., :Dv]
    return q, k, v


def _ok():
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK


# (B, Hq, Hkv, Sq, Skv, D, Dv, num_splits, v_of_k)
DECODE = [
    (2, 16, 1, 1, 1000, 576, 512, 4, True),     # latent cache: V = the first 512 columns of K
    (1, 32, 1, 1, 700, 576, 512, 3, False),     # 32 rows, the most TMEM holds at Dv = 512
    (2, 8, 2, 3, 900, 320, 256, 2, False),
    (1, 32, 8, 8, 1024, 192, 128, 4, False),    # 8 draft rows
    (2, 32, 1, 2, 333, 192, 128, 3, True),      # ragged tail
    (1, 16, 1, 1, 100, 576, 512, 30, True),     # empty splits
]


@pytest.mark.parametrize("case", DECODE, ids=[f"D{c[5]}v{c[6]}g{c[1] // c[2]}Sq{c[3]}x{c[4]}S{c[7]}"
                                              f"{'k' if c[8] else ''}" for c in DECODE])
def test_decode_narrow_v_matches_oracle(case):
    B, Hq, Hkv, Sq, Skv, D, Dv, S, vk = case
    q, k, v = _qkv(B, Hq, Hkv, Sq, Skv, D, Dv, vk, seed=81)
    kc = k.cuda()
    vc = kc[..., :Dv] if vk else v.cuda()
    scale = _scale(D)
    po, pl = ga.decode_split_kv(q.cuda(), kc, vc, S, q_offset=Skv - Sq, scale=scale)
    out, lse = ga.merge(po, pl, out_dtype=torch.float32)
    _ok()
    assert po.shape == (S, B, Sq, Hq, Dv) and out.shape == (B, Sq, Hq, Dv)
    want_o, want_l = oracle.attention_ex(q, k, v, scale=scale, causal=True, q_offset=Skv - Sq)
    assert_o_close(out, want_o, f"decode {case}")
    assert_lse_close(lse, want_l, f"decode {case}")


TERMS = [dict(softcap=20.0, alibi_max_bias=8.0, window=300), dict(mask=True)]


@pytest.mark.parametrize("terms", TERMS, ids=["cap_alibi_w300", "mask"])
@pytest.mark.parametrize("dims", [(576, 512), (192, 128)], ids=["576_512", "192_128"])
def test_decode_narrow_v_with_terms(dims, terms):
    D, Dv = dims
    B, Hq, Hkv, Sq, Skv, S = 2, 16, 1, 2, 800, 3
    q, k, v = _qkv(B, Hq, Hkv, Sq, Skv, D, Dv, D == 576, seed=82)
    sinks = make_sinks(Hq, seed=83)
    terms = dict(terms)
    if terms.pop("mask", False):
        terms["mask"] = make_mask(B, Sq, Skv, seed=84)
    dev = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in terms.items()}
    kc = k.cuda()
    vc = kc[..., :Dv] if D == 576 else v.cuda()
    out, lse = ga.decode_kv(q.cuda(), kc, vc, S, q_offset=Skv - Sq, out_dtype=torch.float32, sinks=sinks.cuda(),
                            **dev)
    _ok()
    want_o, want_l = oracle.attention_ex(q, k, v, scale=_scale(D), causal=True, q_offset=Skv - Sq,
                                         sinks=sinks.numpy(), **terms)
    assert_o_close(out, want_o, f"{dims} {list(terms)}")
    assert_lse_close(lse, want_l, f"{dims} {list(terms)}")


@pytest.mark.parametrize("page_size", [16, 64, 256])
def test_decode_narrow_v_paged_equals_contiguous(page_size):
    """A paged latent cache, V a view of K: partials bit-identical to the
    contiguous run (256-key splits visit the same tiles)."""
    B, Hq, Hkv, Sq, Skv, D, Dv, S = 2, 16, 1, 1, 1024, 576, 512, 4
    q, k, v = _qkv(B, Hq, Hkv, Sq, Skv, D, Dv, True, seed=85)
    kc, _, bt = make_paged(k, k, page_size, seed=86)
    q, k, kc = q.cuda(), k.cuda(), kc.cuda()
    po, pl = ga.decode_split_kv(q, k, k[..., :Dv], S, q_offset=Skv - Sq)
    po2, pl2 = ga.decode_split_kv(q, kc, kc[..., :Dv], S, block_table=bt.cuda(), q_offset=Skv - Sq)
    _ok()
    assert torch.equal(po, po2) and torch.equal(pl, pl2)


def test_decode_narrow_v_seq_lens():
    B, Hq, Hkv, Sq, Skv, D, Dv, S = 3, 16, 1, 1, 1500, 576, 512, 5
    q, k, v = _qkv(B, Hq, Hkv, Sq, Skv, D, Dv, True, seed=87)
    lens = make_seq_lens(B, Skv, seed=88)
    lens[0] = Skv
    kc = k.cuda()
    out, lse = ga.decode_kv(q.cuda(), kc, kc[..., :Dv], S, seq_lens=lens.cuda(), out_dtype=torch.float32)
    _ok()
    for b in range(B):
        n = int(lens[b])
        wo, wl = oracle.attention_ex(q[b:b + 1], k[b:b + 1, :n], v[b:b + 1, :n], scale=_scale(D), causal=True,
                                     q_offset=n - Sq)
        assert_o_close(out[b:b + 1], wo, f"len {n}")
        assert_lse_close(lse[b:b + 1], wl, f"len {n}")


# (B, Hq, Hkv, Sq, Skv, D, Dv, q_offset, causal, v_of_k)
PREFILL = [
    (1, 16, 1, 200, 700, 576, 512, 500, True, True),
    (1, 8, 2, 300, 300, 320, 256, 0, True, False),
    (1, 8, 2, 257, 900, 192, 128, 643, True, False),
    (2, 4, 4, 130, 130, 192, 128, 0, False, False),     # g = 1, non-causal
    (1, 32, 1, 40, 1000, 576, 512, 960, True, True),    # g = 32: 2 query rows per CTA
]


@pytest.mark.parametrize("case", PREFILL, ids=[f"D{c[5]}v{c[6]}g{c[1] // c[2]}Sq{c[3]}x{c[4]}"
                                               f"{'c' if c[8] else 'n'}" for c in PREFILL])
def test_prefill_narrow_v_matches_oracle(case):
    B, Hq, Hkv, Sq, Skv, D, Dv, q_offset, causal, vk = case
    q, k, v = _qkv(B, Hq, Hkv, Sq, Skv, D, Dv, vk, seed=89)
    kc = k.cuda()
    vc = kc[..., :Dv] if vk else v.cuda()
    scale = _scale(D)
    out, lse = ga.prefill_kv(q.cuda(), kc, vc, causal=causal, q_offset=q_offset, scale=scale,
                             out_dtype=torch.float32)
    _ok()
    assert out.shape == (B, Sq, Hq, Dv)
    want_o, want_l = oracle.attention_ex(q, k, v, scale=scale, causal=causal, q_offset=q_offset)
    assert_o_close(out, want_o, f"prefill {case}")
    assert_lse_close(lse, want_l, f"prefill {case}")


def test_prefill_narrow_v_with_terms():
    B, Hq, Hkv, Sq, Skv, D, Dv = 2, 8, 2, 150, 600, 192, 128
    q, k, v = _qkv(B, Hq, Hkv, Sq, Skv, D, Dv, False, seed=90)
    sinks = make_sinks(Hq, seed=91)
    mask = make_mask(B, Sq, Skv, seed=92)
    terms = dict(softcap=25.0, alibi_max_bias=8.0, window=200)
    out, lse = ga.prefill_kv(q.cuda(), k.cuda(), v.cuda(), q_offset=Skv - Sq, out_dtype=torch.float32,
                             sinks=sinks.cuda(), mask=mask.cuda(), **terms)
    _ok()
    want_o, want_l = oracle.attention_ex(q, k, v, scale=_scale(D), causal=True, q_offset=Skv - Sq,
                                         sinks=sinks.numpy(), mask=mask, **terms)
    assert_o_close(out, want_o, "terms")
    assert_lse_close(lse, want_l, "terms")


@pytest.mark.parametrize("D", [64, 128, 256])
def test_prefill_kv_strided_equals_prefill(D):
    """The fast prefill kernel through a view: K and V interleaved in one
    tensor, and a head-major cache, bit-identical to the contiguous call."""
    B, Hq, Hkv, Sq, Skv = 2, 16, 4, 300, 500
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=93)
    q = q.cuda()
    o1, l1 = ga.prefill(q, k.cuda(), v.cuda(), q_offset=Skv - Sq)
    kv = torch.stack([k, v], dim=2).cuda()                # [B, Skv, 2, Hkv, D]
    o2, l2 = ga.prefill_kv(q, kv[:, :, 0], kv[:, :, 1], q_offset=Skv - Sq)
    kh = k.permute(0, 2, 1, 3).contiguous().cuda()        # [B, Hkv, Skv, D]
    vh = v.permute(0, 2, 1, 3).contiguous().cuda()
    o3, l3 = ga.prefill_kv(q, kh.permute(0, 2, 1, 3), vh.permute(0, 2, 1, 3), q_offset=Skv - Sq)
    _ok()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert torch.equal(o1, o3) and torch.equal(l1, l3)


@pytest.mark.parametrize("D,page_size", [(128, 16), (128, 256), (512, 64)])
def test_prefill_kv_paged_seq_lens(D, page_size):
    """Chunked prefill into a paged cache: sequence b's Sq new rows sit at the
    end of its len_b keys."""
    B, Hq, Hkv, Sq, Skv = 3, 8, 1, 70, 768
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=94)
    kc, vc, bt = make_paged(k, v, page_size, seed=95)
    lens = make_seq_lens(B, Skv, seed=96, low=Sq)
    lens[1] = Sq - 5                                      # 5 rows at negative positions see no key
    sinks = make_sinks(Hq, seed=97)
    out, lse = ga.prefill_kv(q.cuda(), kc.cuda(), vc.cuda(), block_table=bt.cuda(), seq_lens=lens.cuda(),
                             out_dtype=torch.float32, sinks=sinks.cuda())
    _ok()
    for b in range(B):
        n = int(lens[b])
        cut = max(0, Sq - n)   # rows at a negative position see no key
        wo, wl = oracle.attention_ex(q[b:b + 1, cut:], k[b:b + 1, :n], v[b:b + 1, :n], scale=_scale(D),
                                     causal=True, q_offset=n - Sq + cut, sinks=sinks.numpy())
        assert_o_close(out[b:b + 1, cut:], wo, f"len {n}")
        assert_lse_close(lse[b:b + 1, :, cut:], wl, f"len {n}")
        if cut:
            assert float(out[b, :cut].abs().max()) == 0.0


@pytest.mark.parametrize("D", [128, 512])
def test_prefill_kv_fp8(D):
    B, Hq, Hkv, Sq, Skv = 1, 16, 2, 180, 640
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=98)
    kc, vc, ks, vs = make_fp8_kv(k, v)
    out, lse = ga.prefill_kv(q.cuda(), kc.cuda(), vc.cuda(), q_offset=Skv - Sq, k_scale=ks.cuda(),
                             v_scale=vs.cuda(), out_dtype=torch.float32)
    _ok()
    want_o, want_l = oracle.attention_fp8(q, kc, vc, ks, vs, scale=_scale(D), causal=True, q_offset=Skv - Sq)
    assert_o_close(out, want_o, f"fp8 D{D}")
    assert_lse_close(lse, want_l, f"fp8 D{D}")


@pytest.mark.parametrize("name", ["mla_decode_d576_v512", "prefill_d192_v128_4k"])
def test_narrow_v_workload_full_size_sampled(name):
    """The timed narrow-V workloads, in their timed launch configuration."""
    w = WORKLOADS[name]
    q, k, v = make_workload_inputs(w, seed=0)
    kc = k.cuda()
    vc = kc[..., :w.dv] if w.v_of_k else v.cuda()
    if w.kind == "decode":
        out, lse = ga.decode_kv(q.cuda(), kc, vc, w.num_splits, causal=w.causal, q_offset=w.q_offset,
                                scale=w.scale)
    else:
        out, lse = ga.prefill_kv(q.cuda(), kc, vc, causal=w.causal, q_offset=w.q_offset, scale=w.scale)
    _ok()
    rows = sample_rows(w, 40, seed=29)
    got_o, got_l = gather_rows(out, lse, rows)
    want_o, want_l = oracle_rows_by_batch(q, k, v, rows, scale=w.scale, causal=w.causal, q_offset=w.q_offset)
    assert_o_close(got_o, want_o, w.name)
    assert_lse_close(got_l, want_l, w.name)


def test_views_with_own_v_strides():
    """K contiguous and V head-major (its own strides): bit-identical to the
    contiguous prefill and decode."""
    B, Hq, Hkv, Sq, Skv, D, S = 2, 16, 4, 8, 600, 128, 3
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=99)
    q, kc = q.cuda(), k.cuda()
    vh = v.permute(0, 2, 1, 3).contiguous().cuda().permute(0, 2, 1, 3)   # [B, Skv, Hkv, D] view, head-major
    o1, l1 = ga.prefill(q, kc, v.cuda(), q_offset=Skv - Sq)
    o2, l2 = ga.prefill_kv(q, kc, vh, q_offset=Skv - Sq)
    p1, m1 = ga.decode_split(q, kc, v.cuda(), S, q_offset=Skv - Sq)
    p2, m2 = ga.decode_split_kv(q, kc, vh, S, q_offset=Skv - Sq)
    _ok()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert torch.equal(p1, p2) and torch.equal(m1, m2)
