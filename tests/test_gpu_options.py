"""Optional logit terms (softcap, ALiBi, sink logits, sliding window) in the
prefill, split-KV decode and merge kernels vs the float64 oracle (B200)."""
import math

import numpy as np
import pytest
import torch

import gqa_flash_attention_attn_b200 as ga
from gqa_flash_attention_attn_b200.inputs import WORKLOADS, make_qkv, make_sinks, make_workload_inputs, sample_rows
import oracle
from parity import assert_lse_close, assert_o_close, gather_rows

pytestmark = pytest.mark.gpu


def _scale(D):
    return float(torch.tensor(1.0 / math.sqrt(D), dtype=torch.float32))


def _sinks(Hq, seed, with_ninf=False):
    s = make_sinks(Hq, seed=seed)
    if with_ninf:
        s[0] = -math.inf          # a head with no sink
        s[-1] = 25.0              # a sink that outweighs every key
    return s


# (B, Hq, Hkv, Sq, Skv, D, q_offset, causal, softcap, alibi, sinks, window, out_dtype)
PREFILL = [
    (1, 8, 2, 300, 300, 128, 0, True, 1.5, 0.0, False, 0, torch.bfloat16),      # softcap bites
    (1, 8, 2, 257, 257, 128, 0, True, 0.0, 8.0, False, 0, torch.float32),       # ALiBi, Hq power of two
    (1, 12, 4, 200, 200, 128, 0, True, 0.0, 8.0, False, 0, torch.float32),      # ALiBi, Hq = 12: second slope base
    (2, 4, 2, 190, 190, 64, 0, True, 0.0, 0.0, True, 0, torch.float32),         # sinks, incl. -inf and dominant
    (1, 4, 2, 400, 400, 128, 0, True, 0.0, 0.0, False, 1, torch.float32),       # window 1: only the diagonal key
    (1, 4, 2, 520, 520, 128, 0, True, 0.0, 0.0, False, 100, torch.bfloat16),    # ragged window edge
    (1, 4, 2, 300, 900, 128, 600, True, 0.0, 0.0, False, 256, torch.bfloat16),  # window at depth: tiles skipped
    (1, 4, 2, 300, 300, 128, 0, True, 0.0, 0.0, False, 4096, torch.float32),    # window wider than the sequence
    (1, 8, 2, 333, 700, 128, 367, True, 30.0, 4.0, True, 128, torch.bfloat16),  # every term
    (1, 4, 2, 256, 500, 64, 0, False, 5.0, 2.0, True, 0, torch.float32),        # non-causal, no window
    (1, 4, 2, 200, 600, 256, 400, True, 2.0, 8.0, True, 160, torch.bfloat16),   # D = 256, every term
    (1, 6, 2, 129, 129, 256, 0, True, 0.0, 1.0, False, 64, torch.float32),      # D = 256, odd group
]


def _pid(c):
    B, Hq, Hkv, Sq, Skv, D, qo, causal, cap, ab, sk, w, od = c
    return f"H{Hq}/{Hkv}S{Sq}x{Skv}D{D}o{qo}{'c' if causal else 'n'}cap{cap}ab{ab}{'s' if sk else ''}w{w}"


@pytest.mark.parametrize("case", PREFILL, ids=[_pid(c) for c in PREFILL])
def test_prefill_options_match_oracle(case):
    B, Hq, Hkv, Sq, Skv, D, q_offset, causal, cap, ab, use_sinks, window, out_dtype = case
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=7)
    scale = _scale(D)
    sinks = _sinks(Hq, seed=8, with_ninf=True) if use_sinks else None
    out, lse = ga.prefill(q.cuda(), k.cuda(), v.cuda(), causal=causal, q_offset=q_offset, scale=scale,
                          out_dtype=out_dtype, softcap=cap, alibi_max_bias=ab,
                          sinks=None if sinks is None else sinks.cuda(), window=window)
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    want_o, want_lse = oracle.attention_ex(q, k, v, scale=scale, causal=causal, q_offset=q_offset, softcap=cap,
                                           alibi_max_bias=ab, sinks=None if sinks is None else sinks.numpy(),
                                           window=window)
    assert_o_close(out, want_o, str(case))
    assert_lse_close(lse, want_lse, str(case))


def test_prefill_options_off_equal_plain_path():
    """All terms zero through the options entry point: bit-identical to attn_prefill."""
    q, k, v = make_qkv(1, 8, 2, 300, 300, 128, seed=9)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o1, l1 = ga.prefill(qc, kc, vc)
    out = torch.empty_like(o1)
    lse = torch.empty_like(l1)
    opt = ga.AttnOptions(0.0, 0.0, None, 0)
    import ctypes
    st = ga.library().attn_prefill_ex(qc.data_ptr(), kc.data_ptr(), vc.data_ptr(), out.data_ptr(),
                                      lse.data_ptr(), 1, 8, 2, 300, 300, 128, 0, 1, _scale(128), 0,
                                      ctypes.byref(opt), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert st == ga.ATTN_OK
    assert torch.equal(o1, out) and torch.equal(l1, lse)


def test_window_rows_ignore_keys_outside():
    """Keys older than the window do not change any row (exact equality)."""
    B, Hq, Hkv, S, D, w = 1, 4, 2, 384, 128, 64
    q, k, v = make_qkv(B, Hq, Hkv, S, S, D, seed=11)
    o1, l1 = ga.prefill(q.cuda(), k.cuda(), v.cuda(), window=w)
    k2, v2 = k.clone(), v.clone()
    # rows >= 200 see keys > 200 - 64 only: rewrite keys 0..136 for them
    k2[:, :137] = torch.randn_like(k2[:, :137].float()).bfloat16()
    v2[:, :137] = torch.randn_like(v2[:, :137].float()).bfloat16()
    o2, l2 = ga.prefill(q.cuda(), k2.cuda(), v2.cuda(), window=w)
    torch.cuda.synchronize()
    assert torch.equal(o1[:, 200:], o2[:, 200:])
    assert torch.equal(l1[:, :, 200:], l2[:, :, 200:])


def test_dominant_sink_drives_output_to_zero():
    """A sink logit far above every key takes nearly all of the probability."""
    q, k, v = make_qkv(1, 4, 2, 130, 130, 128, seed=12)
    sinks = torch.full((4,), 60.0)
    out, lse = ga.prefill(q.cuda(), k.cuda(), v.cuda(), out_dtype=torch.float32, sinks=sinks.cuda())
    torch.cuda.synchronize()
    assert float(out.abs().max()) < 1e-12
    assert torch.allclose(lse.cpu(), torch.full_like(lse.cpu(), 60.0), atol=1e-4)


# (B, Hq, Hkv, Sq, Skv, D, q_offset, causal, num_splits, softcap, alibi, sinks, window)
DECODE = [
    (2, 16, 1, 1, 1000, 512, 999, True, 4, 2.0, 0.0, False, 0),
    (2, 16, 1, 1, 1000, 512, 999, True, 4, 0.0, 8.0, True, 0),
    (1, 16, 2, 1, 2000, 512, 1999, True, 8, 0.0, 0.0, True, 300),   # window: early splits empty
    (1, 32, 8, 8, 700, 128, 692, True, 3, 30.0, 4.0, True, 100),    # verify rows, every term
    (1, 12, 4, 4, 513, 256, 509, True, 5, 0.0, 8.0, False, 17),     # Hq = 12 ALiBi, tiny window
    (1, 8, 1, 1, 777, 128, 0, False, 6, 1.0, 1.0, True, 0),         # non-causal
    (1, 16, 2, 8, 515, 128, 507, True, 1, 5.0, 2.0, True, 1),       # window 1, one split
]


def _did(c):
    B, Hq, Hkv, Sq, Skv, D, qo, causal, S, cap, ab, sk, w = c
    return f"H{Hq}/{Hkv}S{Sq}x{Skv}D{D}S{S}cap{cap}ab{ab}{'s' if sk else ''}w{w}"


@pytest.mark.parametrize("case", DECODE, ids=[_did(c) for c in DECODE])
def test_decode_options_match_oracle(case):
    B, Hq, Hkv, Sq, Skv, D, q_offset, causal, S, cap, ab, use_sinks, window = case
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=13)
    scale = _scale(D)
    sinks = _sinks(Hq, seed=14, with_ninf=True) if use_sinks else None
    po, pl = ga.decode_split(q.cuda(), k.cuda(), v.cuda(), S, causal=causal, q_offset=q_offset, scale=scale,
                             softcap=cap, alibi_max_bias=ab, window=window)
    out, lse = ga.merge(po, pl, out_dtype=torch.float32, sinks=None if sinks is None else sinks.cuda())
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    want_po, want_pl = oracle.split_ex(q, k, v, S, scale=scale, causal=causal, q_offset=q_offset, softcap=cap,
                                       alibi_max_bias=ab, window=window)
    assert_lse_close(pl, want_pl, f"partial lse {case}")
    assert_o_close(po, want_po, f"partial out {case}")
    want_o, want_lse = oracle.attention_ex(q, k, v, scale=scale, causal=causal, q_offset=q_offset, softcap=cap,
                                           alibi_max_bias=ab, sinks=None if sinks is None else sinks.numpy(),
                                           window=window)
    assert_o_close(out, want_o, f"merged {case}")
    assert_lse_close(lse, want_lse, f"merged {case}")


def test_merge_sinks_on_oracle_partials():
    """The merge kernel alone with sinks, on oracle partials that include empty splits."""
    B, Hq, Hkv, Sq, Skv, D, S = 2, 8, 2, 4, 90, 128, 16
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=15)
    po, pl = oracle.split(q, k, v, S, scale=_scale(D), causal=True, q_offset=20)
    sinks = _sinks(Hq, seed=16, with_ninf=True)
    out, lse = ga.merge(torch.from_numpy(po).float().cuda(), torch.from_numpy(pl).float().cuda(),
                        out_dtype=torch.float32, sinks=sinks.cuda())
    want_o, want_lse = oracle.merge_ex(po, pl, sinks=sinks.numpy())
    torch.cuda.synchronize()
    assert_o_close(out, want_o, "merge sinks")
    assert_lse_close(lse, want_lse, "merge sinks")


def _rows_oracle_ex(w, q, k, v, rows, sinks, mask=None):
    rows_np = np.asarray(rows, dtype=np.int64)
    want_o = np.zeros((len(rows), w.D))
    want_l = np.zeros((len(rows),))
    for b in np.unique(rows_np[:, 0]):
        sel = np.nonzero(rows_np[:, 0] == b)[0]
        sub = rows_np[sel].copy()
        sub[:, 0] = 0
        mb = None if mask is None else mask[b:b + 1] if mask.shape[0] > 1 else mask
        o, l = oracle.attention_rows_ex(q[b:b + 1], k[b:b + 1], v[b:b + 1], sub, scale=w.scale, causal=w.causal,
                                        q_offset=w.q_offset, softcap=w.softcap, alibi_max_bias=w.alibi_max_bias,
                                        sinks=None if sinks is None else sinks.numpy(), window=w.window, mask=mb)
        want_o[sel] = o
        want_l[sel] = l
    return want_o, want_l


OPTION_WORKLOADS = [n for n, w in WORKLOADS.items() if w.has_options]


@pytest.mark.parametrize("name", OPTION_WORKLOADS)
def test_option_workload_full_size_sampled(name):
    """Each timed workload with optional terms, at full size and in the timed
    launch configuration, on sampled rows."""
    w = WORKLOADS[name]
    q, k, v = make_workload_inputs(w, seed=0)
    from gqa_flash_attention_attn_b200.inputs import make_mask
    sinks = make_sinks(w.Hq, seed=0) if w.sinks else None
    sk = None if sinks is None else sinks.cuda()
    mask = make_mask(w.mask_batch, w.Sq, w.Skv, seed=0) if w.mask_batch else None
    terms = dict(softcap=w.softcap, alibi_max_bias=w.alibi_max_bias, window=w.window,
                 mask=None if mask is None else mask.cuda())
    if w.kind == "prefill":
        out, lse = ga.prefill(q.cuda(), k.cuda(), v.cuda(), causal=w.causal, q_offset=w.q_offset, scale=w.scale,
                              sinks=sk, **terms)
    else:
        out, lse = ga.decode(q.cuda(), k.cuda(), v.cuda(), w.num_splits, causal=w.causal, q_offset=w.q_offset,
                             scale=w.scale, sinks=sk, **terms)
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    rows = sample_rows(w, 40, seed=21)
    got_o, got_l = gather_rows(out, lse, rows)
    want_o, want_l = _rows_oracle_ex(w, q, k, v, rows, sinks, mask)
    assert_o_close(got_o, want_o, name)
    assert_lse_close(got_l, want_l, name)


def test_headline_prefill_with_every_term_sampled():
    """The 4k causal GQA prefill at full size, every optional term on (window
    included), sampled rows."""
    base = WORKLOADS["gqa_causal_prefill_4k_d128"]
    import dataclasses
    w = dataclasses.replace(base, softcap=30.0, alibi_max_bias=8.0, sinks=True, window=1024)
    q, k, v = make_workload_inputs(w, seed=0)
    sinks = _sinks(w.Hq, seed=17)
    out, lse = ga.prefill(q.cuda(), k.cuda(), v.cuda(), causal=True, q_offset=w.q_offset, scale=w.scale,
                          sinks=sinks.cuda(), softcap=w.softcap, alibi_max_bias=w.alibi_max_bias,
                          window=w.window)
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    rows = sample_rows(w, 48, seed=21)
    got_o, got_l = gather_rows(out, lse, rows)
    want_o, want_l = _rows_oracle_ex(w, q, k, v, rows, sinks)
    assert_o_close(got_o, want_o, "4k prefill, every term")
    assert_lse_close(got_l, want_l, "4k prefill, every term")


# (B, Hq, Hkv, Sq, Skv, D, q_offset, causal, softcap, alibi, sinks, window, mask batch)
MASKED_PREFILL = [
    (2, 8, 2, 200, 384, 128, 184, True, 0.0, 0.0, False, 0, 2),     # per-sequence masks, vector path
    (1, 8, 2, 300, 300, 128, 0, True, 0.0, 0.0, False, 0, 1),       # ragged Skv: scalar tail
    (2, 4, 2, 130, 517, 64, 0, False, 0.0, 0.0, True, 0, 1),        # shared mask, non-causal, sinks
    (1, 8, 2, 256, 640, 128, 384, True, 20.0, 4.0, True, 256, 1),  # every term
    (1, 4, 2, 200, 600, 256, 400, True, 0.0, 8.0, False, 0, 1),     # D = 256 with ALiBi
    (1, 4, 2, 150, 333, 256, 183, True, 10.0, 0.0, True, 0, 1),     # D = 256 softcap, ragged
    # more units than 2 x 148 CTAs: the mask stages carry across units
    (2, 32, 8, 1280, 1280, 128, 0, True, 0.0, 4.0, False, 0, 2),
    (2, 32, 8, 1200, 1280, 64, 80, True, 0.0, 0.0, False, 0, 1),
]


@pytest.mark.parametrize("case", MASKED_PREFILL, ids=[f"c{i}" for i in range(len(MASKED_PREFILL))])
def test_prefill_mask_matches_oracle(case):
    from gqa_flash_attention_attn_b200.inputs import make_mask
    B, Hq, Hkv, Sq, Skv, D, q_offset, causal, cap, ab, use_sinks, window, mb = case
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=51)
    mask = make_mask(mb, Sq, Skv, seed=52)
    mask[0, 3] = float("-inf")                # a fully masked row
    sinks = _sinks(Hq, seed=53) if use_sinks else None
    scale = _scale(D)
    out, lse = ga.prefill(q.cuda(), k.cuda(), v.cuda(), causal=causal, q_offset=q_offset, scale=scale,
                          out_dtype=torch.float32, softcap=cap, alibi_max_bias=ab, window=window,
                          sinks=None if sinks is None else sinks.cuda(), mask=mask.cuda())
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    want_o, want_l = oracle.attention_ex(q, k, v, scale=scale, causal=causal, q_offset=q_offset, softcap=cap,
                                         alibi_max_bias=ab, window=window, mask=mask,
                                         sinks=None if sinks is None else sinks.numpy())
    assert_o_close(out, want_o, str(case))
    assert_lse_close(lse, want_l, str(case))


def test_prefill_mask_of_zeros_equals_no_mask():
    q, k, v = make_qkv(1, 8, 2, 256, 256, 128, seed=54)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    zero = torch.zeros((1, 256, 256), dtype=torch.bfloat16, device="cuda")
    o1, l1 = ga.prefill(qc, kc, vc, alibi_max_bias=2.0)
    o2, l2 = ga.prefill(qc, kc, vc, alibi_max_bias=2.0, mask=zero)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("paged", [False, True])
def test_decode_mask_matches_oracle(paged):
    from gqa_flash_attention_attn_b200.inputs import make_mask, make_paged
    B, Hq, Hkv, Sq, Skv, D, S = 2, 32, 8, 8, 1024, 128, 5
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=55)
    mask = make_mask(B, Sq, Skv, seed=56, p_inf=0.5)     # e.g. a tree of draft tokens
    mask[1, 2] = float("-inf")
    sinks = _sinks(Hq, seed=57)
    kw = dict(causal=True, q_offset=Skv - Sq, softcap=15.0, alibi_max_bias=2.0, mask=mask.cuda())
    if paged:
        kc, vc, bt = make_paged(k, v, 64, seed=58)
        out, lse = ga.decode_kv(q.cuda(), kc.cuda(), vc.cuda(), S, block_table=bt.cuda(), out_dtype=torch.float32,
                                sinks=sinks.cuda(), **kw)
    else:
        out, lse = ga.decode(q.cuda(), k.cuda(), v.cuda(), S, out_dtype=torch.float32, sinks=sinks.cuda(), **kw)
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    want_o, want_l = oracle.attention_ex(q, k, v, scale=_scale(D), causal=True, q_offset=Skv - Sq, softcap=15.0,
                                         alibi_max_bias=2.0, mask=mask, sinks=sinks.numpy())
    assert_o_close(out, want_o, f"decode mask paged={paged}")
    assert_lse_close(lse, want_l, f"decode mask paged={paged}")


@pytest.mark.parametrize("shape", [(1, 8, 1, 4, 1001, 256, 3), (1, 4, 2, 40, 700, 128, 2)],
                         ids=["unaligned_rows", "sq40_unstaged"])
def test_decode_mask_unstaged_paths(shape):
    """Masks the decode kernel reads directly instead of staging them: rows
    that are not 16-byte aligned (Skv = 1001), and more than 32 query rows."""
    from gqa_flash_attention_attn_b200.inputs import make_mask
    B, Hq, Hkv, Sq, Skv, D, S = shape
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=59)
    mask = make_mask(B, Sq, Skv, seed=60)
    out, lse = ga.decode(q.cuda(), k.cuda(), v.cuda(), S, q_offset=Skv - Sq, out_dtype=torch.float32,
                         mask=mask.cuda(), alibi_max_bias=1.0)
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    want_o, want_l = oracle.attention_ex(q, k, v, scale=_scale(D), causal=True, q_offset=Skv - Sq,
                                         alibi_max_bias=1.0, mask=mask)
    assert_o_close(out, want_o, str(shape))
    assert_lse_close(lse, want_l, str(shape))


def test_decode_terms_with_grouped_splits():
    """Short splits and many CTAs (several consecutive splits per CTA), with a
    staged mask, ALiBi (tiles newest first) and a window crossing the splits."""
    from gqa_flash_attention_attn_b200.inputs import make_mask
    B, Hq, Hkv, Sq, Skv, D, S = 64, 16, 2, 4, 512, 128, 8
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=91)
    mask = make_mask(B, Sq, Skv, seed=92)
    terms = dict(alibi_max_bias=4.0, window=300, softcap=25.0)
    po, pl = ga.decode_split(q.cuda(), k.cuda(), v.cuda(), S, q_offset=Skv - Sq, mask=mask.cuda(), **terms)
    out, lse = ga.merge(po, pl, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    want_po, want_pl = oracle.split_ex(q, k, v, S, scale=_scale(D), causal=True, q_offset=Skv - Sq, mask=mask,
                                       **terms)
    assert_lse_close(pl, want_pl, "grouped partial lse")
    assert_o_close(po, want_po, "grouped partial out")
    want_o, want_l = oracle.attention_ex(q, k, v, scale=_scale(D), causal=True, q_offset=Skv - Sq, mask=mask,
                                         **terms)
    assert_o_close(out, want_o, "grouped merged")
    assert_lse_close(lse, want_l, "grouped merged")
