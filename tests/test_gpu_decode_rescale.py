"""Split-KV decode where the running maximum of every row moves again and
again along the keys (B200), against the float64 oracle.

The decode kernel for fp8 K/V and for the optional logit terms checks each
logit against the running maximum as it loads it and runs the row-maximum
reduction, the O and row-sum rescales only on tiles where some row's
maximum moves; with random inputs that is the first tile of a split.  Here
the logits grow along the keys (an additive mask that ramps up, or K whose
magnitude grows), so most tiles move the maximum, with 16 and 32 rows per
CTA and with several splits per CTA (partials published at each split's
end)."""
import math

import pytest
import torch

import gqa_flash_attention_attn_b200 as ga
from gqa_flash_attention_attn_b200.inputs import make_fp8_kv, make_mask, make_qkv
import oracle
from parity import assert_lse_close, assert_o_close

pytestmark = pytest.mark.gpu


def _scale(D):
    return float(torch.tensor(1.0 / math.sqrt(D), dtype=torch.float32))


def _ramp_mask(B, Sq, Skv, top, seed):
    """An additive mask rising linearly from 0 to `top` (natural-log units)
    along the keys, with some -inf entries."""
    ramp = torch.linspace(0.0, top, Skv, dtype=torch.float64).view(1, 1, Skv).expand(B, Sq, Skv).clone()
    holes = make_mask(B, Sq, Skv, seed=seed, p_inf=0.1).double()
    return (ramp + torch.where(torch.isinf(holes), holes, torch.zeros_like(holes))).to(torch.bfloat16)


# (B, Hq, Hkv, Sq, Skv, D, num_splits): 16 rows (g 4 x Sq 4) and 32 rows
# (g 4 x Sq 8) per CTA; the last case has more key ranges than two CTAs per
# SM hold, so each CTA streams two consecutive splits
RAMP = [
    (2, 8, 2, 4, 1300, 128, 2),
    (2, 8, 2, 8, 1300, 128, 3),
    (1, 16, 1, 1, 2100, 512, 4),
    (4, 32, 8, 8, 4096, 128, 16),
]


@pytest.mark.parametrize("case", RAMP, ids=[f"B{c[0]}H{c[1]}/{c[2]}S{c[3]}x{c[4]}D{c[5]}n{c[6]}" for c in RAMP])
def test_mask_ramp_moves_the_maximum(case):
    B, Hq, Hkv, Sq, Skv, D, S = case
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=91)
    # 3 (natural-log) units more per 128-key tile: 4.3 in log2 units, so the
    # bf16 threshold (8) moves a row's maximum every second tile
    mask = _ramp_mask(B, Sq, Skv, 3.0 * Skv / 128, seed=92)
    q_offset = Skv - Sq
    po, pl = ga.decode_split(q.cuda(), k.cuda(), v.cuda(), S, causal=True, q_offset=q_offset, scale=_scale(D),
                             mask=mask.cuda())
    out, lse = ga.merge(po, pl, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    want_o, want_l = oracle.attention_ex(q, k, v, scale=_scale(D), causal=True, q_offset=q_offset, mask=mask)
    assert_o_close(out, want_o, f"mask ramp {case}")
    assert_lse_close(lse, want_l, f"mask ramp {case}")


@pytest.mark.parametrize("case", RAMP, ids=[f"B{c[0]}H{c[1]}/{c[2]}S{c[3]}x{c[4]}D{c[5]}n{c[6]}" for c in RAMP])
def test_fp8_growing_keys_move_the_maximum(case):
    B, Hq, Hkv, Sq, Skv, D, S = case
    q, k, v = make_qkv(B, Hq, Hkv, Sq, Skv, D, seed=93)
    # |k| grows 16-fold along the keys: logits several units larger per tile
    grow = torch.linspace(0.25, 4.0, Skv, dtype=torch.float32).view(1, Skv, 1, 1)
    k = (k.float() * grow).to(torch.bfloat16)
    kc, vc, ks, vs = make_fp8_kv(k, v)
    q_offset = Skv - Sq
    po, pl = ga.decode_split_kv(q.cuda(), kc.cuda(), vc.cuda(), S, causal=True, q_offset=q_offset,
                                scale=_scale(D), k_scale=ks.cuda(), v_scale=vs.cuda())
    out, lse = ga.merge(po, pl, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ga.last_status() == ga.ATTN_OK
    want_o, want_l = oracle.attention_fp8(q, kc, vc, ks, vs, scale=_scale(D), causal=True, q_offset=q_offset)
    assert_o_close(out, want_o, f"fp8 growing keys {case}")
    assert_lse_close(lse, want_l, f"fp8 growing keys {case}")
