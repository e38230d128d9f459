"""The seeded input generators (no attention arithmetic): shapes, seeds,
and the layouts the paged and fp8 helpers promise."""
import torch

from gqa_flash_attention_attn_b200.inputs import (WORKLOADS, make_fp8_kv, make_mask, make_paged, make_qkv,
                                                  make_seq_lens, make_sinks)


def test_make_qkv_is_seeded_bf16():
    a = make_qkv(2, 4, 2, 3, 5, 8, seed=7)
    b = make_qkv(2, 4, 2, 3, 5, 8, seed=7)
    c = make_qkv(2, 4, 2, 3, 5, 8, seed=8)
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    assert not torch.equal(a[0], c[0])
    assert [t.shape for t in a] == [(2, 3, 4, 8), (2, 5, 2, 8), (2, 5, 2, 8)]
    assert all(t.dtype == torch.bfloat16 for t in a)


def test_make_paged_round_trips():
    _, k, v = make_qkv(3, 4, 2, 1, 100, 16, seed=1)
    for ps in (16, 32, 128):
        kc, vc, bt = make_paged(k, v, ps, seed=2)
        mp = (100 + ps - 1) // ps
        assert bt.shape == (3, mp) and bt.dtype == torch.int32
        assert len(set(bt.flatten().tolist())) == 3 * mp            # distinct physical pages
        for b in range(3):
            kg = torch.cat([kc[int(bt[b, j])] for j in range(mp)])[:100]
            vg = torch.cat([vc[int(bt[b, j])] for j in range(mp)])[:100]
            assert torch.equal(kg, k[b]) and torch.equal(vg, v[b])


def test_make_fp8_kv_codes_and_scales():
    _, k, v = make_qkv(2, 4, 2, 1, 64, 32, seed=3)
    kc, vc, ks, vs = make_fp8_kv(k, v)
    assert kc.dtype == torch.uint8 and kc.shape == k.shape and ks.shape == (2,)
    for codes, sc, x in ((kc, ks, k), (vc, vs, v)):
        deq = codes.view(torch.float8_e4m3fn).float() * sc.view(1, 1, -1, 1)
        # largest magnitude maps to 448 exactly; e4m3 keeps 3 mantissa bits
        assert torch.allclose(deq.abs().amax(dim=(0, 1, 3)), x.float().abs().amax(dim=(0, 1, 3)), rtol=1e-6)
        assert float(((deq - x.float()).abs() / x.float().abs().clamp_min(1e-3)).max()) < 0.07
        assert not torch.isnan(deq).any()


def test_make_mask_and_lengths_and_sinks():
    m = make_mask(2, 5, 40, seed=4, p_inf=0.5)
    assert m.dtype == torch.bfloat16 and m.shape == (2, 5, 40)
    assert torch.isinf(m).any() and not torch.isinf(m[:, :, 0]).any()
    lens = make_seq_lens(6, 300, seed=5, low=4)
    assert lens.dtype == torch.int32 and int(lens.min()) >= 4 and int(lens.max()) <= 300
    s = make_sinks(8, seed=6)
    assert s.shape == (8,) and s.dtype == torch.float32


def test_workload_byte_and_flop_counts():
    w = WORKLOADS["gqa_causal_prefill_4k_d128"]
    assert w.visible_pairs_per_head() == 4096 * 4097 // 2
    assert w.flops() == 4 * 128 * (4096 * 4097 // 2) * 32
    f8 = WORKLOADS["fp8_kv_decode_d512"]
    b16 = WORKLOADS["split_kv_decode_d512"]
    kv16 = 2 * 16 * 16384 * 1 * 512 * 2
    assert b16.io_bytes() - f8.io_bytes() == kv16 // 2      # fp8 K/V: one byte per element
    sw = WORKLOADS["sliding_window_prefill_16k_w4096_d128"]
    lo, hi = sw.visible_range(10000)
    assert (lo, hi) == (10000 - 4096 + 1, 10001)


def test_narrow_v_workloads():
    """Workloads with Dv < D: V drawn Dv wide, or a view of K's first Dv columns."""
    from gqa_flash_attention_attn_b200.inputs import make_workload_inputs
    w = WORKLOADS["prefill_d192_v128_4k"]
    assert w.dv == 128
    assert w.flops() == 2 * (192 + 128) * (4096 * 4097 // 2) * 32
    q, k, v = make_qkv(1, 4, 2, 3, 5, 192, seed=9, Dv=128)
    q2, k2, _ = make_qkv(1, 4, 2, 3, 5, 192, seed=9)
    assert v.shape == (1, 5, 2, 128) and torch.equal(q, q2) and torch.equal(k, k2)
    m = WORKLOADS["mla_decode_d576_v512"]
    small = m.__class__(**{**m.__dict__, "B": 2, "Skv": 64, "q_offset": 63})
    q, k, v = make_workload_inputs(small)
    assert v.shape[-1] == 512 and v.data_ptr() == k.data_ptr() and torch.equal(v, k[..., :512])
    # V inside K: only K's bytes are read
    assert m.io_bytes() == (16 * 16 * 576 * 2 + 16 * 16384 * 576 * 2 + 16 * 16 * 512 * 2 + 16 * 16 * 4)
