"""The C-ABI library on the host: it loads, exports every declared entry point,
and rejects bad arguments before any CUDA call (so these run without a GPU)."""
import ctypes

import pytest

import gqa_flash_attention_attn_b200 as ga
from gqa_flash_attention_attn_b200 import build as gbuild


@pytest.fixture(scope="module")
def lib():
    gbuild.build()
    return ga.library()


def test_exports_every_declared_symbol(lib):
    names = ga.declared_functions()
    assert {"attn_prefill", "attn_decode_split", "attn_merge", "attn_last_status"} <= set(names)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/attn.h but not exported"


def test_version_and_status_strings(lib):
    assert ga.version() == 0x000500
    assert ga.status_string(ga.ATTN_OK) == "ok"
    assert ga.status_string(ga.ATTN_ERR_TIMEOUT) == "pipeline wait timed out"
    assert ga.status_string(12345) == "unknown status"


def test_workspace_bytes(lib):
    S, B, Hq, Sq, D = 32, 16, 16, 1, 512
    assert ga.decode_workspace_bytes(B, Hq, Sq, D, S) == 4 * (S * B * Sq * Hq * D + S * B * Hq * Sq)
    assert ga.decode_workspace_bytes(0, Hq, Sq, D, S) == 0
    assert ga.decode_workspace_bytes(B, Hq, Sq, D, 0) == 0


# Fake but 256-byte aligned addresses: the checks must reject before any use.
P = ctypes.c_void_p(0x10000)
P2 = ctypes.c_void_p(0x20000)
MIS = ctypes.c_void_p(0x10008)


def _prefill(lib, **kw):
    a = dict(q=P, k=P, v=P, out=P2, lse=P2, B=1, Hq=8, Hkv=2, Sq=128, Skv=128, D=128, q_offset=0, causal=1,
             scale=0.125, out_dtype=0)
    a.update(kw)
    return lib.attn_prefill(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"], a["Hq"], a["Hkv"], a["Sq"],
                            a["Skv"], a["D"], a["q_offset"], a["causal"], a["scale"], a["out_dtype"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), ga.ATTN_ERR_INVALID_ARG),
    (dict(out=None), ga.ATTN_ERR_INVALID_ARG),
    (dict(B=0), ga.ATTN_ERR_INVALID_ARG),
    (dict(Sq=0), ga.ATTN_ERR_INVALID_ARG),
    (dict(Skv=-1), ga.ATTN_ERR_INVALID_ARG),
    (dict(Hq=6, Hkv=4), ga.ATTN_ERR_INVALID_ARG),
    (dict(q_offset=-1), ga.ATTN_ERR_INVALID_ARG),
    (dict(causal=2), ga.ATTN_ERR_INVALID_ARG),
    (dict(scale=0.0), ga.ATTN_ERR_INVALID_ARG),
    (dict(scale=-0.1), ga.ATTN_ERR_INVALID_ARG),
    (dict(scale=float("inf")), ga.ATTN_ERR_INVALID_ARG),
    (dict(scale=float("nan")), ga.ATTN_ERR_INVALID_ARG),
    (dict(out_dtype=7), ga.ATTN_ERR_INVALID_ARG),
    (dict(D=72), ga.ATTN_ERR_UNSUPPORTED),     # the head size that crashed a staging path
    (dict(D=32), ga.ATTN_ERR_UNSUPPORTED),
    (dict(D=512, Hq=64, Hkv=1), ga.ATTN_ERR_UNSUPPORTED),   # D = 512 needs a group of at most 32
    (dict(D=320), ga.ATTN_ERR_UNSUPPORTED),
    (dict(q=MIS), ga.ATTN_ERR_ALIGNMENT),
    (dict(v=MIS), ga.ATTN_ERR_ALIGNMENT),
    (dict(out=MIS), ga.ATTN_ERR_ALIGNMENT),
    (dict(lse=ctypes.c_void_p(0x20002)), ga.ATTN_ERR_ALIGNMENT),
    (dict(q_offset=2**31 - 100), ga.ATTN_ERR_INVALID_ARG),
])
def test_prefill_rejects(lib, kw, status):
    assert _prefill(lib, **kw) == status


def _decode(lib, **kw):
    a = dict(q=P, k=P, v=P, po=P2, pl=P2, B=16, Hq=16, Hkv=1, Sq=1, Skv=16384, D=512, q_offset=16383, causal=1,
             scale=0.0441941738, S=32)
    a.update(kw)
    return lib.attn_decode_split(a["q"], a["k"], a["v"], a["po"], a["pl"], a["B"], a["Hq"], a["Hkv"], a["Sq"],
                                 a["Skv"], a["D"], a["q_offset"], a["causal"], a["scale"], a["S"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(S=0), ga.ATTN_ERR_INVALID_ARG),
    (dict(S=16385), ga.ATTN_ERR_INVALID_ARG),        # more splits than keys
    (dict(po=None), ga.ATTN_ERR_INVALID_ARG),
    (dict(pl=None), ga.ATTN_ERR_INVALID_ARG),
    (dict(Hq=12, Hkv=8), ga.ATTN_ERR_INVALID_ARG),
    (dict(D=64, Hq=96, Hkv=1), ga.ATTN_ERR_UNSUPPORTED),   # 96 rows x (2 + 1) > 256 TMEM columns
    (dict(D=32), ga.ATTN_ERR_UNSUPPORTED),
    (dict(D=96), ga.ATTN_ERR_UNSUPPORTED),
    (dict(Hq=64, Sq=1), ga.ATTN_ERR_UNSUPPORTED),   # 64 rows x (2 + 512/128) > 256 TMEM columns
    (dict(D=128, Hq=32, Hkv=1, Sq=8), ga.ATTN_ERR_UNSUPPORTED),  # 256 rows
    (dict(D=512, Hq=48, Hkv=1, Sq=1), ga.ATTN_ERR_UNSUPPORTED),  # 48 x (2 + 4) > 256
    (dict(D=256, Hq=80, Hkv=1, Sq=1), ga.ATTN_ERR_UNSUPPORTED),  # 80 x (2 + 2) > 256
    (dict(po=MIS), ga.ATTN_ERR_ALIGNMENT),
    (dict(k=MIS), ga.ATTN_ERR_ALIGNMENT),
    (dict(pl=ctypes.c_void_p(0x20001)), ga.ATTN_ERR_ALIGNMENT),
])
def test_decode_rejects(lib, kw, status):
    assert _decode(lib, **kw) == status


@pytest.mark.parametrize("args,status", [
    ((None, P, P2, P2, 1, 2, 3, 128, 4, 0), ga.ATTN_ERR_INVALID_ARG),
    ((P, P, P2, P2, 1, 2, 3, 130, 4, 0), ga.ATTN_ERR_UNSUPPORTED),
    ((P, P, P2, P2, 1, 2, 3, 2048, 4, 0), ga.ATTN_ERR_UNSUPPORTED),
    ((P, P, P2, P2, 1, 2, 3, 128, 0, 0), ga.ATTN_ERR_INVALID_ARG),
    ((P, P, P2, P2, 1, 2, 3, 128, 4, 3), ga.ATTN_ERR_INVALID_ARG),
    ((MIS, P, P2, P2, 1, 2, 3, 128, 4, 0), ga.ATTN_ERR_ALIGNMENT),
    ((P, P, ctypes.c_void_p(0x20004), P2, 1, 2, 3, 128, 4, 0), ga.ATTN_ERR_ALIGNMENT),
])
def test_merge_rejects(lib, args, status):
    assert lib.attn_merge(*args, None) == status


def _opt(softcap=0.0, alibi=0.0, sinks=None, window=0, mask=None, msb=0, msr=0):
    return ctypes.byref(ga.AttnOptions(softcap, alibi, sinks, window, mask, msb, msr))


@pytest.mark.parametrize("opt,kw,status", [
    (dict(softcap=-1.0), {}, ga.ATTN_ERR_INVALID_ARG),
    (dict(softcap=float("nan")), {}, ga.ATTN_ERR_INVALID_ARG),
    (dict(softcap=float("inf")), {}, ga.ATTN_ERR_INVALID_ARG),
    (dict(softcap=1e-45), {}, ga.ATTN_ERR_INVALID_ARG),          # scale / softcap overflows
    (dict(alibi=-0.5), {}, ga.ATTN_ERR_INVALID_ARG),
    (dict(alibi=float("inf")), {}, ga.ATTN_ERR_INVALID_ARG),
    (dict(window=-3), {}, ga.ATTN_ERR_INVALID_ARG),
    (dict(sinks=0x20002), {}, ga.ATTN_ERR_ALIGNMENT),            # misaligned sink array
    (dict(window=64), dict(causal=0), ga.ATTN_ERR_UNSUPPORTED),
    (dict(window=64), dict(q_offset=1), ga.ATTN_ERR_UNSUPPORTED),  # q_offset + Sq > Skv
    (dict(softcap=30.0), dict(q=None), ga.ATTN_ERR_INVALID_ARG),  # shape checks still apply
    (dict(softcap=30.0), dict(D=72), ga.ATTN_ERR_UNSUPPORTED),
    (dict(mask=0x80001), {}, ga.ATTN_ERR_ALIGNMENT),             # bf16 mask at an odd address
    (dict(mask=0x80000, msr=-128), {}, ga.ATTN_ERR_INVALID_ARG),
    (dict(mask=0x80000, msb=-1, msr=128), {}, ga.ATTN_ERR_INVALID_ARG),
])
def test_prefill_ex_rejects(lib, opt, kw, status):
    a = dict(q=P, k=P, v=P, out=P2, lse=P2, B=1, Hq=8, Hkv=2, Sq=128, Skv=128, D=128, q_offset=0, causal=1,
             scale=0.125, out_dtype=0)
    a.update(kw)
    assert lib.attn_prefill_ex(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"], a["Hq"], a["Hkv"], a["Sq"],
                               a["Skv"], a["D"], a["q_offset"], a["causal"], a["scale"], a["out_dtype"],
                               _opt(**opt), None) == status


@pytest.mark.parametrize("opt,kw,status", [
    (dict(sinks=0x30000), {}, ga.ATTN_ERR_INVALID_ARG),  # sinks belong to the merge
    (dict(softcap=-2.0), {}, ga.ATTN_ERR_INVALID_ARG),
    (dict(window=-1), {}, ga.ATTN_ERR_INVALID_ARG),
    (dict(window=128), dict(causal=0), ga.ATTN_ERR_UNSUPPORTED),
    (dict(window=128), dict(q_offset=16384), ga.ATTN_ERR_UNSUPPORTED),
    (dict(alibi=8.0), dict(D=96), ga.ATTN_ERR_UNSUPPORTED),
])
def test_decode_split_ex_rejects(lib, opt, kw, status):
    a = dict(q=P, k=P, v=P, po=P2, pl=P2, B=16, Hq=16, Hkv=1, Sq=1, Skv=16384, D=512, q_offset=16383, causal=1,
             scale=0.0441941738, S=32)
    a.update(kw)
    assert lib.attn_decode_split_ex(a["q"], a["k"], a["v"], a["po"], a["pl"], a["B"], a["Hq"], a["Hkv"],
                                    a["Sq"], a["Skv"], a["D"], a["q_offset"], a["causal"], a["scale"], a["S"],
                                    _opt(**opt), None) == status


def test_merge_ex_rejects_misaligned_sinks(lib):
    assert lib.attn_merge_ex(P, P, P2, P2, 1, 2, 3, 128, 4, 0, ctypes.c_void_p(0x30002), None) == \
        ga.ATTN_ERR_ALIGNMENT
    # the other checks come first, as in attn_merge
    assert lib.attn_merge_ex(None, P, P2, P2, 1, 2, 3, 128, 4, 0, P, None) == ga.ATTN_ERR_INVALID_ARG


def test_options_struct_matches_header():
    """AttnOptions mirrors attn_options: float, float, pointer, int."""
    import re
    text = open(ga._HEADER).read()
    body = re.search(r"typedef struct attn_options \{(.*?)\} attn_options;", text, re.S).group(1)
    fields = [ln.split(";")[0].split()[-1].lstrip("*") for ln in body.strip().splitlines() if ";" in ln]
    assert fields == [f[0] for f in ga.AttnOptions._fields_]
    assert ctypes.sizeof(ga.AttnOptions) == 48


def _view(view):
    vw = dict(k=0x40000, v=0x50000, stride_seq=1024 * 512, stride_token=512, stride_head=512, block_table=None,
              max_pages=0, page_size=0, num_pages=0, seq_lens=None, kv_dtype=0, k_scale=None, v_scale=None,
              head_dim_v=0, v_stride_seq=0, v_stride_token=0, v_stride_head=0)
    vw.update(view or {})
    return ga.AttnKVView(**vw)


def _kv_decode(lib, view=None, **kw):
    a = dict(q=P, po=P2, pl=P2, B=2, Hq=16, Hkv=1, Sq=1, Skv=1024, D=512, q_offset=1023, causal=1,
             scale=0.0441941738, S=4)
    a.update(kw)
    if view is None:
        view = {}
    v = _view(view)
    return lib.attn_decode_split_kv(a["q"], ctypes.byref(v), a["po"], a["pl"], a["B"], a["Hq"], a["Hkv"], a["Sq"],
                                    a["Skv"], a["D"], a["q_offset"], a["causal"], a["scale"], a["S"], None, None)


@pytest.mark.parametrize("view,kw,status", [
    (dict(k=None), {}, ga.ATTN_ERR_INVALID_ARG),
    (dict(stride_token=0), {}, ga.ATTN_ERR_INVALID_ARG),
    (dict(stride_seq=-512), {}, ga.ATTN_ERR_INVALID_ARG),
    (dict(stride_head=1 << 37), {}, ga.ATTN_ERR_INVALID_ARG),
    (dict(stride_token=516), {}, ga.ATTN_ERR_ALIGNMENT),             # 1032 bytes: not a 16-byte multiple
    (dict(v=0x50008), {}, ga.ATTN_ERR_ALIGNMENT),
    (dict(seq_lens=0x60002), {}, ga.ATTN_ERR_ALIGNMENT),
    (dict(block_table=0x70000, max_pages=8, page_size=100, num_pages=64), {}, ga.ATTN_ERR_INVALID_ARG),
    (dict(block_table=0x70000, max_pages=8, page_size=8, num_pages=64), dict(Skv=64), ga.ATTN_ERR_INVALID_ARG),
    (dict(block_table=0x70000, max_pages=4, page_size=128, num_pages=64), {}, ga.ATTN_ERR_INVALID_ARG),  # 4*128 != Skv
    (dict(block_table=0x70000, max_pages=0, page_size=128, num_pages=64), {}, ga.ATTN_ERR_INVALID_ARG),
    (dict(block_table=0x70000, max_pages=8, page_size=128, num_pages=0), dict(Skv=1024), ga.ATTN_ERR_INVALID_ARG),
    (dict(block_table=0x70002, max_pages=8, page_size=128, num_pages=64), dict(Skv=1024), ga.ATTN_ERR_ALIGNMENT),
    ({}, dict(D=32), ga.ATTN_ERR_UNSUPPORTED),
    (dict(kv_dtype=2, k_scale=0x90000, v_scale=0x90010, stride_token=64, stride_head=64, stride_seq=64 * 1024),
     dict(D=64), ga.ATTN_ERR_UNSUPPORTED),                                    # fp8 at D = 64: no kernel
    (dict(kv_dtype=5), {}, ga.ATTN_ERR_INVALID_ARG),
    (dict(kv_dtype=2), {}, ga.ATTN_ERR_INVALID_ARG),                           # fp8 without scales
    (dict(kv_dtype=2, k_scale=0x90000, v_scale=0x90002), {}, ga.ATTN_ERR_INVALID_ARG),
    (dict(kv_dtype=2, k_scale=0x90000, v_scale=0x90010, stride_head=520,
          stride_token=520, stride_seq=520 * 1024), {}, ga.ATTN_ERR_ALIGNMENT),  # 520 bytes: not 16-byte multiples
    (dict(head_dim_v=-1), {}, ga.ATTN_ERR_INVALID_ARG),
    (dict(v_stride_token=512), {}, ga.ATTN_ERR_INVALID_ARG),                  # own V strides: all three
    (dict(v_stride_token=516, v_stride_head=512, v_stride_seq=1024 * 512), {}, ga.ATTN_ERR_ALIGNMENT),
    (dict(head_dim_v=256), {}, ga.ATTN_ERR_UNSUPPORTED),                       # (512, 256): no kernel
    (dict(head_dim_v=512), dict(D=320), ga.ATTN_ERR_UNSUPPORTED),              # Dv > D
    (dict(head_dim_v=512, stride_token=576, stride_head=576, stride_seq=576 * 1024), dict(D=576, Hq=48),
     ga.ATTN_ERR_UNSUPPORTED),                                                 # 48 rows x (2 + 4) > 256
    (dict(head_dim_v=512, kv_dtype=2, k_scale=0x90000, v_scale=0x90010, stride_token=576, stride_head=576,
          stride_seq=576 * 1024), dict(D=576), ga.ATTN_ERR_UNSUPPORTED),     # fp8 pairs: no kernel
])
def test_decode_split_kv_rejects(lib, view, kw, status):
    assert _kv_decode(lib, view, **kw) == status


def test_decode_split_kv_rejects_null_view(lib):
    assert lib.attn_decode_split_kv(P, None, P2, P2, 1, 8, 1, 1, 128, 128, 127, 1, 0.08, 1, None, None) == \
        ga.ATTN_ERR_INVALID_ARG


def test_kv_view_struct_matches_header():
    import re
    text = open(ga._HEADER).read()
    body = re.search(r"typedef struct attn_kv_view \{(.*?)\} attn_kv_view;", text, re.S).group(1)
    fields = [ln.split(";")[0].split()[-1].lstrip("*") for ln in body.strip().splitlines() if ";" in ln]
    assert fields == [f[0] for f in ga.AttnKVView._fields_]
    assert ctypes.sizeof(ga.AttnKVView) == 128


def _kv_prefill(lib, view=None, opt=None, **kw):
    a = dict(q=P, out=P2, lse=P2, B=2, Hq=16, Hkv=1, Sq=64, Skv=1024, D=512, q_offset=960, causal=1,
             scale=0.0441941738, out_dtype=0)
    a.update(kw)
    v = _view(view)
    return lib.attn_prefill_kv(a["q"], ctypes.byref(v), a["out"], a["lse"], a["B"], a["Hq"], a["Hkv"], a["Sq"],
                               a["Skv"], a["D"], a["q_offset"], a["causal"], a["scale"], a["out_dtype"],
                               None if opt is None else ctypes.byref(opt), None)


@pytest.mark.parametrize("view,kw,status", [
    (dict(k=None), {}, ga.ATTN_ERR_INVALID_ARG),
    ({}, dict(out=None), ga.ATTN_ERR_INVALID_ARG),
    ({}, dict(out_dtype=2), ga.ATTN_ERR_INVALID_ARG),
    ({}, dict(D=96), ga.ATTN_ERR_UNSUPPORTED),
    (dict(block_table=0x70000, max_pages=8, page_size=128, num_pages=64), dict(D=32), ga.ATTN_ERR_UNSUPPORTED),
    (dict(kv_dtype=2, k_scale=0x90000, v_scale=0x90010, stride_token=64, stride_head=64, stride_seq=64 * 1024),
     dict(D=64), ga.ATTN_ERR_UNSUPPORTED),                                    # fp8 at D = 64: no kernel
    ({}, dict(Hq=64), ga.ATTN_ERR_UNSUPPORTED),                                # g = 64 > 32 on the wide path
    (dict(head_dim_v=256), {}, ga.ATTN_ERR_UNSUPPORTED),
    (dict(stride_token=516), {}, ga.ATTN_ERR_ALIGNMENT),
    ({}, dict(q=ctypes.c_void_p(0x10008)), ga.ATTN_ERR_ALIGNMENT),
    ({}, dict(lse=ctypes.c_void_p(0x20002)), ga.ATTN_ERR_ALIGNMENT),
    ({}, dict(scale=0.0), ga.ATTN_ERR_INVALID_ARG),
    ({}, dict(q_offset=-1), ga.ATTN_ERR_INVALID_ARG),
])
def test_prefill_kv_rejects(lib, view, kw, status):
    assert _kv_prefill(lib, view, **kw) == status


def test_prefill_kv_rejects_null_view(lib):
    assert lib.attn_prefill_kv(P, None, P2, P2, 1, 8, 1, 128, 128, 128, 0, 1, 0.08, 0, None, None) == \
        ga.ATTN_ERR_INVALID_ARG


def _kv_fused(lib, view=None, opt=None, **kw):
    a = dict(q=P, out=P2, lse=P2, B=2, Hq=16, Hkv=1, Sq=1, Skv=1024, D=512, q_offset=1023, causal=1,
             scale=0.0441941738, S=16, out_dtype=0)
    a.update(kw)
    v = _view(view)
    return lib.attn_decode_fused(a["q"], ctypes.byref(v), a["out"], a["lse"], a["B"], a["Hq"], a["Hkv"], a["Sq"],
                                 a["Skv"], a["D"], a["q_offset"], a["causal"], a["scale"], a["S"], a["out_dtype"],
                                 None if opt is None else ctypes.byref(opt), None)


@pytest.mark.parametrize("view,kw,status", [
    (dict(k=None), {}, ga.ATTN_ERR_INVALID_ARG),
    ({}, dict(out=None), ga.ATTN_ERR_INVALID_ARG),
    ({}, dict(out_dtype=7), ga.ATTN_ERR_INVALID_ARG),
    ({}, dict(S=0), ga.ATTN_ERR_INVALID_ARG),
    ({}, dict(D=32), ga.ATTN_ERR_UNSUPPORTED),
    (dict(kv_dtype=2, k_scale=0x90000, v_scale=0x90010, stride_token=64, stride_head=64, stride_seq=64 * 1024),
     dict(D=64), ga.ATTN_ERR_UNSUPPORTED),                                    # fp8 at D = 64: no kernel
    ({}, dict(out=ctypes.c_void_p(0x20008)), ga.ATTN_ERR_ALIGNMENT),
    ({}, dict(lse=ctypes.c_void_p(0x20002)), ga.ATTN_ERR_ALIGNMENT),
    (dict(stride_token=128, stride_head=128, stride_seq=128 * 1024), dict(D=128, Hq=64, Hkv=1, Sq=2),
     ga.ATTN_ERR_UNSUPPORTED),   # 128 rows x (2 + 1) TMEM column groups > 256
])
def test_decode_fused_rejects(lib, view, kw, status):
    assert _kv_fused(lib, view, **kw) == status
