"""Seeded synthetic inputs and the named workloads.

This module holds no attention arithmetic.  It draws Q, K, V for both the CUDA
path and the float64 oracle, so the two sides always see identical bf16 values.

Recipe: a ``torch.Generator`` seeded with ``seed`` draws q, k, v in that order
as iid N(0, 1) float32 and casts each to bf16 (round to nearest even).  The
shapes follow the workloads that the pages measure (head dims 64 to 512,
grouped-query heads, 8-row speculative-verify steps, prefill at depth): see
``WORKLOADS``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    """One attention problem: shapes, mask, scale and (for decode) splits."""
    name: str
    kind: str            # "prefill" or "decode"
    B: int
    Hq: int
    Hkv: int
    Sq: int
    Skv: int
    D: int
    q_offset: int
    causal: bool
    out_dtype: str       # "bf16" or "f32"
    num_splits: int = 1
    note: str = ""
    # optional logit terms (0 / False = off); sinks are drawn by make_sinks(Hq, seed=0)
    softcap: float = 0.0
    alibi_max_bias: float = 0.0
    sinks: bool = False
    window: int = 0
    # K/V cache layout: 0 = contiguous [B, Skv, Hkv, D]; else paged with this
    # many keys per page (pages scattered by make_paged(k, v, page_size, seed=0))
    page_size: int = 0
    # additive mask drawn by make_mask(mask_batch, Sq, Skv, seed=0); 0 = none,
    # 1 = one mask shared by the batch, B = one per sequence
    mask_batch: int = 0
    # K/V element type: "bf16", or "fp8" (e4m3 codes with per-head scales from
    # make_fp8_kv of the bf16 draw)
    kv_dtype: str = "bf16"
    # V head size (0: D); v_of_k: V is the first Dv columns of K (one cache
    # holds both, as for multi-head latent attention)
    Dv: int = 0
    v_of_k: bool = False
    # decode: one launch whose thread-block clusters merge the key ranges
    # (num_splits -> the largest power of two <= min(num_splits, 8) ranges)
    fused: bool = False

    @property
    def dv(self) -> int:
        return self.Dv or self.D

    @property
    def has_options(self) -> bool:
        return bool(self.softcap or self.alibi_max_bias or self.sinks or self.window or self.mask_batch)

    @property
    def scale(self) -> float:
        # the float32 value both sides receive
        return float(torch.tensor(1.0 / math.sqrt(self.D), dtype=torch.float32))

    def visible_range(self, s: int) -> tuple[int, int]:
        """Keys [lo, hi) that query row s sees (causal mask and window)."""
        pos = self.q_offset + s
        hi = min(self.Skv, pos + 1) if self.causal else self.Skv
        lo = max(0, pos - self.window + 1) if self.window > 0 else 0
        return lo, max(lo, hi)

    def visible_pairs_per_head(self) -> int:
        """Number of visible (query row, key) pairs for one (batch, head)."""
        if not self.causal:
            return self.Sq * self.Skv
        total = 0
        for s in range(self.Sq):
            lo, hi = self.visible_range(s)
            total += hi - lo
        return total

    def kv_rows_read(self) -> int:
        """Keys that at least one query row sees: the K/V rows a pass must read."""
        lo, _ = self.visible_range(0)
        _, hi = self.visible_range(self.Sq - 1)
        return hi - lo if self.causal else self.Skv

    def flops(self) -> int:
        """Algorithmic FLOPs: 2*D (Q.K) + 2*Dv (P.V) per visible (query, key) pair."""
        return 2 * (self.D + self.dv) * self.visible_pairs_per_head() * self.B * self.Hq

    def io_bytes(self) -> int:
        """Algorithmic bytes: Q, K, V read once (bf16; V counted in K when it
        is a view of K); O and LSE written once."""
        ob = 2 if self.out_dtype == "bf16" else 4
        q = self.B * self.Sq * self.Hq * self.D * 2
        cols = self.D + (0 if self.v_of_k else self.dv)
        kv = self.B * self.kv_rows_read() * self.Hkv * cols * (1 if self.kv_dtype == "fp8" else 2)
        o = self.B * self.Sq * self.Hq * self.dv * ob
        lse = self.B * self.Hq * self.Sq * 4
        return q + kv + o + lse


WORKLOADS = {
    "tiny_causal_gqa_prefill": Workload(
        "tiny_causal_gqa_prefill", "prefill", B=1, Hq=4, Hkv=1, Sq=128, Skv=128, D=64,
        q_offset=0, causal=True, out_dtype="f32",
        note="B1 Hq4 Hkv1 S128 D64, fp32 out"),
    "gqa_causal_prefill_4k_d128": Workload(
        "gqa_causal_prefill_4k_d128", "prefill", B=1, Hq=32, Hkv=8, Sq=4096, Skv=4096, D=128,
        q_offset=0, causal=True, out_dtype="bf16",
        note="B1 Hq32 Hkv8 S4096 D128, bf16 out"),
    "prefill_at_depth_d256": Workload(
        "prefill_at_depth_d256", "prefill", B=1, Hq=16, Hkv=8, Sq=2048, Skv=10240, D=256,
        q_offset=8192, causal=True, out_dtype="bf16",
        note="2048 new queries at depth 8192 over 10240 keys, D256"),
    "split_kv_decode_d512": Workload(
        "split_kv_decode_d512", "decode", B=16, Hq=16, Hkv=1, Sq=1, Skv=16384, D=512,
        q_offset=16383, causal=True, out_dtype="bf16", num_splits=32,
        note="B16 Hq16 Hkv1 Skv16384 D512, 32 splits merged by LSE"),
    "spec_verify_decode_d128": Workload(
        "spec_verify_decode_d128", "decode", B=4, Hq=32, Hkv=8, Sq=8, Skv=32768, D=128,
        q_offset=32760, causal=True, out_dtype="bf16", num_splits=16,
        note="8 draft rows per sequence, causal among themselves, Skv 32768"),
    "prefill_4k_d128_softcap_alibi_sinks": Workload(
        "prefill_4k_d128_softcap_alibi_sinks", "prefill", B=1, Hq=32, Hkv=8, Sq=4096, Skv=4096, D=128,
        q_offset=0, causal=True, out_dtype="bf16", softcap=30.0, alibi_max_bias=8.0, sinks=True,
        note="the 4k causal GQA prefill with logit softcap 30, ALiBi (max bias 8) and per-head sinks"),
    "sliding_window_prefill_16k_w4096_d128": Workload(
        "sliding_window_prefill_16k_w4096_d128", "prefill", B=1, Hq=32, Hkv=8, Sq=16384, Skv=16384, D=128,
        q_offset=0, causal=True, out_dtype="bf16", window=4096,
        note="B1 Hq32 Hkv8 S16384 D128, causal with a 4096-key sliding window"),
    "split_kv_decode_d512_softcap_alibi_sinks": Workload(
        "split_kv_decode_d512_softcap_alibi_sinks", "decode", B=16, Hq=16, Hkv=1, Sq=1, Skv=16384, D=512,
        q_offset=16383, causal=True, out_dtype="bf16", num_splits=32, softcap=30.0, alibi_max_bias=8.0,
        sinks=True, note="the D512 split-KV decode with softcap 30, ALiBi (max bias 8) and sinks in the merge"),
    "prefill_4k_d128_mask": Workload(
        "prefill_4k_d128_mask", "prefill", B=1, Hq=32, Hkv=8, Sq=4096, Skv=4096, D=128,
        q_offset=0, causal=True, out_dtype="bf16", mask_batch=1,
        note="the 4k causal GQA prefill plus a shared additive bf16 mask (20 % of entries -inf)"),
    "spec_verify_decode_d128_mask": Workload(
        "spec_verify_decode_d128_mask", "decode", B=4, Hq=32, Hkv=8, Sq=8, Skv=32768, D=128,
        q_offset=32760, causal=True, out_dtype="bf16", num_splits=16, mask_batch=4,
        note="the 8-row verify decode with a per-sequence additive mask over all keys"),
    "fp8_kv_decode_d512": Workload(
        "fp8_kv_decode_d512", "decode", B=16, Hq=16, Hkv=1, Sq=1, Skv=16384, D=512,
        q_offset=16383, causal=True, out_dtype="bf16", num_splits=32, kv_dtype="fp8",
        note="the D512 split-KV decode over an fp8 e4m3 K/V cache with per-head scales"),
    "fp8_kv_spec_verify_decode_d128": Workload(
        "fp8_kv_spec_verify_decode_d128", "decode", B=4, Hq=32, Hkv=8, Sq=8, Skv=32768, D=128,
        q_offset=32760, causal=True, out_dtype="bf16", num_splits=16, kv_dtype="fp8",
        note="the 8-row verify decode over an fp8 e4m3 K/V cache"),
    "prefill_d512_g16_4k": Workload(
        "prefill_d512_g16_4k", "prefill", B=1, Hq=16, Hkv=1, Sq=4096, Skv=4096, D=512,
        q_offset=0, causal=True, out_dtype="bf16",
        note="B1 Hq16 Hkv1 Sq=Skv=4096 D512, causal: head size 512 with one K/V head (MLA-like width)"),
    "paged_decode_d512_p64": Workload(
        "paged_decode_d512_p64", "decode", B=16, Hq=16, Hkv=1, Sq=1, Skv=16384, D=512,
        q_offset=16383, causal=True, out_dtype="bf16", num_splits=32, page_size=64,
        note="the D512 split-KV decode over a paged cache: 64-key pages in scattered order"),
    "split_kv_decode_d512_fused": Workload(
        "split_kv_decode_d512_fused", "decode", B=16, Hq=16, Hkv=1, Sq=1, Skv=16384, D=512,
        q_offset=16383, causal=True, out_dtype="bf16", num_splits=8, fused=True,
        note="the D512 decode in one launch: 8 key ranges per sequence merged inside an 8-CTA cluster"),
    "spec_verify_decode_d128_fused": Workload(
        "spec_verify_decode_d128_fused", "decode", B=4, Hq=32, Hkv=8, Sq=8, Skv=32768, D=128,
        q_offset=32760, causal=True, out_dtype="bf16", num_splits=8, fused=True,
        note="the verify decode in one launch: 8 key ranges per (sequence, K/V head) merged in a cluster"),
    "mla_decode_d576_v512": Workload(
        "mla_decode_d576_v512", "decode", B=16, Hq=16, Hkv=1, Sq=1, Skv=16384, D=576, Dv=512, v_of_k=True,
        q_offset=16383, causal=True, out_dtype="bf16", num_splits=32,
        note="B16 Hq16 Hkv1 Skv16384, K 576 wide and V its first 512 columns (latent-cache decode)"),
    "prefill_d192_v128_4k": Workload(
        "prefill_d192_v128_4k", "prefill", B=1, Hq=32, Hkv=8, Sq=4096, Skv=4096, D=192, Dv=128,
        q_offset=0, causal=True, out_dtype="bf16",
        note="the 4k causal GQA prefill with Q/K head size 192 and V/O head size 128"),
}


def make_qkv(B, Hq, Hkv, Sq, Skv, D, *, seed=0, device="cpu", Dv=None):
    """Seeded q [B,Sq,Hq,D], k [B,Skv,Hkv,D] and v [B,Skv,Hkv,Dv] (Dv = D by
    default), all bf16, drawn q, k, v in order."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    q = torch.randn((B, Sq, Hq, D), generator=gen, dtype=torch.float32, device=device)
    q = q.to(torch.bfloat16)
    k = torch.randn((B, Skv, Hkv, D), generator=gen, dtype=torch.float32, device=device)
    k = k.to(torch.bfloat16)
    v = torch.randn((B, Skv, Hkv, Dv or D), generator=gen, dtype=torch.float32, device=device)
    v = v.to(torch.bfloat16)
    return q, k, v


def make_sinks(Hq, *, seed=0, std=3.0, device="cpu"):
    """Seeded fp32 sink logits [Hq] ~ N(0, std^2), one per query head."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return torch.randn((Hq,), generator=gen, dtype=torch.float32, device=device) * std


def make_paged(k, v, page_size, *, seed=0, extra_pages=3):
    """Scatter contiguous k, v [B, Skv, Hkv, D] into a paged cache.

    Returns (k_cache, v_cache, block_table): caches [num_pages, page_size, Hkv, D]
    with num_pages = B * ceil(Skv / page_size) + extra_pages, logical page j of
    sequence b stored at physical page block_table[b, j] (a seeded random
    permutation; the extra pages hold unrelated random rows), and the unused
    tail of each sequence's last page filled with random rows too."""
    B, Skv, Hkv, D = k.shape
    mp = (Skv + page_size - 1) // page_size
    n = B * mp + extra_pages
    gen = torch.Generator().manual_seed(seed)
    perm = torch.randperm(n, generator=gen)[: B * mp].reshape(B, mp).to(torch.int32)
    kc = torch.randn((n, page_size, Hkv, D), generator=gen).to(k.dtype)
    vc = torch.randn((n, page_size, Hkv, D), generator=gen).to(v.dtype)
    for b in range(B):
        for j in range(mp):
            t0, t1 = j * page_size, min(Skv, (j + 1) * page_size)
            kc[perm[b, j], : t1 - t0] = k[b, t0:t1]
            vc[perm[b, j], : t1 - t0] = v[b, t0:t1]
    return kc, vc, perm


def make_seq_lens(B, Skv, *, seed=0, low=1):
    """Seeded per-sequence key counts, uniform in [low, Skv], int32 [B]."""
    gen = torch.Generator().manual_seed(seed)
    return torch.randint(low, Skv + 1, (B,), generator=gen, dtype=torch.int64).to(torch.int32)


def make_mask(B, Sq, Skv, *, seed=0, std=2.0, p_inf=0.2, device="cpu"):
    """Seeded additive bf16 mask [B, Sq, Skv]: N(0, std^2) values with a
    fraction p_inf of the entries at -inf (key 0 of every row is kept)."""
    gen = torch.Generator().manual_seed(seed)
    m = torch.randn((B, Sq, Skv), generator=gen) * std
    cut = torch.rand((B, Sq, Skv), generator=gen) < p_inf
    cut[:, :, 0] = False
    m[cut] = float("-inf")
    return m.to(torch.bfloat16).to(device)


def make_fp8_kv(k, v):
    """An fp8 e4m3 K/V cache from bf16 k, v [B, Skv, Hkv, D]: per K/V head
    scale = max |x| / 448 (the largest e4m3 value), codes = x / scale cast to
    float8_e4m3fn (round to nearest even).  Returns (k_codes, v_codes,
    k_scale, v_scale): uint8 [B, Skv, Hkv, D] and fp32 [Hkv]."""
    out = []
    for x in (k, v):
        xf = x.float()
        amax = xf.abs().amax(dim=(0, 1, 3)).clamp_min(1e-12)
        sc = (amax / 448.0).to(torch.float32)
        codes = (xf / sc.view(1, 1, -1, 1)).to(torch.float8_e4m3fn).view(torch.uint8)
        out.append((codes, sc))
    return out[0][0], out[1][0], out[0][1], out[1][1]


def make_workload_inputs(w: Workload, *, seed=0, device="cpu"):
    """q, k, v of a workload; with v_of_k, v is the view k[..., :Dv]."""
    q, k, v = make_qkv(w.B, w.Hq, w.Hkv, w.Sq, w.Skv, w.D, seed=seed, device=device, Dv=w.dv)
    if w.v_of_k:
        v = k[..., :w.dv]
    return q, k, v


def sample_rows(w: Workload, n: int, *, seed=1234, include_edges=True):
    """(b, h, s) triples spread over the problem, including its corners."""
    gen = torch.Generator().manual_seed(seed)
    b = torch.randint(0, w.B, (n,), generator=gen)
    h = torch.randint(0, w.Hq, (n,), generator=gen)
    s = torch.randint(0, w.Sq, (n,), generator=gen)
    rows = torch.stack([b, h, s], dim=1).tolist()
    if include_edges:
        for bb in {0, w.B - 1}:
            for hh in {0, w.Hq - 1}:
                for ss in {0, 1, w.Sq // 2, w.Sq - 1}:
                    if 0 <= ss < w.Sq:
                        rows.append([bb, hh, ss])
    return rows
