"""Pins that tie the float64 oracle to facts fixed outside itself.

Each ``pin_*`` takes a loaded oracle library handle and raises AssertionError
when the oracle disagrees with what the mathematics or a worked example fixes.
They are run against the real oracle (tests/test_oracle_pins.py) and against
planted mutants of it (tests/test_oracle_mutants.py), so every plausible
mistake in the oracle (a dropped term, a wrong sign or index, an off-by-one
mask) is shown to fail at least one of them.

What pins what:
  brute force       textbook softmax in 40-digit decimal arithmetic on tiny
                    integer inputs, GQA by explicit head repetition
  golden            closed-form worked example (tests/golden/three_key_causal.txt)
  single key        a row that sees one key returns that V row exactly
  uniform logits    Q = 0 gives the mean of the visible V rows and LSE = ln|T|
  probs             each row of weights sums to one; masked weights are zero
  causal future     keys after the diagonal cannot change a row
  split merge       merge(split) equals the unsplit result for any split count
  gqa               grouped heads equal MHA with K/V heads repeated
  sdpa              torch's own float64 scaled_dot_product_attention
  permutation       non-causal attention is invariant to a joint (K, V) shuffle
  shift             adding u to every key leaves O and shifts LSE by scale*q.u
  large logits      huge logits give the arg-max V row and LSE = max logit
  scale             (q, scale) and (2q, scale/2) give identical results
  options           softcap, ALiBi, sinks and window: 40-digit decimal brute
                    force, the standard ALiBi slope values, geometric-series and
                    single-key closed forms, limits (huge cap, window 1 / Skv,
                    sink -inf), split/merge identity, torch SDPA with a bias
  narrow V          V with Dv < D columns: 40-digit decimal brute force and
                    torch SDPA with a value head size unlike the key's
"""
from __future__ import annotations

import decimal
import math
import os

import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _normal(rng, shape):
    # bf16-representable values so the same data could feed the GPU
    x = torch.from_numpy(rng.standard_normal(shape).astype(np.float32)).to(torch.bfloat16)
    return x.double().numpy()


def pin_bruteforce_decimal(lib):
    """Textbook softmax attention in 40-digit decimals on tiny integer inputs."""
    decimal.getcontext().prec = 40
    rng = _rng(1)
    for (B, Hq, Hkv, Sq, Skv, D, q_offset, causal) in [
        (1, 2, 1, 3, 4, 3, 1, True),
        (2, 4, 2, 2, 3, 2, 0, False),
        (1, 3, 3, 4, 4, 2, 0, True),
        (1, 2, 1, 2, 5, 4, 3, True),
    ]:
        q = rng.integers(-2, 3, size=(B, Sq, Hq, D)).astype(np.float64)
        k = rng.integers(-2, 3, size=(B, Skv, Hkv, D)).astype(np.float64)
        v = rng.integers(-3, 4, size=(B, Skv, Hkv, D)).astype(np.float64)
        scale = 0.5
        out, lse = oracle.attention(q, k, v, scale=scale, causal=causal, q_offset=q_offset, lib=lib)
        g = Hq // Hkv
        # explicit MHA copy of K and V: head h reads kv head floor(h/g)
        kk = [[[k[b, t, h // g] for h in range(Hq)] for t in range(Skv)] for b in range(B)]
        vv = [[[v[b, t, h // g] for h in range(Hq)] for t in range(Skv)] for b in range(B)]
        for b in range(B):
            for h in range(Hq):
                for s in range(Sq):
                    ts = [t for t in range(Skv) if (not causal) or t <= q_offset + s]
                    ex = []
                    for t in ts:
                        dot = sum(decimal.Decimal(int(q[b, s, h, d])) * decimal.Decimal(int(kk[b][t][h][d]))
                                  for d in range(D))
                        ex.append((decimal.Decimal(scale) * dot).exp())
                    den = sum(ex)
                    want_lse = den.ln()
                    for d in range(D):
                        num = sum(e * decimal.Decimal(int(vv[b][t][h][d])) for e, t in zip(ex, ts))
                        want = num / den
                        assert abs(float(want) - out[b, s, h, d]) < 1e-13, (b, h, s, d)
                    assert abs(float(want_lse) - lse[b, h, s]) < 1e-13, (b, h, s)


def pin_golden_three_keys(lib):
    """Closed-form worked example: logits 0, 1, 2 under a causal mask."""
    rows = []
    with open(os.path.join(GOLDEN, "three_key_causal.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([float(x) for x in line.split()])
    q = np.zeros((1, 3, 1, 3))
    q[0, :, 0, 0] = 1.0
    k = np.zeros((1, 3, 1, 3))
    k[0, 1, 0, 0] = 1.0
    k[0, 2, 0, 0] = 2.0
    v = np.zeros((1, 3, 1, 3))
    for t in range(3):
        v[0, t, 0, t] = 1.0
    out, lse = oracle.attention(q, k, v, scale=1.0, causal=True, q_offset=0, lib=lib)
    for r in rows:
        s = int(r[0])
        np.testing.assert_allclose(out[0, s, 0, :], r[1:4], rtol=0, atol=1e-14)
        assert abs(lse[0, 0, s] - r[4]) < 1e-13


def pin_single_visible_key(lib):
    """Causal row 0 at q_offset 0 (and any row over one key) returns V exactly."""
    rng = _rng(2)
    B, Hq, Hkv, Sq, Skv, D = 2, 4, 2, 5, 7, 16
    q, k, v = _normal(rng, (B, Sq, Hq, D)), _normal(rng, (B, Skv, Hkv, D)), _normal(rng, (B, Skv, Hkv, D))
    scale = 0.25
    out, lse = oracle.attention(q, k, v, scale=scale, causal=True, q_offset=0, lib=lib)
    for b in range(B):
        for h in range(Hq):
            kvh = h // (Hq // Hkv)
            assert np.array_equal(out[b, 0, h], v[b, 0, kvh])
            want = scale * float(np.dot(q[b, 0, h], k[b, 0, kvh]))
            assert abs(lse[b, h, 0] - want) <= 1e-12 * max(1.0, abs(want))
    # one key, non-causal: every row is that key's V row
    out1, lse1 = oracle.attention(q, k[:, :1], v[:, :1], scale=scale, causal=False, lib=lib)
    for b in range(B):
        for h in range(Hq):
            kvh = h // (Hq // Hkv)
            for s in range(Sq):
                assert np.array_equal(out1[b, s, h], v[b, 0, kvh])


def pin_uniform_logits(lib):
    """Q = 0: O is the mean of the visible V rows and LSE = ln(number visible)."""
    rng = _rng(3)
    B, Hq, Hkv, Sq, Skv, D = 1, 2, 1, 6, 9, 8
    q = np.zeros((B, Sq, Hq, D))
    k, v = _normal(rng, (B, Skv, Hkv, D)), _normal(rng, (B, Skv, Hkv, D))
    q_offset = 2
    out, lse = oracle.attention(q, k, v, scale=0.3, causal=True, q_offset=q_offset, lib=lib)
    for s in range(Sq):
        n = min(Skv, q_offset + s + 1)
        for h in range(Hq):
            np.testing.assert_allclose(out[0, s, h], v[0, :n, 0].mean(axis=0), rtol=0, atol=1e-13)
            assert abs(lse[0, h, s] - math.log(n)) < 1e-13


def pin_probs_sum_to_one(lib):
    """Each row of weights is a distribution; masked keys have weight zero."""
    rng = _rng(4)
    B, Hq, Hkv, Sq, Skv, D = 1, 4, 2, 5, 11, 16
    q, k, v = _normal(rng, (B, Sq, Hq, D)), _normal(rng, (B, Skv, Hkv, D)), _normal(rng, (B, Skv, Hkv, D))
    q_offset = 3
    out, _ = oracle.attention(q, k, v, scale=0.25, causal=True, q_offset=q_offset, lib=lib)
    for h in range(Hq):
        for s in range(Sq):
            p = oracle.probs(q, k, 0, h, s, scale=0.25, causal=True, q_offset=q_offset, lib=lib)
            assert abs(p.sum() - 1.0) < 1e-14
            assert np.all(p[q_offset + s + 1:] == 0.0)
            assert np.all(p[: q_offset + s + 1] > 0.0)
            kvh = h // (Hq // Hkv)
            np.testing.assert_allclose(p @ v[0, :, kvh], out[0, s, h], rtol=0, atol=1e-13)


def pin_causal_ignores_future(lib):
    """Changing keys and values after a row's diagonal leaves that row unchanged."""
    rng = _rng(5)
    B, Hq, Hkv, Sq, Skv, D = 1, 2, 1, 8, 8, 16
    q, k, v = _normal(rng, (B, Sq, Hq, D)), _normal(rng, (B, Skv, Hkv, D)), _normal(rng, (B, Skv, Hkv, D))
    out, lse = oracle.attention(q, k, v, scale=0.25, causal=True, lib=lib)
    cut = 4
    k2, v2 = k.copy(), v.copy()
    k2[:, cut + 1:] = _normal(rng, k2[:, cut + 1:].shape)
    v2[:, cut + 1:] = _normal(rng, v2[:, cut + 1:].shape)
    out2, lse2 = oracle.attention(q, k2, v2, scale=0.25, causal=True, lib=lib)
    assert np.array_equal(out[:, : cut + 1], out2[:, : cut + 1])
    assert np.array_equal(lse[:, :, : cut + 1], lse2[:, :, : cut + 1])
    assert not np.allclose(out[:, cut + 1:], out2[:, cut + 1:])


def pin_split_merge(lib):
    """Merging per-split partials reproduces unsplit attention, empty splits included."""
    rng = _rng(6)
    B, Hq, Hkv, Sq, Skv, D = 2, 4, 2, 3, 37, 16
    q, k, v = _normal(rng, (B, Sq, Hq, D)), _normal(rng, (B, Skv, Hkv, D)), _normal(rng, (B, Skv, Hkv, D))
    for causal, q_offset in [(True, 20), (False, 0), (True, 0)]:
        out, lse = oracle.attention(q, k, v, scale=0.25, causal=causal, q_offset=q_offset, lib=lib)
        for S in (1, 2, 7, 32, Skv):
            po, pl = oracle.split(q, k, v, S, scale=0.25, causal=causal, q_offset=q_offset, lib=lib)
            mo, ml = oracle.merge(po, pl, lib=lib)
            np.testing.assert_allclose(mo, out, rtol=0, atol=1e-12)
            np.testing.assert_allclose(ml, lse, rtol=0, atol=1e-12)
            chunk = -(-Skv // S)
            for sg in range(S):
                lo = sg * chunk
                for s in range(Sq):
                    last = Skv if not causal else min(Skv, q_offset + s + 1)
                    if lo >= last:  # no visible key: must publish (-inf, 0)
                        assert np.all(np.isneginf(pl[sg, :, :, s]))
                        assert np.all(po[sg, :, s] == 0.0)
        # one key per split: partial O is that V row, partial LSE its logit
        po, pl = oracle.split(q, k, v, Skv, scale=0.25, causal=False, lib=lib)
        for t in (0, 5, Skv - 1):
            for h in range(Hq):
                kvh = h // (Hq // Hkv)
                assert np.array_equal(po[t, 0, 0, h], v[0, t, kvh])
                want = 0.25 * float(np.dot(q[0, 0, h], k[0, t, kvh]))
                assert abs(pl[t, 0, h, 0] - want) < 1e-12


def pin_gqa_equals_repeated_mha(lib):
    """Hq heads over Hkv groups equal MHA with each K/V head repeated g times."""
    rng = _rng(7)
    B, Hq, Hkv, Sq, Skv, D = 1, 6, 2, 5, 9, 8
    q, k, v = _normal(rng, (B, Sq, Hq, D)), _normal(rng, (B, Skv, Hkv, D)), _normal(rng, (B, Skv, Hkv, D))
    g = Hq // Hkv
    kr, vr = np.repeat(k, g, axis=2), np.repeat(v, g, axis=2)
    out, lse = oracle.attention(q, k, v, scale=0.3, causal=True, q_offset=2, lib=lib)
    out2, lse2 = oracle.attention(q, kr, vr, scale=0.3, causal=True, q_offset=2, lib=lib)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


def pin_torch_sdpa(lib):
    """torch's float64 scaled_dot_product_attention with an explicit bottom-right mask."""
    rng = _rng(8)
    B, Hq, Hkv, Sq, Skv, D = 2, 8, 2, 7, 19, 32
    q, k, v = _normal(rng, (B, Sq, Hq, D)), _normal(rng, (B, Skv, Hkv, D)), _normal(rng, (B, Skv, Hkv, D))
    g = Hq // Hkv
    for causal, q_offset in [(True, 12), (True, 0), (False, 0)]:
        out, lse = oracle.attention(q, k, v, scale=0.2, causal=causal, q_offset=q_offset, lib=lib)
        tq = torch.from_numpy(q).permute(0, 2, 1, 3)                      # B,Hq,Sq,D
        tk = torch.from_numpy(k).permute(0, 2, 1, 3).repeat_interleave(g, dim=1)
        tv = torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(g, dim=1)
        mask = None
        if causal:
            s_idx = torch.arange(Sq).view(-1, 1) + q_offset
            t_idx = torch.arange(Skv).view(1, -1)
            mask = t_idx <= s_idx
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=0.2)
        np.testing.assert_allclose(out, ref.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)
        logits = (tq @ tk.transpose(-1, -2)) * 0.2
        if mask is not None:
            logits = logits.masked_fill(~mask, float("-inf"))
        np.testing.assert_allclose(lse, torch.logsumexp(logits, dim=-1).numpy(), rtol=0, atol=1e-12)


def pin_key_permutation(lib):
    """Non-causal attention does not depend on the order of the (key, value) pairs."""
    rng = _rng(9)
    B, Hq, Hkv, Sq, Skv, D = 1, 4, 4, 6, 23, 16
    q, k, v = _normal(rng, (B, Sq, Hq, D)), _normal(rng, (B, Skv, Hkv, D)), _normal(rng, (B, Skv, Hkv, D))
    perm = rng.permutation(Skv)
    out, lse = oracle.attention(q, k, v, scale=0.25, causal=False, lib=lib)
    out2, lse2 = oracle.attention(q, k[:, perm], v[:, perm], scale=0.25, causal=False, lib=lib)
    np.testing.assert_allclose(out, out2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, lse2, rtol=0, atol=1e-13)


def pin_shift_invariance(lib):
    """k_t -> k_t + u for every t: O is unchanged and LSE moves by scale * q.u."""
    rng = _rng(10)
    B, Hq, Hkv, Sq, Skv, D = 1, 2, 1, 5, 12, 8
    q, k, v = _normal(rng, (B, Sq, Hq, D)), _normal(rng, (B, Skv, Hkv, D)), _normal(rng, (B, Skv, Hkv, D))
    u = rng.integers(-3, 4, size=(D,)).astype(np.float64)
    out, lse = oracle.attention(q, k, v, scale=0.5, causal=True, q_offset=3, lib=lib)
    out2, lse2 = oracle.attention(q, k + u, v, scale=0.5, causal=True, q_offset=3, lib=lib)
    np.testing.assert_allclose(out2, out, rtol=0, atol=1e-12)
    shift = 0.5 * np.einsum("bshd,d->bhs", q, u)
    np.testing.assert_allclose(lse2, lse + shift, rtol=0, atol=1e-12)


def pin_large_logits(lib):
    """Logits spread by thousands: O is the arg-max V row, LSE the largest logit."""
    rng = _rng(11)
    B, Hq, Hkv, Sq, Skv, D = 1, 2, 1, 4, 16, 8
    q, k, v = _normal(rng, (B, Sq, Hq, D)), _normal(rng, (B, Skv, Hkv, D)), _normal(rng, (B, Skv, Hkv, D))
    q = q * 4096.0
    out, lse = oracle.attention(q, k, v, scale=1.0, causal=False, lib=lib)
    for h in range(Hq):
        for s in range(Sq):
            z = np.array([float(np.dot(q[0, s, h], k[0, t, 0])) for t in range(Skv)])
            top = np.argsort(z)
            assert z[top[-1]] - z[top[-2]] > 800.0  # the rest underflow in fp64
            np.testing.assert_allclose(out[0, s, h], v[0, top[-1], 0], rtol=0, atol=1e-12)
            assert abs(lse[0, h, s] - z[top[-1]]) <= 1e-12 * abs(z[top[-1]])


def pin_scale_power_of_two(lib):
    """(q, scale) and (2q, scale/2) are the same logits, so results are identical."""
    rng = _rng(12)
    B, Hq, Hkv, Sq, Skv, D = 1, 4, 2, 6, 10, 16
    q, k, v = _normal(rng, (B, Sq, Hq, D)), _normal(rng, (B, Skv, Hkv, D)), _normal(rng, (B, Skv, Hkv, D))
    out, lse = oracle.attention(q, k, v, scale=0.125, causal=True, q_offset=4, lib=lib)
    out2, lse2 = oracle.attention(2.0 * q, k, v, scale=0.0625, causal=True, q_offset=4, lib=lib)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)
    out3, _ = oracle.attention(q, k, v, scale=0.25, causal=True, q_offset=4, lib=lib)
    assert not np.allclose(out, out3)


# ---------------------------------------------------------------- options ----
# Pins for the optional logit terms (softcap, ALiBi, sinks, sliding window).

def _alibi_pow2(h, n, max_bias):
    """ALiBi slope for a power-of-two head count n: 2^(-max_bias (h+1) / n)."""
    return 2.0 ** (-max_bias * (h + 1) / n)


def pin_ext_bruteforce_decimal(lib):
    """Textbook softmax in 40-digit decimals with softcap, ALiBi, a sink and a window."""
    decimal.getcontext().prec = 40
    Dd = decimal.Decimal
    rng = _rng(21)

    def tanh(x):
        e2 = (2 * x).exp()
        return (e2 - 1) / (e2 + 1)

    for (B, Hq, Hkv, Sq, Skv, D, q_offset, causal, cap, mb, window, use_sink) in [
        (1, 4, 2, 3, 6, 2, 3, True, 1.5, 8.0, 0, True),
        (1, 2, 1, 4, 5, 3, 1, True, 0.0, 4.0, 2, False),
        (2, 2, 2, 2, 4, 2, 0, False, 0.75, 0.0, 0, True),
        (1, 4, 1, 3, 7, 2, 4, True, 0.0, 0.0, 3, True),
    ]:
        q = rng.integers(-2, 3, size=(B, Sq, Hq, D)).astype(np.float64)
        k = rng.integers(-2, 3, size=(B, Skv, Hkv, D)).astype(np.float64)
        v = rng.integers(-3, 4, size=(B, Skv, Hkv, D)).astype(np.float64)
        sinks = rng.integers(-2, 3, size=(Hq,)).astype(np.float64) if use_sink else None
        scale = 0.5
        out, lse = oracle.attention_ex(q, k, v, scale=scale, causal=causal, q_offset=q_offset, softcap=cap,
                                       alibi_max_bias=mb, sinks=sinks, window=window, lib=lib)
        g = Hq // Hkv
        for b in range(B):
            for h in range(Hq):
                slope = Dd(_alibi_pow2(h, Hq, mb)) if mb > 0 else Dd(0)
                for s in range(Sq):
                    pos = q_offset + s
                    ts = [t for t in range(Skv) if ((not causal) or t <= pos) and (window == 0 or t > pos - window)]
                    ex = []
                    for t in ts:
                        z = Dd(scale) * sum(Dd(int(q[b, s, h, d])) * Dd(int(k[b, t, h // g, d])) for d in range(D))
                        if cap > 0:
                            z = Dd(cap) * tanh(z / Dd(cap))
                        z = z + slope * (t - pos)
                        ex.append(z.exp())
                    den = sum(ex) + (Dd(int(sinks[h])).exp() if use_sink else Dd(0))
                    for d in range(D):
                        num = sum(e * Dd(int(v[b, t, h // g, d])) for e, t in zip(ex, ts))
                        assert abs(float(num / den) - out[b, s, h, d]) < 1e-13, (b, h, s, d)
                    assert abs(float(den.ln()) - lse[b, h, s]) < 1e-13, (b, h, s)


def pin_alibi_slopes(lib):
    """Geometric ALiBi slopes: 2^-1..2^-8 for 8 heads at max_bias 8; for 12 heads
    the first 8 as for 8 heads, then the odd powers of 2^-1/2."""
    for h in range(8):
        assert oracle.alibi_slope(h, 8, 8.0, lib=lib) == 2.0 ** -(h + 1)
    want12 = [2.0 ** -(h + 1) for h in range(8)] + [2.0 ** -(0.5 + j) for j in range(4)]
    for h in range(12):
        assert abs(oracle.alibi_slope(h, 12, 8.0, lib=lib) - want12[h]) < 1e-15


def pin_alibi_geometric_closed_form(lib):
    """Q = 0: the logits are slope*(t - pos), a geometric series in closed form."""
    rng = _rng(22)
    B, Hq, Hkv, Sq, Skv, D = 1, 4, 1, 5, 9, 4
    q = np.zeros((B, Sq, Hq, D))
    k, v = _normal(rng, (B, Skv, Hkv, D)), _normal(rng, (B, Skv, Hkv, D))
    q_offset = 3
    out, lse = oracle.attention_ex(q, k, v, scale=0.3, causal=True, q_offset=q_offset, alibi_max_bias=8.0, lib=lib)
    for h in range(Hq):
        r = math.exp(-_alibi_pow2(h, Hq, 8.0))
        for s in range(Sq):
            pos = q_offset + s
            n = min(Skv, pos + 1)
            w = np.array([r ** (pos - t) for t in range(n)])
            np.testing.assert_allclose(out[0, s, h], (w[:, None] * v[0, :n, 0]).sum(0) / w.sum(), rtol=0, atol=1e-13)
            assert abs(lse[0, h, s] - math.log((1 - r ** n) / (1 - r))) < 1e-13


def pin_sink_closed_form(lib):
    """A row that sees one key z with a sink s: O = V e^z/(e^z + e^s), LSE = log(e^z + e^s);
    a sink of -inf changes nothing."""
    rng = _rng(23)
    B, Hq, Hkv, Sq, Skv, D = 1, 4, 2, 3, 6, 8
    q, k, v = _normal(rng, (B, Sq, Hq, D)), _normal(rng, (B, Skv, Hkv, D)), _normal(rng, (B, Skv, Hkv, D))
    sinks = np.array([0.5, -1.0, 2.0, 0.0])
    out, lse = oracle.attention_ex(q, k, v, scale=0.25, causal=True, sinks=sinks, lib=lib)
    for h in range(Hq):
        kvh = h // 2
        z = 0.25 * float(np.dot(q[0, 0, h], k[0, 0, kvh]))
        w = math.exp(z) / (math.exp(z) + math.exp(sinks[h]))
        np.testing.assert_allclose(out[0, 0, h], w * v[0, 0, kvh], rtol=0, atol=1e-14)
        assert abs(lse[0, h, 0] - math.log(math.exp(z) + math.exp(sinks[h]))) < 1e-13
    o0, l0 = oracle.attention(q, k, v, scale=0.25, causal=True, lib=lib)
    o1, l1 = oracle.attention_ex(q, k, v, scale=0.25, causal=True, sinks=np.full(Hq, -np.inf), lib=lib)
    assert np.array_equal(o0, o1) and np.array_equal(l0, l1)


def pin_softcap_limits(lib):
    """A huge cap changes nothing; a small cap bounds every logit by +-cap."""
    rng = _rng(24)
    B, Hq, Hkv, Sq, Skv, D = 1, 2, 1, 4, 10, 8
    q, k, v = _normal(rng, (B, Sq, Hq, D)), _normal(rng, (B, Skv, Hkv, D)), _normal(rng, (B, Skv, Hkv, D))
    o0, l0 = oracle.attention(q, k, v, scale=0.5, causal=False, lib=lib)
    o1, l1 = oracle.attention_ex(q, k, v, scale=0.5, causal=False, softcap=1e9, lib=lib)
    np.testing.assert_allclose(o1, o0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l1, l0, rtol=0, atol=1e-12)
    cap = 0.25
    o2, l2 = oracle.attention_ex(100.0 * q, k, v, scale=0.5, causal=False, softcap=cap, lib=lib)
    assert np.all(l2 <= cap + math.log(Skv) + 1e-12) and np.all(l2 >= -cap + math.log(Skv) - 1e-12)


def pin_window_limits(lib):
    """Window 1: each row sees only its own position; a window of Skv is plain causal."""
    rng = _rng(25)
    B, Hq, Hkv, Sq, Skv, D = 1, 4, 2, 6, 9, 8
    q, k, v = _normal(rng, (B, Sq, Hq, D)), _normal(rng, (B, Skv, Hkv, D)), _normal(rng, (B, Skv, Hkv, D))
    q_offset = 3
    out, lse = oracle.attention_ex(q, k, v, scale=0.3, causal=True, q_offset=q_offset, window=1, lib=lib)
    for s in range(Sq):
        pos = q_offset + s
        for h in range(Hq):
            kvh = h // 2
            assert np.array_equal(out[0, s, h], v[0, pos, kvh])
            assert abs(lse[0, h, s] - 0.3 * float(np.dot(q[0, s, h], k[0, pos, kvh]))) < 1e-12
    o0, l0 = oracle.attention(q, k, v, scale=0.3, causal=True, q_offset=q_offset, lib=lib)
    o1, l1 = oracle.attention_ex(q, k, v, scale=0.3, causal=True, q_offset=q_offset, window=Skv, lib=lib)
    assert np.array_equal(o0, o1) and np.array_equal(l0, l1)


def pin_split_merge_ex(lib):
    """Merging split partials (sinks added once, by the merge) reproduces the unsplit result."""
    rng = _rng(26)
    B, Hq, Hkv, Sq, Skv, D = 1, 4, 2, 3, 29, 8
    q, k, v = _normal(rng, (B, Sq, Hq, D)), _normal(rng, (B, Skv, Hkv, D)), _normal(rng, (B, Skv, Hkv, D))
    sinks = np.array([0.3, -0.7, 1.1, 0.0])
    kw = dict(scale=0.3, causal=True, q_offset=Skv - Sq, softcap=2.0, alibi_max_bias=4.0, window=11)
    out, lse = oracle.attention_ex(q, k, v, sinks=sinks, lib=lib, **kw)
    for S in (1, 3, 7):
        po, pl = oracle.split_ex(q, k, v, S, lib=lib, **kw)
        mo, ml = oracle.merge_ex(po, pl, sinks=sinks, lib=lib)
        np.testing.assert_allclose(mo, out, rtol=0, atol=1e-12)
        np.testing.assert_allclose(ml, lse, rtol=0, atol=1e-12)


def pin_torch_sdpa_bias(lib):
    """torch's float64 SDPA with an additive ALiBi + window bias (masked keys at -inf)."""
    rng = _rng(27)
    B, Hq, Hkv, Sq, Skv, D = 1, 8, 2, 5, 13, 16
    q, k, v = _normal(rng, (B, Sq, Hq, D)), _normal(rng, (B, Skv, Hkv, D)), _normal(rng, (B, Skv, Hkv, D))
    q_offset, window, mb = 8, 6, 8.0
    out, lse = oracle.attention_ex(q, k, v, scale=0.2, causal=True, q_offset=q_offset, alibi_max_bias=mb,
                                   window=window, lib=lib)
    g = Hq // Hkv
    tq = torch.from_numpy(q).permute(0, 2, 1, 3)
    tk = torch.from_numpy(k).permute(0, 2, 1, 3).repeat_interleave(g, dim=1)
    tv = torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(g, dim=1)
    pos = torch.arange(Sq, dtype=torch.float64).view(-1, 1) + q_offset
    t = torch.arange(Skv, dtype=torch.float64).view(1, -1)
    slopes = torch.tensor([_alibi_pow2(h, Hq, mb) for h in range(Hq)], dtype=torch.float64).view(1, -1, 1, 1)
    bias = slopes * (t - pos)
    visible = (t <= pos) & (t > pos - window)
    bias = bias.masked_fill(~visible, float("-inf"))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=bias, scale=0.2)
    np.testing.assert_allclose(out, ref.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)
    logits = (tq @ tk.transpose(-1, -2)) * 0.2 + bias
    np.testing.assert_allclose(lse, torch.logsumexp(logits, dim=-1).numpy(), rtol=0, atol=1e-12)


def _mask(rng, B, Sq, Skv, p_inf=0.2):
    """A random additive mask [B, Sq, Skv] with some -inf entries (never a full row)."""
    m = _normal(rng, (B, Sq, Skv)) * 2.0
    cut = rng.random((B, Sq, Skv)) < p_inf
    cut[:, :, 0] = False
    m[cut] = -np.inf
    return m


def pin_mask_torch_sdpa(lib):
    """torch's float64 SDPA with the same additive mask (-inf entries included),
    per-batch and shared across the batch."""
    rng = _rng(31)
    B, Hq, Hkv, Sq, Skv, D = 2, 4, 2, 5, 9, 8
    q, k, v = _normal(rng, (B, Sq, Hq, D)), _normal(rng, (B, Skv, Hkv, D)), _normal(rng, (B, Skv, Hkv, D))
    g = Hq // Hkv
    tq = torch.from_numpy(q).permute(0, 2, 1, 3)
    tk = torch.from_numpy(k).permute(0, 2, 1, 3).repeat_interleave(g, dim=1)
    tv = torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(g, dim=1)
    for mask in (_mask(rng, B, Sq, Skv), _mask(rng, 1, Sq, Skv)):
        out, lse = oracle.attention_ex(q, k, v, scale=0.3, causal=False, mask=mask, lib=lib)
        tm = torch.from_numpy(mask)[:, None]          # broadcast over heads
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=tm, scale=0.3)
        np.testing.assert_allclose(out, ref.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)
        logits = (tq @ tk.transpose(-1, -2)) * 0.3 + tm
        np.testing.assert_allclose(lse, torch.logsumexp(logits, dim=-1).numpy(), rtol=0, atol=1e-12)


def pin_mask_removes_keys_and_shifts(lib):
    """A -inf mask entry removes that key (same as dropping the key row); a mask
    constant along a row leaves O unchanged and adds the constant to the LSE,
    also under softcap and ALiBi."""
    rng = _rng(32)
    B, Hq, Hkv, Sq, Skv, D = 1, 2, 1, 3, 7, 4
    q, k, v = _normal(rng, (B, Sq, Hq, D)), _normal(rng, (B, Skv, Hkv, D)), _normal(rng, (B, Skv, Hkv, D))
    keep = np.array([0, 2, 3, 6])
    mask = np.full((1, Sq, Skv), -np.inf)
    mask[:, :, keep] = 0.0
    out, lse = oracle.attention_ex(q, k, v, scale=0.5, causal=False, mask=mask, lib=lib)
    ref_o, ref_l = oracle.attention(q, k[:, keep], v[:, keep], scale=0.5, causal=False, lib=lib)
    np.testing.assert_allclose(out, ref_o, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, ref_l, rtol=0, atol=1e-14)
    c = np.array([0.75, -2.5, 4.0]).reshape(1, Sq, 1) * np.ones((1, Sq, Skv))
    kw = dict(scale=0.5, causal=True, q_offset=Skv - Sq, softcap=1.5, alibi_max_bias=2.0, lib=lib)
    o0, l0 = oracle.attention_ex(q, k, v, **kw)
    o1, l1 = oracle.attention_ex(q, k, v, mask=c, **kw)
    np.testing.assert_allclose(o1, o0, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l0 + np.array([0.75, -2.5, 4.0]).reshape(1, 1, Sq), rtol=0, atol=1e-13)


def pin_mask_fully_masked_row(lib):
    """A row whose every visible key is masked: O = 0 and LSE = -inf, or
    LSE = the sink logit when a sink is present."""
    rng = _rng(33)
    B, Hq, Hkv, Sq, Skv, D = 1, 2, 2, 2, 5, 4
    q, k, v = _normal(rng, (B, Sq, Hq, D)), _normal(rng, (B, Skv, Hkv, D)), _normal(rng, (B, Skv, Hkv, D))
    mask = np.zeros((1, Sq, Skv))
    mask[0, 1] = -np.inf
    out, lse = oracle.attention_ex(q, k, v, scale=0.5, causal=False, mask=mask, lib=lib)
    assert np.all(out[0, 1] == 0.0) and np.all(np.isneginf(lse[0, :, 1]))
    assert np.all(np.isfinite(lse[0, :, 0]))
    sinks = np.array([0.5, -1.0])
    out, lse = oracle.attention_ex(q, k, v, scale=0.5, causal=False, mask=mask, sinks=sinks, lib=lib)
    assert np.all(out[0, 1] == 0.0)
    np.testing.assert_allclose(lse[0, :, 1], sinks, rtol=0, atol=1e-15)


def pin_split_merge_mask(lib):
    """Split-then-merge with a mask equals the unsplit result."""
    rng = _rng(34)
    B, Hq, Hkv, Sq, Skv, D = 2, 4, 1, 3, 23, 8
    q, k, v = _normal(rng, (B, Sq, Hq, D)), _normal(rng, (B, Skv, Hkv, D)), _normal(rng, (B, Skv, Hkv, D))
    mask = _mask(rng, B, Sq, Skv, p_inf=0.4)
    kw = dict(scale=0.3, causal=True, q_offset=Skv - Sq, mask=mask, lib=lib)
    out, lse = oracle.attention_ex(q, k, v, **kw)
    for S in (1, 4, 23):
        po, pl = oracle.split_ex(q, k, v, S, **kw)
        mo, ml = oracle.merge(po, pl, lib=lib)
        np.testing.assert_allclose(mo, out, rtol=0, atol=1e-12)
        np.testing.assert_allclose(ml, lse, rtol=0, atol=1e-12)


def pin_e4m3_codes_match_torch(lib):
    """The oracle's e4m3 decoder against torch's float8_e4m3fn for all 256 codes."""
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).double().numpy()
    got = np.array([oracle.e4m3_value(c, lib=lib) for c in range(256)])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert got[0x7e] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x08] == 2.0 ** -6 and got[0xb8] == -1.0


def pin_fp8_attention_equals_dequantized(lib):
    """Attention over fp8 codes with per-head scales equals attention over the
    values torch decodes, times the scales (non-unit, per head)."""
    rng = _rng(41)
    B, Hq, Hkv, Sq, Skv, D = 2, 4, 2, 3, 9, 8
    q = _normal(rng, (B, Sq, Hq, D))
    kc = torch.from_numpy(rng.integers(0, 256, (B, Skv, Hkv, D), dtype=np.uint8))
    vc = torch.from_numpy(rng.integers(0, 256, (B, Skv, Hkv, D), dtype=np.uint8))
    kc[(kc & 0x7f) == 0x7f] = 0x3c                   # no NaN codes
    vc[(vc & 0x7f) == 0x7f] = 0x41
    ks, vs = np.array([0.01, 0.003]), np.array([0.5, 0.02])
    kd = kc.view(torch.float8_e4m3fn).double().numpy() * ks.reshape(1, 1, -1, 1)
    vd = vc.view(torch.float8_e4m3fn).double().numpy() * vs.reshape(1, 1, -1, 1)
    kw = dict(scale=0.3, causal=True, q_offset=Skv - Sq, lib=lib)
    out, lse = oracle.attention_fp8(q, kc, vc, ks, vs, **kw)
    ref_o, ref_l = oracle.attention(q, kd, vd, **kw)
    np.testing.assert_array_equal(out, ref_o)
    np.testing.assert_array_equal(lse, ref_l)


def pin_narrow_v_bruteforce_decimal(lib):
    """V with fewer columns than K (Dv < D): textbook softmax in 40-digit
    decimals, through attention_ex and attention_rows_ex."""
    decimal.getcontext().prec = 40
    Dd = decimal.Decimal
    rng = _rng(41)
    for (B, Hq, Hkv, Sq, Skv, D, Dv, q_offset, causal, window, use_sink) in [
        (1, 2, 1, 3, 5, 3, 2, 2, True, 0, False),
        (2, 4, 2, 2, 4, 4, 1, 0, False, 0, True),
        (1, 4, 1, 3, 6, 5, 2, 3, True, 2, True),
    ]:
        q = rng.integers(-2, 3, size=(B, Sq, Hq, D)).astype(np.float64)
        k = rng.integers(-2, 3, size=(B, Skv, Hkv, D)).astype(np.float64)
        v = rng.integers(-3, 4, size=(B, Skv, Hkv, Dv)).astype(np.float64)
        sinks = rng.integers(-2, 3, size=(Hq,)).astype(np.float64) if use_sink else None
        scale = 0.5
        kw = dict(scale=scale, causal=causal, q_offset=q_offset, sinks=sinks, window=window, lib=lib)
        out, lse = oracle.attention_ex(q, k, v, **kw)
        assert out.shape == (B, Sq, Hq, Dv)
        rows = [(b, h, s) for b in range(B) for h in range(Hq) for s in range(Sq)]
        ro, rl = oracle.attention_rows_ex(q, k, v, rows, **kw)
        assert ro.shape == (len(rows), Dv)
        g = Hq // Hkv
        for i, (b, h, s) in enumerate(rows):
            pos = q_offset + s
            ts = [t for t in range(Skv) if ((not causal) or t <= pos) and (window == 0 or t > pos - window)]
            ex = [(Dd(scale) * sum(Dd(int(q[b, s, h, d])) * Dd(int(k[b, t, h // g, d])) for d in range(D))).exp()
                  for t in ts]
            den = sum(ex) + (Dd(int(sinks[h])).exp() if use_sink else Dd(0))
            for d in range(Dv):
                want = float(sum(e * Dd(int(v[b, t, h // g, d])) for e, t in zip(ex, ts)) / den)
                assert abs(want - out[b, s, h, d]) < 1e-13 and abs(want - ro[i, d]) < 1e-13, (b, h, s, d)
            assert abs(float(den.ln()) - lse[b, h, s]) < 1e-13 and abs(float(den.ln()) - rl[i]) < 1e-13


def pin_narrow_v_torch_sdpa(lib):
    """V with Dv < D columns against torch's float64 SDPA, which takes a value
    head size unlike the key's."""
    rng = _rng(42)
    B, Hq, Hkv, Sq, Skv, D, Dv = 2, 6, 2, 5, 11, 12, 8
    q = _normal(rng, (B, Sq, Hq, D))
    k = _normal(rng, (B, Skv, Hkv, D))
    v = _normal(rng, (B, Skv, Hkv, Dv))
    out, _ = oracle.attention_ex(q, k, v, scale=0.3, causal=False, lib=lib)
    g = Hq // Hkv
    tq = torch.from_numpy(q).permute(0, 2, 1, 3)
    tk = torch.from_numpy(k).permute(0, 2, 1, 3).repeat_interleave(g, dim=1)
    tv = torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(g, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=0.3).permute(0, 2, 1, 3).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


ALL_PINS = [
    pin_bruteforce_decimal,
    pin_golden_three_keys,
    pin_single_visible_key,
    pin_uniform_logits,
    pin_probs_sum_to_one,
    pin_causal_ignores_future,
    pin_split_merge,
    pin_gqa_equals_repeated_mha,
    pin_torch_sdpa,
    pin_key_permutation,
    pin_shift_invariance,
    pin_large_logits,
    pin_scale_power_of_two,
    pin_ext_bruteforce_decimal,
    pin_alibi_slopes,
    pin_alibi_geometric_closed_form,
    pin_sink_closed_form,
    pin_softcap_limits,
    pin_window_limits,
    pin_split_merge_ex,
    pin_torch_sdpa_bias,
    pin_mask_torch_sdpa,
    pin_mask_removes_keys_and_shifts,
    pin_mask_fully_masked_row,
    pin_split_merge_mask,
    pin_e4m3_codes_match_torch,
    pin_fp8_attention_equals_dequantized,
    pin_narrow_v_bruteforce_decimal,
    pin_narrow_v_torch_sdpa,
]
