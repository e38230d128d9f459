"""The softmax's polynomial exp2 (exp2_poly2 in csrc/ptx.cuh), replayed step by
step in numpy float32 from the coefficients in the source: its relative error
bound on the range the softmax feeds it, and exact zeros for masked keys (CPU)."""
import os
import re

import numpy as np

PTX = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "gqa_flash_attention_attn_b200",
                   "csrc", "ptx.cuh")


def _coefficients():
    src = open(PTX).read()
    body = src[src.index("float2 exp2_poly2("):]
    body = body[:body.index("\n}\n")]
    vals = [float(x) for x in re.findall(r"make_float2\(([0-9.]+)f, \1f\)", body)]
    # Horner from the top: c3, c2, c1, then the constant 1
    c3, c2, c1, one = vals[:4]
    assert one == 1.0
    return np.float32(c1), np.float32(c2), np.float32(c3)


def _exp2_poly(x):
    c1, c2, c3 = _coefficients()
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-127.0))
    t = (x + f32(12582912.0)).astype(f32)
    n = (t + f32(-12582912.0)).astype(f32)
    f = (x - n).astype(f32)
    q = (c3 * f + c2).astype(f32)
    q = (q * f + c1).astype(f32)
    q = (q * f + f32(1.0)).astype(f32)
    bits = ((t.view(np.int32).astype(np.int64) << 23) + 0x3F800000) & 0xFFFFFFFF
    scale = bits.astype(np.uint32).view(np.float32)
    return (q * scale).astype(f32)


def test_relative_error_bound():
    x = np.linspace(-126.0, 9.0, 1_000_001).astype(np.float32)
    y = _exp2_poly(x)
    rel = np.abs(y.astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1.1e-4, rel.max()


def test_masked_and_underflowing_inputs_give_zero():
    x = np.array([-np.inf, -1e30, -200.0, -127.0, -126.6], dtype=np.float32)
    assert np.all(_exp2_poly(x) == 0.0)


def test_integers_are_exact():
    x = np.arange(-126, 9, dtype=np.float32)
    np.testing.assert_array_equal(_exp2_poly(x), np.exp2(x.astype(np.float64)).astype(np.float32))
