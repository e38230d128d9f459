"""The float64 oracle against what the definition of attention fixes (CPU only)."""
import pytest

import oracle
from oracle_pins import ALL_PINS


@pytest.fixture(scope="module")
def lib():
    return oracle.load()


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_pin(lib, pin):
    pin(lib)


def test_attention_rows_equals_attention(lib):
    """attention_rows runs the pinned per-row routine; it must agree bitwise with attention."""
    import numpy as np
    rng = np.random.default_rng(13)
    B, Hq, Hkv, Sq, Skv, D = 2, 4, 2, 7, 15, 8
    q = rng.standard_normal((B, Sq, Hq, D))
    k = rng.standard_normal((B, Skv, Hkv, D))
    v = rng.standard_normal((B, Skv, Hkv, D))
    out, lse = oracle.attention(q, k, v, scale=0.3, causal=True, q_offset=5, lib=lib)
    rows = [(b, h, s) for b in range(B) for h in range(Hq) for s in range(Sq)][::3]
    ro, rl = oracle.attention_rows(q, k, v, rows, scale=0.3, causal=True, q_offset=5, lib=lib)
    for i, (b, h, s) in enumerate(rows):
        assert np.array_equal(ro[i], out[b, s, h]) and rl[i] == lse[b, h, s]
