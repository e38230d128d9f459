"""Fail-demo acceptance for the oracle's pins.

Each case plants one plausible mistake in a copy of oracle.c (CPU only), builds
it, and requires that at least one pin rejects it.  A pin set that let any of
these through would not be pinning the oracle.
"""
import os

import pytest

import oracle
from oracle_pins import ALL_PINS

SRC = os.path.join(os.path.dirname(os.path.abspath(oracle.__file__)), "oracle.c")

# (name, text in oracle.c, replacement); every occurrence is replaced
MUTANTS = [
    ("causal_off_by_one", "if (causal && pos + 1 < last) last = pos + 1;",
     "if (causal && pos < last) last = pos;"),
    ("causal_sees_one_more", "if (causal && pos + 1 < last) last = pos + 1;",
     "if (causal && pos + 2 < last) last = pos + 2;"),
    ("no_max_subtraction", "const double p = exp(z[t - t_lo] - m);", "const double p = exp(z[t - t_lo]);"),
    ("lse_drops_max", "return m + log(l);", "return log(l);"),
    ("lse_base_two", "return m + log(l);", "return m + log2(l);"),
    ("scale_dropped", "const double zt = scale * acc;", "const double zt = acc;"),
    ("scale_squared", "const double zt = scale * acc;", "const double zt = scale * scale * acc;"),
    ("gqa_modulo_mapping", "const int64_t kvh = h / g;", "const int64_t kvh = h % Hkv;"),
    ("value_row_from_key_zero", "const double* vr = v + kv_index(b, t, kvh, Skv, Hkv, D);",
     "const double* vr = v + kv_index(b, t_lo, kvh, Skv, Hkv, D);"),
    ("unnormalised_output", "const double w = z[t - t_lo] / l;", "const double w = z[t - t_lo];"),
    ("merge_weight_sign", "const double w = exp(x - M);", "const double w = exp(M - x);"),
    ("merge_lse_no_max", "lse[r] = M + log(wsum);", "lse[r] = log(wsum);"),
    ("split_chunk_floor", "const int64_t chunk = (Skv + num_splits - 1) / num_splits;",
     "const int64_t chunk = Skv / num_splits;"),
    ("alibi_sign", "z[t - t_lo] = zc + slope * (double)(t - pos);", "z[t - t_lo] = zc - slope * (double)(t - pos);"),
    ("alibi_slope_exponent", "pow(m0, (double)(h + 1))", "pow(m0, (double)h)"),
    ("softcap_ignored", "softcap * tanh(zt / softcap) : zt;", "zt : zt;"),
    ("sink_not_in_denominator", "double l = has_sink ? exp(opt->sinks[h] - m) : 0.0;", "double l = 0.0;"),
    ("mask_sign", "z[t - t_lo] += opt->mask[b * opt->mask_sb + s * opt->mask_ss + t];",
     "z[t - t_lo] -= opt->mask[b * opt->mask_sb + s * opt->mask_ss + t];"),
    ("mask_row_ignored", "z[t - t_lo] += opt->mask[b * opt->mask_sb + s * opt->mask_ss + t];",
     "z[t - t_lo] += opt->mask[b * opt->mask_sb + t];"),
    ("mask_batch_ignored", "z[t - t_lo] += opt->mask[b * opt->mask_sb + s * opt->mask_ss + t];",
     "z[t - t_lo] += opt->mask[s * opt->mask_ss + t];"),
    ("masked_row_not_empty", "if (m == -INFINITY) return -INFINITY;", ""),
    ("e4m3_bias_8", "else mag = ldexp(1.0 + (double)m / 8.0, e - 7);", "else mag = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    ("e4m3_subnormal_as_normal", "if (e == 0) mag = ldexp((double)m / 8.0, -6);",
     "if (e == 0) mag = ldexp(1.0 + (double)m / 8.0, -7);"),
    ("e4m3_sign_dropped", "return sign ? -mag : mag;", "return mag;"),
    ("fp8_v_scale_from_k", "v[i] = oracle_e4m3_value(v_codes[i]) * v_scale[kvh];",
     "v[i] = oracle_e4m3_value(v_codes[i]) * k_scale[kvh];"),
    ("window_off_by_one", "if (opt && opt->window > 0 && pos - opt->window + 1 > first) first = pos - opt->window + 1;",
     "if (opt && opt->window > 0 && pos - opt->window > first) first = pos - opt->window;"),
    ("merge_sink_dropped", "double wsum = sinks ? exp(sinks[h] - M) : 0.0;", "double wsum = 0.0;"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mutant = tmp_path / "oracle_mutant.c"
    mutant.write_text(src.replace(old, new))
    so = oracle.build(str(mutant), str(tmp_path / "liboracle_mutant.so"))
    lib = oracle.load(so)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(lib)
        except (AssertionError, ValueError, FloatingPointError):
            caught.append(pin.__name__)
    assert caught, f"no pin rejects the planted mistake {name}"


def _pad_v_at_end(k, v):
    import numpy as np
    pad = np.zeros(v.shape[:-1] + (k.shape[-1],))
    pad[..., k.shape[-1] - v.shape[-1]:] = v
    return pad, v.shape[-1]


def _pad_v_unsliced(k, v):
    import numpy as np
    pad = np.zeros(v.shape[:-1] + (k.shape[-1],))
    pad[..., :v.shape[-1]] = v
    return pad, k.shape[-1]


@pytest.mark.parametrize("mutant", [_pad_v_at_end, _pad_v_unsliced], ids=["v_at_end", "unsliced"])
def test_narrow_v_mutant_is_caught(monkeypatch, mutant):
    """A wrong widening of a narrow V (values in the last columns; O returned
    D wide with the padding columns) fails a narrow-V pin."""
    from oracle_pins import pin_narrow_v_bruteforce_decimal, pin_narrow_v_torch_sdpa
    monkeypatch.setattr(oracle, "_pad_v", mutant)
    lib = oracle.load()
    caught = 0
    for pin in (pin_narrow_v_bruteforce_decimal, pin_narrow_v_torch_sdpa):
        try:
            pin(lib)
        except AssertionError:
            caught += 1
    assert caught > 0
