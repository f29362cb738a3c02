"""Pins of the 8-bit latent-cache oracle (oracle/fp8_cache.py) to things other than itself: torch's
own float8_e4m3fn type (a conversion written by others), the format's closed-form properties,
and the error bound that three mantissa bits allow. The planted slips at the end must fail them."""
import numpy as np
import pytest
import torch

from oracle import fp8_cache as F
from oracle import mla_oracle as O


def _torch_values(codes):
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_every_code_decodes_like_torch():
    codes = np.arange(256, dtype=np.uint8)
    got, ref = F.e4m3_decode(codes), _torch_values(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert np.isnan(got).sum() == 2                       # 0x7F and 0xFF
    assert F.e4m3_decode(np.array([0x7E]))[0] == 448.0    # largest finite value
    assert F.e4m3_decode(np.array([0x01]))[0] == 2.0 ** -9   # smallest subnormal


def test_encoding_rounds_like_torch_including_every_midpoint():
    """torch converts to float8 through float32, so the sweep holds float32 values (there both
    round once): every code's value, every midpoint between neighbours (ties to even) and the
    float32 values just either side of it."""
    vals = np.unique(F.e4m3_decode(np.arange(0x7F, dtype=np.uint8))).astype(np.float32)
    mids = (vals[:-1] + vals[1:]) / np.float32(2)
    r = np.random.default_rng(50)
    sweep = np.concatenate([vals, mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9)),
                            r.uniform(0, 448, 4000).astype(np.float32), r.uniform(0, 0.02, 2000).astype(np.float32)])
    sweep = np.concatenate([sweep, -sweep]).astype(np.float64)
    got = F.e4m3_decode(F.e4m3_encode(sweep))
    ref = torch.from_numpy(sweep).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(got, ref)


def test_codes_round_trip_and_saturate():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF, 0x80)], np.uint8)
    assert np.array_equal(F.e4m3_encode(F.e4m3_decode(codes)), codes)
    assert F.e4m3_encode(np.array([1e6, -500.0]))[0] == 0x7E
    assert F.e4m3_encode(np.array([-500.0]))[0] == 0xFE


def test_row_quantisation_error_within_half_a_unit_of_the_last_place():
    """Three mantissa bits: a normal code is within 2^-4 of its value's magnitude; below the
    normal range (|c/s| < 2^-6) the spacing is 2^-9, so the error is at most 2^-10 · s."""
    r = np.random.default_rng(51)
    c = r.standard_normal((64, 512)) * r.uniform(0.01, 30, (64, 1))
    c[5] = 0.0                                             # a zero row
    codes, s = F.quantize_rows(c)
    deq = F.dequantize_rows(codes, s)
    assert s[5] == 0 and not deq[5].any()
    live = s > 0
    rel = c[live] / s[live, None]
    err = np.abs(deq[live] - c[live])
    normal = np.abs(rel) >= 2.0 ** -6
    assert (err[normal] <= 2.0 ** -4 * np.abs(c[live][normal]) * (1 + 1e-12)).all()
    assert (err[~normal] <= (2.0 ** -10 * np.broadcast_to(s[live, None], rel.shape))[~normal] * (1 + 1e-12)).all()
    # each row's largest magnitude lands on the largest code
    np.testing.assert_allclose(np.abs(deq[live]).max(axis=1), np.abs(c[live]).max(axis=1), rtol=1e-15)


def test_decode_over_the_8bit_cache_stays_close_to_the_16bit_one():
    """Attention over dequantised rows: the latent part of every value moves by at most 2^-4 of
    its size, so the output (a convex combination of rows) moves by a comparable fraction."""
    r = np.random.default_rng(52)
    L, H, d_c, d_r = 300, 8, 64, 16
    c = r.standard_normal((L, d_c))
    k_r = r.standard_normal((L, d_r))
    q = r.standard_normal((1, H, d_c + d_r)) * 0.2
    codes, s = F.quantize_rows(c)
    o8, l8 = F.absorbed_decode_fp8(q, codes, s, k_r, L, 1 / np.sqrt(192))
    o, l = O.absorbed_decode(q, c, k_r, L, 1 / np.sqrt(192))
    assert np.abs(o8 - o).max() <= 2.0 ** -4 * np.abs(c).max()
    assert np.abs(l8 - l).max() < 0.05


def test_float32_decision_equals_the_exact_one_where_no_rounding_intervenes():
    """Rows whose largest magnitude is 448·2^k and whose values are E4M3 values times 2^k: the scale
    2^k and every quotient are exact in float32, so both quantisations give the same codes, and
    dequantising gives the rows back."""
    r = np.random.default_rng(53)
    codes = r.integers(0, 0x7F, (16, 512)).astype(np.uint8) | (r.integers(0, 2, (16, 512)).astype(np.uint8) << 7)
    codes[:, 0] = 0x7E                                     # each row reaches 448
    k = r.integers(-20, 20, 16)
    c = F.e4m3_decode(codes) * np.ldexp(1.0, k)[:, None]
    c32, s32 = F.quantize_rows_f32(c)
    c64, s64 = F.quantize_rows(c)
    assert np.array_equal(s32, np.ldexp(1.0, k)) and np.array_equal(s32, s64)
    assert np.array_equal(F.e4m3_decode(c32), F.e4m3_decode(c64))   # +0 and -0 may differ as codes
    np.testing.assert_array_equal(F.dequantize_rows(c32, s32), c)


def test_float32_decision_differs_from_the_exact_one_only_at_ties():
    """On bf16-valued random rows the two precisions agree except where the exact quotient lies within
    a float32 rounding of a midpoint between two E4M3 values (a tie that float32 can move)."""
    r = np.random.default_rng(54)
    c = torch.from_numpy(r.standard_normal((256, 512)) * r.uniform(0.01, 30, (256, 1))).to(torch.bfloat16)
    c = c.to(torch.float64).numpy()
    c32, s32 = F.quantize_rows_f32(c)
    c64, s64 = F.quantize_rows(c)
    np.testing.assert_allclose(s32, s64, rtol=2.0 ** -24)
    diff = F.e4m3_decode(c32) != F.e4m3_decode(c64)
    assert diff.mean() < 1e-3
    if diff.any():
        exact = np.abs(c / s64[:, None])[diff]
        v32, v64 = np.abs(F.e4m3_decode(c32)[diff]), np.abs(F.e4m3_decode(c64)[diff])
        mid = (v32 + v64) / 2                                # the two candidates are neighbours
        assert (np.abs(exact - mid) <= 2.0 ** -22 * mid).all()


# planted slips ------------------------------------------------------------------------------

def test_planted_wrong_exponent_bias_is_caught(monkeypatch):
    monkeypatch.setattr(F, "_BIAS", 8)
    with pytest.raises(AssertionError):
        test_every_code_decodes_like_torch()


def test_planted_ties_away_from_zero_is_caught(monkeypatch):
    good = F.e4m3_encode

    def bad(v):
        v = np.asarray(v, float)
        up = good(np.nextafter(np.abs(v), np.inf)) & 0x7F   # a midpoint nudged up: ties away from zero
        return np.where(v < 0, up | 0x80, up).astype(np.uint8)
    monkeypatch.setattr(F, "e4m3_encode", bad)
    with pytest.raises(AssertionError):
        test_encoding_rounds_like_torch_including_every_midpoint()
