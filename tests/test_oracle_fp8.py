"""Pins for the FP8 (e4m3) part of the oracle: the code format, the quantiser
and attention over a dequantised cache.

The format is pinned by values that follow from its field layout and are
quoted for E4M3 everywhere (largest finite 448, smallest subnormal 2**-9,
smallest normal 2**-6, two NaN codes) and by PyTorch's own float8_e4m3fn type
(a library routine).  Attention over an FP8 cache is pinned by reduction to
the bf16 oracle and by closed forms in the scales.  The last tests plant
plausible mistakes and check that a pin catches each.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from oracle import fp8

ALL = np.arange(256, dtype=np.uint8)
FINITE = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)


@pytest.mark.parametrize("code,value", [
    (0x00, 0.0), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9), (0x08, 2.0 ** -6), (0x09, 1.125 * 2.0 ** -6),
    (0x38, 1.0), (0x3C, 1.5), (0x40, 2.0), (0x77, 240.0), (0x78, 256.0), (0x7E, 448.0),
    (0xB8, -1.0), (0xFE, -448.0), (0x81, -(2.0 ** -9)),
])
def test_e4m3_closed_form_codes(code, value):
    assert fp8.e4m3_decode([code])[0] == value


def test_e4m3_special_codes():
    v = fp8.e4m3_decode(ALL)
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF])
    assert np.isnan(v).sum() == 2                   # no other NaN, and no infinities
    assert not np.isinf(v).any()
    assert v[0x80] == 0.0 and np.signbit(v[0x80])   # negative zero
    pos = v[:0x7F]
    assert (np.diff(pos) > 0).all()                 # codes 0x00..0x7E increase strictly
    assert np.array_equal(v[0x80:0xFF], -pos)       # sign bit only flips the sign


def test_e4m3_matches_torch_float8():
    ref = torch.from_numpy(ALL.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = fp8.e4m3_decode(ALL)
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], got[ok])
    assert np.array_equal(np.signbit(ref[ok]), np.signbit(got[ok]))


def test_encode_roundtrips_every_finite_code():
    assert np.array_equal(fp8.e4m3_encode(fp8.e4m3_decode(FINITE)), FINITE)


def test_encode_ties_go_to_the_even_code():
    pos = fp8.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    for c in range(0x7E):
        mid = 0.5 * (pos[c] + pos[c + 1])            # exact in float64
        even = c if c % 2 == 0 else c + 1
        assert fp8.e4m3_encode([mid])[0] == even, hex(c)
        gap = pos[c + 1] - pos[c]
        assert fp8.e4m3_encode([mid - gap / 8])[0] == c
        assert fp8.e4m3_encode([mid + gap / 8])[0] == c + 1
        assert fp8.e4m3_encode([-mid])[0] == (even | 0x80)


def test_encode_saturates_and_keeps_nan():
    x = [448.0, 449.0, 464.0, 476.0, 1e9, math.inf, -500.0, -math.inf]
    assert list(fp8.e4m3_encode(x)) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]
    assert fp8.e4m3_encode([math.nan])[0] == 0x7F


def test_encode_small_values_and_signed_zero():
    x = [0.0, -0.0, 1e-6, -1e-6, 2.0 ** -10, 2.0 ** -10 * 1.0001, 3 * 2.0 ** -10, -(2.0 ** -10)]
    # 2**-10 is the tie between 0 and 2**-9 (even code 0x00); 3 * 2**-10 ties 0x01 / 0x02
    assert list(fp8.e4m3_encode(x)) == [0x00, 0x80, 0x00, 0x80, 0x00, 0x01, 0x02, 0x80]


def test_encode_matches_torch_cast_in_range():
    g = torch.Generator().manual_seed(5)
    x = torch.cat([torch.randn(20000, generator=g) * s for s in (1e-3, 0.05, 1.0, 30.0, 150.0)])
    x = x.clamp(-448.0, 448.0)
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = fp8.e4m3_encode(x.to(torch.float64).numpy())
    assert np.array_equal(ref, got)


def test_quantize_error_is_within_half_a_step():
    """Three mantissa bits: in the normal range the rounding error is at most
    2**-4 of the value; below 2**-6 it is at most half the subnormal step 2**-9."""
    g = np.random.default_rng(3)
    x = g.standard_normal((7, 3, 64)).astype(np.float32) * 10      # |x / s| stays below 448
    s = np.array([0.25, 1.0, 2.0], dtype=np.float32)
    assert (np.abs(x) / s[:, None] < 448).all()
    codes = fp8.quantize_rows(x, s)
    back = fp8.dequantize(codes, s)
    q = x.astype(np.float64) / s[:, None]
    err = np.abs(back / s[:, None] - q)
    bound = np.where(np.abs(q) >= 2.0 ** -6, np.abs(q) * 2.0 ** -4, 2.0 ** -10)
    assert (err <= bound * (1 + 1e-12)).all()


def test_quantize_uses_each_heads_scale():
    x = np.ones((2, 3, 8), dtype=np.float32)
    s = np.array([1.0, 2.0, 4.0], dtype=np.float32)
    v = fp8.e4m3_decode(fp8.quantize_rows(x, s))
    assert np.array_equal(v[:, 0], np.full((2, 8), 1.0))
    assert np.array_equal(v[:, 1], np.full((2, 8), 0.5))
    assert np.array_equal(v[:, 2], np.full((2, 8), 0.25))


def _codes(shape, seed):
    g = np.random.default_rng(seed)
    c = g.integers(0, 256, size=shape).astype(np.uint8)
    c[(c == 0x7F) | (c == 0xFF)] = 0x38
    # keep magnitudes moderate so that softmax weights are not all on one key
    v = fp8.e4m3_decode(c)
    c[np.abs(v) > 8] = 0x30
    return c


def test_decode_fp8_with_unit_scales_is_plain_decode():
    B, T, Hq, Hkv, d, L = 2, 3, 4, 2, 16, 40
    g = np.random.default_rng(1)
    q = g.standard_normal((B, T, Hq, d))
    kc, vc = _codes((B, L, Hkv, d), 2), _codes((B, L, Hkv, d), 3)
    one = np.ones(Hkv, dtype=np.float32)
    lens = np.array([L, 25])
    o8, l8 = fp8.decode_fp8(q, kc, vc, one, one, lens, 0.25, True)
    o, lse = oracle.decode(q, fp8.e4m3_decode(kc), fp8.e4m3_decode(vc), lens, 0.25, True)
    assert np.array_equal(o8, o) and np.array_equal(l8, lse)


@pytest.mark.parametrize("ka,vb", [(1, 0), (-2, 3), (0, -1)])
def test_decode_fp8_scales_are_closed_forms(ka, vb):
    """A K scale of 2**a is the softmax scale times 2**a; a V scale of 2**b
    multiplies O by 2**b and leaves LSE alone (exact: powers of two)."""
    B, T, Hq, Hkv, d, L = 2, 2, 6, 3, 16, 33
    g = np.random.default_rng(7)
    q = g.standard_normal((B, T, Hq, d))
    kc, vc = _codes((B, L, Hkv, d), 8), _codes((B, L, Hkv, d), 9)
    ks = np.full(Hkv, 2.0 ** ka, dtype=np.float32)
    vs = np.full(Hkv, 2.0 ** vb, dtype=np.float32)
    lens = np.array([L, 17])
    o8, l8 = fp8.decode_fp8(q, kc, vc, ks, vs, lens, 0.125, True)
    o, lse = oracle.decode(q, fp8.e4m3_decode(kc), fp8.e4m3_decode(vc), lens, 0.125 * 2.0 ** ka, True)
    np.testing.assert_allclose(o8, o * 2.0 ** vb, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(l8, lse, rtol=1e-12, atol=1e-14)


def test_decode_fp8_per_head_scales_follow_the_gqa_mapping():
    """Head g's scale applies exactly to the query heads that read KV head g."""
    B, T, Hq, Hkv, d, L = 1, 1, 4, 2, 8, 12
    g = np.random.default_rng(11)
    q = g.standard_normal((B, T, Hq, d))
    kc, vc = _codes((B, L, Hkv, d), 12), _codes((B, L, Hkv, d), 13)
    lens = np.array([L])
    base_o, _ = fp8.decode_fp8(q, kc, vc, np.ones(2, np.float32), np.ones(2, np.float32), lens, 0.3, True)
    o, _ = fp8.decode_fp8(q, kc, vc, np.ones(2, np.float32), np.array([1.0, 4.0], np.float32), lens, 0.3, True)
    np.testing.assert_allclose(o[:, :, :2], base_o[:, :, :2], rtol=1e-13)
    np.testing.assert_allclose(o[:, :, 2:], 4 * base_o[:, :, 2:], rtol=1e-13)


def test_paged_fp8_equals_contiguous_fp8():
    B, T, Hq, Hkv, d = 3, 2, 4, 2, 16
    lens = np.array([5, 33, 48])
    nblk = [(int(L) + 15) // 16 for L in lens]
    perm = np.random.default_rng(2).permutation(sum(nblk) + 2).astype(np.int32)
    table = np.full((B, max(nblk)), -1, np.int32)
    off = 0
    for b in range(B):
        table[b, :nblk[b]] = perm[off:off + nblk[b]]
        off += nblk[b]
    kp, vp = _codes((sum(nblk) + 2, 16, Hkv, d), 4), _codes((sum(nblk) + 2, 16, Hkv, d), 5)
    ks = np.array([0.5, 0.75], np.float32)
    vs = np.array([1.5, 0.25], np.float32)
    q = np.random.default_rng(6).standard_normal((B, T, Hq, d))
    op, lp = fp8.decode_paged_fp8(q, kp, vp, ks, vs, table, lens, 0.2, True)
    kc = oracle.gather_paged(kp, table, lens)
    vc = oracle.gather_paged(vp, table, lens)
    oc, lc = fp8.decode_fp8(q, kc, vc, ks, vs, lens, 0.2, True)
    assert np.array_equal(op, oc) and np.array_equal(lp, lc)


def test_append_fp8_writes_the_quantised_rows():
    B, T, Hkv, d, cap = 2, 3, 2, 8, 10
    g = np.random.default_rng(21)
    kc = np.zeros((B, cap, Hkv, d), np.uint8)
    vc = np.zeros((B, cap, Hkv, d), np.uint8)
    kn = g.standard_normal((B, T, Hkv, d)).astype(np.float32)
    vn = g.standard_normal((B, T, Hkv, d)).astype(np.float32)
    ks = np.array([0.01, 0.02], np.float32)
    vs = np.array([0.03, 0.04], np.float32)
    lens = np.array([0, 7])
    k2, v2 = fp8.kv_append_fp8(kc, vc, kn, vn, ks, vs, lens)
    assert k2.dtype == np.uint8
    for b in range(B):
        p = int(lens[b])
        back = fp8.dequantize(k2[b, p:p + T], ks)
        np.testing.assert_allclose(back, kn[b], rtol=2.0 ** -4)
        assert not k2[b, :p].any() and not k2[b, p + T:].any()
        np.testing.assert_allclose(fp8.dequantize(v2[b, p:p + T], vs), vn[b], rtol=2.0 ** -4)


# ------------------------------------------------------------ planted mistakes
def test_wrong_exponent_bias_is_caught(monkeypatch):
    def bad_value(code):
        v = fp8.e4m3_value(code)
        return v * 2.0 if (code >> 3) & 0xF else v      # bias 6 for normal codes
    table = np.array([bad_value(c) for c in range(256)])
    monkeypatch.setattr(fp8, "_TABLE", table)
    monkeypatch.setattr(fp8, "_POS", table[:0x7F])
    with pytest.raises(AssertionError):
        test_e4m3_closed_form_codes(0x38, 1.0)
    with pytest.raises(AssertionError):
        test_e4m3_matches_torch_float8()


def test_ties_away_from_zero_is_caught(monkeypatch):
    good = fp8.e4m3_encode

    def bad_encode(x):
        x = np.asarray(x, dtype=np.float64)
        c = good(x)
        pos = fp8._POS
        a = np.abs(x)
        up = (c & 0x7F) < 0x7E
        nxt = pos[np.minimum((c & 0x7F).astype(int) + 1, 0x7E)]
        tie = up & np.isfinite(a) & (a - pos[(c & 0x7F).astype(int)] == nxt - a)
        return np.where(tie, c + 1, c).astype(np.uint8)

    monkeypatch.setattr(fp8, "e4m3_encode", bad_encode)
    with pytest.raises(AssertionError):
        test_encode_ties_go_to_the_even_code()


def test_swapped_scales_are_caught(monkeypatch):
    good = fp8.decode_fp8

    def swapped(q, kc, vc, ks, vs, lens, scale, causal=True):
        return good(q, kc, vc, vs, ks, lens, scale, causal)

    monkeypatch.setattr(fp8, "decode_fp8", swapped)
    with pytest.raises(AssertionError):
        test_decode_fp8_scales_are_closed_forms(-2, 3)
