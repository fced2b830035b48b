"""FP8 (e4m3) KV cache: the code format, the quantiser and attention over it.

TEST INFRASTRUCTURE ONLY (see the package docstring): the CUDA library never
imports this module and this module never imports the library.

Sources (page title, section):

* "KV cache, flash attention and inference optimisation" lesson, section "用它"
  (production serving with ``--kv-cache-dtype fp8``: the cache is stored in an
  8-bit float format).
* "[BEE-30062] FlashAttention 與高效注意力核心", FlashAttention-3 paragraph of
  "背景" and the related-reading entry on quantisation (FP8 mode combines
  quantisation with the tiled kernel).

The pages name FP8 but fix neither the encoding nor the scaling.  Readings
taken here:

* Encoding: the OCP 8-bit float E4M3 ("FN" variant): 1 sign bit, 4 exponent
  bits with bias 7, 3 mantissa bits; exponent field 0 holds the subnormals
  ``m / 8 * 2**-6``; there are no infinities; ``S.1111.111`` is NaN, so the
  largest finite magnitude is ``1.75 * 2**8 = 448``.
* Scaling: one float32 scale per KV head for K and one for V; a stored code
  ``c`` of head ``g`` stands for ``value(c) * scale[g]``.
* Quantisation of a new token (the append path): ``x / scale[g]`` computed in
  float32 (one IEEE division), then rounded to the nearest e4m3 value, ties to
  the even code, saturating to +-448 (values beyond, infinities included);
  NaN gives the NaN code 0x7F.  A negative value that rounds to zero keeps its
  sign (code 0x80).
* Attention over an FP8 cache is exact attention over the dequantised cache.
"""

from __future__ import annotations

import numpy as np

from .attention import decode, decode_paged, kv_append, kv_append_paged

E4M3_MAX = 448.0
E4M3_NAN = 0x7F


def e4m3_value(code: int) -> float:
    """Value of one e4m3 code, from the field definition."""
    code = int(code) & 0xFF
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** (1 - 7)
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


# all 256 codes, decoded once (a plain table of the definition above)
_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)
# non-negative finite values in code order 0x00 .. 0x7E (strictly increasing)
_POS = _TABLE[:0x7F]


def e4m3_decode(codes) -> np.ndarray:
    """Array of uint8 codes -> float64 values (NaN for the two NaN codes)."""
    return _TABLE[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(x) -> np.ndarray:
    """float values -> uint8 codes: nearest e4m3 value, ties to the even code,
    saturating to +-448; NaN -> 0x7F."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    out = np.zeros(x.shape, dtype=np.uint8)
    finite = np.isfinite(a)
    sat = ~finite | (a >= E4M3_MAX)
    mag = np.where(sat, 0.0, a)
    hi = np.clip(np.searchsorted(_POS, mag, side="left"), 1, 0x7E)   # first value >= mag
    lo = hi - 1
    d_lo = mag - _POS[lo]
    d_hi = _POS[hi] - mag
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(mag == 0.0, 0, code)
    code = np.where(sat, 0x7E, code).astype(np.uint8)
    code = code | np.where(np.signbit(x), 0x80, 0).astype(np.uint8)
    code = np.where(np.isnan(x), E4M3_NAN, code).astype(np.uint8)
    out[...] = code
    return out


def quantize_rows(x, scale) -> np.ndarray:
    """Codes of new K or V rows ``[..., Hkv, d]`` with per-KV-head ``scale[Hkv]``.

    The division is done in float32, as the reading above fixes, so that the
    rounding decision is taken on the same float32 quotient on every side.
    """
    x32 = np.asarray(x, dtype=np.float32)
    s32 = np.asarray(scale, dtype=np.float32)
    q = (x32 / s32[:, None]).astype(np.float32)
    return e4m3_encode(q.astype(np.float64))


def dequantize(codes, scale) -> np.ndarray:
    """float64 values of a cache ``[..., Hkv, d]`` of codes with per-KV-head scales."""
    s = np.asarray(scale, dtype=np.float32).astype(np.float64)
    return e4m3_decode(codes) * s[:, None]


def decode_fp8(q, k_codes, v_codes, k_scale, v_scale, seqlens_k, scale: float, causal: bool = True):
    """Decode over a contiguous FP8 cache ``[B, Lcap, Hkv, d]``: exact attention
    over the dequantised K and V (see ``attention.decode``)."""
    return decode(q, dequantize(k_codes, k_scale), dequantize(v_codes, v_scale), seqlens_k, scale, causal)


def decode_paged_fp8(q, k_codes, v_codes, k_scale, v_scale, page_table, seqlens_k, scale: float,
                     causal: bool = True):
    """Decode over paged FP8 pools ``[num_blocks, 16, Hkv, d]``."""
    return decode_paged(q, dequantize(k_codes, k_scale), dequantize(v_codes, v_scale), page_table, seqlens_k,
                        scale, causal)


def kv_append_fp8(k_codes, v_codes, k_new, v_new, k_scale, v_scale, cache_lens):
    """Quantise ``T`` new tokens and write their codes into a contiguous cache
    (returns new arrays; see ``attention.kv_append`` for the placement)."""
    return kv_append(k_codes, v_codes, quantize_rows(k_new, k_scale), quantize_rows(v_new, v_scale), cache_lens)


def kv_append_paged_fp8(k_codes, v_codes, k_new, v_new, k_scale, v_scale, cache_lens, page_table):
    """Quantise and write into paged pools (see ``attention.kv_append_paged``)."""
    return kv_append_paged(k_codes, v_codes, quantize_rows(k_new, k_scale), quantize_rows(v_new, v_scale),
                           cache_lens, page_table)
