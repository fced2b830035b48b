"""Plant plausible mistakes in the oracle (on the CPU) and check that a pin catches each.

A pin that still passes with a dropped term, a wrong sign or index, or a
transposed operand would not be pinning anything.
"""

import sys

import numpy as np
import pytest

import oracle
import oracle.kv_bytes as kvb
from tests import test_oracle_pins as pins

att = sys.modules["oracle.attention"]  # the submodule (the package re-exports a function of that name)


def _attend_variant(mistake):
    def attend(q, k, v, scale, causal):
        q = np.asarray(q, dtype=np.float64)
        k = np.asarray(k, dtype=np.float64)
        v = np.asarray(v, dtype=np.float64)
        Nq, Lk = q.shape[0], k.shape[0]
        vis = att.visible_mask(Nq, Lk, causal)
        s = (q @ k.T) * (1.0 if mistake == "no_scale" else scale)
        if mistake == "transposed_scores" and Nq == Lk:
            s = s.T
        s = np.where(vis, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        w = np.exp(s - m) if mistake != "sign" else np.exp(m - s)
        w = np.where(vis, w, 0.0)
        z = w.sum(axis=1, keepdims=True)
        o = (w @ v) / z if mistake != "no_normalise" else (w @ v)
        lse = (np.log(z) if mistake == "lse_drops_max" else m + np.log(z))[:, 0]
        return o, lse
    return attend


def _expect_failure(fn, *args):
    with pytest.raises((AssertionError, ValueError, IndexError)):
        fn(*args)


@pytest.mark.parametrize("mistake,pin,args", [
    ("no_scale", pins.test_prefill_matches_torch_sdpa, (True, 7, 16)),
    ("transposed_scores", pins.test_prefill_matches_torch_sdpa, (False, 7, 16)),
    ("sign", pins.test_prefill_matches_torch_sdpa, (False, 7, 16)),
    ("no_normalise", pins.test_identical_v_rows_give_that_row, ()),
    ("lse_drops_max", pins.test_dominant_score_selects_its_v_row, ()),
])
def test_attend_mistakes_are_caught(monkeypatch, mistake, pin, args):
    bad = _attend_variant(mistake)
    monkeypatch.setattr(att, "attend_head", bad)
    monkeypatch.setattr(oracle, "attend_head", bad)
    _expect_failure(pin, *args)


def test_wrong_gqa_mapping_is_caught(monkeypatch):
    monkeypatch.setattr(att, "kv_head_for", lambda h, Hq, Hkv: h % Hkv)
    _expect_failure(pins.test_gqa_equals_mha_with_repeat_interleave)


def test_top_left_mask_is_caught(monkeypatch):
    def top_left(Nq, Lk, causal):
        t = np.arange(Nq)[:, None]
        j = np.arange(Lk)[None, :]
        return np.ones((Nq, Lk), bool) if not causal else j <= t
    monkeypatch.setattr(att, "visible_mask", top_left)
    monkeypatch.setattr(oracle, "visible_mask", top_left)
    _expect_failure(pins.test_decode_equals_last_rows_of_causal_prefill, 2, 17)
    _expect_failure(pins.test_zero_query_gives_mean_and_log_count, 4, 9)


def test_off_by_one_mask_is_caught(monkeypatch):
    def shifted(Nq, Lk, causal):
        t = np.arange(Nq)[:, None]
        j = np.arange(Lk)[None, :]
        return np.ones((Nq, Lk), bool) if not causal else j < (Lk - Nq) + t
    monkeypatch.setattr(att, "visible_mask", shifted)
    monkeypatch.setattr(oracle, "visible_mask", shifted)
    _expect_failure(pins.test_zero_query_gives_mean_and_log_count, 4, 9)


def test_wrong_page_slot_is_caught(monkeypatch):
    orig = att.gather_paged

    def bad_gather(pool, table, seqlens, page_tokens=16):
        out = orig(pool, table, seqlens, page_tokens)
        return out[:, ::-1].copy()  # tokens read in the wrong order
    monkeypatch.setattr(att, "gather_paged", bad_gather)
    _expect_failure(pins.test_paged_equals_contiguous)


def test_missing_kv_factor_is_caught(monkeypatch):
    monkeypatch.setattr(kvb, "bytes_per_token_per_layer", lambda h, d, e: h * d * e)
    monkeypatch.setattr(oracle, "bytes_per_token_per_layer", lambda h, d, e: h * d * e)
    rows = list(pins._golden_rows("kv_cache_bytes.txt"))
    per_token = [r for r in rows if r[0][0] == "per_token"][0]
    _expect_failure(pins.test_kv_bytes_golden, *per_token)
