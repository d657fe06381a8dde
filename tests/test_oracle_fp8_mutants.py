"""Planted mistakes in the fp8 base oracle (on the CPU only): each must make one of the
pins of tests/test_oracle_fp8.py fail — a wrong exponent bias, ties rounded away from
zero, truncation, the wrong saturation value, a dropped per-row scale."""

import numpy as np
import pytest

import oracle as O
import oracle.fp8 as OF
import test_oracle_fp8 as T

REAL_VALUE = OF.e4m3_value
REAL_ROUND = OF.e4m3_round


def _patch(monkeypatch, name, fn):
    monkeypatch.setattr(O, name, fn)
    monkeypatch.setattr(OF, name, fn)


def _caught(*pins):
    for pin in pins:
        try:
            pin()
        except AssertionError:
            return True
    return False


ALL = (T.test_code_table_landmarks, T.test_code_table_matches_torch, T.test_rounding_matches_torch_in_range,
       T.test_rounding_hand_cases_and_saturation, T.test_rounding_is_nearest_by_brute_force,
       lambda: T.test_quantize_base_invariants("bf16"), T.test_quantize_codes_by_brute_force,
       T.test_apply_with_fp8_base_reduces_to_bf16_apply)


def test_pins_pass_on_the_real_oracle():
    for pin in ALL:
        pin()


def test_exponent_bias_eight(monkeypatch):
    def value(codes):
        return REAL_VALUE(codes) / 2.0
    _patch(monkeypatch, "e4m3_value", value)
    assert _caught(*ALL)


def test_ties_away_from_zero(monkeypatch):
    def rnd(v):
        v = np.asarray(v, dtype=np.float32)
        c = REAL_ROUND(v)
        mags = REAL_VALUE(np.arange(0x7F, dtype=np.uint8))
        a = np.abs(v.astype(np.float64))
        m = (c & 0x7F).astype(np.int64)
        up = np.minimum(m + 1, 126)
        tie = (m < 126) & (np.abs(a - mags[m]) == np.abs(mags[up] - a)) & (a > mags[m])
        m = np.where(tie, up, m)
        return (m | (c & 0x80)).astype(np.uint8)
    _patch(monkeypatch, "e4m3_round", rnd)
    assert _caught(*ALL)


def test_truncation(monkeypatch):
    def rnd(v):
        v = np.asarray(v, dtype=np.float32)
        mags = REAL_VALUE(np.arange(0x7F, dtype=np.uint8))
        a = np.abs(v.astype(np.float64))
        m = np.clip(np.searchsorted(mags, a, side="right") - 1, 0, 126)
        return np.where(np.signbit(v), m | 0x80, m).astype(np.uint8)
    _patch(monkeypatch, "e4m3_round", rnd)
    assert _caught(*ALL)


def test_saturates_to_the_wrong_value(monkeypatch):
    def rnd(v):
        c = REAL_ROUND(v)
        return np.where((c & 0x7F) == 0x7E, c - 1, c).astype(np.uint8)
    _patch(monkeypatch, "e4m3_round", rnd)
    assert _caught(*ALL)


def test_scale_dropped_from_the_dequantized_base(monkeypatch):
    def deq(codes, scales):
        return REAL_VALUE(codes)
    _patch(monkeypatch, "dequantize_base", deq)
    assert _caught(*ALL)
