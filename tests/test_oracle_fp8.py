"""Pins of the fp8 (e4m3) base oracle: the code table against the OCP E4M3 definition's
landmark values and against PyTorch's float8_e4m3fn, the rounding against PyTorch's
conversion (round to nearest even) and hand-made ties, saturation, the per-row
quantizer's invariants and brute force on small rows, and the apply with an fp8 base
reduced to the already pinned bf16 apply."""

import numpy as np
import pytest

import oracle as O
from workloads import activations, bf16_bits, random_tenant


def test_code_table_landmarks():
    # OCP E4M3: zero, smallest subnormal 2^-9, largest subnormal 7 * 2^-9, smallest
    # normal 2^-6, one, 1.5, two, largest finite 448, NaN at S.1111.111, signed zero
    v = O.e4m3_value(np.array([0x00, 0x01, 0x07, 0x08, 0x38, 0x3C, 0x40, 0x7E, 0xFE, 0x7F, 0xFF, 0x80],
                              dtype=np.uint8))
    assert list(v[:9]) == [0.0, 2.0 ** -9, 7 * 2.0 ** -9, 2.0 ** -6, 1.0, 1.5, 2.0, 448.0, -448.0]
    assert np.isnan(v[9]) and np.isnan(v[10])
    assert v[11] == 0.0 and np.signbit(v[11])
    mags = O.e4m3_value(np.arange(0x7F, dtype=np.uint8))
    assert np.all(np.diff(mags) > 0)  # strictly increasing with the code
    assert len(np.unique(np.abs(O.e4m3_value(np.arange(256, dtype=np.uint8))[~np.isnan(
        O.e4m3_value(np.arange(256, dtype=np.uint8)))]))) == 127


def test_code_table_matches_torch():
    import torch
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.e4m3_value(np.arange(256, dtype=np.uint8))
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], got[ok])
    assert np.array_equal(np.signbit(ref[ok]), np.signbit(got[ok]))


def test_rounding_matches_torch_in_range():
    import torch
    rng = np.random.default_rng(0)
    mags = O.e4m3_value(np.arange(0x7F, dtype=np.uint8))
    # random values over the whole range, every exact midpoint, values next to them
    v = np.concatenate([rng.uniform(-464, 464, 20000), rng.normal(0, 1e-2, 20000),
                        (mags[:-1] + mags[1:]) / 2, -(mags[:-1] + mags[1:]) / 2, mags, -mags,
                        [0.0, -0.0, 1e-30, -1e-30, 464.0, -464.0]]).astype(np.float32)
    v = np.concatenate([v, np.nextafter(v, np.float32(np.inf)), np.nextafter(v, np.float32(-np.inf))])
    v = v[np.abs(v) <= 464]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = O.e4m3_round(v)
    assert np.array_equal(got, ref)


def test_rounding_hand_cases_and_saturation():
    f = lambda xs: list(O.e4m3_round(np.array(xs, dtype=np.float32)))  # noqa: E731
    # 1.0625 is halfway between 1.0 (m=0) and 1.125 (m=1): even -> 1.0; 1.1875 between
    # 1.125 (m=1) and 1.25 (m=2): even -> 1.25; 15/8 * 2^-7 between 7 * 2^-9 and 2^-6
    assert f([1.0625, 1.1875, 7.5 * 2 ** -9]) == [0x38, 0x3A, 0x08]
    # above the largest finite value: 448 (satfinite), sign kept
    assert f([449.0, 480.0, 1e30, -1e30]) == [0x7E, 0x7E, 0x7E, 0xFE]
    # below half the smallest subnormal: signed zero
    assert f([2.0 ** -11, -(2.0 ** -11)]) == [0x00, 0x80]


def test_rounding_is_nearest_by_brute_force():
    rng = np.random.default_rng(1)
    v = rng.uniform(-448, 448, 3000).astype(np.float32)
    got = O.e4m3_value(O.e4m3_round(v))
    table = O.e4m3_value(np.arange(0x7F, dtype=np.uint8))
    table = np.concatenate([table, -table])
    best = np.min(np.abs(v[:, None].astype(np.float64) - table[None, :]), axis=1)
    assert np.array_equal(np.abs(v - got), best)


@pytest.mark.parametrize("w_dtype", ["bf16", "f32"])
def test_quantize_base_invariants(w_dtype):
    rng = np.random.default_rng(2)
    w = rng.normal(0, 0.02, size=(37, 160))
    w[3] = 0.0                      # a zero row
    w[5, :] = rng.normal(0, 1e-30, 160)  # tiny values
    w = bf16_bits(w) if w_dtype == "bf16" else w.astype(np.float32)
    codes, scales = O.quantize_base(w, w_dtype)
    wd = O.decode(w, w_dtype)
    assert codes.dtype == np.uint8 and scales.dtype == np.float32
    assert scales[3] == 0 and np.all(codes[3] == 0)
    for o in range(w.shape[0]):
        if scales[o] == 0:
            continue
        # the row's largest magnitude maps to +-448
        i = int(np.argmax(np.abs(wd[o])))
        assert codes[o, i] & 0x7F == 0x7E
        # the scale is the fp32 quotient max / 448
        assert scales[o] == np.float32(np.float32(np.max(np.abs(wd[o]))) / np.float32(448))
    wh = O.dequantize_base(codes, scales)
    q = wd / np.where(scales > 0, scales, 1)[:, None]
    # relative error 2^-4 in the normal range, absolute 2^-10 * s below it (+ fp32 slack)
    bound = np.where(np.abs(q) >= 2 ** -6, np.abs(q) * 2 ** -4, 2 ** -10) * 1.0001 + 1e-6 * np.abs(q)
    err = np.abs(wh - wd) / np.where(scales > 0, scales, 1)[:, None]
    assert np.all(err <= bound)


def test_quantize_codes_by_brute_force():
    rng = np.random.default_rng(3)
    w = rng.normal(0, 0.02, size=(4, 64)).astype(np.float32)
    codes, scales = O.quantize_base(w, "f32")
    table = O.e4m3_value(np.arange(0x7F, dtype=np.uint8))
    for o in range(4):
        for i in range(64):
            q = np.float32(w[o, i] / scales[o])  # fp32 quotient
            a = abs(float(q))
            d = np.abs(table - a)
            cands = np.flatnonzero(d == d.min())
            want = int(cands[0] if len(cands) == 1 else [c for c in cands if c % 2 == 0][0])
            want |= 0x80 if np.signbit(q) else 0
            assert codes[o, i] == want


def test_apply_with_fp8_base_reduces_to_bf16_apply():
    """With power-of-two row scales the dequantized base (<= 4 significant bits times a
    power of two) is exactly a bf16 matrix, so the fp8-base apply must equal the pinned
    bf16 apply on that matrix."""
    rng = np.random.default_rng(4)
    d_out, d_in, B = 48, 256, 6
    codes = rng.integers(0, 256, size=(d_out, d_in), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x38  # no NaN codes
    scales = (2.0 ** rng.integers(-12, -4, size=d_out)).astype(np.float32)
    wb = O.dequantize_base(codes, scales)
    wb_bits = bf16_bits(wb)
    assert np.array_equal(O.decode(wb_bits, "bf16"), wb)
    tenants = [random_tenant(rng, d_out, d_in, m) for m in (0, 1, 2, 3)]
    ids = np.array([0, 1, -1, 2, 3, 0], dtype=np.int32)
    x = activations(rng, B, d_in)
    y8 = O.apply_multi_fp8(codes, scales, tenants, ids, x, "bf16")
    yb = O.apply_multi(wb_bits, "bf16", tenants, ids, x, "bf16")
    np.testing.assert_allclose(y8, yb, rtol=0, atol=1e-15)
