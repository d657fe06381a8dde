"""Pins for the float64 oracle, against what the pages and the mathematics fix.

Each test names the passage it follows. None of them re-types the oracle's own
formula: they use the pages' printed numbers, closed forms, brute force over tiny
inputs, pure-Python loops, or invariants that a dropped term, a wrong sign or index
or a transposed operand would break.
"""

import json
import math
import os

import numpy as np
import pytest

import oracle as O
from workloads import bf16_bits, bf16_bits_to_f32, random_tenant, tiny_config

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")))


# --------------------------------------------------------------------------------
# worked examples ("bitdelta" page, "How BitDelta Works" 1-4)
# --------------------------------------------------------------------------------
def test_worked_delta():
    g = GOLD["delta"]
    d = O.delta(g["base_weight"], g["fine_tuned_weight"])
    np.testing.assert_allclose(d, g["delta"], rtol=0, atol=1e-12)


def test_worked_group_scale():
    g = GOLD["group_scale"]
    s = O.abs_mean_scales(np.array(g["delta_group"]), O.MODE_GROUP, g["group_size"])
    assert s.shape == (1,)
    assert abs(s[0] - g["scale"]) < 1e-12


@pytest.mark.parametrize("case", GOLD["signs"]["cases"])
def test_worked_signs(case):
    bits = O.sign_bits(np.array(case["delta_group"]))
    assert list(np.where(bits, 1, -1)) == case["signs"]


def test_worked_reconstruction():
    g = GOLD["reconstruction"]
    # pack the 4 signs into a 1 x 32 row (remaining columns +1, scale 0 irrelevant)
    bits = np.ones((1, 32), dtype=bool)
    bits[0, :4] = np.array(g["signs"]) > 0
    words = O.pack_bits(bits)
    rec = O.reconstruct(words, np.array(g["scales"] * 8), O.MODE_GROUP, 4, 1, 32)
    np.testing.assert_allclose(rec[0, :4], g["reconstructed"], rtol=0, atol=1e-12)
    err = np.abs(rec[0, :4] - np.array(g["original"])).mean()
    assert abs(err - 0.05) < 1e-12  # |0|+|0|+|0.1|+|0.1| over 4


@pytest.mark.parametrize("case,word", [
    (GOLD["signs"]["cases"][0], 0xFFFFFFFF),
    (GOLD["signs"]["cases"][1], 0x55555555),
])
def test_worked_example_tiled_to_128(case, word):
    """The printed group of 4, repeated 32 times into one 1 x 128 row with G = 128:
    the abs-mean is unchanged and every packed word is the 4-sign pattern repeated
    8 times, least significant bit first."""
    row = np.tile(np.array(case["delta_group"]), 32)[None, :]
    base = np.zeros_like(row)
    out = O.compress(base.astype(np.float32), row.astype(np.float32), "f32", O.MODE_GROUP, 128)
    assert out["signs"].shape == (1, 4)
    assert all(int(w) == word for w in out["signs"].ravel())
    expected = np.abs(np.array(case["delta_group"], dtype=np.float32).astype(np.float64)).mean()
    assert abs(out["scales"][0, 0] - expected) < 1e-15


# --------------------------------------------------------------------------------
# sign and packing conventions
# --------------------------------------------------------------------------------
def test_sign_of_zero_is_plus_one():
    d = np.array([0.0, -0.0, 1e-300, -1e-300, -5e-324, 5e-324])
    assert list(O.sign_bits(d)) == [True, True, True, False, False, True]


def test_pack_bit_positions():
    """Column c lands in bit c % 32 of word c // 32, independently of numpy's
    packbits: checked by building each word with integer shifts."""
    rng = np.random.default_rng(5)
    bits = rng.random((3, 96)) < 0.5
    words = O.pack_bits(bits)
    for o in range(3):
        for w in range(3):
            expect = 0
            for j in range(32):
                if bits[o, 32 * w + j]:
                    expect |= 1 << j
            assert int(words[o, w]) == expect
    assert np.array_equal(O.unpack_bits(words, 96), bits)


def test_pack_rejects_ragged():
    with pytest.raises(ValueError):
        O.pack_bits(np.ones((2, 40), dtype=bool))


# --------------------------------------------------------------------------------
# closed form: mean |delta| is the L2-optimal scale for fixed signs
# ("BitDelta Guide", "2. Optimal L2 Norm Initialization")
# --------------------------------------------------------------------------------
@pytest.mark.parametrize("g", [4, 7, 16])
def test_abs_mean_is_l2_optimal_brute_force(g):
    rng = np.random.default_rng(100 + g)
    for _ in range(5):
        d = rng.normal(0, 1, size=g)
        sgn = np.where(d >= 0, 1.0, -1.0)
        grid = np.linspace(0.0, np.abs(d).max(), 100001)
        err = ((d[None, :] - grid[:, None] * sgn[None, :]) ** 2).sum(axis=1)
        best = grid[np.argmin(err)]
        step = grid[1] - grid[0]
        s = O.abs_mean_scales(d, O.MODE_GROUP, g)[0]
        assert abs(best - s) <= step


def test_tensor_mode_is_scalar_alpha():
    rng = np.random.default_rng(7)
    d = rng.normal(size=(6, 64))
    a = O.abs_mean_scales(d, O.MODE_TENSOR)
    total = 0.0
    for v in d.ravel():
        total += abs(float(v))
    assert a.shape == (1,)
    assert abs(a[0] - total / d.size) < 1e-14


# --------------------------------------------------------------------------------
# per-axis scales by pure-Python loops on a non-square matrix
# ("Per-Axis Weight Deltas", "Key Contributions" 1)
# --------------------------------------------------------------------------------
def test_row_col_group_by_loops():
    rng = np.random.default_rng(11)
    d_out, d_in, G = 5, 64, 32
    d = rng.normal(size=(d_out, d_in))
    rows = O.abs_mean_scales(d, O.MODE_ROW)
    cols = O.abs_mean_scales(d, O.MODE_COL)
    grp = O.abs_mean_scales(d, O.MODE_GROUP, G)
    assert rows.shape == (d_out,) and cols.shape == (d_in,) and grp.shape == (d_out, d_in // G)
    for o in range(d_out):
        acc = 0.0
        for i in range(d_in):
            acc += abs(d[o, i])
        assert abs(rows[o] - acc / d_in) < 1e-14
        for g in range(d_in // G):
            acc = 0.0
            for i in range(g * G, (g + 1) * G):
                acc += abs(d[o, i])
            assert abs(grp[o, g] - acc / G) < 1e-14
    for i in range(d_in):
        acc = 0.0
        for o in range(d_out):
            acc += abs(d[o, i])
        assert abs(cols[i] - acc / d_out) < 1e-14


# --------------------------------------------------------------------------------
# blockwise scales ("Per-Axis Weight Deltas", Future Directions: blockwise per-group
# scaling), square G x G blocks, by pure-Python loops with a ragged last row block
# --------------------------------------------------------------------------------
def test_block_by_loops():
    rng = np.random.default_rng(12)
    d_out, d_in, G = 70, 96, 32
    d = rng.normal(size=(d_out, d_in))
    blk = O.abs_mean_scales(d, O.MODE_BLOCK, G)
    assert blk.shape == (3, 3)
    for rb in range(3):
        for g in range(3):
            acc, n = 0.0, 0
            for o in range(rb * G, min((rb + 1) * G, d_out)):
                for i in range(g * G, (g + 1) * G):
                    acc += abs(d[o, i])
                    n += 1
            assert n == (G * G if rb < 2 else 6 * G)
            assert abs(blk[rb, g] - acc / n) < 1e-14


def test_block_special_cases():
    rng = np.random.default_rng(13)
    G = 32
    # one row: a block is a group
    d = rng.normal(size=(1, 128))
    assert np.array_equal(O.abs_mean_scales(d, O.MODE_BLOCK, G), O.abs_mean_scales(d, O.MODE_GROUP, G))
    # rows repeated within each block: the block scale is the group scale of any row
    base = rng.normal(size=(2, 64))
    d = np.repeat(base, G, axis=0)
    blk = O.abs_mean_scales(d, O.MODE_BLOCK, G)
    grp = O.abs_mean_scales(base, O.MODE_GROUP, G)
    np.testing.assert_allclose(blk, grp, rtol=1e-14, atol=0)
    # expand: entry (o, i) takes block (o // G, i // G)
    e = O.expand_scales(blk, O.MODE_BLOCK, G, 2 * G, 64)
    for o in (0, G - 1, G, 2 * G - 1):
        for i in (0, G - 1, G, 63):
            assert e[o, i] == blk[o // G, i // G]


# --------------------------------------------------------------------------------
# clip ("bitdelta" page, "Safety Benefits: 1. Outlier Clipping")
# --------------------------------------------------------------------------------
@pytest.mark.parametrize("n,k", [(16, 1.0), (100, 3.0), (9, 2.0)])
def test_clip_closed_form_single_spike(n, k):
    """n-1 zeros and one 1: mean 1/n; unbiased variance ((n-1)/n) / (n-1) = 1/n."""
    d = np.zeros(n)
    d[-1] = 1.0
    mean, std, lo, hi = O.clip_stats(d, k)
    assert abs(mean - 1.0 / n) < 1e-15
    assert abs(std - 1.0 / math.sqrt(n)) < 1e-15
    c = O.clip(d, lo, hi)
    assert abs(c[-1] - min(1.0, 1.0 / n + k / math.sqrt(n))) < 1e-15
    assert np.all(c[:-1] == max(0.0, 1.0 / n - k / math.sqrt(n)))


def test_clip_inclusive_and_sign_after_clip():
    d = np.array([-2.0, -1.0, 0.5, 1.0, 3.0])
    c = O.clip(d, -1.0, 1.0)
    assert list(c) == [-1.0, -1.0, 0.5, 1.0, 1.0]
    # with lo > 0 every clamped negative becomes positive: sign follows the clip
    c2 = O.clip(d, 0.25, 1.0)
    assert list(O.sign_bits(c2)) == [True] * 5


def test_clip_single_entry_is_identity():
    mean, std, lo, hi = O.clip_stats(np.array([0.3]), 3.0)
    assert std == 0.0 and lo == hi == mean == 0.3


# --------------------------------------------------------------------------------
# invariants of sign x abs-mean reconstruction, per group
# --------------------------------------------------------------------------------
@pytest.mark.parametrize("mode", [O.MODE_GROUP, O.MODE_ROW, O.MODE_COL, O.MODE_TENSOR, O.MODE_BLOCK])
def test_reconstruction_invariants(mode):
    rng = np.random.default_rng(21 + mode)
    d_out, d_in, G = (6, 256, 64) if mode != O.MODE_BLOCK else (40, 128, 16)
    wb = rng.normal(0, 0.02, size=(d_out, d_in)).astype(np.float32)
    wf = (wb + rng.normal(0, 0.002, size=(d_out, d_in))).astype(np.float32)
    out = O.compress(wb, wf, "f32", mode, G)
    dc = out["delta_c"]
    rec = O.reconstruct(out["signs"], out["scales"], mode, G, d_out, d_in)
    if mode == O.MODE_GROUP:
        slices = [(slice(o, o + 1), slice(g * G, (g + 1) * G)) for o in range(d_out)
                  for g in range(d_in // G)]
    elif mode == O.MODE_ROW:
        slices = [(slice(o, o + 1), slice(None)) for o in range(d_out)]
    elif mode == O.MODE_COL:
        slices = [(slice(None), slice(i, i + 1)) for i in range(d_in)]
    elif mode == O.MODE_BLOCK:
        slices = [(slice(rb * G, (rb + 1) * G), slice(g * G, (g + 1) * G))
                  for rb in range(-(-d_out // G)) for g in range(d_in // G)]
    else:
        slices = [(slice(None), slice(None))]
    for sl in slices:
        a, r = dc[sl], rec[sl]
        # abs-mean keeps the L1 norm of the slice
        assert abs(np.abs(r).sum() - np.abs(a).sum()) < 1e-12
        # magnitude constant within the slice
        assert np.ptp(np.abs(r)) < 1e-15
        # residual energy: sum d^2 - n s^2
        s = np.abs(r).ravel()[0]
        assert abs(((a - r) ** 2).sum() - ((a ** 2).sum() - a.size * s * s)) < 1e-12
        # signs agree with the clipped delta (sign(0) = +1)
        assert np.all((r >= 0) == (a >= 0))


def test_tiny_config_validation_threshold():
    """The tiny workload passes the pages' reconstruction check (mean abs error
    below 0.01, "Best Practices: 3. Compression Validation")."""
    cfg = tiny_config()
    thr = GOLD["validation_threshold"]["max_mean_abs_error"]
    for wf in cfg["w_fine"]:
        out = O.compress(cfg["w_base"], wf, "f32", O.MODE_GROUP, 128, True, 3.0)
        rec = O.reconstruct(out["signs"], out["scales"], O.MODE_GROUP, 128, 256, 512)
        d = O.delta(cfg["w_base"], wf)
        assert np.abs(rec - d).mean() < thr
        # the outliers are really clipped: at least the planted ones exceed hi
        mean, std, lo, hi = out["stats"]
        assert (d > hi).sum() + (d < lo).sum() >= 100


# --------------------------------------------------------------------------------
# decoding of stored formats
# --------------------------------------------------------------------------------
def test_decode_bf16_known_values():
    bits = np.array([0x3F80, 0xC000, 0x0000, 0x8000, 0x3E80, 0x0001], dtype=np.uint16)
    v = O.decode(bits, "bf16")
    assert list(v[:5]) == [1.0, -2.0, 0.0, -0.0, 0.25]
    assert v[5] == 2.0 ** -133  # smallest bf16 subnormal, decoded exactly
    assert math.copysign(1.0, v[3]) == -1.0


def test_decode_roundtrip_with_generator():
    rng = np.random.default_rng(3)
    x = rng.normal(size=1000).astype(np.float32)
    b = bf16_bits(x)
    assert np.array_equal(O.decode(b, "bf16"), bf16_bits_to_f32(b).astype(np.float64))
    # round-to-nearest: error at most half a bf16 ulp (2^-9 relative)
    assert np.all(np.abs(bf16_bits_to_f32(b) - x) <= np.abs(x) * 2.0 ** -8)


# --------------------------------------------------------------------------------
# multi-tenant apply ("BitDelta Guide", "Systems Mechanics: 1. Decoupled Forward Pass")
# --------------------------------------------------------------------------------
def _small_problem(seed=0, d_out=6, d_in=64, B=5, T=3, modes=(0, 1, 2)):
    rng = np.random.default_rng(seed)
    wb = bf16_bits(rng.normal(0, 0.02, size=(d_out, d_in)))
    tenants = [random_tenant(rng, d_out, d_in, modes[u % len(modes)], 32) for u in range(T)]
    x = bf16_bits(rng.normal(0, 1, size=(B, d_in)))
    ids = rng.integers(-1, T, size=B).astype(np.int32)
    ids[0] = 0
    return wb, tenants, x, ids


def test_apply_pure_python_loops():
    """Every y[t, o] by explicit loops over the definition: sum_i (W_base[o,i] +
    sign_u[o,i] * s_u(o,i)) * x[t,i], sign unpacked bit by bit."""
    wb, tenants, x, ids = _small_problem()
    y = O.apply_multi(wb, "bf16", tenants, ids, x, "bf16")
    W = bf16_bits_to_f32(wb).astype(np.float64)
    X = bf16_bits_to_f32(x).astype(np.float64)
    d_out, d_in = W.shape
    for t in range(X.shape[0]):
        u = int(ids[t])
        for o in range(d_out):
            acc = 0.0
            for i in range(d_in):
                w = W[o, i]
                if u >= 0:
                    tn = tenants[u]
                    bit = (int(tn["signs"][o, i // 32]) >> (i % 32)) & 1
                    sc = tn["scales"].astype(np.float64)
                    if tn["mode"] == 0:
                        s = sc[o, i // tn["group_size"]]
                    elif tn["mode"] == 1:
                        s = sc[o]
                    else:
                        s = sc[i]
                    w += s if bit else -s
                acc += w * X[t, i]
            assert abs(y[t, o] - acc) < 1e-12 * (1 + abs(acc))


def test_apply_equals_merged_weight():
    """Decomposition: W_base x + Delta_hat x == (W_base + Delta_hat) x per tenant."""
    wb, tenants, x, ids = _small_problem(seed=1, d_out=8, d_in=128, B=7)
    y = O.apply_multi(wb, "bf16", tenants, ids, x, "bf16")
    W = O.decode(wb, "bf16")
    X = O.decode(x, "bf16")
    for t in range(len(ids)):
        u = int(ids[t])
        Wu = W if u < 0 else O.reconstruct(
            tenants[u]["signs"], O.decode(tenants[u]["scales"], "f16"), tenants[u]["mode"],
            32, 8, 128, w_base=W)
        np.testing.assert_allclose(y[t], Wu @ X[t], rtol=1e-13, atol=1e-15)


def test_apply_properties():
    wb, tenants, x, ids = _small_problem(seed=2, d_out=7, d_in=96, B=9)
    y = O.apply_multi(wb, "bf16", tenants, ids, x, "bf16")
    # permuting tokens permutes outputs
    p = np.random.default_rng(0).permutation(len(ids))
    yp = O.apply_multi(wb, "bf16", tenants, ids[p], x[p], "bf16")
    np.testing.assert_allclose(yp, y[p], rtol=1e-14, atol=1e-16)
    # x = 0 gives 0
    z = O.apply_multi(wb, "bf16", tenants, ids, np.zeros_like(x), "bf16")
    assert np.all(z == 0)
    # linearity in x (exact inputs in f64)
    xf = O.decode(x, "bf16")
    y2 = O.apply_multi(wb, "bf16", tenants, ids, (2 * xf), "f64")
    np.testing.assert_allclose(y2, 2 * y, rtol=1e-14, atol=1e-16)
    # tenant -1 is the base product alone
    base = O.apply_multi(wb, "bf16", tenants, np.full_like(ids, -1), x, "bf16")
    np.testing.assert_allclose(base, xf @ O.decode(wb, "bf16").T, rtol=1e-14, atol=1e-16)
    # out-of-range id is an error in the definition
    bad = ids.copy()
    bad[0] = len(tenants)
    with pytest.raises(ValueError):
        O.apply_multi(wb, "bf16", tenants, bad, x, "bf16")


def test_apply_rows_matches_full():
    wb, tenants, x, ids = _small_problem(seed=4, d_out=9, d_in=64, B=4)
    y = O.apply_multi(wb, "bf16", tenants, ids, x, "bf16")
    rows = np.array([0, 3, 8])
    yr = O.apply_rows(wb, "bf16", tenants, ids, x, "bf16", rows)
    np.testing.assert_array_equal(yr, y[:, rows])
