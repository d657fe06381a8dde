"""Planted mistakes: each test patches one plausible error into the oracle (on the CPU
only) and checks that the pins of tests/test_oracle.py catch it — a dropped term, a
wrong sign or index, a reversed bit order, a transposed axis, a biased estimator."""

import numpy as np

import oracle as O
import oracle.bitdelta as OB
import test_oracle as T

GOLD = T.GOLD


def _patch(monkeypatch, name, fn):
    monkeypatch.setattr(O, name, fn)
    monkeypatch.setattr(OB, name, fn)


def _caught(*pins):
    """True when at least one pin fails under the planted mistake."""
    for pin in pins:
        try:
            pin()
        except AssertionError:
            return True
    return False


def _all_worked_signs():
    for case in GOLD["signs"]["cases"]:
        T.test_worked_signs(case)


def _l2_pins():
    for g in (4, 7, 16):
        T.test_abs_mean_is_l2_optimal_brute_force(g)


def _clip_pins():
    for n, k in [(16, 1.0), (100, 3.0), (9, 2.0)]:
        T.test_clip_closed_form_single_spike(n, k)
    T.test_clip_inclusive_and_sign_after_clip()


def _reconstruction_pins():
    T.test_worked_reconstruction()
    for mode in (O.MODE_GROUP, O.MODE_ROW, O.MODE_COL, O.MODE_TENSOR, O.MODE_BLOCK):
        T.test_reconstruction_invariants(mode)


def _block_pins():
    T.test_block_by_loops()
    T.test_block_special_cases()


def _apply_pins():
    T.test_apply_pure_python_loops()
    T.test_apply_equals_merged_weight()
    T.test_apply_properties()


def test_pins_pass_on_the_real_oracle():
    for pins in (T.test_worked_delta, T.test_worked_group_scale, _all_worked_signs,
                 T.test_sign_of_zero_is_plus_one, T.test_pack_bit_positions, _l2_pins,
                 T.test_row_col_group_by_loops, _clip_pins, _reconstruction_pins, _apply_pins,
                 _block_pins):
        pins()


def test_reversed_delta(monkeypatch):
    orig = O.delta
    _patch(monkeypatch, "delta", lambda wb, wf: orig(wf, wb))
    assert _caught(T.test_worked_delta)


def test_sign_of_zero_negative(monkeypatch):
    _patch(monkeypatch, "sign_bits", lambda dc: np.asarray(dc, dtype=np.float64) > 0)
    assert _caught(T.test_sign_of_zero_is_plus_one, _all_worked_signs)


def test_sign_inverted(monkeypatch):
    _patch(monkeypatch, "sign_bits", lambda dc: np.asarray(dc, dtype=np.float64) < 0)
    assert _caught(_all_worked_signs)


def test_msb_first_packing(monkeypatch):
    def pack(bits):
        bits = np.asarray(bits, dtype=bool)
        if bits.ndim == 1:
            bits = bits[None, :]
        b8 = np.packbits(bits, axis=1, bitorder="big")
        return np.ascontiguousarray(b8).view("<u4").reshape(bits.shape[0], bits.shape[1] // 32)
    _patch(monkeypatch, "pack_bits", pack)
    assert _caught(T.test_pack_bit_positions)


def test_scale_without_abs(monkeypatch):
    # the mean of the signed delta instead of the mean of its magnitude
    _patch(monkeypatch, "abs_mean_scales",
           lambda dc, mode, group_size=128: _signed_mean(dc, mode, group_size))
    assert _caught(T.test_worked_group_scale, _l2_pins, T.test_row_col_group_by_loops)


def _signed_mean(dc, mode, group_size):
    dc = np.asarray(dc, dtype=np.float64)
    if mode == O.MODE_GROUP:
        s = dc.reshape(-1, group_size).mean(axis=1)
        return s.reshape(dc.shape[0], -1) if dc.ndim == 2 else s
    if mode == O.MODE_ROW:
        return dc.mean(axis=1)
    if mode == O.MODE_COL:
        return dc.mean(axis=0)
    return np.array([dc.mean()])


def test_groups_along_the_wrong_axis(monkeypatch):
    orig = O.abs_mean_scales

    def scales(dc, mode, group_size=128):
        dc = np.asarray(dc, dtype=np.float64)
        if mode == O.MODE_GROUP and dc.ndim == 2 and dc.shape[0] % group_size == 0:
            # groups of G consecutive rows of one column, laid out [d_out/G, d_in]
            return np.abs(dc).reshape(-1, group_size, dc.shape[1]).mean(axis=1).T.reshape(
                dc.shape[0], -1)[:, : dc.shape[1] // group_size]
        if mode == O.MODE_ROW:
            return orig(dc, O.MODE_COL, group_size)[: dc.shape[0]]
        return orig(dc, mode, group_size)
    _patch(monkeypatch, "abs_mean_scales", scales)
    assert _caught(T.test_row_col_group_by_loops)


def test_biased_std(monkeypatch):
    def stats(d, k):
        d = np.asarray(d, dtype=np.float64).ravel()
        m = float(d.mean())
        s = float(np.sqrt(np.mean((d - m) ** 2)))  # N instead of N - 1
        return m, s, m - k * s, m + k * s
    _patch(monkeypatch, "clip_stats", stats)
    assert _caught(_clip_pins)


def test_clip_dropped(monkeypatch):
    _patch(monkeypatch, "clip", lambda d, lo, hi: np.asarray(d, dtype=np.float64))
    assert _caught(_clip_pins)


def test_reconstruct_flips_signs(monkeypatch):
    orig = O.reconstruct

    def rec(signs, scales, mode, group_size, d_out, d_in, w_base=None, rows=None):
        words = np.asarray(signs, dtype="<u4")
        return orig(~words, scales, mode, group_size, d_out, d_in, w_base=w_base, rows=rows)
    _patch(monkeypatch, "reconstruct", rec)
    assert _caught(_reconstruction_pins)


def test_apply_drops_the_base(monkeypatch):
    orig = O.apply_multi

    def apply(w_base, w_dtype, tenants, tenant_ids, x, x_dtype, rows=None):
        return orig(np.zeros_like(np.asarray(w_base)), w_dtype, tenants, tenant_ids, x, x_dtype,
                    rows=rows)
    _patch(monkeypatch, "apply_multi", apply)
    assert _caught(_apply_pins)


def test_apply_uses_the_wrong_tenant(monkeypatch):
    orig = O.apply_multi

    def apply(w_base, w_dtype, tenants, tenant_ids, x, x_dtype, rows=None):
        ids = np.asarray(tenant_ids)
        n = len(tenants)
        shifted = np.where(ids >= 0, (ids + 1) % max(n, 1), ids).astype(np.int32)
        return orig(w_base, w_dtype, tenants, shifted, x, x_dtype, rows=rows)
    _patch(monkeypatch, "apply_multi", apply)
    assert _caught(_apply_pins)


def test_block_rows_off_by_one(monkeypatch):
    real = OB.abs_mean_scales

    def scales(dc, mode, group_size=128):
        if mode != O.MODE_BLOCK:
            return real(dc, mode, group_size)
        a = np.abs(np.asarray(dc, dtype=np.float64))
        G = group_size
        nrb = -(-a.shape[0] // G)
        out = np.empty((nrb, a.shape[1] // G))
        for rb in range(nrb):
            blk = a[rb * G:(rb + 1) * G - 1] if rb * G + 1 < a.shape[0] else a[rb * G:]
            out[rb] = blk.reshape(blk.shape[0], -1, G).mean(axis=(0, 2))
        return out
    _patch(monkeypatch, "abs_mean_scales", scales)
    assert _caught(_block_pins, _reconstruction_pins)


def test_block_index_transposed(monkeypatch):
    real = OB.expand_scales

    def expand(scales, mode, group_size, d_out, d_in, rows=None):
        if mode != O.MODE_BLOCK:
            return real(scales, mode, group_size, d_out, d_in, rows)
        nrb, ngc = -(-d_out // group_size), d_in // group_size
        s = np.asarray(scales, dtype=np.float64).reshape(nrb, ngc)
        r = np.arange(d_out) if rows is None else np.asarray(rows)
        # block row taken from the column and block column from the row
        bi = np.minimum(np.arange(d_in)[None, :] // group_size, nrb - 1) + 0 * r[:, None]
        bj = np.minimum(r[:, None] // group_size, ngc - 1) + 0 * np.arange(d_in)[None, :]
        return s[bi, bj]
    _patch(monkeypatch, "expand_scales", expand)
    assert _caught(_block_pins, _reconstruction_pins)
