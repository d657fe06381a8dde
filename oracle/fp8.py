"""float64 reference of an FP8 (e4m3) base model under the 1-bit delta path.

TEST INFRASTRUCTURE ONLY, like the rest of this package: the product path never imports
it and it never imports the product.

"BitDelta Guide", "3. Quantized Base Model Compatibility (BitDelta + GPTQ / QuIP#)": the
1-bit delta is computed against, and applied on top of, quantized base weights.
"Per-Axis Weight Deltas for Frequent Model Updates", Future Directions: INT4/FP8
co-design. The pages fix neither the 8-bit format nor the scale rule. The readings taken
here (the plainest ones):

* Format: the OCP 8-bit floating point E4M3 encoding: 1 sign bit, 4 exponent bits with
  bias 7, 3 mantissa bits; exponent field 0 holds the subnormals m/8 * 2^-6; the
  pattern S.1111.111 is NaN; there are no infinities; the largest finite value is 448.
* Per-channel scales: one fp32 scale per output row o, s_o = max_i |W[o, i]| / 448,
  computed as an fp32 division.
* Codes: q[o, i] = e4m3 rounding of the fp32 quotient W[o, i] / s_o (fp32 division),
  to nearest with ties to the even mantissa, magnitudes above 448 saturating to 448, the
  sign kept (a negative value that rounds to zero gives -0). A row of zeros has s_o = 0
  and all codes 0. The quotient and the rounding are taken in fp32 because they decide
  an integer code, and fp32 is the precision of the kernel that encodes.
* Dequantized base: W_hat[o, i] = s_o * value(q[o, i]); the apply is the decomposed
  forward of :func:`oracle.bitdelta.apply_multi` with W_hat as the base.
"""

from __future__ import annotations

import numpy as np

from .bitdelta import apply_multi, decode

E4M3_MAX = 448.0


def e4m3_value(codes) -> np.ndarray:
    """Value of each e4m3 code (uint8), from the bit fields; NaN for S.1111.111."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * 2.0 ** (e - 7.0))
    v = sign * mag
    return np.where((c & 0x7F) == 0x7F, np.nan, v)


def _magnitudes():
    """The 127 finite non-negative e4m3 magnitudes, indexed by code 0x00 .. 0x7E
    (increasing with the code)."""
    return e4m3_value(np.arange(0x7F, dtype=np.uint8))


def e4m3_round(v) -> np.ndarray:
    """e4m3 codes of float32 values: nearest finite magnitude, ties to the even code
    (even mantissa), saturation at 448, sign kept. Inputs must be finite."""
    v = np.asarray(v, dtype=np.float32)
    if not np.all(np.isfinite(v)):
        raise ValueError("finite inputs only")
    a = np.abs(v.astype(np.float64))
    mags = _magnitudes()
    hi = np.searchsorted(mags, a, side="left")          # first magnitude >= a
    hi = np.minimum(hi, len(mags) - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - mags[lo]
    d_hi = mags[hi] - a
    pick = np.where(d_lo < d_hi, lo, hi)
    tie = (d_lo == d_hi) & (lo != hi)
    pick = np.where(tie, np.where(lo % 2 == 0, lo, hi), pick)
    pick = np.where(a >= E4M3_MAX, len(mags) - 1, pick)  # saturate
    code = pick.astype(np.uint8)
    return np.where(np.signbit(v), code | 0x80, code).astype(np.uint8)


def quantize_base(w, w_dtype: str):
    """Per-row fp32 scales and e4m3 codes of a base weight matrix ``[d_out, d_in]``
    (``w_dtype`` "bf16" bit patterns or "f32")."""
    w32 = decode(w, w_dtype).astype(np.float32)  # exact: bf16 and f32 values are f32 values
    amax = np.max(np.abs(w32), axis=1)
    scales = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    codes = np.zeros(w32.shape, dtype=np.uint8)
    nz = scales > 0
    q = (w32[nz] / scales[nz][:, None]).astype(np.float32)
    codes[nz] = e4m3_round(q)
    return codes, scales


def dequantize_base(codes, scales) -> np.ndarray:
    """W_hat = s_o * value(q) in float64."""
    return np.asarray(scales, dtype=np.float64)[:, None] * e4m3_value(codes)


def apply_multi_fp8(codes, scales, tenants, tenant_ids, x, x_dtype: str, rows=None):
    """y_t = W_hat x_t + Delta_hat_u x_t with the dequantized fp8 base (float64)."""
    return apply_multi(dequantize_base(codes, scales), "f64", tenants, tenant_ids, x, x_dtype, rows=rows)
