"""float64 reference of BitDelta compress / reconstruct / multi-tenant apply.

TEST INFRASTRUCTURE ONLY (see the package docstring): the product path never imports
this module and this module never imports the product.

Conventions shared with the CUDA library only through the *definition* of the method,
never through code:

* A weight matrix is ``[d_out, d_in]`` row-major, the ``[Out, In]`` layout of the
  ``BitDeltaLinear`` listing in "BitDelta Guide", section "1. Computing the Binary
  Sign Delta and Initial Scale in PyTorch".
* The sign mask is packed along the input axis ("Per-Axis Weight Deltas",
  "Methodology": masks stay packed at 1 bit along the input axis), 32 signs per
  ``uint32`` word, word ``w`` of row ``o`` holding columns ``32w .. 32w+31`` with
  column ``32w + j`` in bit ``j`` (least significant bit first). Bit 1 means +1 and
  bit 0 means -1 ("BitDelta Guide", "1. Mathematical Formulation": one bit, 0 for -1
  and 1 for +1).
* sign(0) is +1, -0.0 included: bit = not (delta < 0). The pages disagree here
  ("bitdelta" page, "3. 1-bit Quantization", uses a sign function with sign(0) = 0,
  which has no 1-bit code; "BitDelta Guide" maps delta <= 0 to -1); the plainest
  reading that gives every entry a 1-bit code and matches the required rule is
  delta >= 0 -> +1.
"""

from __future__ import annotations

import numpy as np

MODE_GROUP = 0   # one scale per contiguous run of G entries along d_in
MODE_ROW = 1     # one scale per output row (a 1 x d_out vector)
MODE_COL = 2     # one scale per input column (a d_in x 1 vector)
MODE_TENSOR = 3  # one scalar for the whole matrix (the original per-matrix alpha)
MODE_BLOCK = 4   # one scale per square block of G rows x G columns

_MODES = (MODE_GROUP, MODE_ROW, MODE_COL, MODE_TENSOR, MODE_BLOCK)


# ----------------------------------------------------------------------------------
# exact decoding of the storage formats the library accepts
# ----------------------------------------------------------------------------------
def decode(a, dtype: str) -> np.ndarray:
    """Widen stored values to float64 without rounding.

    ``bf16`` arrays are carried as their uint16 bit patterns; a bf16 value is the
    float32 whose upper half is those 16 bits and whose lower half is zero, so the
    widening is exact. ``f16`` may be given as float16 values or uint16 bits. ``f32``
    and ``f64`` widen exactly by definition.
    """
    a = np.asarray(a)
    if dtype == "bf16":
        if a.dtype != np.uint16:
            raise TypeError("bf16 data must be given as uint16 bit patterns")
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if dtype == "f16":
        if a.dtype == np.uint16:
            a = a.view(np.float16)
        if a.dtype != np.float16:
            raise TypeError("f16 data must be float16 values or uint16 bit patterns")
        return a.astype(np.float64)
    if dtype == "f32":
        if a.dtype != np.float32:
            raise TypeError("f32 data must be float32")
        return a.astype(np.float64)
    if dtype == "f64":
        return a.astype(np.float64)
    raise ValueError(f"unknown dtype {dtype!r}")


# ----------------------------------------------------------------------------------
# compress
# ----------------------------------------------------------------------------------
def delta(w_base: np.ndarray, w_fine: np.ndarray) -> np.ndarray:
    """Delta = W_fine - W_base, elementwise ("bitdelta" page, "1. Delta Computation";
    "BitDelta Guide", "1. Mathematical Formulation"). Exact in float64 for inputs
    decoded from bf16 / fp16 / fp32."""
    w_base = np.asarray(w_base, dtype=np.float64)
    w_fine = np.asarray(w_fine, dtype=np.float64)
    if w_base.shape != w_fine.shape:
        raise ValueError("base and fine-tuned weights differ in shape")
    return w_fine - w_base


def clip_stats(d: np.ndarray, k: float):
    """Mean and standard deviation of the whole delta matrix and the clip bounds
    ``mean -/+ k*std`` ("bitdelta" page, "Safety Benefits: 1. Outlier Clipping",
    default k = 3; "3. Safety-First Configuration" uses k = 2).

    The page calls ``delta.std()``, whose default is the unbiased (N - 1) estimator.
    For a single entry that estimator is undefined; this oracle takes std = 0 there
    (the clip then maps the entry onto itself).
    Returns ``(mean, std, lo, hi)`` as Python floats.
    """
    d = np.asarray(d, dtype=np.float64).ravel()
    n = d.size
    if n == 0:
        raise ValueError("empty delta")
    mean = float(np.mean(d))
    if n > 1:
        var = float(np.sum((d - mean) ** 2)) / (n - 1)
        std = float(np.sqrt(var))
    else:
        std = 0.0
    return mean, std, mean - k * std, mean + k * std


def clip(d: np.ndarray, lo: float, hi: float) -> np.ndarray:
    """clamp(delta, lo, hi) with inclusive bounds: a value equal to a bound stays."""
    return np.minimum(np.maximum(np.asarray(d, dtype=np.float64), lo), hi)


def abs_mean_scales(dc: np.ndarray, mode: int, group_size: int = 128) -> np.ndarray:
    """Absolute-mean scales of the (clipped) delta.

    * group: the page's recipe ("bitdelta", "2. Group Quantization") flattens the
      delta, cuts it into ``numel // G`` contiguous groups of G entries and takes
      ``mean(|delta|)`` of each. For a ``[d_out, d_in]`` matrix with ``d_in % G == 0``
      the groups are contiguous runs along d_in, so the result is shaped
      ``[d_out, d_in // G]``; for 1-D input (the page's worked example) it is
      ``[numel // G]``.
    * row: one scale per output row (``[d_out]``); column: one per input column
      (``[d_in]``) ("Per-Axis Weight Deltas", "Key Contributions" 1). The pages learn
      these vectors from calibration data; here each is the analytic abs-mean of its
      slice, the L2-optimal value for fixed signs ("BitDelta Guide",
      "2. Optimal L2 Norm Initialization", applied per slice).
    * tensor: one scalar, ``alpha = (1 / (n m)) sum |delta_ij|`` (same section).
    * block: "Per-Axis Weight Deltas", Future Directions, names blockwise per-group
      scaling without defining the block. Reading: the group of G entries along a row
      extended to a square block of G rows x G columns (rows ``G rb .. G rb + G - 1``,
      columns ``G g .. G g + G - 1``), one abs-mean per block; the last row block holds
      the ``d_out % G`` remaining rows when G does not divide d_out. Shape
      ``[ceil(d_out / G), d_in // G]``.
    """
    dc = np.asarray(dc, dtype=np.float64)
    a = np.abs(dc)
    if mode == MODE_GROUP:
        if group_size <= 0 or a.size % group_size != 0:
            raise ValueError("group size must divide the number of entries")
        if a.ndim == 2 and a.shape[1] % group_size != 0:
            raise ValueError("group size must divide d_in")
        s = a.reshape(-1, group_size).mean(axis=1)
        if a.ndim == 2:
            s = s.reshape(a.shape[0], a.shape[1] // group_size)
        return s
    if mode == MODE_ROW:
        return a.mean(axis=1)
    if mode == MODE_COL:
        return a.mean(axis=0)
    if mode == MODE_TENSOR:
        return np.array([a.mean()])
    if mode == MODE_BLOCK:
        if a.ndim != 2 or group_size <= 0 or a.shape[1] % group_size != 0:
            raise ValueError("block scales need a [d_out, d_in] matrix with G dividing d_in")
        d_out, d_in = a.shape
        G = group_size
        nrb = -(-d_out // G)
        s = np.empty((nrb, d_in // G))
        for rb in range(nrb):
            blk = a[rb * G:(rb + 1) * G]
            s[rb] = blk.reshape(blk.shape[0], d_in // G, G).mean(axis=(0, 2))
        return s
    raise ValueError(f"unknown scale mode {mode}")


def sign_bits(dc: np.ndarray) -> np.ndarray:
    """Boolean sign mask: True (+1) where the clipped delta is >= 0, -0.0 included."""
    return ~(np.asarray(dc, dtype=np.float64) < 0)


def pack_bits(bits: np.ndarray) -> np.ndarray:
    """Pack a boolean ``[d_out, d_in]`` mask into ``uint32[d_out, d_in // 32]``,
    column ``32w + j`` in bit ``j`` of word ``w`` (LSB first)."""
    bits = np.asarray(bits, dtype=bool)
    if bits.ndim == 1:
        bits = bits[None, :]
    d_out, d_in = bits.shape
    if d_in % 32 != 0:
        raise ValueError("d_in must be a multiple of 32 to pack signs into uint32 words")
    b8 = np.packbits(bits, axis=1, bitorder="little")
    return np.ascontiguousarray(b8).view("<u4").reshape(d_out, d_in // 32)


def unpack_bits(words: np.ndarray, d_in: int) -> np.ndarray:
    """Inverse of :func:`pack_bits`: ``uint32[d_out, d_in // 32]`` -> bool."""
    words = np.ascontiguousarray(np.asarray(words, dtype="<u4"))
    if words.ndim == 1:
        words = words[None, :]
    b8 = words.view(np.uint8).reshape(words.shape[0], -1)
    return np.unpackbits(b8, axis=1, bitorder="little")[:, :d_in].astype(bool)


def compress(w_base, w_fine, dtype: str, mode: int = MODE_GROUP, group_size: int = 128,
             clip_on: bool = False, clip_k: float = 3.0):
    """The compress half of the method in the order clip -> scale -> sign.

    Steps: delta ("1. Delta Computation"); optional whole-matrix k-sigma clamp
    ("Outlier Clipping"); abs-mean scales per the chosen granularity ("2. Group
    Quantization" / per-axis vectors / per-matrix alpha); sign bits of the clipped
    delta ("3. 1-bit Quantization"), packed as described in the module docstring.

    Returns a dict with ``signs`` (uint32 ``[d_out, d_in//32]``), ``scales``
    (float64, shape per :func:`abs_mean_scales`), ``stats`` (``(mean, std, lo, hi)``
    or ``None`` when clip is off) and ``delta_c`` (the clipped delta, float64).
    """
    d = delta(decode(w_base, dtype), decode(w_fine, dtype))
    if d.ndim != 2:
        raise ValueError("compress expects a [d_out, d_in] matrix")
    stats = None
    dc = d
    if clip_on:
        stats = clip_stats(d, clip_k)
        dc = clip(d, stats[2], stats[3])
    scales = abs_mean_scales(dc, mode, group_size)
    signs = pack_bits(sign_bits(dc))
    return {"signs": signs, "scales": scales, "stats": stats, "delta_c": dc}


# ----------------------------------------------------------------------------------
# reconstruct
# ----------------------------------------------------------------------------------
def expand_scales(scales: np.ndarray, mode: int, group_size: int, d_out: int, d_in: int,
                  rows=None) -> np.ndarray:
    """Per-entry scale matrix ``[len(rows) or d_out, d_in]`` for the given granularity."""
    s = np.asarray(scales, dtype=np.float64)
    r = np.arange(d_out) if rows is None else np.asarray(rows)
    if mode == MODE_GROUP:
        s = s.reshape(d_out, d_in // group_size)[r]
        return np.repeat(s, group_size, axis=1)
    if mode == MODE_ROW:
        return np.repeat(s.reshape(d_out)[r][:, None], d_in, axis=1)
    if mode == MODE_COL:
        return np.repeat(s.reshape(1, d_in), len(r), axis=0)
    if mode == MODE_TENSOR:
        return np.full((len(r), d_in), float(s.reshape(-1)[0]))
    if mode == MODE_BLOCK:
        s = s.reshape(-(-d_out // group_size), d_in // group_size)[r // group_size]
        return np.repeat(s, group_size, axis=1)
    raise ValueError(f"unknown scale mode {mode}")


def reconstruct(signs, scales, mode: int, group_size: int, d_out: int, d_in: int,
                w_base=None, rows=None) -> np.ndarray:
    """Delta_hat = signs * scales ("4. Reconstruction"); with ``w_base`` given, the
    personalised weight W_base + Delta_hat ("5. Serving"). ``signs`` are packed words;
    ``scales`` are float64 values (decode stored fp16 / fp32 scales first)."""
    r = np.arange(d_out) if rows is None else np.asarray(rows)
    bits = unpack_bits(np.asarray(signs).reshape(d_out, d_in // 32)[r], d_in)
    dh = np.where(bits, 1.0, -1.0) * expand_scales(scales, mode, group_size, d_out, d_in, r)
    if w_base is not None:
        dh = dh + np.asarray(w_base, dtype=np.float64).reshape(d_out, d_in)[r]
    return dh


# ----------------------------------------------------------------------------------
# multi-tenant apply
# ----------------------------------------------------------------------------------
def apply_multi(w_base, w_dtype: str, tenants, tenant_ids, x, x_dtype: str, rows=None):
    """Decomposed multi-tenant forward ("BitDelta Guide", "Systems Mechanics:
    1. Decoupled Forward Pass"): for every token t of tenant u,
    ``y_t = W_base x_t + Delta_hat_u x_t``, the base shared by all tokens and the delta
    chosen per token.

    ``tenants`` is a list of dicts ``{signs, scales, scale_dtype, mode, group_size}``
    holding the bytes the library receives (scales decoded exactly here). A tenant id
    of -1 means "base model only"; any other id outside ``[0, len(tenants))`` is an
    error. ``rows`` (optional) restricts the output to those rows of ``d_out``.
    Each tenant's tokens are handled together by a float64 matmul. Returns float64
    ``[B, len(rows) or d_out]``.
    """
    wb = decode(w_base, w_dtype)
    d_out, d_in = wb.shape
    xs = decode(x, x_dtype).reshape(-1, d_in)
    ids = np.asarray(tenant_ids, dtype=np.int64).reshape(-1)
    if ids.size != xs.shape[0]:
        raise ValueError("one tenant id per token is required")
    r = np.arange(d_out) if rows is None else np.asarray(rows)
    y = xs @ wb[r].T
    for u in np.unique(ids):
        if u == -1:
            continue
        if u < 0 or u >= len(tenants):
            raise ValueError(f"tenant id {u} out of range")
        t = tenants[u]
        s = decode(t["scales"], t["scale_dtype"])
        dh = reconstruct(t["signs"], s, t["mode"], t.get("group_size", 128), d_out, d_in,
                         rows=r)
        sel = ids == u
        y[sel] += xs[sel] @ dh.T
    return y


def apply_rows(w_base, w_dtype, tenants, tenant_ids, x, x_dtype, rows):
    """:func:`apply_multi` restricted to the output rows ``rows``; used to check
    sampled outputs of full-size workloads one row at a time."""
    return apply_multi(w_base, w_dtype, tenants, tenant_ids, x, x_dtype, rows=rows)
