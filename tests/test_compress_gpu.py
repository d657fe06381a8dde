"""GPU parity of bd_compress / bd_reconstruct against the fp64 oracle, through the C ABI.

Signs must be bit-exact; scales within 1e-5 relative; clip statistics close to the
oracle's. Sizes span several warp chunks and ragged tails (d_in % 256 != 0, odd d_out)."""

import json
import os

import numpy as np
import pytest

import oracle as O
from helpers import assert_scales_close, dev, host
from workloads import bf16_bits, tiny_config, weight_pair

pytestmark = pytest.mark.gpu

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")))


@pytest.fixture(scope="module")
def bd():
    from tenant_serving_b200 import build
    build.build()
    import tenant_serving_b200 as m
    return m


def _gpu_compress(bd, wb, wf, dtype, mode, G=128, clip=False, k=3.0):
    cfg = bd.compress_cfg(mode=mode, group_size=G, clip=clip, clip_k=k)
    signs, scales, stats = bd.bd_compress(dev(wb, dtype), dev(wf, dtype), cfg)
    return host(signs), host(scales), (host(stats) if stats is not None else None)


def _check(bd, wb, wf, dtype, mode, G=128, clip=False, k=3.0):
    ref = O.compress(wb, wf, dtype, mode, G, clip, k)
    signs, scales, stats = _gpu_compress(bd, wb, wf, dtype, mode, G, clip, k)
    np.testing.assert_array_equal(signs, ref["signs"])
    assert_scales_close(scales.reshape(ref["scales"].shape), ref["scales"])
    if clip:
        m, s, lo, hi = ref["stats"]
        assert abs(stats[0] - m) <= 1e-9 * max(1.0, abs(m)) + 1e-12 * s
        assert abs(stats[1] - s) <= 1e-9 * s
        assert abs(stats[2] - lo) <= 1e-9 * abs(lo) + 1e-12
        assert abs(stats[3] - hi) <= 1e-9 * abs(hi) + 1e-12
    return ref, signs, scales


def test_worked_examples_tiled(bd):
    """The pages' groups of 4 ("3. 1-bit Quantization"), each repeated 32 times into a
    1 x 128 row (G = 128): scale = abs-mean, words = 0xFFFFFFFF / 0x55555555."""
    rows = []
    for case in GOLD["signs"]["cases"]:
        rows.append(np.tile(np.array(case["delta_group"], dtype=np.float32), 32))
    wf = np.stack(rows).astype(np.float32)
    wb = np.zeros_like(wf)
    ref, signs, scales = _check(bd, wb, wf, "f32", O.MODE_GROUP, 128)
    assert all(int(w) == 0xFFFFFFFF for w in signs[0])
    assert all(int(w) == 0x55555555 for w in signs[1])
    assert abs(scales[0, 0] - 0.2) < 1e-7


@pytest.mark.parametrize("tenant", [0, 1])
def test_tiny_config(bd, tenant):
    cfg = tiny_config()
    _check(bd, cfg["w_base"], cfg["w_fine"][tenant], "f32", O.MODE_GROUP, 128, True, 3.0)


SHAPES = [(1, 32), (3, 96), (37, 256), (64, 544), (129, 1024), (300, 4096 + 96)]


@pytest.mark.parametrize("d_out,d_in", SHAPES)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("mode", [O.MODE_GROUP, O.MODE_ROW, O.MODE_COL, O.MODE_TENSOR, O.MODE_BLOCK])
@pytest.mark.parametrize("clip", [False, True])
def test_random_shapes(bd, d_out, d_in, dtype, mode, clip):
    seed = d_out * 7 + d_in + mode * 1000 + int(clip) * 10000 + (dtype == "f32")
    wb, wf = weight_pair(seed, d_out, d_in, dtype, 0.02, 0.002, 0.01, 20.0)
    G = 32 if d_in % 64 else (64 if d_in % 128 else 128)
    _check(bd, wb, wf, dtype, mode, G, clip, 3.0)


@pytest.mark.parametrize("G", [32, 64, 128, 256, 512, 1024])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_group_sizes(bd, G, dtype):
    wb, wf = weight_pair(G, 40, 2048, dtype, 0.02, 0.002, 0.001, 20.0)
    _check(bd, wb, wf, dtype, O.MODE_GROUP, G, True, 2.0)


@pytest.mark.parametrize("G", [32, 64, 128, 256, 512, 1024])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_block_sizes(bd, G, dtype):
    """G x G blocks over 1100 rows (a ragged last row block for every G)."""
    wb, wf = weight_pair(G + 1, 1100, 2048, dtype, 0.02, 0.002, 0.001, 20.0)
    _check(bd, wb, wf, dtype, O.MODE_BLOCK, G, G == 128, 3.0)


def test_zero_and_negative_zero(bd):
    """delta exactly 0 (and -0.0 = -0.0 - 0.0) gives sign +1 and scale 0."""
    d_out, d_in = 4, 256
    wb = np.zeros((d_out, d_in), dtype=np.float32)
    wf = np.zeros((d_out, d_in), dtype=np.float32)
    wf[1] = -0.0
    wb[2] = 1.0
    wf[2] = 1.0
    wf[3, :128] = -1e-30  # a tiny negative group next to a zero group
    for mode in (O.MODE_GROUP, O.MODE_ROW, O.MODE_COL, O.MODE_TENSOR):
        ref, signs, scales = _check(bd, wb, wf, "f32", mode, 128)
    signs, scales, _ = _gpu_compress(bd, wb, wf, "f32", O.MODE_GROUP, 128)
    assert all(int(w) == 0xFFFFFFFF for w in signs[:3].ravel())
    assert all(int(w) == 0 for w in signs[3, :4])
    assert np.all(scales[:3] == 0) and scales[3, 1] == 0


def test_clip_flips_signs_when_bound_positive(bd):
    """If the whole delta is shifted so lo > 0, every clamped negative becomes positive."""
    rng = np.random.default_rng(9)
    d_out, d_in = 16, 512
    wb = rng.normal(0, 0.02, size=(d_out, d_in)).astype(np.float32)
    d = 5.0 + rng.normal(0, 1.0, size=(d_out, d_in))
    d[0, :10] = -4.0  # far below mean - 3 std
    wf = (wb + d).astype(np.float32)
    ref, signs, _ = _check(bd, wb, wf, "f32", O.MODE_GROUP, 128, True, 3.0)
    assert ref["stats"][2] > 0
    assert int(signs[0, 0]) == 0xFFFFFFFF


@pytest.mark.parametrize("mode", [O.MODE_GROUP, O.MODE_BLOCK])
@pytest.mark.parametrize("side", [1.0, -1.0])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_clip_bound_past_zero_rewrites_signs(bd, mode, side, dtype):
    """A delta shifted so far that lo > 0 (side +1) or hi < 0 (side -1): the clamp moves
    the far tail across zero, so the signs of every group with a clamped entry change;
    G = 64 and 512 column groups (G x G blocks) over 130 rows."""
    rng = np.random.default_rng(19 + int(side > 0) + 2 * mode)
    for G in (64, 512):
        d_out, d_in = 130, 1024
        wb = rng.normal(0, 0.02, size=(d_out, d_in))
        d = side * (5.0 + rng.normal(0, 1.0, size=(d_out, d_in)))
        d[7, 3:40] = -side * 4.0  # far on the other side of zero
        wf = wb + d
        if dtype == "bf16":
            wb, wf = bf16_bits(wb), bf16_bits(wf)
        else:
            wb, wf = wb.astype(np.float32), wf.astype(np.float32)
        ref, signs, _ = _check(bd, wb, wf, dtype, mode, G, True, 3.0)
        lo, hi = ref["stats"][2], ref["stats"][3]
        assert (lo > 0) if side > 0 else (hi < 0)
        assert int(signs[7, 1]) == (0xFFFFFFFF if side > 0 else 0)


def test_bf16_llama_k_proj_full(bd):
    """Full k_proj shape (1024 x 4096, bf16), delta ~ N(0, 0.001), 0.05% outliers x30,
    group 128 with the 3-sigma clip; compared element by element."""
    wb, wf = weight_pair(2024, 1024, 4096, "bf16")
    ref, signs, _ = _check(bd, wb, wf, "bf16", O.MODE_GROUP, 128, True, 3.0)
    # about 3.6% of stored deltas are exactly zero in bf16 (sign +1 must hold there)
    zero = O.delta(O.decode(wb, "bf16"), O.decode(wf, "bf16")) == 0
    assert zero.mean() > 0.01


@pytest.mark.parametrize("mode", [O.MODE_ROW, O.MODE_COL])
def test_bf16_llama_down_proj_axis(bd, mode):
    wb, wf = weight_pair(77, 4096, 14336, "bf16")
    _check(bd, wb, wf, "bf16", mode, 128, mode == O.MODE_COL, 3.0)


def test_reconstruct_matches_oracle(bd):
    rng = np.random.default_rng(4)
    d_out, d_in = 70, 768
    words = rng.integers(0, 2 ** 32, size=(d_out, d_in // 32), dtype=np.uint64).astype(np.uint32)
    wb = bf16_bits(rng.normal(0, 0.02, size=(d_out, d_in)))
    for mode, G in ((O.MODE_GROUP, 64), (O.MODE_ROW, 128), (O.MODE_COL, 128), (O.MODE_TENSOR, 128),
                    (O.MODE_BLOCK, 32), (O.MODE_BLOCK, 128)):
        shape = bd.scales_shape(mode, d_out, d_in, G)
        s16 = (rng.random(shape) * 0.01).astype(np.float16)
        for sd, s in (("f16", s16), ("f32", s16.astype(np.float32) * 1.5)):
            ref = O.reconstruct(words, O.decode(s, sd), mode, G, d_out, d_in)
            out = bd.bd_reconstruct(dev(words), dev(s), mode, G, d_out, d_in)
            np.testing.assert_array_equal(host(out).astype(np.float64), ref)  # exact in fp32
            refw = O.reconstruct(words, O.decode(s, sd), mode, G, d_out, d_in,
                                 w_base=O.decode(wb, "bf16"))
            import torch
            outw = bd.bd_reconstruct(dev(words), dev(s), mode, G, d_out, d_in, w_base=dev(wb),
                                     out_dtype=torch.bfloat16)
            # bf16 output: rounded once from the fp32 sum
            got = O.decode(host(outw), "bf16")
            assert np.all(np.abs(got - refw) <= np.abs(refw) * 2.0 ** -8 + 1e-30)


def test_compress_then_reconstruct_validation_threshold(bd):
    """Round trip on the GPU passes the pages' check mean |rec - delta| < 0.01."""
    cfg = tiny_config()
    wb, wf = cfg["w_base"], cfg["w_fine"][0]
    c = bd.compress_cfg(mode=bd.BD_SCALE_GROUP, group_size=128, clip=True, clip_k=3.0)
    signs, scales, _ = bd.bd_compress(dev(wb), dev(wf), c)
    rec = host(bd.bd_reconstruct(signs, scales, bd.BD_SCALE_GROUP, 128, 256, 512))
    d = O.delta(wb, wf)
    assert np.abs(rec - d).mean() < GOLD["validation_threshold"]["max_mean_abs_error"]


@pytest.mark.parametrize("clip", [False, True])
def test_bf16_llama_gate_full_sampled(bd, clip):
    """The bench's compress configuration on its largest matrix: gate_proj 14336 x 4096
    bf16, group 128, with and without the 3-sigma clip. The clip statistics are checked
    over the whole matrix; signs (bit-exact) and scales on 256 sampled rows."""
    d_out, d_in = 14336, 4096
    wb, wf = weight_pair(14336, d_out, d_in, "bf16")
    signs, scales, stats = _gpu_compress(bd, wb, wf, "bf16", O.MODE_GROUP, 128, clip, 3.0)
    d = O.delta(O.decode(wb, "bf16"), O.decode(wf, "bf16"))
    rows = np.sort(np.random.default_rng(3).choice(d_out, 256, replace=False))
    dr = d[rows]
    if clip:
        m, s, lo, hi = O.clip_stats(d, 3.0)
        assert abs(stats[0] - m) <= 1e-9 * max(1.0, abs(m)) + 1e-12 * s
        assert abs(stats[1] - s) <= 1e-9 * s
        dr = O.clip(dr, lo, hi)
    ref_scales = O.abs_mean_scales(dr, O.MODE_GROUP, 128)
    ref_signs = O.pack_bits(O.sign_bits(dr))
    np.testing.assert_array_equal(signs.reshape(d_out, d_in // 32)[rows], ref_signs)
    assert_scales_close(scales.reshape(d_out, d_in // 128)[rows], ref_scales)
