"""GPU parity of bd_apply_multi against the fp64 oracle, through the C ABI.

Tolerance (apply outputs, bf16 inputs, fp32 accumulation):
    |y - y_ref| <= 1e-2 * (|y_ref| + rms(y_ref)), rms over the output tensor,
checked on the full output, plus cases where W_base = 0 so that the same bound applies
to the delta product alone, and fp32-output cases held to 1e-5 with the rms taken per
token (fp32 rounding scales with each token's own outputs)."""

import numpy as np
import pytest

import oracle as O
from helpers import APPLY_TOL, assert_apply_close, dev, host
from workloads import (LLAMA3_8B_FUSED, LLAMA3_8B_PROJECTIONS, activations, bf16_bits,
                       random_tenant, tiny_config, weight_pair, zipf_ids)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bd():
    from tenant_serving_b200 import build
    build.build()
    import tenant_serving_b200 as m
    return m


def _table(bd, tenants, layout=0):
    """Device tenant table; layout 1 stores every tenant in the tiled serving layout
    written by bd_prepare_tenant (the oracle always receives the row-major words)."""
    recs = []
    for t in tenants:
        s, sc = dev(t["signs"]), dev(t["scales"])
        if layout == 1:
            d_out, wpr = t["signs"].shape
            s, sc = bd.bd_prepare_tenant(s, sc, t["mode"], t["group_size"], d_out, wpr * 32)
        recs.append((s, sc, t["mode"], t["group_size"], layout))
    return bd.TenantTable(recs, "cuda")


def _run(bd, wb, tenants, ids, x, y_dtype="bf16", w_dtype="bf16", layout=0):
    import torch
    table = _table(bd, tenants, layout)
    y, ws = bd.bd_apply_multi(dev(wb, w_dtype), table, dev(ids), dev(x, w_dtype),
                              y_dtype=torch.bfloat16 if y_dtype == "bf16" else torch.float32)
    rc, flags = bd.bd_get_status(ws)
    yh = host(y)
    yv = O.decode(yh, "bf16") if y_dtype == "bf16" else yh.astype(np.float64)
    return yv, rc, flags


def _problem(seed, d_out, d_in, B, T, modes=(0,), G=128, zero_base=False, ids=None):
    rng = np.random.default_rng(seed)
    wb = bf16_bits(rng.normal(0, 0.02, size=(d_out, d_in)))
    if zero_base:
        wb[:] = 0
    tenants = [random_tenant(rng, d_out, d_in, modes[u % len(modes)], G) for u in range(T)]
    x = activations(rng, B, d_in)
    if ids is None:
        ids = rng.integers(0, T, size=B).astype(np.int32)
    return wb, tenants, np.asarray(ids, dtype=np.int32), x


# -----------------------------------------------------------------------------------
def test_tiny_config_end_to_end(bd):
    """Compress both tenants on the GPU and in the oracle, then apply the 4 fp32 tokens
    (ids [0, 1, 0, 1]); each side uses only its own compress results."""
    import torch
    cfg = tiny_config()
    wb = cfg["w_base"]
    ref_t, gpu_t = [], []
    for wf in cfg["w_fine"]:
        r = O.compress(wb, wf, "f32", O.MODE_GROUP, 128, True, 3.0)
        ref_t.append({"signs": r["signs"], "scales": r["scales"].astype(np.float32),
                      "scale_dtype": "f32", "mode": 0, "group_size": 128})
        c = bd.compress_cfg(mode=0, group_size=128, clip=True, clip_k=3.0)
        s, sc, _ = bd.bd_compress(dev(wb), dev(wf), c)
        gpu_t.append((s, sc, 0, 128))
    y_ref = O.apply_multi(wb, "f32", ref_t, cfg["tenant_ids"], cfg["x"], "f32")
    table = bd.TenantTable(gpu_t, "cuda")
    y, ws = bd.bd_apply_multi(dev(wb), table, dev(cfg["tenant_ids"]), dev(cfg["x"]),
                              y_dtype=torch.float32)
    assert bd.bd_get_status(ws)[0] == bd.BD_OK
    assert_apply_close(host(y), y_ref)
    assert_apply_close(host(y), y_ref, tol=1e-5, per_token=True, what="y (fp32 path, tight)")


@pytest.mark.parametrize("layout", [0, 1])
@pytest.mark.parametrize("B", [1, 4, 16, 63, 200, 300])
@pytest.mark.parametrize("mode", [0, 1, 2, 3, 4])
def test_random_batches(bd, B, mode, layout):
    d_out, d_in = 384 + 8, 1024
    wb, tenants, ids, x = _problem(B * 10 + mode, d_out, d_in, B, 5, (mode,))
    ids[0] = -1  # base only
    y, rc, _ = _run(bd, wb, tenants, ids, x, layout=layout)
    assert rc == bd.BD_OK
    y_ref = O.apply_multi(wb, "bf16", tenants, ids, x, "bf16")
    assert_apply_close(y, y_ref)


@pytest.mark.parametrize("layout", [0, 1])
@pytest.mark.parametrize("mode", [0, 1, 2, 3, 4])
@pytest.mark.parametrize("d_out,d_in", [(1100, 544), (64, 4096), (2050, 256), (130, 96), (600, 640)])
def test_delta_only_tight(bd, mode, d_out, d_in, layout):
    """W_base = 0: the bound now constrains the delta product by itself; with fp32
    outputs it must also hold at 1e-5."""
    G = 32 if d_in % 128 else 128
    wb, tenants, ids, x = _problem(d_out + d_in + mode, d_out, d_in, 9, 3, (mode,), G=G,
                                   zero_base=True)
    y_ref = O.apply_multi(wb, "bf16", tenants, ids, x, "bf16")
    y, rc, _ = _run(bd, wb, tenants, ids, x, y_dtype="f32", layout=layout)
    assert rc == bd.BD_OK
    assert_apply_close(y, y_ref)
    assert_apply_close(y, y_ref, tol=1e-5, per_token=True, what="delta only (fp32 out)")


@pytest.mark.parametrize("layout", [0, 1])
@pytest.mark.parametrize("d_out,d_in", [(600, 8224), (1100, 14336), (520, 4096)])
def test_k_chunks(bd, d_out, d_in, layout):
    """Few (tenant group, 512-row tile) units: the lookup-table kernel cuts each unit
    into K chunks of whole 256-column windows (33 ragged windows into 3 chunks, 56 into 8,
    16 into 8), and the CTA that completes a tile adds the chunks' partial sums. Every
    scale mode, groups of 1-4 tokens and a 6-token tenant (two passes); W_base = 0 and
    fp32 outputs, held to 1e-5 per token as well."""
    G = 32 if d_in % 128 else 128
    ids = np.array([0] * 4 + [1] * 3 + [2] * 2 + [3] + [4] * 6 + [-1] * 2, dtype=np.int32)
    np.random.default_rng(d_in).shuffle(ids)
    wb, tenants, ids, x = _problem(d_out * 3 + d_in, d_out, d_in, len(ids), 5, (0, 1, 2, 3, 4), G=G,
                                   zero_base=True, ids=ids)
    y_ref = O.apply_multi(wb, "bf16", tenants, ids, x, "bf16")
    y, rc, flags = _run(bd, wb, tenants, ids, x, y_dtype="f32", layout=layout)
    assert rc == bd.BD_OK and flags == 0
    assert_apply_close(y, y_ref)
    assert_apply_close(y, y_ref, tol=1e-5, per_token=True, what="delta only (fp32 out)")


@pytest.mark.parametrize("layout", [0, 1])
def test_mixed_modes_and_group_sizes(bd, layout):
    rng = np.random.default_rng(12)
    d_out, d_in = 520, 2048
    wb = bf16_bits(rng.normal(0, 0.02, size=(d_out, d_in)))
    tenants = [random_tenant(rng, d_out, d_in, 0, g) for g in (32, 64, 128, 256, 512, 2048)]
    tenants += [random_tenant(rng, d_out, d_in, m) for m in (1, 2, 3)]
    tenants += [random_tenant(rng, d_out, d_in, 4, g) for g in (32, 64, 128, 512)]
    B = 40
    x = activations(rng, B, d_in)
    ids = rng.integers(-1, len(tenants), size=B).astype(np.int32)
    y, rc, _ = _run(bd, wb, tenants, ids, x, y_dtype="f32", layout=layout)
    assert rc == bd.BD_OK
    assert_apply_close(y, O.apply_multi(wb, "bf16", tenants, ids, x, "bf16"), tol=1e-5, per_token=True)


def test_single_tenant_equals_merged_weight(bd):
    """All tokens of one tenant: y = (W_base + Delta_hat) X, a plain matmul."""
    wb, tenants, _, x = _problem(3, 640, 1024, 48, 1, (0,))
    ids = np.zeros(48, dtype=np.int32)
    y, rc, _ = _run(bd, wb, tenants, ids, x, y_dtype="f32")
    t = tenants[0]
    W = O.reconstruct(t["signs"], O.decode(t["scales"], "f16"), 0, 128, 640, 1024,
                      w_base=O.decode(wb, "bf16"))
    assert_apply_close(y, O.decode(x, "bf16") @ W.T, tol=1e-5, per_token=True)


def test_zero_input_and_permutation(bd):
    wb, tenants, ids, x = _problem(5, 256, 512, 24, 4, (0, 1, 2))
    y0, _, _ = _run(bd, wb, tenants, ids, np.zeros_like(x), y_dtype="f32")
    assert np.all(y0 == 0)
    y, _, _ = _run(bd, wb, tenants, ids, x, y_dtype="f32")
    p = np.random.default_rng(1).permutation(len(ids))
    yp, _, _ = _run(bd, wb, tenants, ids[p], x[p], y_dtype="f32")
    np.testing.assert_array_equal(yp, y[p])  # per-token results do not depend on order


def test_out_of_range_ids_flag_and_base_only(bd):
    wb, tenants, ids, x = _problem(6, 256, 512, 10, 3, (0,))
    ids[2] = 3
    ids[5] = -7
    y, rc, flags = _run(bd, wb, tenants, ids, x, y_dtype="f32")
    assert rc == bd.BD_ERR_TENANT_RANGE and flags & bd.BD_DEV_TENANT_RANGE
    fixed = ids.copy()
    fixed[2] = -1
    fixed[5] = -1
    assert_apply_close(y, O.apply_multi(wb, "bf16", tenants, fixed, x, "bf16"), tol=1e-5, per_token=True)
    # the next good call clears the status word
    _, rc2, flags2 = _run(bd, wb, tenants, fixed, x, y_dtype="f32")
    assert rc2 == bd.BD_OK and flags2 == 0


def test_bad_tenant_record_flag(bd):
    import torch
    wb, tenants, ids, x = _problem(8, 256, 512, 6, 2, (0,))
    ids[:] = [0, 1, 0, 1, 0, 1]
    t0 = tenants[0]
    good = (dev(t0["signs"]), dev(t0["scales"]), 0, 128)
    bad = (dev(tenants[1]["signs"]), dev(tenants[1]["scales"]), 0, 96)  # 96 is not a power of 2
    table = bd.TenantTable([good, bad], "cuda")
    y, ws = bd.bd_apply_multi(dev(wb), table, dev(ids), dev(x), y_dtype=torch.float32)
    rc, flags = bd.bd_get_status(ws)
    assert rc == bd.BD_ERR_TENANT_RECORD and flags & bd.BD_DEV_TENANT_RECORD
    fixed = np.where(ids == 1, -1, ids).astype(np.int32)
    assert_apply_close(host(y), O.apply_multi(wb, "bf16", tenants, fixed, x, "bf16"), tol=1e-5, per_token=True)


def test_tenant_without_tokens_and_many_tenants(bd):
    wb, tenants, _, x = _problem(10, 300, 768, 33, 40, (0, 1, 2, 3))
    ids = np.array([39] * 20 + list(range(13)), dtype=np.int32)  # tenants 13..38 idle
    y, rc, _ = _run(bd, wb, tenants, ids, x)
    assert rc == bd.BD_OK
    assert_apply_close(y, O.apply_multi(wb, "bf16", tenants, ids, x, "bf16"))


def _sampled_rows_check(bd, d_out, d_in, tenants, ids, x, wb, rows, y):
    sub = []
    for t in tenants:
        s = t["scales"]
        if t["mode"] == 0:
            s = s[rows]
        elif t["mode"] == 1:
            s = s[rows]
        sub.append(dict(t, signs=t["signs"][rows], scales=s))
    y_ref = O.apply_multi(wb[rows], "bf16", sub, ids, x, "bf16")
    assert_apply_close(y[:, rows], y_ref)


@pytest.mark.parametrize("layout", [0, 1])
def test_decode_config_up_proj(bd, layout):
    """Decode GEMV at full size: up_proj 14336 x 4096 bf16 base, 64 resident tenants with
    group-128 fp16 scales, 64 tokens, one per tenant (a seeded permutation). Checked on
    256 sampled output rows plus full-tensor properties."""
    rng = np.random.default_rng(2000)
    d_out, d_in, T = 14336, 4096, 64
    wb = bf16_bits(rng.normal(0, 0.02, size=(d_out, d_in)))
    tenants = [random_tenant(rng, d_out, d_in, 0, 128) for _ in range(T)]
    ids = rng.permutation(T).astype(np.int32)
    x = activations(rng, T, d_in)
    y, rc, _ = _run(bd, wb, tenants, ids, x, layout=layout)
    assert rc == bd.BD_OK
    rows = np.sort(rng.choice(d_out, 256, replace=False))
    _sampled_rows_check(bd, d_out, d_in, tenants, ids, x, wb, rows, y)
    assert np.isfinite(y).all()


def test_mixed_config_layer(bd):
    """One Llama-3-8B-shaped layer (7 projections), 32 tenants with per-axis fp16 scales
    (row or column per (tenant, projection) by seed), 256 tokens with Zipf(1.1) ids.
    Sampled rows per projection."""
    rng = np.random.default_rng(3000)
    B, T = 256, 32
    ids = zipf_ids(rng, B, T, 1.1)
    for name, d_out, d_in in LLAMA3_8B_PROJECTIONS:
        wb = bf16_bits(rng.normal(0, 0.02, size=(d_out, d_in)))
        tenants = [random_tenant(rng, d_out, d_in, int(rng.integers(1, 3))) for _ in range(T)]
        x = activations(rng, B, d_in)
        y, rc, _ = _run(bd, wb, tenants, ids, x, layout=1)
        assert rc == bd.BD_OK, name
        rows = np.sort(rng.choice(d_out, 64, replace=False))
        _sampled_rows_check(bd, d_out, d_in, tenants, ids, x, wb, rows, y)


@pytest.mark.parametrize("call", ["qkv", "o", "gate_up", "down"])
def test_serving_config_fused_call(bd, call):
    """The serving bench's launch configuration at full size: one fused call of a layer
    (qkv 6144x4096, o 4096x4096, gate_up 28672x4096, down 4096x14336), bf16 base, 100
    tenants with fp16 group-128 scales in the tiled serving layout, 512 tokens with
    Zipf(1.1) ids (both delta kernels and the split-K base product take part). Checked
    on 64 sampled output rows."""
    shapes = {n: (o, i) for n, o, i in LLAMA3_8B_FUSED}
    d_out, d_in = shapes[call]
    rng = np.random.default_rng(7000 + d_out + d_in)
    B, T = 512, 100
    ids = zipf_ids(rng, B, T, 1.1)
    wb = bf16_bits(rng.normal(0, 0.02, size=(d_out, d_in)))
    tenants = [random_tenant(rng, d_out, d_in, 0, 128) for _ in range(T)]
    x = activations(rng, B, d_in)
    y, rc, flags = _run(bd, wb, tenants, ids, x, layout=1)
    assert rc == bd.BD_OK and flags == 0
    rows = np.sort(rng.choice(d_out, 64, replace=False))
    _sampled_rows_check(bd, d_out, d_in, tenants, ids, x, wb, rows, y)
    assert np.isfinite(y).all()


def test_launches_are_counted(bd):
    n0 = bd.bd_launch_count()
    wb, tenants, ids, x = _problem(1, 128, 256, 4, 2, (0,))
    _run(bd, wb, tenants, ids, x)
    assert bd.bd_launch_count() - n0 == 3  # bucket, base product, lookup-table delta
    # a tenant with at least bd_tc_min_tokens() tokens in the batch takes the tensor-core
    # delta (gather + product): two launches more
    n0 = bd.bd_launch_count()
    wb, tenants, ids, x = _problem(1, 128, 256, 16, 2, (0,))
    _run(bd, wb, tenants, ids, x)
    assert bd.bd_launch_count() - n0 == 5


@pytest.mark.parametrize("d_out,d_in,mode,G", [(1100, 640, 0, 128), (513, 544, 0, 32),
                                               (300, 4096, 1, 128), (70, 256, 2, 128),
                                               (9, 128, 3, 128), (1024, 4096, 0, 128)])
@pytest.mark.parametrize("sdt", ["f16", "f32"])
def test_prepare_tenant_layout(bd, d_out, d_in, mode, G, sdt):
    """bd_prepare_tenant writes exactly the documented tiled layout: tile (rb, w) of
    512 rows x 8 words at word offset (rb * ceil(d_in/256) + w) * 4096, zero padding;
    group-128 scales tiled as [row][2] per tile; other scales copied unchanged."""
    rng = np.random.default_rng(d_out + d_in + mode)
    t = random_tenant(rng, d_out, d_in, mode, G, sdt)
    s_t, sc_t = bd.bd_prepare_tenant(dev(t["signs"]), dev(t["scales"]), mode, G, d_out, d_in)
    got_s, got_sc = host(s_t), host(sc_t)
    nrt, nwin, wpr = -(-d_out // 512), -(-d_in // 256), d_in // 32
    want = np.zeros((nrt, nwin, 512, 8), dtype=np.uint32)
    for rb in range(nrt):
        for w in range(nwin):
            rows = t["signs"][rb * 512:(rb + 1) * 512, w * 8:min((w + 1) * 8, wpr)]
            want[rb, w, :rows.shape[0], :rows.shape[1]] = rows
    np.testing.assert_array_equal(got_s, want.reshape(-1))
    sc = np.asarray(t["scales"])
    if mode == 0 and G == 128:
        ws = np.zeros((nrt, nwin, 512, 2), dtype=sc.dtype)
        for rb in range(nrt):
            for w in range(nwin):
                blk = sc[rb * 512:(rb + 1) * 512, w * 2:min((w + 1) * 2, d_in // 128)]
                ws[rb, w, :blk.shape[0], :blk.shape[1]] = blk
        np.testing.assert_array_equal(got_sc.view(sc.dtype), ws.reshape(-1))
    else:
        np.testing.assert_array_equal(got_sc.view(sc.dtype)[:sc.size], sc.reshape(-1))


# -----------------------------------------------------------------------------------
# tenants with many tokens in the batch: the tensor-core delta product
def _many_token_problem(seed, d_out, d_in, counts, mode, G, zero_base=False, x_scales=True):
    """Tenant u gets counts[u] tokens (shuffled, plus 5 base-only tokens). Some tokens
    are scaled far outside the usual activation range (x 3e4, x 1e-20) and one is all
    zero, so the per-token power-of-two scaling into fp16 is exercised."""
    rng = np.random.default_rng(seed)
    wb = bf16_bits(rng.normal(0, 0.02, size=(d_out, d_in)))
    if zero_base:
        wb[:] = 0
    tenants = [random_tenant(rng, d_out, d_in, mode, G) for _ in counts]
    ids = np.concatenate([np.full(c, u, dtype=np.int32) for u, c in enumerate(counts)] +
                         [np.full(5, -1, dtype=np.int32)])
    rng.shuffle(ids)
    B = len(ids)
    xf = rng.normal(0, 1, size=(B, d_in))
    if x_scales:
        xf[1] *= 3e4
        xf[2] *= 1e-20
        xf[3] = 0
    return wb, tenants, ids, bf16_bits(xf)


@pytest.mark.parametrize("layout", [0, 1])
@pytest.mark.parametrize("mode,G", [(0, 128), (0, 64), (0, 256), (1, 128), (3, 128), (2, 128), (4, 64),
                                    (4, 128)])
def test_many_token_tenants_delta_only(bd, mode, G, layout):
    """300 tokens (five tensor-core segments), 9 (the smallest many-token tenant), 8 (two
    passes of the lookup-table kernel), 20 and 1 token; 200 rows (a partial 128-row tile),
    384 columns (a partial 256-column tile of the serving layout; 768 for groups of 256).
    Column scales (mode 2) in the tiled layout take the tensor-core path with the scales
    folded into the fp16 activations: that product rounds once per element (relative
    2^-11), so its fp32 check is 1e-3 per token instead of 1e-5."""
    d_out, d_in = 200, (768 if G == 256 else 384)
    wb, tenants, ids, x = _many_token_problem(mode * 7 + G + layout, d_out, d_in,
                                              [300, 9, 8, 20, 1], mode, G, zero_base=True)
    y_ref = O.apply_multi(wb, "bf16", tenants, ids, x, "bf16")
    y, rc, flags = _run(bd, wb, tenants, ids, x, y_dtype="f32", layout=layout)
    assert rc == bd.BD_OK and flags == 0
    assert_apply_close(y, y_ref)
    tight = 1e-3 if (mode == 2 and layout == 1) else 1e-5
    assert_apply_close(y, y_ref, tol=tight, per_token=True, what="delta only (fp32 out)")


@pytest.mark.parametrize("layout", [0, 1])
@pytest.mark.parametrize("y_dtype", ["bf16", "f32"])
def test_many_token_tenants_with_base(bd, y_dtype, layout):
    d_out, d_in = 1100, 1024
    wb, tenants, ids, x = _many_token_problem(77 + layout, d_out, d_in, [512, 40, 9, 3, 130], 0, 128)
    y_ref = O.apply_multi(wb, "bf16", tenants, ids, x, "bf16")
    y, rc, flags = _run(bd, wb, tenants, ids, x, y_dtype=y_dtype, layout=layout)
    assert rc == bd.BD_OK and flags == 0
    assert_apply_close(y, y_ref)


def test_many_token_tenant_counts_sweep(bd):
    """Every segment size from 1 to 40 tokens (the tensor-core N from 16 to 48 and the
    switch between the two delta kernels) in one batch."""
    d_out, d_in = 384, 512
    counts = list(range(1, 41))
    wb, tenants, ids, x = _many_token_problem(5, d_out, d_in, counts, 1, 128, zero_base=True,
                                              x_scales=False)
    y_ref = O.apply_multi(wb, "bf16", tenants, ids, x, "bf16")
    y, rc, flags = _run(bd, wb, tenants, ids, x, y_dtype="f32", layout=1)
    assert rc == bd.BD_OK and flags == 0
    assert_apply_close(y, y_ref, tol=1e-5, per_token=True, what="delta only (fp32 out)")


def test_many_token_f32_scales_use_lookup_path(bd):
    """fp32 scales are not exact in fp16: such tenants stay on the lookup-table kernel and
    must still agree at the fp32 bound."""
    d_out, d_in = 256, 512
    rng = np.random.default_rng(9)
    wb = np.zeros((d_out, d_in), dtype=np.uint16)
    tenants = [random_tenant(rng, d_out, d_in, 0, 128, scale_dtype="f32") for _ in range(2)]
    ids = np.array([0] * 40 + [1] * 24, dtype=np.int32)
    x = activations(rng, len(ids), d_in)
    y_ref = O.apply_multi(wb, "bf16", tenants, ids, x, "bf16")
    y, rc, flags = _run(bd, wb, tenants, ids, x, y_dtype="f32")
    assert rc == bd.BD_OK and flags == 0
    assert_apply_close(y, y_ref, tol=1e-5, per_token=True, what="delta only (fp32 out)")


def test_max_batch_many_segments(bd):
    """The largest batch the call accepts (65536 tokens): two tenants in the tiled layout
    with 40000 and 20000 tokens (938 tensor-core segments), one with 5 tokens (lookup
    table) and 5531 base-only tokens, shuffled."""
    import torch
    rng = np.random.default_rng(65536)
    d_out, d_in = 128, 256
    wb = bf16_bits(rng.normal(0, 0.02, size=(d_out, d_in)))
    tenants = [random_tenant(rng, d_out, d_in, 0, 128) for _ in range(3)]
    ids = np.concatenate([np.full(40000, 0), np.full(20000, 1), np.full(5, 2),
                          np.full(65536 - 60005, -1)]).astype(np.int32)
    rng.shuffle(ids)
    x = activations(rng, len(ids), d_in)
    y, rc, flags = _run(bd, wb, tenants, ids, x, y_dtype="f32", layout=1)
    assert rc == bd.BD_OK and flags == 0
    assert_apply_close(y, O.apply_multi(wb, "bf16", tenants, ids, x, "bf16"))


def test_max_tenants(bd):
    """The largest tenant table the call accepts (16384 records, one device buffer of
    sign words and one of scales), 2048 tokens spread over it."""
    import torch
    rng = np.random.default_rng(16384)
    d_out, d_in, T, B = 64, 256, 16384, 2048
    wb = bf16_bits(rng.normal(0, 0.02, size=(d_out, d_in)))
    words = rng.integers(0, 2 ** 32, size=(T, d_out, d_in // 32), dtype=np.uint64).astype(np.uint32)
    z = rng.normal(0.0, 1.0, size=(T, d_out, d_in // 128))
    scales = (0.001 * np.sqrt(2 / np.pi) * np.exp(0.1 * z)).astype(np.float16)
    words_d, scales_d = dev(words), dev(scales)
    recs = [(words_d[u], scales_d[u], 0, 128) for u in range(T)]
    table = bd.TenantTable(recs, "cuda")
    ids = rng.integers(-1, T, size=B).astype(np.int32)
    x = activations(rng, B, d_in)
    y, ws = bd.bd_apply_multi(dev(wb), table, dev(ids), dev(x), y_dtype=torch.float32)
    assert bd.bd_get_status(ws) == (bd.BD_OK, 0)
    used = sorted(set(int(u) for u in ids if u >= 0))
    ref_t = [{"signs": words[u], "scales": scales[u], "scale_dtype": "f16", "mode": 0,
              "group_size": 128} for u in used]
    remap = {u: i for i, u in enumerate(used)}
    ids_ref = np.array([remap[int(u)] if u >= 0 else -1 for u in ids], dtype=np.int32)
    assert_apply_close(host(y), O.apply_multi(wb, "bf16", ref_t, ids_ref, x, "bf16"))
