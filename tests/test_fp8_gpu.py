"""GPU parity of the e4m3 base path against the fp64 oracle (oracle.fp8), through the C ABI.

bd_quantize_base_fp8 must give the oracle's codes and scales bit for bit (both take the
fp32 quotients and round them the same way). bd_apply_multi_fp8 is held to the apply
tolerance |y - y_ref| <= 1e-2 * (|y_ref| + rms(y_ref)); the oracle quantizes the base
itself (its codes never come from the GPU) and the GPU path uses its own codes."""

import numpy as np
import pytest

import oracle as O
from helpers import assert_apply_close, dev, host
from workloads import activations, bf16_bits, random_tenant

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bd():
    from tenant_serving_b200 import build
    build.build()
    import tenant_serving_b200 as m
    return m


def _weights(rng, d_out, d_in, dtype):
    w = rng.normal(0, 0.02, size=(d_out, d_in))
    w[min(3, d_out - 1)] = 0.0                                # a zero row
    if d_out > 5:
        w[5] = rng.normal(0, 1e-30, d_in)                      # tiny values (subnormal codes)
        w[4, :7] = [1e-3, -2e-5, 3e-9, 0.0, -0.0, 5e-2, -5e-2]
    return bf16_bits(w) if dtype == "bf16" else w.astype(np.float32)


@pytest.mark.parametrize("d_out,d_in", [(1100, 640), (513, 544), (7, 4096), (128, 32)])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_quantize_is_bit_exact(bd, d_out, d_in, dtype):
    rng = np.random.default_rng(d_out + d_in)
    w = _weights(rng, d_out, d_in, dtype)
    codes, scales = bd.bd_quantize_base_fp8(dev(w, dtype))
    c_ref, s_ref = O.quantize_base(w, dtype)
    got_c = codes.cpu().numpy()
    got_s = scales.cpu().numpy()
    assert np.array_equal(got_s.view(np.uint32), s_ref.view(np.uint32))
    bad = np.argwhere(got_c != c_ref)
    assert bad.size == 0, (bad[:5], got_c[tuple(bad[0])], c_ref[tuple(bad[0])])


def _table(bd, tenants):
    recs = []
    for t in tenants:
        s, sc = dev(t["signs"]), dev(t["scales"])
        d_out, wpr = t["signs"].shape
        s, sc = bd.bd_prepare_tenant(s, sc, t["mode"], t["group_size"], d_out, wpr * 32)
        recs.append((s, sc, t["mode"], t["group_size"], 1))
    return bd.TenantTable(recs, "cuda")


@pytest.mark.parametrize("d_out,d_in,B,counts", [
    (1100, 640, 1, None), (1100, 640, 7, None), (513, 544, 40, None),
    (700, 512, 300, (20, 3, 1, 0, 12)), (256, 1024, 700, None), (130, 4096, 64, (64,))])
def test_apply_fp8_base_matches_oracle(bd, d_out, d_in, B, counts):
    import torch
    rng = np.random.default_rng(7 * d_out + B)
    w = _weights(rng, d_out, d_in, "bf16")
    T = 5
    G = 128 if d_in % 128 == 0 else 32
    tenants = [random_tenant(rng, d_out, d_in, u % 4, G) for u in range(T)]
    if counts is None:
        ids = rng.integers(-1, T, size=B).astype(np.int32)
    else:
        ids = np.concatenate([np.full(c, u, dtype=np.int32) for u, c in enumerate(counts)])
        ids = np.concatenate([ids, np.full(B - len(ids), -1, dtype=np.int32)])
        rng.shuffle(ids)
    x = activations(rng, B, d_in)
    codes, scales = bd.bd_quantize_base_fp8(dev(w))
    y, ws = bd.bd_apply_multi_fp8(codes, scales, _table(bd, tenants), dev(ids), dev(x))
    rc, flags = bd.bd_get_status(ws)
    assert rc == bd.BD_OK and flags == 0
    c_ref, s_ref = O.quantize_base(w, "bf16")
    y_ref = O.apply_multi_fp8(c_ref, s_ref, tenants, ids, x, "bf16")
    assert_apply_close(O.decode(host(y), "bf16"), y_ref)
    # the fp32 output, held to the same bound with the rms of each token
    y32, _ = bd.bd_apply_multi_fp8(codes, scales, _table(bd, tenants), dev(ids), dev(x), y_dtype=torch.float32)
    assert_apply_close(host(y32), y_ref, per_token=True)


def test_every_code_and_extreme_activations(bd):
    """Random codes over all 254 finite patterns (subnormals included) with random row
    scales, given to both sides as inputs; activations whose per-token maxima span 2^-100
    to 2^100 and a zero token exercise the power-of-two limb scaling."""
    rng = np.random.default_rng(9)
    d_out, d_in, B = 300, 768, 24
    codes = rng.integers(0, 256, size=(d_out, d_in), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x01
    scales = (rng.uniform(0.5, 2.0, d_out) * 1e-4).astype(np.float32)
    tenants = [random_tenant(rng, d_out, d_in, m) for m in (0, 1)]
    ids = rng.integers(-1, 2, size=B).astype(np.int32)
    x = O.decode(activations(rng, B, d_in), "bf16")
    x *= (2.0 ** rng.integers(-100, 100, size=B))[:, None]
    x[3] = 0.0
    xb = bf16_bits(x)
    import torch
    y, ws = bd.bd_apply_multi_fp8(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(),
                                  _table(bd, tenants), dev(ids), dev(xb), y_dtype=torch.float32)
    assert bd.bd_get_status(ws)[0] == bd.BD_OK
    y_ref = O.apply_multi_fp8(codes, scales, tenants, ids, xb, "bf16")
    assert_apply_close(host(y), y_ref, per_token=True)
    assert np.all(host(y)[3] == O.apply_multi_fp8(codes, scales, tenants, ids, xb, "bf16")[3])


def test_decode_config_fp8_base_sampled_rows(bd):
    """The decode workload with an e4m3 base: up_proj 14336 x 4096, 64 tenants (fp16
    group-128 scales, tiled), 64 tokens one per tenant; 64 sampled output rows."""
    rng = np.random.default_rng(2000)
    d_out, d_in, T = 14336, 4096, 64
    w = bf16_bits(rng.normal(0, 0.02, size=(d_out, d_in)))
    tenants = [random_tenant(rng, d_out, d_in, 0, 128) for _ in range(T)]
    ids = rng.permutation(T).astype(np.int32)
    x = activations(rng, T, d_in)
    codes, scales = bd.bd_quantize_base_fp8(dev(w))
    y, ws = bd.bd_apply_multi_fp8(codes, scales, _table(bd, tenants), dev(ids), dev(x))
    assert bd.bd_get_status(ws)[0] == bd.BD_OK
    rows = np.sort(rng.choice(d_out, 64, replace=False))
    c_ref, s_ref = O.quantize_base(w[rows], "bf16")  # per-row: the sampled rows alone
    full = np.zeros((d_out, d_in), dtype=np.uint8)
    full_s = np.zeros(d_out, dtype=np.float32)
    full[rows], full_s[rows] = c_ref, s_ref
    y_ref = O.apply_multi_fp8(full, full_s, tenants, ids, x, "bf16", rows=rows)
    assert_apply_close(O.decode(host(y), "bf16")[:, rows], y_ref)


def test_host_errors(bd):
    import torch
    w = torch.zeros((64, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(bd.BitDeltaError) as e:
        bd.bd_quantize_base_fp8(w[:, :80])  # d_in % 32 != 0
    assert e.value.code in (bd.BD_ERR_SHAPE, bd.BD_ERR_ALIGN)
    codes, scales = bd.bd_quantize_base_fp8(w)
    assert int(codes.to(torch.int32).sum()) == 0 and float(scales.abs().sum()) == 0.0
