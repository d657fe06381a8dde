"""GPU checks of the host-resident tenant cache: the packed host records are the bytes
bd_prepare_tenant writes on the device; batches served through the cache's slots (with
evictions, prefetch one batch ahead on a copy stream) give the fp64 oracle's outputs;
the slots hold exactly the host records of their tenants."""

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


@pytest.mark.parametrize("d_out,d_in,mode,G", [(1100, 640, 0, 128), (513, 544, 0, 32), (300, 4096, 1, 128),
                                               (70, 256, 2, 128), (9, 128, 3, 128)])
def test_host_record_is_the_device_layout(bd, d_out, d_in, mode, G):
    rng = np.random.default_rng(d_out + 3 * d_in + mode)
    t = random_tenant(rng, d_out, d_in, mode, G)
    rec = bd.bd_prepare_record_host(t["signs"], t["scales"], mode, G, d_out, d_in).numpy()
    s_t, sc_t = bd.bd_prepare_tenant(dev(t["signs"]), dev(t["scales"]), mode, G, d_out, d_in)
    sb = host(s_t).view(np.uint8)
    scb = sc_t.cpu().numpy().view(np.uint8)
    assert np.array_equal(rec[:sb.size], sb)
    # tiled group-128 scales are written whole; other modes are copied, and the device
    # buffer's padding past the scales is left as allocated
    n = scb.size if (mode == 0 and G == 128) else np.asarray(t["scales"]).nbytes
    assert np.array_equal(rec[sb.size:sb.size + n], scb[:n])


MODULES = [(1100, 640, 64), (700, 512, 128)]


def _host_tenants(bd, n_host, seed):
    """Per (tenant, module): the tenant (oracle input) and its pinned packed record."""
    rng = np.random.default_rng(seed)
    tenants, records = {}, {}
    for u in range(n_host):
        for m, (d_out, d_in, g) in enumerate(MODULES):
            mode = int(rng.integers(0, 4))
            G = [64, 128][int(rng.integers(0, 2))] if m == 0 else 128
            t = random_tenant(rng, d_out, d_in, mode, G if mode == 0 else 128)
            tenants[(u, m)] = t
            records[(u, m)] = bd.bd_prepare_record_host(t["signs"], t["scales"], mode, t["group_size"],
                                                        d_out, d_in, pin=True)
    return tenants, records


def test_serving_through_the_cache(bd):
    import torch
    n_host, n_slots = 9, 4
    tenants, records = _host_tenants(bd, n_host, 11)
    cache = bd.TenantCache(MODULES, n_host_tenants=n_host, n_slots=n_slots, device="cuda")
    for (u, m), rec in records.items():
        t = tenants[(u, m)]
        cache.register(u, m, rec, t["mode"], t["group_size"])
    rng = np.random.default_rng(12)
    wbs = [bf16_bits(rng.normal(0, 0.02, size=(d_out, d_in))) for d_out, d_in, _ in MODULES]
    # batches of 40 tokens over <= 2 tenants each (one of them often with >= 9 tokens, the
    # tensor-core path), base-only tokens mixed in; consecutive batches share few tenants,
    # so slots are evicted and refilled while the previous batch may still be computing
    batches = []
    for k in range(8):
        us = rng.choice(n_host, size=2, replace=False)
        ids = rng.choice(np.concatenate([us, [-1]]), size=40, p=[0.6, 0.3, 0.1]).astype(np.int32)
        batches.append(ids)
    copy_s = torch.cuda.Stream()
    comp_s = torch.cuda.current_stream()
    ticket_next = cache.prefetch(batches[0], stream=copy_s)
    for k, ids in enumerate(batches):
        slots, n_loads, ticket = ticket_next
        assert n_loads <= 2
        if k + 1 < len(batches):
            # the next batch is loaded while this one computes; the slots this batch holds
            # are not taken (4 slots: 2 held here, 2 free for the next batch's tenants)
            ticket_next = cache.prefetch(batches[k + 1], stream=copy_s)
        cache.acquire(ticket, stream=comp_s)
        slot_dev = dev(slots)
        x = [activations(np.random.default_rng(100 + k * 2 + m), len(ids), d_in)
             for m, (_, d_in, _) in enumerate(MODULES)]
        outs = []
        for m, (d_out, d_in, _) in enumerate(MODULES):
            y, ws = bd.bd_apply_multi(dev(wbs[m]), cache.table(m), slot_dev, dev(x[m]), stream=comp_s)
            outs.append((y, ws))
        cache.release(ticket, stream=comp_s)
        for m, (d_out, d_in, _) in enumerate(MODULES):
            y, ws = outs[m]
            rc, flags = bd.bd_get_status(ws)
            assert rc == bd.BD_OK and flags == 0
            ts = [tenants[(u, m)] for u in range(n_host)]
            y_ref = O.apply_multi(wbs[m], "bf16", ts, ids, x[m], "bf16")
            assert_apply_close(O.decode(host(y), "bf16"), y_ref, what=f"batch {k} module {m}")
    torch.cuda.synchronize()
    # the slots hold exactly the host records of their tenants
    resident, stats = cache.resident()
    assert stats["misses"] >= 8 and stats["hits"] >= 1
    pool = cache.pool.cpu().numpy()
    for s, u in enumerate(resident):
        if u < 0:
            continue
        for m in range(len(MODULES)):
            rec = records[(u, m)].numpy()
            p = cache.table(m).ptr().value
            # the device table's record of slot s points into the pool
            tab = np.frombuffer(pool[p - cache.pool.data_ptr():][:32 * n_slots].tobytes(), dtype=np.uint64)
            signs_addr = int(tab[4 * s])
            off = signs_addr - cache.pool.data_ptr()
            assert np.array_equal(pool[off:off + rec.size], rec)
    cache.close()


def test_prefetch_errors_change_nothing(bd):
    import torch
    n_host, n_slots = 4, 2
    tenants, records = _host_tenants(bd, n_host, 21)
    cache = bd.TenantCache(MODULES, n_host_tenants=n_host, n_slots=n_slots, device="cuda")
    for (u, m), rec in records.items():
        cache.register(u, m, rec, tenants[(u, m)]["mode"], tenants[(u, m)]["group_size"])
    s = torch.cuda.Stream()
    _, _, t0 = cache.prefetch(np.array([0, 1], dtype=np.int32), stream=s)
    before = cache.resident()
    with pytest.raises(bd.BitDeltaError) as e:
        cache.prefetch(np.array([2], dtype=np.int32), stream=s)  # both slots held by t0
    assert e.value.code == bd.BD_ERR_CONFIG
    with pytest.raises(bd.BitDeltaError) as e:
        cache.prefetch(np.array([4], dtype=np.int32), stream=s)
    assert e.value.code == bd.BD_ERR_TENANT_RANGE
    assert cache.resident() == before
    cache.acquire(t0)
    cache.release(t0)
    slots, n, t1 = cache.prefetch(np.array([2, 3], dtype=np.int32), stream=s)
    assert n == 2 and sorted(slots) == [0, 1]
    cache.acquire(t1)
    cache.release(t1)
    torch.cuda.synchronize()
    cache.close()
