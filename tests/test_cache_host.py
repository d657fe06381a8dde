"""Host-side parts of the tenant cache (no GPU): the packed record layout written by
bd_prepare_record_host, the pool sizing, and the slot assignment (least recently used
eviction, batch holds, error cases) checked against a plain Python model of the policy
the header states."""

import numpy as np
import pytest

from workloads import random_tenant


@pytest.fixture(scope="module")
def bd():
    from tenant_serving_b200 import build
    build.build()
    import tenant_serving_b200 as m
    return m


def _want_record(t, d_out, d_in):
    """The documented record: TILED signs, then TILED (group-128) or plain scales."""
    nrt, nwin, wpr = -(-d_out // 512), -(-d_in // 256), d_in // 32
    want = np.zeros((nrt, nwin, 512, 8), dtype=np.uint32)
    for rb in range(nrt):
        for w in range(nwin):
            blk = t["signs"][rb * 512:(rb + 1) * 512, w * 8:min((w + 1) * 8, wpr)]
            want[rb, w, :blk.shape[0], :blk.shape[1]] = blk
    sc = np.asarray(t["scales"])
    if t["mode"] == 0 and t["group_size"] == 128:
        ws = np.zeros((nrt, nwin, 512, 2), dtype=sc.dtype)
        for rb in range(nrt):
            for w in range(nwin):
                blk = sc[rb * 512:(rb + 1) * 512, w * 2:min((w + 1) * 2, d_in // 128)]
                ws[rb, w, :blk.shape[0], :blk.shape[1]] = blk
        scb = ws.reshape(-1).tobytes()
    else:
        scb = sc.reshape(-1).tobytes()
    return want.reshape(-1).tobytes(), scb


@pytest.mark.parametrize("d_out,d_in,mode,G", [(1100, 640, 0, 128), (513, 544, 0, 32), (300, 4096, 1, 128),
                                               (70, 256, 2, 128), (9, 128, 3, 128), (1024, 512, 0, 64),
                                               (70, 256, 4, 32)])
@pytest.mark.parametrize("sdt", ["f16", "f32"])
def test_record_layout(bd, d_out, d_in, mode, G, sdt):
    rng = np.random.default_rng(d_out * 7 + d_in + mode)
    t = random_tenant(rng, d_out, d_in, mode, G, sdt)
    rec = bd.bd_prepare_record_host(t["signs"], t["scales"], mode, G, d_out, d_in).numpy().tobytes()
    sb, scb = _want_record(t, d_out, d_in)
    assert len(rec) == bd.bd_cache_record_bytes(d_out, d_in, mode, G, bd.BD_F16 if sdt == "f16" else bd.BD_F32)
    assert rec[:len(sb)] == sb
    assert rec[len(sb):len(sb) + len(scb)] == scb
    assert set(rec[len(sb) + len(scb):]) <= {0}  # padding is zero


def test_record_errors(bd):
    rng = np.random.default_rng(0)
    t = random_tenant(rng, 64, 256, 0, 128)
    with pytest.raises(bd.BitDeltaError) as e:
        bd.bd_prepare_record_host(t["signs"], t["scales"], 0, 96, 64, 256)  # not a power of two
    assert e.value.code == bd.BD_ERR_CONFIG
    assert bd.bd_cache_record_bytes(64, 250, 1, 0) == 0  # d_in % 32


def test_pool_holds_the_largest_record_of_every_module(bd):
    mods = [(1100, 640, 32), (4096, 4096, 128), (70, 256, 0)]
    c = bd.TenantCache(mods, n_host_tenants=3, n_slots=2, device=None)
    import torch
    for m, (d_out, d_in, g) in enumerate(mods):
        for mode in range(4):
            if mode == 0 and not g:
                continue  # the module takes no GROUP records
            for G in ([g, 128, d_in] if mode == 0 else [0]):
                if mode == 0 and (d_in % G or G & (G - 1)):
                    continue
                n = bd.bd_cache_record_bytes(d_out, d_in, mode, G, bd.BD_F16)
                assert n > 0
                c.register(0, m, torch.zeros(n, dtype=torch.uint8), mode, G)
    # every record fits its module's region: the slot is at least the sum of the largest
    slot = (c.pool.numel() - 256 * (-(-3 * 2 * 32 // 256))) // 2
    largest = [bd.bd_cache_record_bytes(1100, 640, 0, 32, bd.BD_F16),
               max(bd.bd_cache_record_bytes(4096, 4096, 0, 128, bd.BD_F16),
                   bd.bd_cache_record_bytes(4096, 4096, 1, 0, bd.BD_F16)),
               max(bd.bd_cache_record_bytes(70, 256, md, 0, bd.BD_F16) for md in (1, 2, 3))]
    assert slot >= sum(largest)
    # a GROUP record finer than the module allows is refused
    with pytest.raises(bd.BitDeltaError) as e:
        c.register(1, 2, torch.zeros(1 << 16, dtype=torch.uint8), 0, 128)
    assert e.value.code == bd.BD_ERR_CONFIG
    c.close()


class LruModel:
    """The policy the header states, written out: hits keep their slot; each missing
    tenant takes the free slot (not holding a tenant of this batch, not held by an
    unreleased batch) with the oldest last use, never-used first, lowest index on ties."""

    def __init__(self, n_slots):
        self.slot_tenant = [-1] * n_slots
        self.stamp = [-1] * n_slots
        self.held = {}  # ticket -> set of slots
        self.next = 0

    def assign(self, ids):
        distinct = list(dict.fromkeys(u for u in ids if u != -1))
        where = {u: s for s, u in enumerate(self.slot_tenant) if u >= 0}
        taken = {where[u] for u in distinct if u in where}
        busy = set().union(*self.held.values()) if self.held else set()
        cand = [s for s in range(len(self.slot_tenant)) if s not in taken and s not in busy]
        missing = [u for u in distinct if u not in where]
        if len(cand) < len(missing):
            return None
        cand.sort(key=lambda s: (self.stamp[s], s))
        loads = []
        for u, s in zip(missing, cand):
            old = self.slot_tenant[s]
            if old >= 0:
                where.pop(old, None)
            self.slot_tenant[s] = u
            where[u] = s
            loads.append((u, s))
        t = self.next
        self.next += 1
        for u in distinct:
            self.stamp[where[u]] = t
        self.held[t] = {where[u] for u in distinct}
        return [where[u] if u != -1 else -1 for u in ids], loads, t

    def release(self, t):
        self.held.pop(t)


def _cache_over(bd, n_host, n_slots, mods=((512, 256, 128),)):
    import torch
    c = bd.TenantCache(list(mods), n_host_tenants=n_host, n_slots=n_slots, device=None)
    for u in range(n_host):
        for m, (d_out, d_in, g) in enumerate(mods):
            n = bd.bd_cache_record_bytes(d_out, d_in, 0, g, bd.BD_F16)
            c.register(u, m, torch.zeros(n, dtype=torch.uint8), 0, g)
    return c


def test_assign_follows_lru_with_holds(bd):
    rng = np.random.default_rng(5)
    n_host, n_slots = 12, 5
    c = _cache_over(bd, n_host, n_slots)
    model = LruModel(n_slots)
    open_tickets = []
    for step in range(300):
        pool = rng.choice(n_host, size=int(rng.integers(1, 5)), replace=False)
        ids = [int(u) for u in rng.choice(pool, size=int(rng.integers(1, 9)))]
        if rng.random() < 0.3:
            ids.append(-1)
        if len(open_tickets) >= 4:
            t = open_tickets.pop(0)
            c.release(t)
            model.release(t)
        want = model.assign(ids)  # None (and no change) when the free slots are too few
        if want is None:
            with pytest.raises(bd.BitDeltaError) as e:
                c.assign(ids)
            assert e.value.code == bd.BD_ERR_CONFIG
            t = open_tickets.pop(0)
            c.release(t)
            model.release(t)
            continue
        slots, loads, ticket = c.assign(ids)
        assert ticket == want[2]
        assert list(slots) == want[0]
        assert loads == want[1]
        assert c.resident()[0] == model.slot_tenant
        open_tickets.append(ticket)
        # most batches are released at once, some stay held for a while
        while open_tickets and (len(open_tickets) > 2 or rng.random() < 0.6):
            t = open_tickets.pop(0)
            c.release(t)
            model.release(t)
    st = c.resident()[1]
    assert st["hits"] > 50 and st["misses"] > 50
    c.close()


def test_assign_errors_leave_the_state_unchanged(bd):
    c = _cache_over(bd, 6, 3)
    s0, _, t0 = c.assign([0, 1, 0])
    before = c.resident()
    for ids, code in (([0, 6], bd.BD_ERR_TENANT_RANGE), ([-2], bd.BD_ERR_TENANT_RANGE),
                      ([2, 3, 4], bd.BD_ERR_CONFIG)):  # 0, 1 held: one free slot for three
        with pytest.raises(bd.BitDeltaError) as e:
            c.assign(ids)
        assert e.value.code == code
        assert c.resident() == before
    c.release(t0)
    s, loads, _ = c.assign([2, 3, 4])  # now every slot may be taken, oldest first
    assert sorted(u for u, _ in loads) == [2, 3, 4] and sorted(s) == [0, 1, 2]
    c.close()


def test_unregistered_tenant_is_refused(bd):
    import torch
    c = bd.TenantCache([(512, 256, 128), (256, 512, 128)], n_host_tenants=2, n_slots=2, device=None)
    n = bd.bd_cache_record_bytes(512, 256, 0, 128, bd.BD_F16)
    c.register(0, 0, torch.zeros(n, dtype=torch.uint8), 0, 128)  # module 1 missing
    with pytest.raises(bd.BitDeltaError) as e:
        c.assign([0])
    assert e.value.code == bd.BD_ERR_TENANT_RECORD
    c.close()


def test_four_batches_may_be_held(bd):
    c = _cache_over(bd, 8, 8)
    tickets = [c.assign([u])[2] for u in range(4)]
    with pytest.raises(bd.BitDeltaError) as e:
        c.assign([5])
    assert e.value.code == bd.BD_ERR_CONFIG
    c.release(tickets[1])
    assert c.assign([5])[2] == 4
    with pytest.raises(bd.BitDeltaError):
        c.release(tickets[1])  # released already
    c.close()
