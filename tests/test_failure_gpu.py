"""Failure detection on the GPU without a fault: a bounded wait that nothing satisfies
gives up, the status word says BD_ERR_TIMEOUT, and the same context keeps working."""

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


def test_wait_runs_out_and_context_stays_usable(bd):
    import torch
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    # ~1 ms at the B200's clock: nothing arrives, so the wait must give up
    assert bd.bd_selftest_wait_timeout(ws, 2_000_000) == bd.BD_OK
    rc, flags = bd.bd_get_status(ws)
    assert rc == bd.BD_ERR_TIMEOUT and flags & bd.BD_DEV_TIMEOUT
    torch.cuda.synchronize()  # the kernel ended; no sticky error on the context

    # the next calls on the same context run and are correct
    rng = np.random.default_rng(5)
    d_out, d_in = 256, 512
    wb = bf16_bits(rng.normal(0, 0.02, size=(d_out, d_in)))
    tenants = [random_tenant(rng, d_out, d_in, 0, 128)]
    ids = np.zeros(16, dtype=np.int32)
    x = activations(rng, 16, d_in)
    table = bd.TenantTable([(dev(t["signs"]), dev(t["scales"]), t["mode"], t["group_size"])
                            for t in tenants], "cuda")
    y, ws2 = bd.bd_apply_multi(dev(wb), table, dev(ids), dev(x), y_dtype=torch.float32)
    assert bd.bd_get_status(ws2)[0] == bd.BD_OK
    assert_apply_close(host(y), O.apply_multi(wb, "bf16", tenants, ids, x, "bf16"))
    # and a fresh self-test call clears the old flag before it sets it again
    assert bd.bd_selftest_wait_timeout(ws, 1000) == bd.BD_OK
    assert bd.bd_get_status(ws)[0] == bd.BD_ERR_TIMEOUT
