"""bd_compress_noalloc: the entry point for callers that cannot allocate device memory
(for example code inside a runtime that owns all GPU memory, or a loop that must not
pay for an allocation). It runs the same kernels as bd_compress with scratch taken from
a fixed array inside the library, so its results must match bd_compress's exactly.

This file is collected last on purpose: a failure here leaves every other test run."""

import ctypes

import numpy as np
import pytest

from helpers import SCALE_RTOL, assert_scales_close, dev, host
from workloads import weight_pair

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bd():
    from tenant_serving_b200 import build
    build.build()
    import tenant_serving_b200 as m
    return m


CASES = [
    # (seed, d_out, d_in, dtype, mode, group, clip)
    (11, 1024, 4096, "bf16", 0, 128, True),   # group scales, 3-sigma clip
    (12, 300, 4096 + 96, "f32", 1, 128, True),  # row scales use the scratch partials
]


@pytest.mark.parametrize("case", CASES)
def test_noalloc_matches_workspace_version_twice(bd, case):
    seed, d_out, d_in, dtype, mode, G, clip = case
    cfg = bd.compress_cfg(mode=mode, group_size=G, clip=clip, clip_k=3.0)
    # two calls in a row on different inputs: the second must not see the first's data
    for call in range(2):
        wb, wf = weight_pair(seed + 100 * call, d_out, d_in, dtype, 0.02, 0.002, 0.001, 20.0)
        a = bd.bd_compress(dev(wb, dtype), dev(wf, dtype), cfg)
        b = bd.bd_compress_noalloc(dev(wb, dtype), dev(wf, dtype), cfg)
        np.testing.assert_array_equal(host(b[0]), host(a[0]))
        assert_scales_close(host(b[1]), host(a[1]), rtol=SCALE_RTOL)
        if clip:
            np.testing.assert_allclose(host(b[2]), host(a[2]), rtol=1e-12, atol=0)


def test_noalloc_rejects_scratch_beyond_maximum(bd):
    import torch
    # column scales of a 14336 x 4096 matrix need far more than the fixed scratch
    cfg = bd.compress_cfg(mode=bd.BD_SCALE_COL, clip=True)
    assert bd.bd_compress_workspace_size(14336, 4096, cfg) > (1 << 20)
    wb = torch.zeros((14336, 4096), dtype=torch.bfloat16, device="cuda")
    signs = torch.empty((14336, 128), dtype=torch.int32, device="cuda")
    scales = torch.empty(4096, dtype=torch.float32, device="cuda")
    rc = bd.lib().bd_compress_noalloc(ctypes.c_void_p(wb.data_ptr()), ctypes.c_void_p(wb.data_ptr()),
                                      bd.BD_BF16, 14336, 4096, ctypes.byref(cfg),
                                      ctypes.c_void_p(signs.data_ptr()),
                                      ctypes.c_void_p(scales.data_ptr()), None, None)
    assert rc == bd.BD_ERR_WORKSPACE
