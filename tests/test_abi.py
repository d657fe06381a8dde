"""The C-ABI library loads and exports every entry point declared in include/*.h, and the
host-side argument checks answer without touching a GPU (no compute calls here)."""

import ctypes
import glob
import os
import re

import pytest

import tenant_serving_b200 as bd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"\b(bd_[a-z0-9_]+)\s*\(", src):
            names.add(m.group(1))
    return names


@pytest.fixture(scope="module")
def lib():
    from tenant_serving_b200 import build
    build.build()
    return bd.lib()


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert {"bd_compress", "bd_reconstruct", "bd_apply_multi"} <= names
    for n in sorted(names):
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
    # and the binding wraps every one of them by the same name
    assert set(bd.EXPORTS) == names


def test_status_strings(lib):
    for code in range(0, 12):
        s = bd.status_string(code)
        assert s and s != "unknown status"
    assert bd.status_string(999) == "unknown status"


def _cfg(**kw):
    return bd.compress_cfg(**kw)


def test_compress_host_validation(lib):
    fake = ctypes.c_void_p(0x1000)  # never dereferenced: validation fails first
    cfg = _cfg(mode=bd.BD_SCALE_GROUP, group_size=128)
    # bad dtype
    assert lib.bd_compress(fake, fake, 7, 4, 128, ctypes.byref(cfg), fake, fake, None, fake, 1 << 20, None) == bd.BD_ERR_DTYPE
    # d_in not a multiple of 32
    assert lib.bd_compress(fake, fake, bd.BD_BF16, 4, 100, ctypes.byref(cfg), fake, fake, None, fake, 1 << 20, None) == bd.BD_ERR_SHAPE
    # group size not a power of two / not dividing d_in
    for g in (0, 16, 96, 512):
        c = _cfg(mode=bd.BD_SCALE_GROUP, group_size=g)
        assert lib.bd_compress(fake, fake, bd.BD_BF16, 4, 256, ctypes.byref(c), fake, fake, None, fake, 1 << 20, None) == bd.BD_ERR_CONFIG
    # block sizes follow the group rules
    for g in (16, 96, 512):
        c = _cfg(mode=bd.BD_SCALE_BLOCK, group_size=g)
        assert lib.bd_compress(fake, fake, bd.BD_BF16, 4, 256, ctypes.byref(c), fake, fake, None, fake, 1 << 20, None) == bd.BD_ERR_CONFIG
    # bad mode, bad clip flag
    c = bd.bd_compress_cfg(128, 9, 0, 3.0)
    assert lib.bd_compress(fake, fake, bd.BD_BF16, 4, 256, ctypes.byref(c), fake, fake, None, fake, 1 << 20, None) == bd.BD_ERR_CONFIG
    c = bd.bd_compress_cfg(128, 0, 2, 3.0)
    assert lib.bd_compress(fake, fake, bd.BD_BF16, 4, 256, ctypes.byref(c), fake, fake, None, fake, 1 << 20, None) == bd.BD_ERR_CONFIG
    # NULL inputs
    assert lib.bd_compress(None, fake, bd.BD_BF16, 4, 256, ctypes.byref(cfg), fake, fake, None, fake, 1 << 20, None) == bd.BD_ERR_NULL
    # misaligned pointer
    mis = ctypes.c_void_p(0x1004)
    assert lib.bd_compress(mis, fake, bd.BD_BF16, 4, 256, ctypes.byref(cfg), fake, fake, None, fake, 1 << 20, None) == bd.BD_ERR_ALIGN
    # workspace too small (clip needs room for the statistics)
    c = _cfg(mode=bd.BD_SCALE_ROW, clip=True)
    need = lib.bd_compress_workspace_size(4, 256, ctypes.byref(c))
    assert need > 0
    assert lib.bd_compress(fake, fake, bd.BD_BF16, 4, 256, ctypes.byref(c), fake, fake, None, fake, need - 1, None) == bd.BD_ERR_WORKSPACE
    # NULL cfg
    assert lib.bd_compress(fake, fake, bd.BD_BF16, 4, 256, None, fake, fake, None, fake, 1 << 20, None) == bd.BD_ERR_NULL


def test_workspace_sizes(lib):
    cfg = _cfg(mode=bd.BD_SCALE_COL, clip=True)
    a = lib.bd_compress_workspace_size(14336, 4096, ctypes.byref(cfg))
    b = lib.bd_compress_workspace_size(1024, 4096, ctypes.byref(cfg))
    assert a >= b > 0
    assert lib.bd_compress_workspace_size(4, 100, ctypes.byref(cfg)) == 0  # invalid shape
    w1 = lib.bd_apply_workspace_size(14336, 4096, 512, 100)
    w2 = lib.bd_apply_workspace_size(14336, 4096, 64, 100)
    assert w1 > w2 > 0
    # at least the fp32 base partial sums of the batch
    assert w1 >= 512 * 14336 * 4


def test_reconstruct_and_apply_host_validation(lib):
    fake = ctypes.c_void_p(0x1000)
    assert lib.bd_reconstruct(None, fake, bd.BD_F16, 0, 128, 4, 256, None, 0, fake, bd.BD_F32, None) == bd.BD_ERR_NULL
    assert lib.bd_reconstruct(fake, fake, bd.BD_BF16, 0, 128, 4, 256, None, 0, fake, bd.BD_F32, None) == bd.BD_ERR_DTYPE
    assert lib.bd_reconstruct(fake, fake, bd.BD_F16, 0, 100, 4, 256, None, 0, fake, bd.BD_F32, None) == bd.BD_ERR_CONFIG
    assert lib.bd_reconstruct(fake, fake, bd.BD_F16, 0, 128, 4, 200, None, 0, fake, bd.BD_F32, None) == bd.BD_ERR_SHAPE
    ap = lib.bd_apply_multi
    # batch 0 is a no-op
    assert ap(fake, bd.BD_BF16, 8, 256, fake, 1, bd.BD_F16, fake, fake, 0, fake, bd.BD_BF16, fake, 0, None) == bd.BD_OK
    assert ap(fake, 5, 8, 256, fake, 1, bd.BD_F16, fake, fake, 4, fake, bd.BD_BF16, fake, 1 << 30, None) == bd.BD_ERR_DTYPE
    assert ap(fake, bd.BD_BF16, 8, 250, fake, 1, bd.BD_F16, fake, fake, 4, fake, bd.BD_BF16, fake, 1 << 30, None) == bd.BD_ERR_SHAPE
    assert ap(fake, bd.BD_BF16, 8, 256, fake, 20000, bd.BD_F16, fake, fake, 4, fake, bd.BD_BF16, fake, 1 << 30, None) == bd.BD_ERR_SHAPE
    assert ap(fake, bd.BD_BF16, 8, 256, fake, 1, bd.BD_F16, None, fake, 4, fake, bd.BD_BF16, fake, 1 << 30, None) == bd.BD_ERR_NULL
    assert ap(fake, bd.BD_BF16, 8, 256, fake, 1, bd.BD_F16, fake, fake, 4, fake, bd.BD_BF16, fake, 16, None) == bd.BD_ERR_WORKSPACE
    mis = ctypes.c_void_p(0x1008)
    assert ap(fake, bd.BD_BF16, 8, 256, fake, 1, bd.BD_F16, fake, mis, 4, fake, bd.BD_BF16, fake, 1 << 30, None) == bd.BD_ERR_ALIGN


def test_launch_count_starts_at_zero_without_gpu_work(lib):
    assert bd.bd_launch_count() >= 0


def test_selftest_wait_timeout_host_validation(lib):
    fake = ctypes.c_void_p(0x1000)
    st = lib.bd_selftest_wait_timeout
    assert st(None, 256, 1000, None) == bd.BD_ERR_NULL
    assert st(fake, 64, 1000, None) == bd.BD_ERR_WORKSPACE
    assert st(ctypes.c_void_p(0x1008), 256, 1000, None) == bd.BD_ERR_ALIGN
    assert st(fake, 256, 0, None) == bd.BD_ERR_CONFIG
    assert st(fake, 256, 5_000_000_000, None) == bd.BD_ERR_CONFIG


def test_apply_limits(lib):
    fake = ctypes.c_void_p(0x1000)
    ap = lib.bd_apply_multi
    # one past the largest batch and the largest tenant table
    assert ap(fake, bd.BD_BF16, 8, 256, fake, 1, bd.BD_F16, fake, fake, 65537, fake, bd.BD_BF16, fake, 1 << 40, None) == bd.BD_ERR_SHAPE
    assert ap(fake, bd.BD_BF16, 8, 256, fake, 16385, bd.BD_F16, fake, fake, 4, fake, bd.BD_BF16, fake, 1 << 40, None) == bd.BD_ERR_SHAPE
    assert lib.bd_apply_workspace_size(8, 256, 65536, 16384) > 0
