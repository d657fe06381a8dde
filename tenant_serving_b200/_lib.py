"""ctypes binding of libbitdelta.so: argument marshalling only.

Every function here forwards to the C entry point of the same name. PyTorch provides
device memory (``torch.empty`` on the GPU) and the current CUDA stream; all arithmetic of
the method runs in the library's kernels. There is no CPU path: if the library or a GPU
is missing, the calls raise.
"""

from __future__ import annotations

import ctypes
import os
from ctypes import c_double, c_float, c_int32, c_int64, c_size_t, c_uint32, c_void_p, POINTER

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libbitdelta.so")

# status codes (include/bitdelta.h)
BD_OK = 0
BD_ERR_NULL = 1
BD_ERR_SHAPE = 2
BD_ERR_DTYPE = 3
BD_ERR_ALIGN = 4
BD_ERR_CONFIG = 5
BD_ERR_CUDA = 6
BD_ERR_TENANT_RANGE = 7
BD_ERR_TIMEOUT = 8
BD_ERR_WORKSPACE = 9
BD_ERR_TENANT_RECORD = 10
BD_ERR_INTERNAL = 11

BD_F32, BD_BF16, BD_F16 = 0, 1, 2
BD_SCALE_GROUP, BD_SCALE_ROW, BD_SCALE_COL, BD_SCALE_TENSOR, BD_SCALE_BLOCK = 0, 1, 2, 3, 4
BD_DEV_TENANT_RANGE, BD_DEV_TIMEOUT, BD_DEV_TENANT_RECORD, BD_DEV_INTERNAL = 0x1, 0x2, 0x4, 0x8
BD_LAYOUT_ROWMAJOR, BD_LAYOUT_TILED = 0, 1

EXPORTS = (
    "bd_compress", "bd_compress_noalloc", "bd_compress_workspace_size", "bd_reconstruct",
    "bd_apply_multi", "bd_prepared_signs_bytes", "bd_prepared_scales_bytes", "bd_prepare_tenant",
    "bd_apply_workspace_size", "bd_get_status", "bd_status_string", "bd_launch_count",
    "bd_profile_enable", "bd_profile_collect", "bd_kernel_name", "bd_selftest_wait_timeout",
    "bd_tc_min_tokens", "bd_cache_record_bytes", "bd_prepare_record_host", "bd_cache_pool_bytes",
    "bd_cache_staging_bytes", "bd_cache_create", "bd_cache_destroy", "bd_cache_register",
    "bd_cache_table", "bd_cache_slots", "bd_cache_assign", "bd_cache_prefetch", "bd_cache_acquire",
    "bd_cache_release", "bd_cache_resident", "bd_quantize_base_fp8", "bd_apply_fp8_workspace_size",
    "bd_apply_multi_fp8",
)


class bd_compress_cfg(ctypes.Structure):
    _fields_ = [("group_size", c_int32), ("mode", c_int32), ("clip", c_int32), ("clip_k", c_float)]


class bd_tenant(ctypes.Structure):
    _fields_ = [("signs", c_void_p), ("scales", c_void_p), ("mode", c_int32),
                ("group_size", c_int32), ("layout", c_int32), ("reserved", c_int32)]


class bd_cache_module(ctypes.Structure):
    _fields_ = [("d_out", c_int64), ("d_in", c_int64), ("min_group_size", c_int32),
                ("reserved", c_int32)]


class BitDeltaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} (status {code})")


_LIB = None


def lib():
    """Load (once) and return the shared library; raise if it is not built."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libbitdelta.so is not built ({LIB_PATH}); run "
                           "`python -m tenant_serving_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    L.bd_compress.argtypes = [c_void_p, c_void_p, c_int32, c_int64, c_int64,
                              POINTER(bd_compress_cfg), c_void_p, c_void_p, c_void_p, c_void_p,
                              c_size_t, c_void_p]
    L.bd_compress.restype = c_int32
    L.bd_compress_noalloc.argtypes = [c_void_p, c_void_p, c_int32, c_int64, c_int64,
                                      POINTER(bd_compress_cfg), c_void_p, c_void_p, c_void_p,
                                      c_void_p]
    L.bd_compress_noalloc.restype = c_int32
    L.bd_compress_workspace_size.argtypes = [c_int64, c_int64, POINTER(bd_compress_cfg)]
    L.bd_compress_workspace_size.restype = c_size_t
    L.bd_reconstruct.argtypes = [c_void_p, c_void_p, c_int32, c_int32, c_int32, c_int64, c_int64,
                                 c_void_p, c_int32, c_void_p, c_int32, c_void_p]
    L.bd_reconstruct.restype = c_int32
    L.bd_apply_multi.argtypes = [c_void_p, c_int32, c_int64, c_int64, c_void_p, c_int32, c_int32,
                                 c_void_p, c_void_p, c_int64, c_void_p, c_int32, c_void_p,
                                 c_size_t, c_void_p]
    L.bd_apply_multi.restype = c_int32
    L.bd_prepared_signs_bytes.argtypes = [c_int64, c_int64]
    L.bd_prepared_signs_bytes.restype = c_size_t
    L.bd_prepared_scales_bytes.argtypes = [c_int64, c_int64, c_int32, c_int32, c_int32]
    L.bd_prepared_scales_bytes.restype = c_size_t
    L.bd_prepare_tenant.argtypes = [c_void_p, c_void_p, c_int32, c_int32, c_int32, c_int64, c_int64,
                                    c_void_p, c_void_p, c_void_p]
    L.bd_prepare_tenant.restype = c_int32
    L.bd_apply_workspace_size.argtypes = [c_int64, c_int64, c_int64, c_int32]
    L.bd_apply_workspace_size.restype = c_size_t
    L.bd_get_status.argtypes = [c_void_p, POINTER(c_uint32), c_void_p]
    L.bd_get_status.restype = c_int32
    L.bd_status_string.argtypes = [c_int32]
    L.bd_status_string.restype = ctypes.c_char_p
    L.bd_launch_count.argtypes = []
    L.bd_launch_count.restype = c_int64
    L.bd_profile_enable.argtypes = [c_int32, c_int32]
    L.bd_profile_enable.restype = c_int32
    L.bd_profile_collect.argtypes = [POINTER(c_int64), POINTER(c_double), c_int32]
    L.bd_profile_collect.restype = c_int32
    L.bd_kernel_name.argtypes = [c_int32]
    L.bd_kernel_name.restype = ctypes.c_char_p
    L.bd_selftest_wait_timeout.argtypes = [c_void_p, c_size_t, c_int64, c_void_p]
    L.bd_selftest_wait_timeout.restype = c_int32
    L.bd_tc_min_tokens.argtypes = []
    L.bd_tc_min_tokens.restype = c_int32
    L.bd_cache_record_bytes.argtypes = [c_int64, c_int64, c_int32, c_int32, c_int32]
    L.bd_cache_record_bytes.restype = c_size_t
    L.bd_prepare_record_host.argtypes = [c_void_p, c_void_p, c_int32, c_int32, c_int32, c_int64,
                                         c_int64, c_void_p, c_size_t]
    L.bd_prepare_record_host.restype = c_int32
    L.bd_cache_pool_bytes.argtypes = [POINTER(bd_cache_module), c_int32, c_int32, c_int32]
    L.bd_cache_pool_bytes.restype = c_size_t
    L.bd_cache_staging_bytes.argtypes = [c_int32, c_int32]
    L.bd_cache_staging_bytes.restype = c_size_t
    L.bd_cache_create.argtypes = [POINTER(bd_cache_module), c_int32, c_int32, c_int32, c_int32,
                                  c_void_p, c_size_t, c_void_p, c_size_t, POINTER(c_void_p)]
    L.bd_cache_create.restype = c_int32
    L.bd_cache_destroy.argtypes = [c_void_p]
    L.bd_cache_destroy.restype = c_int32
    L.bd_cache_register.argtypes = [c_void_p, c_int32, c_int32, c_void_p, c_int32, c_int32]
    L.bd_cache_register.restype = c_int32
    L.bd_cache_table.argtypes = [c_void_p, c_int32]
    L.bd_cache_table.restype = c_void_p
    L.bd_cache_slots.argtypes = [c_void_p]
    L.bd_cache_slots.restype = c_int32
    L.bd_cache_assign.argtypes = [c_void_p, c_void_p, c_int64, c_void_p, c_void_p,
                                  POINTER(c_int32), POINTER(c_int64)]
    L.bd_cache_assign.restype = c_int32
    L.bd_cache_prefetch.argtypes = [c_void_p, c_void_p, c_int64, c_void_p, POINTER(c_int32),
                                    POINTER(c_int64), c_void_p]
    L.bd_cache_prefetch.restype = c_int32
    L.bd_cache_acquire.argtypes = [c_void_p, c_int64, c_void_p]
    L.bd_cache_acquire.restype = c_int32
    L.bd_cache_release.argtypes = [c_void_p, c_int64, c_void_p]
    L.bd_cache_release.restype = c_int32
    L.bd_cache_resident.argtypes = [c_void_p, c_void_p, c_void_p]
    L.bd_cache_resident.restype = c_int32
    L.bd_quantize_base_fp8.argtypes = [c_void_p, c_int32, c_int64, c_int64, c_void_p, c_void_p, c_void_p]
    L.bd_quantize_base_fp8.restype = c_int32
    L.bd_apply_fp8_workspace_size.argtypes = [c_int64, c_int64, c_int64, c_int32]
    L.bd_apply_fp8_workspace_size.restype = c_size_t
    L.bd_apply_multi_fp8.argtypes = [c_void_p, c_void_p, c_int64, c_int64, c_void_p, c_int32, c_int32,
                                     c_void_p, c_void_p, c_int64, c_void_p, c_int32, c_void_p, c_size_t,
                                     c_void_p]
    L.bd_apply_multi_fp8.restype = c_int32
    _LIB = L
    return L


def status_string(code: int) -> str:
    try:
        return lib().bd_status_string(int(code)).decode()
    except Exception:
        return "unknown"


def check(code: int, where: str):
    if code != BD_OK:
        raise BitDeltaError(code, where)


# ----------------------------------------------------------------------------------
# torch marshalling
# ----------------------------------------------------------------------------------
def _torch():
    import torch
    return torch


def dtype_code(t) -> int:
    torch = _torch()
    m = {torch.float32: BD_F32, torch.bfloat16: BD_BF16, torch.float16: BD_F16}
    if t.dtype not in m:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return m[t.dtype]


def _ptr(t):
    return None if t is None else c_void_p(t.data_ptr())


def _stream(stream):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return c_void_p(s.cuda_stream)


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("tensors passed to the library must live on the GPU")


def compress_cfg(mode=BD_SCALE_GROUP, group_size=128, clip=False, clip_k=3.0) -> bd_compress_cfg:
    return bd_compress_cfg(int(group_size), int(mode), 1 if clip else 0, float(clip_k))


def scales_shape(mode, d_out, d_in, group_size):
    if mode == BD_SCALE_GROUP:
        return (d_out, d_in // group_size)
    if mode == BD_SCALE_ROW:
        return (d_out,)
    if mode == BD_SCALE_COL:
        return (d_in,)
    if mode == BD_SCALE_BLOCK:
        return (-(-d_out // group_size), d_in // group_size)
    return (1,)


def bd_compress_workspace_size(d_out, d_in, cfg: bd_compress_cfg) -> int:
    return int(lib().bd_compress_workspace_size(int(d_out), int(d_in), ctypes.byref(cfg)))


def bd_compress(w_base, w_fine, cfg: bd_compress_cfg, signs=None, scales=None, stats=None,
                workspace=None, stream=None):
    """Wrap ``bd_compress``. Allocates missing outputs with torch on the inputs' device.
    Returns ``(signs int32[d_out, d_in//32] holding the uint32 words, scales fp32,
    stats fp64[4] or None)``."""
    torch = _torch()
    _require_cuda(w_base, w_fine)
    d_out, d_in = w_base.shape
    dev = w_base.device
    if signs is None:
        signs = torch.empty((d_out, d_in // 32), dtype=torch.int32, device=dev)
    if scales is None:
        scales = torch.empty(scales_shape(cfg.mode, d_out, d_in, cfg.group_size),
                             dtype=torch.float32, device=dev)
    if stats is None and cfg.clip:
        stats = torch.zeros(4, dtype=torch.float64, device=dev)
    ws = bd_compress_workspace_size(d_out, d_in, cfg)
    if workspace is None:
        workspace = torch.empty(max(ws, 16), dtype=torch.uint8, device=dev)
    rc = lib().bd_compress(_ptr(w_base), _ptr(w_fine), dtype_code(w_base), d_out, d_in,
                           ctypes.byref(cfg), _ptr(signs), _ptr(scales), _ptr(stats),
                           _ptr(workspace), workspace.numel(), _stream(stream))
    check(rc, "bd_compress")
    return signs, scales, stats


def bd_compress_noalloc(w_base, w_fine, cfg: bd_compress_cfg, signs=None, scales=None,
                        stats=None, stream=None):
    """Wrap ``bd_compress_noalloc``: the library allocates nothing and uses its fixed
    device scratch array (outputs missing here are still allocated by torch)."""
    torch = _torch()
    _require_cuda(w_base, w_fine)
    d_out, d_in = w_base.shape
    dev = w_base.device
    if signs is None:
        signs = torch.empty((d_out, d_in // 32), dtype=torch.int32, device=dev)
    if scales is None:
        scales = torch.empty(scales_shape(cfg.mode, d_out, d_in, cfg.group_size),
                             dtype=torch.float32, device=dev)
    if stats is None and cfg.clip:
        stats = torch.zeros(4, dtype=torch.float64, device=dev)
    rc = lib().bd_compress_noalloc(_ptr(w_base), _ptr(w_fine), dtype_code(w_base), d_out, d_in,
                                   ctypes.byref(cfg), _ptr(signs), _ptr(scales), _ptr(stats),
                                   _stream(stream))
    check(rc, "bd_compress_noalloc")
    return signs, scales, stats


def bd_reconstruct(signs, scales, mode, group_size, d_out, d_in, w_base=None, out=None,
                   out_dtype=None, stream=None):
    torch = _torch()
    _require_cuda(signs, scales, w_base)
    if out is None:
        out = torch.empty((d_out, d_in), dtype=out_dtype or torch.float32, device=signs.device)
    rc = lib().bd_reconstruct(_ptr(signs), _ptr(scales), dtype_code(scales), int(mode),
                              int(group_size), int(d_out), int(d_in), _ptr(w_base),
                              dtype_code(w_base) if w_base is not None else BD_F32, _ptr(out),
                              dtype_code(out), _stream(stream))
    check(rc, "bd_reconstruct")
    return out


def bd_prepare_tenant(signs, scales, mode, group_size, d_out, d_in, stream=None):
    """Wrap ``bd_prepare_tenant``: returns (tiled sign words int32, tiled/plain scales) in
    the serving layout, allocated with torch."""
    torch = _torch()
    _require_cuda(signs, scales)
    sdt = dtype_code(scales)
    nb = int(lib().bd_prepared_signs_bytes(int(d_out), int(d_in)))
    ns = int(lib().bd_prepared_scales_bytes(int(d_out), int(d_in), int(mode), int(group_size), sdt))
    if nb == 0 or ns == 0:
        raise BitDeltaError(BD_ERR_CONFIG, "bd_prepare_tenant")
    so = torch.empty(nb // 4, dtype=torch.int32, device=signs.device)
    sc = torch.empty(ns // scales.element_size(), dtype=scales.dtype, device=signs.device)
    rc = lib().bd_prepare_tenant(_ptr(signs), _ptr(scales), sdt, int(mode), int(group_size),
                                 int(d_out), int(d_in), _ptr(so), _ptr(sc), _stream(stream))
    check(rc, "bd_prepare_tenant")
    return so, sc


class TenantTable:
    """A device array of ``bd_tenant`` records for one projection. Keeps references to
    the tensors it points at so they stay alive as long as the table does. Entries are
    (signs, scales, mode, group_size) or (signs, scales, mode, group_size, layout)."""

    def __init__(self, tenants, device):
        torch = _torch()
        self._keep = []
        n = len(tenants)
        arr = (bd_tenant * max(n, 1))()
        for i, rec in enumerate(tenants):
            signs, scales, mode, group_size = rec[:4]
            layout = rec[4] if len(rec) > 4 else BD_LAYOUT_ROWMAJOR
            _require_cuda(signs, scales)
            arr[i] = bd_tenant(signs.data_ptr(), scales.data_ptr(), int(mode), int(group_size),
                               int(layout), 0)
            self._keep.append((signs, scales))
        raw = bytes(arr)
        self.n = n
        self.scale_dtype = dtype_code(tenants[0][1]) if n else BD_F16
        host = torch.frombuffer(bytearray(raw), dtype=torch.uint8)
        self.dev = host.to(device)

    def ptr(self):
        return c_void_p(self.dev.data_ptr())


def bd_apply_workspace_size(d_out, d_in, batch, n_tenants) -> int:
    return int(lib().bd_apply_workspace_size(int(d_out), int(d_in), int(batch), int(n_tenants)))


def bd_apply_multi(w_base, table: TenantTable, tenant_ids, x, y=None, y_dtype=None,
                   workspace=None, stream=None):
    """Wrap ``bd_apply_multi``: y[t] = W_base x[t] + Delta_hat_{ids[t]} x[t]."""
    torch = _torch()
    _require_cuda(w_base, tenant_ids, x)
    d_out, d_in = w_base.shape
    batch = x.shape[0]
    if y is None:
        y = torch.empty((batch, d_out), dtype=y_dtype or torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = torch.empty(max(bd_apply_workspace_size(d_out, d_in, batch, table.n), 16),
                                dtype=torch.uint8, device=x.device)
    rc = lib().bd_apply_multi(_ptr(w_base), dtype_code(w_base), d_out, d_in, table.ptr(), table.n,
                              table.scale_dtype, _ptr(tenant_ids), _ptr(x), batch, _ptr(y),
                              dtype_code(y), _ptr(workspace), workspace.numel(), _stream(stream))
    check(rc, "bd_apply_multi")
    return y, workspace


def bd_quantize_base_fp8(w, codes=None, scales=None, stream=None):
    """Wrap ``bd_quantize_base_fp8``: (codes uint8 [d_out, d_in], scales fp32 [d_out])."""
    torch = _torch()
    _require_cuda(w)
    d_out, d_in = w.shape
    if codes is None:
        codes = torch.empty((d_out, d_in), dtype=torch.uint8, device=w.device)
    if scales is None:
        scales = torch.empty(d_out, dtype=torch.float32, device=w.device)
    rc = lib().bd_quantize_base_fp8(_ptr(w), dtype_code(w), d_out, d_in, _ptr(codes), _ptr(scales), _stream(stream))
    check(rc, "bd_quantize_base_fp8")
    return codes, scales


def bd_apply_fp8_workspace_size(d_out, d_in, batch, n_tenants) -> int:
    return int(lib().bd_apply_fp8_workspace_size(int(d_out), int(d_in), int(batch), int(n_tenants)))


def bd_apply_multi_fp8(w_codes, w_scales, table, tenant_ids, x, y=None, y_dtype=None, workspace=None,
                       stream=None):
    """Wrap ``bd_apply_multi_fp8``: y[t] = W_hat x[t] + Delta_hat_{ids[t]} x[t], W_hat the
    e4m3 base with per-row scales."""
    torch = _torch()
    _require_cuda(w_codes, w_scales, tenant_ids, x)
    d_out, d_in = w_codes.shape
    batch = x.shape[0]
    if y is None:
        y = torch.empty((batch, d_out), dtype=y_dtype or torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = torch.empty(max(bd_apply_fp8_workspace_size(d_out, d_in, batch, table.n), 16),
                                dtype=torch.uint8, device=x.device)
    rc = lib().bd_apply_multi_fp8(_ptr(w_codes), _ptr(w_scales), d_out, d_in, table.ptr(), table.n,
                                  table.scale_dtype, _ptr(tenant_ids), _ptr(x), batch, _ptr(y), dtype_code(y),
                                  _ptr(workspace), workspace.numel(), _stream(stream))
    check(rc, "bd_apply_multi_fp8")
    return y, workspace


def bd_get_status(workspace, stream=None):
    """Returns (status code, flags). Synchronises the stream."""
    f = c_uint32(0)
    rc = lib().bd_get_status(_ptr(workspace), ctypes.byref(f), _stream(stream))
    return int(rc), int(f.value)


def bd_tc_min_tokens() -> int:
    """The library's many-token threshold (tensor-core delta from this token count on)."""
    return int(lib().bd_tc_min_tokens())


def bd_launch_count() -> int:
    return int(lib().bd_launch_count())


def bd_selftest_wait_timeout(workspace, limit_cycles: int, stream=None) -> int:
    """Wrap ``bd_selftest_wait_timeout``: returns the host status of the launch; the
    device outcome is read with bd_get_status(workspace)."""
    _require_cuda(workspace)
    return int(lib().bd_selftest_wait_timeout(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                              int(limit_cycles), _stream(stream)))


def bd_profile_enable(on: bool, capacity: int = 65536):
    check(lib().bd_profile_enable(1 if on else 0, int(capacity)), "bd_profile_enable")


def bd_profile_collect():
    """{kernel name: (timed launches, total ms)} for kernels launched while enabled."""
    n = 32
    la = (c_int64 * n)()
    ms = (c_double * n)()
    k = lib().bd_profile_collect(la, ms, n)
    out = {}
    for i in range(k):
        if la[i]:
            out[lib().bd_kernel_name(i).decode()] = (int(la[i]), float(ms[i]))
    return out


# ----------------------------------------------------------------------------------
# host-resident tenant cache
# ----------------------------------------------------------------------------------
def bd_cache_record_bytes(d_out, d_in, mode, group_size, scale_dtype=BD_F16) -> int:
    return int(lib().bd_cache_record_bytes(int(d_out), int(d_in), int(mode), int(group_size),
                                           int(scale_dtype)))


def bd_prepare_record_host(signs, scales, mode, group_size, d_out, d_in, out=None, pin=False):
    """Wrap ``bd_prepare_record_host``. signs: host int32/uint32 array [d_out, d_in//32];
    scales: host fp16/fp32 array (plain layout). Returns a host uint8 torch tensor holding
    the packed record (pinned if ``pin``)."""
    import numpy as np
    torch = _torch()
    sg = np.ascontiguousarray(np.asarray(signs).view(np.uint32))
    sc = np.ascontiguousarray(np.asarray(scales))
    sdt = {np.dtype(np.float16): BD_F16, np.dtype(np.float32): BD_F32}.get(sc.dtype)
    if sdt is None:
        raise TypeError(f"unsupported scale dtype {sc.dtype}")
    n = bd_cache_record_bytes(d_out, d_in, mode, group_size, sdt)
    if n == 0:
        raise BitDeltaError(BD_ERR_CONFIG, "bd_prepare_record_host")
    if out is None:
        out = torch.empty(n, dtype=torch.uint8)
        if pin:
            out = out.pin_memory()
    rc = lib().bd_prepare_record_host(sg.ctypes.data, sc.ctypes.data, sdt, int(mode), int(group_size),
                                      int(d_out), int(d_in), c_void_p(out.data_ptr()), out.numel())
    check(rc, "bd_prepare_record_host")
    return out


class CacheTable:
    """The device table of one module of a TenantCache, accepted by bd_apply_multi."""

    def __init__(self, ptr, n, scale_dtype):
        self._p, self.n, self.scale_dtype = ptr, n, scale_dtype

    def ptr(self):
        return c_void_p(self._p)


class TenantCache:
    """Wrap ``bd_cache_*``: modules = [(d_out, d_in, min_group_size)]. The device pool and
    the pinned staging are torch allocations kept by this object. ``device=None`` builds
    the cache over host buffers; only ``assign`` (no CUDA) may be used then."""

    def __init__(self, modules, n_host_tenants, n_slots, scale_dtype=BD_F16, device="cuda"):
        torch = _torch()
        L = lib()
        self.n_modules = len(modules)
        arr = (bd_cache_module * self.n_modules)()
        for i, (d_out, d_in, g) in enumerate(modules):
            arr[i] = bd_cache_module(int(d_out), int(d_in), int(g), 0)
        self._mods = arr
        self.scale_dtype = scale_dtype
        pb = int(L.bd_cache_pool_bytes(arr, self.n_modules, int(n_slots), int(scale_dtype)))
        sb = int(L.bd_cache_staging_bytes(self.n_modules, int(n_slots)))
        if pb == 0 or sb == 0:
            raise BitDeltaError(BD_ERR_SHAPE, "bd_cache_pool_bytes")
        if device is None:
            self.pool = torch.empty(pb + 256, dtype=torch.uint8)
            off = (-self.pool.data_ptr()) % 256
            self.pool = self.pool[off:off + pb]
            self.staging = torch.empty(sb, dtype=torch.uint8)
        else:
            self.pool = torch.empty(pb, dtype=torch.uint8, device=device)
            self.staging = torch.empty(sb, dtype=torch.uint8).pin_memory()
        h = c_void_p()
        rc = L.bd_cache_create(arr, self.n_modules, int(scale_dtype), int(n_host_tenants), int(n_slots),
                               c_void_p(self.pool.data_ptr()), pb, c_void_p(self.staging.data_ptr()), sb,
                               ctypes.byref(h))
        check(rc, "bd_cache_create")
        self._h = h
        self._host_only = device is None
        self.n_slots = int(n_slots)
        self.n_host = int(n_host_tenants)
        self._records = {}

    def register(self, tenant, module, record, mode, group_size):
        rc = lib().bd_cache_register(self._h, int(tenant), int(module), c_void_p(record.data_ptr()),
                                     int(mode), int(group_size))
        check(rc, "bd_cache_register")
        self._records[(int(tenant), int(module))] = record

    def table(self, module) -> CacheTable:
        p = lib().bd_cache_table(self._h, int(module))
        if not p:
            raise BitDeltaError(BD_ERR_SHAPE, "bd_cache_table")
        return CacheTable(p, self.n_slots, self.scale_dtype)

    def assign(self, tenant_ids):
        """Host-only slot assignment: (slot_ids int32 array, [(tenant, slot)] loads, ticket)."""
        import numpy as np
        ids = np.ascontiguousarray(np.asarray(tenant_ids, dtype=np.int32))
        slots = np.empty_like(ids)
        loads = np.empty(2 * self.n_slots, dtype=np.int32)
        n = c_int32(0)
        t = c_int64(-1)
        rc = lib().bd_cache_assign(self._h, ids.ctypes.data, ids.size, slots.ctypes.data, loads.ctypes.data,
                                   ctypes.byref(n), ctypes.byref(t))
        check(rc, "bd_cache_assign")
        return slots, [(int(loads[2 * k]), int(loads[2 * k + 1])) for k in range(n.value)], int(t.value)

    def prefetch(self, tenant_ids, stream=None):
        """Assign + loads on ``stream``: (slot_ids int32 array, number of loads, ticket)."""
        import numpy as np
        ids = np.ascontiguousarray(np.asarray(tenant_ids, dtype=np.int32))
        slots = np.empty_like(ids)
        n = c_int32(0)
        t = c_int64(-1)
        rc = lib().bd_cache_prefetch(self._h, ids.ctypes.data, ids.size, slots.ctypes.data, ctypes.byref(n),
                                     ctypes.byref(t), _stream(stream))
        check(rc, "bd_cache_prefetch")
        return slots, int(n.value), int(t.value)

    def _s(self, stream):
        # a host-only cache never issued a copy: its acquire / release touch no stream
        return c_void_p(None) if self._host_only else _stream(stream)

    def acquire(self, ticket, stream=None):
        check(lib().bd_cache_acquire(self._h, int(ticket), self._s(stream)), "bd_cache_acquire")

    def release(self, ticket, stream=None):
        check(lib().bd_cache_release(self._h, int(ticket), self._s(stream)), "bd_cache_release")

    def resident(self):
        """(tenant per slot, {hits, misses, bytes, copies})."""
        import numpy as np
        st = np.zeros(self.n_slots, dtype=np.int32)
        stats = np.zeros(4, dtype=np.int64)
        check(lib().bd_cache_resident(self._h, st.ctypes.data, stats.ctypes.data), "bd_cache_resident")
        return st.tolist(), dict(zip(("hits", "misses", "bytes", "copies"), stats.tolist()))

    def close(self):
        if getattr(self, "_h", None):
            rc = lib().bd_cache_destroy(self._h)
            self._h = None
            check(rc, "bd_cache_destroy")

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
