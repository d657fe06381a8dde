"""B200-native (sm_100a) BitDelta: compress fine-tune deltas to signs + scales and serve
many tenants that share one base model.

The compute lives in ``libbitdelta.so`` (``include/bitdelta.h``); this package is the thin
ctypes binding plus the in-tree build step.
"""

from ._lib import (  # noqa: F401
    BD_OK, BD_ERR_NULL, BD_ERR_SHAPE, BD_ERR_DTYPE, BD_ERR_ALIGN, BD_ERR_CONFIG, BD_ERR_CUDA,
    BD_ERR_TENANT_RANGE, BD_ERR_TIMEOUT, BD_ERR_WORKSPACE, BD_ERR_TENANT_RECORD, BD_ERR_INTERNAL,
    BD_F32, BD_BF16, BD_F16,
    BD_SCALE_GROUP, BD_SCALE_ROW, BD_SCALE_COL, BD_SCALE_TENSOR, BD_SCALE_BLOCK,
    BD_DEV_TENANT_RANGE, BD_DEV_TIMEOUT, BD_DEV_TENANT_RECORD, BD_DEV_INTERNAL,
    BD_LAYOUT_ROWMAJOR, BD_LAYOUT_TILED, bd_prepare_tenant,
    EXPORTS, LIB_PATH, BitDeltaError, TenantTable, bd_compress_cfg, bd_tenant,
    lib, check, status_string, compress_cfg, scales_shape,
    bd_compress, bd_compress_noalloc, bd_compress_workspace_size, bd_reconstruct, bd_apply_multi,
    bd_apply_workspace_size, bd_get_status, bd_launch_count, bd_profile_enable,
    bd_profile_collect, bd_selftest_wait_timeout, bd_tc_min_tokens,
    bd_cache_module, bd_cache_record_bytes, bd_prepare_record_host, CacheTable, TenantCache,
    bd_quantize_base_fp8, bd_apply_fp8_workspace_size, bd_apply_multi_fp8,
)
