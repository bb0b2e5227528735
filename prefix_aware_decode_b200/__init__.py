"""Prefix-aware batched decode attention for B200 (sm_100a).

Pack (host planner), forward and merge (sm_100a kernels) behind the C ABI of
include/pa.h; this package is the thin Python binding over it.
"""
from ._binding import (PA_ERR_CUDA, PA_ERR_DEVICE, PA_ERR_INVALID, PA_ERR_NOMEM, PA_ERR_TIMEOUT,  # noqa: F401
                       PA_ERR_UNSUPPORTED, PA_OK, PA_PLAN_ALWAYS_SHARE, PA_PLAN_DEBUG_CHECKS,
                       PA_PLAN_FAULT_DROP_LOAD, PA_PLAN_KEEP_PACK, PA_PLAN_NO_SHARING, DecodeStep, PaError, PaImageHeader, Plan, attend, merge_rows,
                       lib)
