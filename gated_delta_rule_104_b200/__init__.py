"""Gated delta-rule decode step on B200 (sm_100a): eager and DeltaLog-deferred.

The compute path is libdeltalog.so (CUDA kernels behind the C ABI in
include/deltalog.h); this package is its Python binding plus the host-side
schedule driver. PyTorch provides device memory and streams only.
"""
from ._binding import (  # noqa: F401
    DL_BF16, DL_DECAY_CHANNEL, DL_DECAY_HEAD, DL_F32, DL_I8, DL_MAX_LOG, DL_RWKV6, EXPORTS, DeltaLogError, I8State, Log,
    dl_device_faults, dl_gdn_decode_step, dl_index_guard_build, dl_kda_decode_step, dl_log_append_read, dl_log_append_read_noalloc, dl_log_merge,
    dl_log_merge_read, dl_pool_flush, dl_pool_step, dl_rwkv6_decode_step, dl_state_from_i8, dl_state_to_i8,
    dl_status_string, load, Pool,
)
from .schedule import DeferredDecoder  # noqa: F401
