"""ISPA hot path on NVIDIA B200 (sm_100a): decomposable dual-stream attention, warmup statistics and
the closed-form ridge absorb, behind the C ABI of include/ispa.h (libispa.so, built in-tree)."""
from .ispa import (  # noqa: F401
    AttnArgs, IspaError, LIB_PATH, SYMBOLS, TempCache, absorb, absorb_static, absorb_workspace_size, accum_stats, dual_stream_attn,
    get_device_status, launch_count, lib, project, project_w8a8, quantize_e4m3, select_layers, status_string,
    test_set_flags, version,
)
