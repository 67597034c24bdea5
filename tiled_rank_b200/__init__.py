"""TileQ fused MoE-layer forward for NVIDIA B200 (sm_100a).

The computation lives in libtileq.so (C ABI, include/tileq.h); this package is
its thin ctypes binding plus a helper that keeps a layer's device tensors.
"""
from ._lib import (  # noqa: F401
    TILEQ_LINEAR, TILEQ_SWIGLU, TILEQ_ROUTE_FULL_SOFTMAX, TILEQ_ROUTE_TOPK_SOFTMAX, TileQError,
    TILEQ_ERR_TIMEOUT, TILEQ_ERR_RANGE,
    status_string, tileq_device_status,
    tileq_moe_forward, tileq_moe_forward_unfused, tileq_pack, tileq_pack_per_expert,
    tileq_packed_per_expert_size, tileq_packed_size, tileq_route, tileq_route_static,
    tileq_selftest_bounded_wait,
    tileq_workspace_size, tileq_set_stage_events, tileq_launch_count,
    tileq_wbig, tileq_sketch_workspace_size, tileq_sketch_lowrank,
    tileq_place_in, tileq_place_out, place_in, tileq_place_workspace_size, tileq_place_experts,
)
from .layer import DeviceLayer  # noqa: F401
