"""B200-native fused grouped W4A16 routed-expert MoE layer.

The compute lives in libexactmoe.so (hand-written CUDA for sm_100a behind the
C ABI of include/exactmoe.h). This package is its thin Python binding:
`_native` marshals arguments for the C entry points (same names), `layer`
holds device-buffer plumbing for a whole layer. The library is loaded on first
use of any of these names; if it was not built, that access raises.
"""
from __future__ import annotations

import importlib

_NATIVE_NAMES = {
    "moe_last_error", "moe_abi_version", "moe_launch_counter", "moe_expert_record_layout", "moe_quantize_pack", "moe_route_topk", "moe_route_topk_x16",
    "moe_group_workspace_size", "moe_group_tokens", "moe_group_tokens_noalloc", "MOE_NOALLOC_MAX_PAIRS", "moe_ffn_workspace_size", "moe_grouped_w4a16_ffn",
    "moe_combine", "moe_read_device_error", "moe_debug_stall_next_tc_ffn", "SlotCache", "MoeError",
    "moe_pool_save", "moe_pool_file_info", "moe_pool_load",
    "MOE_RENORM", "MOE_LOGITS_GIVEN", "MOE_IDS_GIVEN", "MOE_PATH_AUTO", "MOE_PATH_GEMV", "MOE_PATH_TC", "MOE_PATH_SEQUENTIAL", "MOE_SLOT_SKIP", "MOE_FFN_X_F16",
    "moe_bf16_record_layout", "moe_bf16_ffn_workspace_size", "moe_grouped_bf16_ffn",
    "MOE_DEVERR_NONE", "MOE_DEVERR_EXPERT_ID", "MOE_DEVERR_NOT_RESIDENT", "MOE_DEVERR_TIMEOUT", "MOE_DEVERR_RANGE",
}
_LAYER_NAMES = {"ExpertBank", "Bf16Bank", "LayerBuffers", "moe_layer_forward"}


def __getattr__(name):
    if name in _NATIVE_NAMES:
        return getattr(importlib.import_module("._native", __name__), name)
    if name in _LAYER_NAMES:
        return getattr(importlib.import_module(".layer", __name__), name)
    raise AttributeError(name)
