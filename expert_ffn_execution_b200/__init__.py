"""B200-native routed-expert FFN layer (libstrata_moe.so + a thin binding).

The C ABI is declared in include/strata_moe.h; `_binding` exposes each call
under the same name.  Build the library with
`python -m expert_ffn_execution_b200.build`.
"""
from ._binding import (DECODE_MAX_T, DEV_BOUNDS, DEV_TIMEOUT, DTYPE_BF16, DTYPE_F16, DTYPE_F32,
                       FMT_Q2_32,
                       FMT_MXFP4_32, FMT_Q4CB_32, QWeights, StrataError, abi_version, exported_symbols, load,
                       moe_bucket, moe_bucket_workspace_size, moe_combine, moe_experts,
                       moe_experts_static_scratch, moe_gather_rows,
                       moe_experts_workspace_size, moe_layer_forward, moe_layer_workspace_size,
                       moe_rmsnorm, moe_route, moe_route_workspace_size, moe_router_topk,
                       moe_router_topk_workspace_size,
                       moe_shared_expert, moe_shared_expert_workspace_size, qweights,
                       status_string, strata_expert_bytes, strata_read_status,
                       strata_selftest_wait)
from .layer import ExpertWeights, MoELayer

__all__ = [n for n in dir() if not n.startswith("_")]
