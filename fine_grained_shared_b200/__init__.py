"""B200 (sm_100a) forward pass of a DeepSeekMoE layer behind a small C ABI.

The layer: fine-grained routed experts (mK of mN active per token) plus
always-active shared experts (DeepSeekMoE, arXiv 2401.06066, Abstract).
Every step runs in ``libfgs_moe.so`` (hand-written CUDA for sm_100a); the
Python side in :mod:`fine_grained_shared_b200.moe` only marshals arguments.
"""
from .moe import (  # noqa: F401
    LIB_PATH, MOE_ERR_ALIGNMENT, MOE_ERR_CUDA, MOE_ERR_INVALID_ARG, MOE_ERR_NOMEM, MOE_ERR_SHAPE,
    MOE_ERR_TIMEOUT, MOE_ERR_UNSUPPORTED, MOE_FLAG_DEBUG_WAIT_TIMEOUT, MOE_FLAG_NO_RESIDUAL,
    MOE_FLAG_NO_ROUTED, MOE_FLAG_NO_SHARED, MOE_GATE_SIGMOID_BIASED, MOE_GATE_SOFTMAX, MOE_OK,
    MoEError, MoELayer, lib, moe_config, moe_create, moe_destroy, moe_experts, moe_forward,
    moe_forward_host, moe_get_routing, moe_router, moe_shared, moe_status_query, moe_workspace_bytes, moe_set_timing, moe_kernel_times, moe_update_bias, KERNEL_NAMES,
    status_string, ExpertParallelLayer, connect_emulated, connect_ipc, forward_emulated, nccl_barrier,
    moe_ep_plan,
)
