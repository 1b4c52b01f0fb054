"""B200-native Agent Attention forward pass.

The compute path is the C-ABI library ``libagentattn.so`` (hand-written
sm_100a CUDA kernels), declared in ``include/agent_attn.h``.  ``binding``
marshals arguments to it; nothing here computes the method in Python, and the
package raises if the library is missing.
"""
from .binding import (  # noqa: F401
    AA_BF16,
    AA_FP32,
    AgentAttnError,
    agent_attn_forward,
    agent_attn_forward_agents,
    agent_attn_forward_bias,
    agent_attn_forward_host,
    agent_attn_backward,
    agent_attn_check_device_error,
    agent_attn_dwc,
    agent_attn_forward_dwc,
    agent_attn_forward_ws,
    agent_attn_selftest_exp2,
    agent_attn_stage_pool,
    agent_attn_stage_aggregate,
    agent_attn_stage_aggregate_static,
    agent_attn_stage_broadcast,
    agent_attn_status_string,
    agent_attn_workspace_bytes,
    library_path,
    load_library,
)
