"""ReLU linear attention with 3D RoPE for video DiTs, on B200 (sm_100a).

The op (SANA-Video paper-graph page, section 3.4, Eq. 2):
    out_i = RoPE(phi(q_i)) S / (phi(q_i) . z + eps),  phi = ReLU,
    S = sum_j RoPE(phi(k_j))^T v_j,  z = sum_j phi(k_j),
optionally times sigmoid(gate), bidirectional or block-causal with a carried
constant-memory state (S, z) ("Block Linear Attention with Constant-Memory KV
Cache", Eq. 3, Algorithm 1).

The computation is the C-ABI CUDA library ``liblinattn.so`` (include/linattn.h);
``_native`` binds it with the same names and ``api`` wraps it for torch tensors.
"""
from . import _native
from .api import (BlockState, Workspace, cross_forward, forward, make_params, temporal_conv,
                  uses_tensor_cores, workspace_for)

__all__ = ["BlockState", "Workspace", "cross_forward", "forward", "make_params", "temporal_conv",
           "uses_tensor_cores", "workspace_for", "_native"]
