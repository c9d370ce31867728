"""B200 (sm_100a) fused Mixture-of-Experts expert layer.

The computation lives in the CUDA library ``libmoe_b200.so`` behind the C
ABI of ``include/moe.h``; :mod:`grouped_gemm_gating_b200.moe` is its Python
binding (argument marshalling only) and
:mod:`grouped_gemm_gating_b200.workloads` draws the seeded synthetic inputs.
"""
from .moe import (ACT_RELU2, ACT_SWIGLU, GROUP_MAX, GROUP_TOP2SUM, MoEBuffers,  # noqa: F401
                  MoEError, load_library, moe_align, moe_align_workspace_size, moe_forward,
                  moe_max_padded, moe_read_status, moe_route, moe_workspace_size)
