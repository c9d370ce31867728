"""CPU fp64 oracle of the fused MoE expert layer (test infrastructure only).

Only the test suite, the package smoke check and the benchmark's CPU-baseline
leg may import this package; the product path never does.
"""
from .moe_oracle import (ACT_RELU2, ACT_SWIGLU, GROUP_MAX, GROUP_TOP2SUM,  # noqa: F401
                         align, backward, backward_values, bf16_to_f64, dequant_mxfp8, e4m3_to_f64,
                         expert_backward_hidden,
                         expert_backward_values, expert_hidden,
                         expert_mlp, forward, forward_values, group_scores, hidden_values, max_padded, route,
                         router_logits, silu, silu_grad)
