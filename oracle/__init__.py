"""fp64 CPU oracle of the DeepSeekMoE layer forward (test infrastructure only).

Only the tests, the package's smoke check and the benchmark's CPU-baseline / reference leg
import this package.  It never imports the CUDA library or its binding.
"""
from .moe_oracle import (  # noqa: F401
    silu, linear, expert_ffn, swiglu_hidden, route, gates_from_indices, permute, layer,
    linear_macs, linear_params, expert_macs, expert_params, hit_entropy, n_routings,
    split_expert, GATE_SOFTMAX_TOPK, GATE_TOPK_SOFTMAX, GATE_SIGMOID_BIAS,
    E4M3_MAX, e4m3_decode, e4m3_round, bf16_round, quantize_rows_e4m3, dequantized_rows, e4m3_weights,
    silu_grad, expert_backward, gate_backward, layer_backward, balance_stats, balance_scores,
)
