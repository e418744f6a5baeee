"""CPU oracle of the hybrid MoE feed-forward block (fp64, numpy).

Test infrastructure only: the tests, the package smoke check and the benchmark's
CPU-baseline leg import it; the product path must never route through it.
"""
from .moe_block import *  # noqa: F401,F403
from .moe_block import (Experts, block_forward, bf16, dense_route, dequantize, gated_mlp,
                        gelu_tanh, moe_all_experts_dense, moe_sparse, permute,
                        quantize_int8_per_channel, rms_norm, router, softmax, topk_gaps)
