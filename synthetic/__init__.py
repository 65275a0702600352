"""Seeded synthetic workloads for the ZAYA1 decoder block.

This package only draws random numbers: shapes, seeds and value
distributions of the workloads, and the tensors drawn from them.  It holds
none of the block's arithmetic, so both the CPU oracle (``oracle/``) and the
CUDA path (``top_moe_block_b200``) can take their inputs from it without
sharing any computation.
"""
from .configs import CONFIGS, BlockConfig, get_config  # noqa: F401
from .gen import (  # noqa: F401
    gen_block_weights,
    gen_prefill_inputs,
    gen_decode_state,
    gen_stack_weights_extra,
    gen_token_ids,
    bf16_values,
)
