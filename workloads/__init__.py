"""Seeded synthetic workloads for one EAGLE tree-verification step.

This package only draws random numbers and encodes them (fp32 -> bf16 bits).
It holds none of the method's arithmetic: no softmax, no top-k, no tree
expansion, no attention, no acceptance.  Both the CPU oracle (through the
tests) and the CUDA path consume what it produces; it imports neither.
"""
from .configs import CONFIGS, Config, get_config  # noqa: F401
from .gen import (  # noqa: F401
    Workload,
    bf16_bits_from_f32,
    f32_from_bf16_bits,
    make_workload,
    make_target_logits,
    draft_rows_count,
    gen_attention_inputs,
    gen_draft_logits,
    gen_prefix_len,
    gen_uniforms,
    stored_to_f32,
)
