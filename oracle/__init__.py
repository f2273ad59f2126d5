"""fp64 CPU oracle of the fused MoE layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  The CUDA library and its binding never do.
"""
from .formats import (  # noqa: F401
    E4M3_MAX,
    bf16_bits_to_f64,
    e4m3_code_to_f64,
    e4m3_value_to_code,
    round_to_bf16,
    round_to_e4m3_satfinite,
)
from .moe_ref import (  # noqa: F401
    act_quant_ref,
    align_ref,
    bf16_tolerance_violation,
    decode_weight,
    exact_logit_scaled,
    moe_forward_ref,
    rel_l2,
    route_ref,
    router_logits,
    silu_mul,
)
from .rope_ref import inv_rope_fp8_ref, inv_rope_ref, per_head_fp8_ref  # noqa: F401
