"""CPU fp64 oracle of the routed MoE SwiGLU layer -- test infrastructure only.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  See ``moe_oracle`` for the functions
and the passages each one follows.
"""

from .moe_oracle import (  # noqa: F401
    LayerResult, Permutation, Selection, dequant_int4_g128, dequant_nvfp4, e2m1_value, e4m3_value, expert_ffn,
    expert_hidden, expert_weights64, moe_forward, moe_partial, override_selection, permute, router_logits,
    select_topk, sigmoid, swiglu_clamped,
)
