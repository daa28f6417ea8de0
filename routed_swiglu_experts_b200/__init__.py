"""B200 (sm_100a) routed Mixture-of-Experts SwiGLU layer forward.

The compute path is the CUDA library ``libmoe_b200.so`` behind the C ABI in
``include/moe.h``; ``_abi`` binds it with ctypes under the same names.
``MoELayer`` below only holds device tensors (torch) and a workspace, and
forwards them to those entry points.  There is no CPU fallback: without the
built library every call raises.
"""

from __future__ import annotations

import math
from typing import Optional

from . import _abi
from ._abi import (  # noqa: F401
    EXPORTED, MOE_ERR_CUDA, MOE_ERR_DEVICE_TIMEOUT, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED,
    MOE_ERR_WORKSPACE, MOE_MAX_EXPERTS, MOE_MAX_TOP_K, MOE_OK, MOE_W_BF16, MOE_W_INT4_G128, MOE_W_NVFP4, MoEError,
    load_library, make_config, make_weights, moe_combine, moe_config, moe_config_validate, moe_forward,
    moe_grouped_swiglu_ffn, moe_grouped_swiglu_ffn_gather, moe_permute, moe_read_device_error, moe_router_topk,
    moe_weights,
    moe_workspace_init, moe_workspace_size, status_name,
)

__all__ = ["MoELayer", "load_library", "moe_forward", "moe_router_topk", "moe_permute",
           "moe_grouped_swiglu_ffn", "moe_grouped_swiglu_ffn_gather", "moe_combine", "moe_workspace_size", "MoEError"]


class MoELayer:
    """Device-resident weights + workspace of one routed MoE layer.

    Tensors (torch, CUDA, contiguous): router_w fp32 [E, H]; correction_bias
    fp32 [E] or None; w_gate_up bf16 [E, 2I, H] (or uint8 [E, 2I, H/2] with
    s_gate_up bf16 [E, 2I, H/128]); w_down bf16 [E, H, I] (or uint8
    [E, H, I/2] with s_down bf16 [E, H, I/128]); shared_w_gate_up bf16
    [2I_s, H] and shared_w_down bf16 [H, I_s] (None when I_s == 0).
    NVFP4 experts: uint8 E2M1 codes as above, s_gate_up / s_down uint8 E4M3
    scales [E, 2I, H/16] / [E, H, I/16], and g_gate_up / g_down fp32 [E]
    tensor scales (their presence selects the format)."""

    def __init__(self, *, hidden, num_experts, top_k, expert_inter, shared_inter, swiglu_limit,
                 routed_scaling_factor, renormalize, router_w, correction_bias, w_gate_up, w_down,
                 s_gate_up=None, s_down=None, shared_w_gate_up=None, shared_w_down=None,
                 g_gate_up=None, g_down=None, max_tokens: int = 0):
        fmt = _abi.weight_format(w_gate_up, g_gate_up)
        self.cfg = make_config(hidden, num_experts, top_k, expert_inter, shared_inter, swiglu_limit,
                               routed_scaling_factor, renormalize, fmt)
        st = moe_config_validate(self.cfg)
        if st != MOE_OK:
            raise MoEError(st, "moe_config_validate")
        self.tensors = dict(router_w=router_w, correction_bias=correction_bias, w_gate_up=w_gate_up,
                            s_gate_up=s_gate_up, w_down=w_down, s_down=s_down,
                            shared_w_gate_up=shared_w_gate_up, shared_w_down=shared_w_down,
                            g_gate_up=g_gate_up, g_down=g_down)
        self.w = make_weights(**self.tensors)
        self.device = router_w.device
        self.ws = None
        self.max_tokens = 0
        if max_tokens:
            self.reserve(max_tokens)

    @property
    def H(self):
        return self.cfg.hidden

    @property
    def k(self):
        return self.cfg.top_k

    def reserve(self, max_tokens: int):
        """Allocate (torch) a workspace big enough for ``max_tokens``."""
        import torch
        if self.ws is not None and max_tokens <= self.max_tokens:
            return
        n = moe_workspace_size(self.cfg, max_tokens)
        self.ws = torch.empty(max(n, 256), dtype=torch.uint8, device=self.device)
        moe_workspace_init(self.ws)
        self.max_tokens = max_tokens

    def forward(self, x, out=None, topk_ids=None, topk_w=None, stream=None):
        import torch
        T = x.shape[0]
        self.reserve(T)
        if out is None:
            out = torch.empty(T, self.H, dtype=torch.bfloat16, device=x.device)
        moe_forward(self.cfg, self.w, x, T, out, topk_ids, topk_w, self.ws, stream)
        return out

    def device_error(self, stream=None) -> int:
        return moe_read_device_error(self.ws, stream)
