"""Expert parallelism across ranks: partition, weight slicing and the one
all-reduce ("Module glm5next_mlp", §One all-reduce for both EP and TP).

Every rank holds the full router and ranks all E experts, runs only the
routed experts of its own contiguous range (the ranges partition [0, E), as
the page's invariant on local expert ranges states) and its slice of the
shared expert's intermediate dimension (the SwiGLU is per feature, so a slice
is a narrower shared expert whose down projection gives a partial sum).  The
CUDA entry point ``moe_forward_ep`` writes each rank's partial
``shared_r + sum of its local routed slots``; one all-reduce (NCCL over NVLink
under ``torch.distributed``) adds the partials into the layer output.

This module is host-side plumbing only: index arithmetic, tensor slicing and
the collective call.  All layer arithmetic runs in the CUDA library.
"""

from __future__ import annotations

from typing import List, Optional, Tuple

from . import _abi


def expert_ranges(num_experts: int, world: int) -> List[Tuple[int, int]]:
    """Contiguous, balanced [begin, end) expert ranges of the ranks; they
    partition [0, num_experts) (the first num_experts % world ranks hold one
    expert more; ranks past num_experts hold none)."""
    if num_experts < 1 or world < 1:
        raise ValueError("need num_experts >= 1 and world >= 1")
    base, extra = divmod(num_experts, world)
    out, b = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        out.append((b, b + n))
        b += n
    return out


def shared_slices(shared_inter: int, world: int, unit: int = 8) -> List[Tuple[int, int]]:
    """Contiguous [begin, end) slices of the shared expert's intermediate
    dimension, in whole units of `unit` features (16-byte rows), balanced;
    they partition [0, shared_inter)."""
    if shared_inter % unit != 0:
        raise ValueError("shared_inter must be a multiple of the unit")
    units = expert_ranges(shared_inter // unit, world) if shared_inter > 0 else [(0, 0)] * world
    return [(b * unit, e * unit) for b, e in units]


def local_tensors(rank: int, world: int, num_experts: int, shared_inter: int, *, w_gate_up, w_down,
                  s_gate_up=None, s_down=None, shared_w_gate_up=None, shared_w_down=None,
                  g_gate_up=None, g_down=None) -> dict:
    """The weight tensors rank `rank` holds: its experts' rows of the routed
    tensors ([E, ...] -> [E_local, ...]) and its slice of the shared expert
    (gate rows [s0, s1) then up rows [I_s + s0, I_s + s1) of the fused gate/up
    weight; columns [s0, s1) of the down weight).  Router tensors are not
    sliced (every rank ranks every expert)."""
    import torch
    b, e = expert_ranges(num_experts, world)[rank]
    s0, s1 = shared_slices(shared_inter, world)[rank]
    out = {
        "w_gate_up": w_gate_up[b:e].contiguous(),
        "w_down": w_down[b:e].contiguous(),
        "s_gate_up": None if s_gate_up is None else s_gate_up[b:e].contiguous(),
        "s_down": None if s_down is None else s_down[b:e].contiguous(),
        "g_gate_up": None if g_gate_up is None else g_gate_up[b:e].contiguous(),
        "g_down": None if g_down is None else g_down[b:e].contiguous(),
        "shared_w_gate_up": None,
        "shared_w_down": None,
        "expert_range": (b, e),
        "shared_slice": (s0, s1),
    }
    if shared_inter > 0 and s1 > s0:
        out["shared_w_gate_up"] = torch.cat([shared_w_gate_up[s0:s1], shared_w_gate_up[shared_inter + s0:
                                                                                       shared_inter + s1]]).contiguous()
        out["shared_w_down"] = shared_w_down[:, s0:s1].contiguous()
    return out


class ExpertParallelLayer:
    """One rank's share of a routed MoE layer: the full router, its local
    experts and its shared-expert slice, and a workspace.  ``forward`` runs
    ``moe_forward_ep`` and, with a process group, the one all-reduce that
    turns the partial into the layer output on every rank."""

    def __init__(self, *, hidden, num_experts, top_k, expert_inter, shared_inter, swiglu_limit,
                 routed_scaling_factor, renormalize, router_w, correction_bias, w_gate_up, w_down,
                 s_gate_up=None, s_down=None, shared_w_gate_up=None, shared_w_down=None,
                 g_gate_up=None, g_down=None, rank: int = 0, world: int = 1, max_tokens: int = 0,
                 group=None):
        loc = local_tensors(rank, world, num_experts, shared_inter, w_gate_up=w_gate_up, w_down=w_down,
                            s_gate_up=s_gate_up, s_down=s_down, shared_w_gate_up=shared_w_gate_up,
                            shared_w_down=shared_w_down, g_gate_up=g_gate_up, g_down=g_down)
        self.expert_range = loc["expert_range"]
        s0, s1 = loc["shared_slice"]
        fmt = _abi.weight_format(w_gate_up, g_gate_up)
        self.cfg = _abi.make_config(hidden, num_experts, top_k, expert_inter, s1 - s0, swiglu_limit,
                                    routed_scaling_factor, renormalize, fmt)
        st = _abi.moe_config_validate(self.cfg)
        if st != _abi.MOE_OK:
            raise _abi.MoEError(st, "moe_config_validate")
        empty = self.expert_range[1] == self.expert_range[0]
        self.tensors = dict(router_w=router_w, correction_bias=correction_bias,
                            w_gate_up=None if empty else loc["w_gate_up"], w_down=None if empty else loc["w_down"],
                            s_gate_up=None if empty else loc["s_gate_up"], s_down=None if empty else loc["s_down"],
                            g_gate_up=None if empty else loc["g_gate_up"], g_down=None if empty else loc["g_down"],
                            shared_w_gate_up=loc["shared_w_gate_up"], shared_w_down=loc["shared_w_down"])
        self.w = _abi.make_weights(**self.tensors)
        self.device = router_w.device
        self.group = group
        self.ws = None
        self.max_tokens = 0
        if max_tokens:
            self.reserve(max_tokens)

    def reserve(self, max_tokens: int):
        import torch
        if self.ws is not None and max_tokens <= self.max_tokens:
            return
        n = _abi.moe_workspace_size(self.cfg, max_tokens)
        self.ws = torch.empty(max(n, 256), dtype=torch.uint8, device=self.device)
        _abi.moe_workspace_init(self.ws)
        self.max_tokens = max_tokens

    def forward_partial(self, x, out=None, topk_ids=None, topk_w=None, stream=None):
        """This rank's partial sum (no collective)."""
        import torch
        T = x.shape[0]
        self.reserve(T)
        if out is None:
            out = torch.empty(T, self.cfg.hidden, dtype=torch.bfloat16, device=x.device)
        b, e = self.expert_range
        _abi.moe_forward_ep(self.cfg, self.w, b, e, x, T, out, topk_ids, topk_w, self.ws, stream)
        return out

    def forward(self, x, out=None, stream=None):
        """The layer output on every rank: partial, then one all-reduce."""
        out = self.forward_partial(x, out=out, stream=stream)
        if self.group is not None:
            import torch.distributed as dist
            dist.all_reduce(out, op=dist.ReduceOp.SUM, group=self.group)
        return out

    def device_error(self, stream=None) -> int:
        return _abi.moe_read_device_error(self.ws, stream)


def all_reduce_partials(partial, group: Optional[object] = None):
    """Sum `partial` over the ranks of `group` in place (the one collective)."""
    import torch.distributed as dist
    dist.all_reduce(partial, op=dist.ReduceOp.SUM, group=group)
    return partial
