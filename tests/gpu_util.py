"""Helpers for the GPU tests: move seeded inputs to the device, run the C-ABI
stages, and compare against the oracle with the stated tolerances."""

from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional

import torch

import routed_swiglu_experts_b200 as rse

# Layer-output tolerance: max|gpu - oracle| <= TOL * max|oracle| over the
# compared rows (bf16 weights), doubled for 4-bit (W4A16, NVFP4) weights:
# their kernels run on fp16 activations.
TOL_BF16 = 2e-2
TOL_W4A16 = 4e-2
# Near-tie exemption on the oracle's k-th vs (k+1)-th biased-score gap.
TIE_GAP = 1e-6


def cuda_available() -> bool:
    return torch.cuda.is_available()


def gpu_layer(inp, max_tokens: Optional[int] = None) -> rse.MoELayer:
    c = inp.cfg
    dev = torch.device("cuda")

    def mv(t):
        return None if t is None else t.to(dev).contiguous()
    return rse.MoELayer(
        hidden=c.H, num_experts=c.E, top_k=c.k, expert_inter=c.I, shared_inter=c.I_s,
        swiglu_limit=c.swiglu_limit, routed_scaling_factor=c.alpha, renormalize=c.renorm,
        router_w=mv(inp.router_w), correction_bias=mv(inp.correction_bias), w_gate_up=mv(inp.w_gate_up),
        w_down=mv(inp.w_down), s_gate_up=mv(inp.s_gate_up), s_down=mv(inp.s_down),
        shared_w_gate_up=mv(inp.shared_w_gate_up), shared_w_down=mv(inp.shared_w_down),
        g_gate_up=mv(inp.g_gate_up), g_down=mv(inp.g_down),
        max_tokens=max_tokens if max_tokens is not None else inp.x.shape[0])


@dataclass
class StageOut:
    ids: torch.Tensor
    topk_w: torch.Tensor
    offsets: torch.Tensor
    row_of: torch.Tensor
    src: torch.Tensor
    w_perm: torch.Tensor
    x_perm: torch.Tensor
    y_perm: torch.Tensor
    shared_out: Optional[torch.Tensor]
    out: torch.Tensor
    # the fused-gather variant: maps-only permute, then the FFN reading x
    maps: tuple = ()
    y_perm_g: Optional[torch.Tensor] = None
    shared_out_g: Optional[torch.Tensor] = None


def run_stages(layer: rse.MoELayer, x: torch.Tensor) -> StageOut:
    """router -> permute -> grouped FFN (+ shared) -> combine, one C-ABI call
    each; then the maps-only permute and the gathered FFN on the same ids."""
    cfg = layer.cfg
    T, H, E, k = x.shape[0], cfg.hidden, cfg.num_experts, cfg.top_k
    R = T * k
    dev = x.device
    layer.reserve(T)
    i32, f32, bf = torch.int32, torch.float32, torch.bfloat16
    ids = torch.empty(T, k, dtype=i32, device=dev)
    tw = torch.empty(T, k, dtype=f32, device=dev)
    rse.moe_router_topk(cfg, layer.w, x, T, ids, tw, layer.ws)
    offsets = torch.empty(E + 1, dtype=i32, device=dev)
    row_of = torch.empty(R, dtype=i32, device=dev)
    src = torch.empty(R, dtype=i32, device=dev)
    w_perm = torch.empty(R, dtype=f32, device=dev)
    x_perm = torch.empty(R, H, dtype=bf, device=dev)
    rse.moe_permute(cfg, ids, tw, x, T, offsets, row_of, src, w_perm, x_perm, layer.ws)
    y_perm = torch.empty(R, H, dtype=bf, device=dev)
    shared_out = torch.empty(T, H, dtype=bf, device=dev) if cfg.shared_inter > 0 else None
    rse.moe_grouped_swiglu_ffn(cfg, layer.w, x_perm, offsets, w_perm, T, y_perm,
                               x if cfg.shared_inter > 0 else None, shared_out, layer.ws)
    out = torch.empty(T, H, dtype=bf, device=dev)
    rse.moe_combine(cfg, y_perm, row_of, None, shared_out, T, out)
    maps = tuple(torch.full_like(a, -7) if a.dtype == i32 else torch.full_like(a, -7.0)
                 for a in (offsets, row_of, src, w_perm))
    rse.moe_permute(cfg, ids, tw, None, T, *maps, None, layer.ws)
    y_perm_g = torch.empty(R, H, dtype=bf, device=dev)
    shared_out_g = torch.empty(T, H, dtype=bf, device=dev) if cfg.shared_inter > 0 else None
    rse.moe_grouped_swiglu_ffn_gather(cfg, layer.w, x, T, maps[2], maps[0], maps[3], y_perm_g, shared_out_g, layer.ws)
    torch.cuda.synchronize()
    return StageOut(ids, tw, offsets, row_of, src, w_perm, x_perm, y_perm, shared_out, out, maps, y_perm_g,
                    shared_out_g)


def rel_err(got: torch.Tensor, want: torch.Tensor) -> float:
    """max|got - want| / max|want| (fp64, CPU)."""
    g = got.detach().to("cpu", torch.float64)
    w = want.detach().to("cpu", torch.float64)
    denom = float(w.abs().max())
    if denom == 0.0:
        return float((g - w).abs().max())
    return float((g - w).abs().max()) / denom


def check_ids(gpu_ids: torch.Tensor, sel, tie_gap: float = TIE_GAP):
    """Ids bit-exact except for tokens whose oracle gap is below tie_gap.
    Returns (near_tie_count, mismatches_among_near_ties)."""
    g = gpu_ids.detach().cpu().to(torch.int64)
    o = sel.ids
    mism = (g != o).any(dim=1)
    exempt = sel.gap < tie_gap
    bad = mism & ~exempt
    assert not bool(bad.any()), f"{int(bad.sum())} tokens select different experts, e.g. {bad.nonzero()[:5].flatten().tolist()}"
    # every emitted id list is still a valid selection: distinct, in range
    E = sel.scores.shape[1]
    assert int(g.min()) >= 0 and int(g.max()) < E
    srt = torch.sort(g, dim=1).values
    assert bool((srt[:, 1:] != srt[:, :-1]).all()) if g.shape[1] > 1 else True
    return int(exempt.sum()), int((mism & exempt).sum())


def tol_for(cfg) -> float:
    return TOL_W4A16 if (cfg.w4a16 or cfg.nvfp4) else TOL_BF16
