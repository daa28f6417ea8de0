"""Expert parallelism through the C ABI (moe_forward_ep), with the ranks run
one after another on one GPU (no collective on the GPU: the all-reduce of
the ranks' partials is a plain sum here; its host side is tested with gloo
ranks in tests/test_ep_ranks.py).

Each rank holds the full router, its own experts and its slice of the
shared expert ("Module glm5next_mlp", §One all-reduce for both EP and TP).
Checked: every rank selects the same experts; each rank's partial equals
the oracle's partial for its expert range and shared slice; and the sum of
the partials equals the single-rank layer, within the layer tolerance."""

import pytest
import torch

import moe_inputs
import oracle
from moe_inputs.configs import LayerConfig
from routed_swiglu_experts_b200 import ep

from gpu_util import cuda_available, rel_err, tol_for

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]

CASES = {
    # tcgen05 grouped GEMMs, shared expert as an extra problem
    "ep_bf16": LayerConfig("ep_bf16", T=333, H=256, E=8, k=3, I=128, I_s=64, alpha=2.5, renorm=True),
    # few tokens: shared slice on the split-K path
    "ep_bf16_few": LayerConfig("ep_bf16_few", T=20, H=256, E=6, k=2, I=128, I_s=48),
    # W4A16 GEMV with the shared slice inside its launches
    "ep_w4a16_gemv": LayerConfig("ep_w4a16_gemv", T=20, H=256, E=6, k=2, I=128, I_s=128, alpha=2.5, renorm=True,
                                 w4a16=True),
    # W4A16 grouped prefill GEMM
    "ep_w4a16_prefill": LayerConfig("ep_w4a16_prefill", T=300, H=256, E=4, k=2, I=256, I_s=128, w4a16=True),
    # NVFP4 grouped GEMM (tensor scales sliced with the experts); shared slice on
    # the tcgen05 launches, then on the split-K path
    "ep_nvfp4": LayerConfig("ep_nvfp4", T=300, H=256, E=4, k=2, I=256, I_s=128, nvfp4=True),
    "ep_nvfp4_few": LayerConfig("ep_nvfp4_few", T=20, H=256, E=6, k=2, I=128, I_s=128, alpha=2.5, renorm=True,
                                nvfp4=True),
    # more ranks than experts: the last rank has no expert, only a shared slice
    "ep_sparse": LayerConfig("ep_sparse", T=150, H=128, E=3, k=2, I=64, I_s=32),
}
WORLDS = {"ep_bf16": [1, 2, 3, 8], "ep_bf16_few": [2], "ep_w4a16_gemv": [2], "ep_w4a16_prefill": [2],
          "ep_nvfp4": [2], "ep_nvfp4_few": [3], "ep_sparse": [4]}


@pytest.mark.parametrize("name,world", [(n, w) for n in CASES for w in WORLDS[n]])
def test_rank_partials_add_up_to_the_layer(name, world):
    cfg = CASES[name]
    inp = moe_inputs.make_layer(cfg, seed=0)
    dev = torch.device("cuda")
    mv = lambda t: None if t is None else t.to(dev).contiguous()  # noqa: E731
    x = inp.x.to(dev)
    total = torch.zeros(cfg.T, cfg.H, dtype=torch.float32, device=dev)
    ids0 = None
    partials = []
    for r in range(world):
        layer = ep.ExpertParallelLayer(
            hidden=cfg.H, num_experts=cfg.E, top_k=cfg.k, expert_inter=cfg.I, shared_inter=cfg.I_s,
            swiglu_limit=cfg.swiglu_limit, routed_scaling_factor=cfg.alpha, renormalize=cfg.renorm,
            router_w=mv(inp.router_w), correction_bias=mv(inp.correction_bias), w_gate_up=mv(inp.w_gate_up),
            w_down=mv(inp.w_down), s_gate_up=mv(inp.s_gate_up), s_down=mv(inp.s_down),
            shared_w_gate_up=mv(inp.shared_w_gate_up), shared_w_down=mv(inp.shared_w_down),
            g_gate_up=mv(inp.g_gate_up), g_down=mv(inp.g_down),
            rank=r, world=world, max_tokens=cfg.T)
        ids = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=dev)
        part = layer.forward_partial(x, topk_ids=ids)
        torch.cuda.synchronize()
        assert layer.device_error() == 0
        if ids0 is None:
            ids0 = ids.clone()
        assert torch.equal(ids, ids0), f"rank {r} selected other experts"
        total += part.float()
        partials.append((layer.expert_range, ep.shared_slices(cfg.I_s, world)[r], part.cpu()))
    gpu_ids = ids0.cpu().long()
    full = oracle.moe_forward(inp, ids_override=gpu_ids).out
    scale = float(full.abs().max())
    tol = tol_for(cfg)
    err = rel_err(total.cpu(), full)
    assert err <= tol, f"{name} x{world}: sum of partials vs layer {err:.3e}"
    for (b, e), (s0, s1), part in partials:
        want = oracle.moe_partial(inp, b, e, s0, s1, ids_override=gpu_ids)
        perr = float((part.double() - want).abs().max()) / scale
        assert perr <= tol, f"{name} x{world}: rank experts [{b}, {e}) shared [{s0}, {s1}) error {perr:.3e}"


def test_single_rank_partial_is_the_forward():
    """With the whole expert range and the whole shared expert, the EP entry
    point gives moe_forward's bits."""
    import routed_swiglu_experts_b200 as rse
    cfg = CASES["ep_bf16"]
    inp = moe_inputs.make_layer(cfg, seed=0)
    dev = torch.device("cuda")
    mv = lambda t: None if t is None else t.to(dev).contiguous()  # noqa: E731
    kw = dict(hidden=cfg.H, num_experts=cfg.E, top_k=cfg.k, expert_inter=cfg.I, shared_inter=cfg.I_s,
              swiglu_limit=cfg.swiglu_limit, routed_scaling_factor=cfg.alpha, renormalize=cfg.renorm,
              router_w=mv(inp.router_w), correction_bias=mv(inp.correction_bias), w_gate_up=mv(inp.w_gate_up),
              w_down=mv(inp.w_down), shared_w_gate_up=mv(inp.shared_w_gate_up), shared_w_down=mv(inp.shared_w_down),
              max_tokens=cfg.T)
    x = inp.x.to(dev)
    a = ep.ExpertParallelLayer(**kw).forward_partial(x)
    b = rse.MoELayer(**kw).forward(x)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
