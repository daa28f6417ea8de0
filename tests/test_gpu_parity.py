"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Small layers (spanning several tiles, ragged tails, empty experts, one hot
expert, exact router ties, the largest supported E and k) are compared in
full at every stage.  The benchmark layers are compared at full size:
router ids for every token, the permutation for every slot, and the layer
output, the shared-expert output and every routed row of the compared
tokens: all tokens of the mid and decode layers, and on the larger layers a
sample of at least 1024 tokens chosen per token tile (the first and last
rows of every tile of every expert, and the rows where a tile's two CTA
halves meet).  The maps-only permute and the grouped FFN with the gather
fused into its loads are compared bit for bit with the x_perm path on every
layer.  Near-tie counts go into every assertion message and the test's
printed line.

Bars: expert ids and permutation indices bit-exact (router ids exempt only
where the oracle's k-th vs (k+1)-th biased-score gap is below 1e-6; those
are counted); routed weights within 1e-5 relative; outputs within
max|gpu - oracle| <= 2e-2 * max|oracle| (bf16 weights) or 4e-2 (W4A16 and
NVFP4 weights).
"""

import math

import pytest
import torch

import moe_inputs
from moe_inputs.configs import CONFIGS, LayerConfig
import oracle
from gpu_util import check_ids, gpu_layer, rel_err, run_stages, tol_for

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    torch.cuda.init()


EDGE = {
    "tiny": CONFIGS["tiny"],
    "ragged": LayerConfig("ragged", T=333, H=200, E=5, k=3, I=72, I_s=40, alpha=1.7, renorm=True),
    "clamp_small": LayerConfig("clamp_small", T=257, H=256, E=8, k=2, I=128, I_s=128, swiglu_limit=0.5),
    "no_clamp": LayerConfig("no_clamp", T=190, H=192, E=6, k=2, I=136, I_s=64, swiglu_limit=math.inf),
    "one_token": LayerConfig("one_token", T=1, H=512, E=16, k=4, I=256, I_s=256, alpha=2.5, renorm=True),
    "no_shared": LayerConfig("no_shared", T=200, H=256, E=8, k=2, I=192, I_s=0),
    "k_equals_e": LayerConfig("k_equals_e", T=100, H=128, E=4, k=4, I=64, I_s=64),
    "single_expert": LayerConfig("single_expert", T=130, H=128, E=1, k=1, I=128, I_s=64, alpha=2.5, renorm=True),
    "max_experts": LayerConfig("max_experts", T=64, H=256, E=1024, k=16, I=64, I_s=0),
    "wide_tiles": LayerConfig("wide_tiles", T=600, H=640, E=4, k=2, I=384, I_s=320, alpha=2.5, renorm=True),
    "w4a16_small": LayerConfig("w4a16_small", T=20, H=256, E=6, k=2, I=128, I_s=128, alpha=2.5, renorm=True,
                               bias_range=0.05, w4a16=True),
    "w4a16_many_tokens": LayerConfig("w4a16_many_tokens", T=96, H=384, E=3, k=2, I=256, I_s=0, w4a16=True),
    # fewer than 32 rows per expert on average: the GEMV path, several 8-token chunks per expert
    "w4a16_chunks": LayerConfig("w4a16_chunks", T=40, H=256, E=8, k=2, I=128, I_s=0, w4a16=True),
    # 32 rows per expert or more: the grouped prefill GEMM (int4 dequantised in shared memory)
    "w4a16_prefill": LayerConfig("w4a16_prefill", T=700, H=512, E=8, k=2, I=384, I_s=256, alpha=2.5, renorm=True,
                                 bias_range=0.05, w4a16=True),
    "w4a16_prefill_clamp": LayerConfig("w4a16_prefill_clamp", T=300, H=256, E=4, k=2, I=256, I_s=128,
                                       swiglu_limit=0.5, w4a16=True),
    # the widest clamp the int4 paths accept (|h| <= L^2 finite in fp16) with
    # activations 50x the benchmark's: GEMV path, then grouped prefill GEMM
    "w4a16_wide_limit": LayerConfig("w4a16_wide_limit", T=20, H=256, E=6, k=2, I=128, I_s=128,
                                    swiglu_limit=255.0, x_scale=50.0, w4a16=True),
    "w4a16_prefill_wide_limit": LayerConfig("w4a16_prefill_wide_limit", T=300, H=256, E=4, k=2, I=256,
                                            I_s=128, swiglu_limit=255.0, x_scale=50.0, w4a16=True),
    # NVFP4 experts.  Fewer than 32 rows per expert: the register-dequant GEMV
    # (shared expert in its launches), with several 8-token chunks per expert,
    # and at the widest clamp with large activations.  32 or more: the grouped
    # tensor-core GEMM over several token and weight tiles with ragged tails
    # (K = 384: the second code copy half past the row), many tiles per
    # expert, the clamp, and the widest clamp with large activations
    "nvfp4_small": LayerConfig("nvfp4_small", T=20, H=256, E=6, k=2, I=128, I_s=128, alpha=2.5, renorm=True,
                               bias_range=0.05, nvfp4=True),
    "nvfp4_chunks": LayerConfig("nvfp4_chunks", T=40, H=384, E=8, k=2, I=256, I_s=0, nvfp4=True),
    "nvfp4_gemv_wide_limit": LayerConfig("nvfp4_gemv_wide_limit", T=20, H=256, E=6, k=2, I=128, I_s=128,
                                         swiglu_limit=255.0, x_scale=50.0, nvfp4=True),
    "nvfp4_prefill": LayerConfig("nvfp4_prefill", T=700, H=512, E=8, k=2, I=384, I_s=256, alpha=2.5, renorm=True,
                                 bias_range=0.05, nvfp4=True),
    "nvfp4_wide": LayerConfig("nvfp4_wide", T=1500, H=1024, E=16, k=4, I=640, I_s=384, alpha=2.5, renorm=True,
                              nvfp4=True),
    "nvfp4_clamp": LayerConfig("nvfp4_clamp", T=300, H=256, E=4, k=2, I=256, I_s=128, swiglu_limit=0.5,
                               nvfp4=True),
    "nvfp4_wide_limit": LayerConfig("nvfp4_wide_limit", T=300, H=256, E=4, k=2, I=256, I_s=0,
                                    swiglu_limit=255.0, x_scale=50.0, nvfp4=True),
    # enough tokens for the row-block top-k kernel: E not a multiple of 4
    # (scalar partial sums), and k >= 8 (17 kept values per thread)
    "rows_e5": LayerConfig("rows_e5", T=1300, H=128, E=5, k=3, I=64, I_s=32, alpha=1.5, renorm=True),
    "rows_k10": LayerConfig("rows_k10", T=1250, H=256, E=40, k=10, I=64, I_s=0),
    "shared_small_t32": LayerConfig("shared_small_t32", T=32, H=256, E=4, k=2, I=64, I_s=96, alpha=2.5,
                                    renorm=True),
    "shared_tc_t33": LayerConfig("shared_tc_t33", T=33, H=256, E=4, k=2, I=64, I_s=96),
}


def _edge_inputs(name):
    cfg = EDGE[name]
    inp = moe_inputs.make_layer(cfg, seed=0)
    if cfg.x_scale != 1.0:
        # keep the router's logits at the benchmark's scale: these layers
        # stress the expert FFN's range, not the router's fp32 rounding
        inp.router_w = inp.router_w / cfg.x_scale
    return inp


def _hot_expert_inputs():
    cfg = LayerConfig("hot_expert", T=300, H=256, E=8, k=1, I=128, I_s=64)
    inp = moe_inputs.make_layer(cfg, seed=2)
    b = torch.zeros(cfg.E)
    b[3] = 10.0                      # every token picks expert 3
    inp.correction_bias = b
    return inp


def _tied_router_inputs():
    cfg = LayerConfig("tied_router", T=128, H=256, E=8, k=3, I=64, I_s=64, bias_kind="zero")
    inp = moe_inputs.make_layer(cfg, seed=4)
    inp.router_w[4:8] = inp.router_w[0:4]   # experts e and e+4 tie exactly
    return inp


def _tied_router_rows_inputs():
    # enough tokens for the row-block top-k kernel (one token per thread),
    # whose exact ties must fall back to the warp path and its fp64 re-order
    cfg = LayerConfig("tied_router_rows", T=1400, H=256, E=8, k=3, I=64, I_s=0, bias_kind="zero")
    inp = moe_inputs.make_layer(cfg, seed=6)
    inp.router_w[4:8] = inp.router_w[0:4]
    return inp


def _all_small_inputs():
    out = {n: _edge_inputs(n) for n in EDGE}
    out["hot_expert"] = _hot_expert_inputs()
    out["tied_router"] = _tied_router_inputs()
    out["tied_router_rows"] = _tied_router_rows_inputs()
    return out


SMALL = sorted(list(EDGE) + ["hot_expert", "tied_router", "tied_router_rows"])


@pytest.fixture(scope="module")
def small_inputs():
    return _all_small_inputs()


@pytest.mark.parametrize("name", SMALL)
def test_stages_match_oracle(small_inputs, name):
    inp = small_inputs[name]
    cfg = inp.cfg
    layer = gpu_layer(inp)
    x = inp.x.cuda()
    st = run_stages(layer, x)
    res = oracle.moe_forward(inp, keep_hidden=True)
    k, E, T = cfg.k, cfg.E, cfg.T

    # router: ids bit-exact outside near-ties; weights of the GPU's ids
    n_tie, n_tie_mis = check_ids(st.ids, res.selection)
    gpu_ids = st.ids.cpu().to(torch.int64)
    res = oracle.moe_forward(inp, keep_hidden=True, ids_override=gpu_ids)
    w_ref = res.selection.weights
    assert torch.allclose(st.topk_w.cpu().double(), w_ref, rtol=1e-5, atol=1e-7)

    # permutation: bit-exact against the oracle's stable sort of the GPU ids
    assert torch.equal(st.offsets.cpu().long(), res.perm.expert_offsets)
    assert torch.equal(st.row_of.cpu().long(), res.perm.row_of)
    assert torch.equal(st.src.cpu().long(), res.perm.src)
    assert torch.equal(st.w_perm.cpu(), st.topk_w.cpu().reshape(-1)[res.perm.src])
    assert torch.equal(st.x_perm.cpu(), inp.x[res.perm.src // k])
    # maps-only permute: the same maps and weights
    for got, want in zip(st.maps, (st.offsets, st.row_of, st.src, st.w_perm)):
        assert torch.equal(got, want)

    tol = tol_for(cfg)
    # routed rows: y_perm[r] = w_perm[r] * FFN_e(x[src[r] / k])
    y_ref = res.y_perm * st.w_perm.cpu().double()[:, None]
    assert rel_err(st.y_perm, y_ref) <= tol, rel_err(st.y_perm, y_ref)
    if cfg.I_s > 0:
        assert rel_err(st.shared_out, res.shared) <= tol
    err = rel_err(st.out, res.out)
    assert err <= tol, f"{name}: layer output error {err:.3e} (near-ties {n_tie}, mismatched {n_tie_mis})"
    # the gather fused into the FFN's loads: the same operands, so the same bits
    assert torch.equal(st.y_perm_g, st.y_perm)
    if cfg.I_s > 0:
        assert torch.equal(st.shared_out_g, st.shared_out)

    # the one-call forward gives the same bits as the staged calls
    out2 = layer.forward(x)
    torch.cuda.synchronize()
    assert torch.equal(out2, st.out)
    assert layer.device_error() == 0


def test_forward_is_deterministic(small_inputs):
    inp = small_inputs["ragged"]
    layer = gpu_layer(inp)
    x = inp.x.cuda()
    a = layer.forward(x).clone()
    b = layer.forward(x).clone()
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("name", ["ragged", "w4a16_prefill", "nvfp4_prefill"])
def test_tile_queues_are_left_at_zero(small_inputs, name):
    """The persistent grouped GEMMs hand tiles out from counters in the
    workspace header; every launch must leave them at zero, so that the next
    call on the same workspace (or a graph replay) starts from tile 0."""
    inp = small_inputs[name]
    layer = gpu_layer(inp)
    x = inp.x.cuda()
    outs = []
    for _ in range(3):
        outs.append(layer.forward(x).clone())
        torch.cuda.synchronize()
        header = layer.ws[:256].view(torch.int32).cpu()
        assert header[0].item() == 0, "device error word set"
        assert torch.count_nonzero(header[2:10]).item() == 0, f"tile queue words {header[2:10].tolist()}"
        assert header[10].item() == 0, "permute ticket counter left non-zero"
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])


@pytest.mark.parametrize("name", ["ragged", "w4a16_small", "w4a16_prefill", "nvfp4_small", "shared_small_t32"])
def test_forward_replays_from_a_cuda_graph(small_inputs, name):
    """The forward enqueues only device work on the given stream (no host
    sync, no allocation): captured once into a CUDA graph, its replay gives
    the eager forward's bits, also on a non-default stream."""
    inp = small_inputs[name]
    layer = gpu_layer(inp)
    x = inp.x.cuda()
    eager = layer.forward(x).clone()
    side = torch.cuda.Stream()
    out = torch.empty_like(eager)
    with torch.cuda.stream(side):
        layer.forward(x, out=out, stream=side)   # warm: every one-time setup happens here
    side.synchronize()
    assert torch.equal(out, eager)
    out.zero_()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        layer.forward(x, out=out, stream=side)
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager)
    assert layer.device_error() == 0
    del graph


@pytest.mark.parametrize("T", [300, 16])
def test_nvfp4_every_scale_byte(T):
    """The down weight's E4M3 block scales vary by output row and take every
    finite E4M3 pattern (both signs, the subnormals, 448): output column n of
    y_perm is one scale value times an unscaled sum, so each column is
    compared with the oracle's on its own.  The E4M3 NaN patterns are left
    out (they make NaN weights by definition).  T = 300: the grouped GEMM;
    T = 16 (8 rows per expert): the GEMV."""
    cfg = LayerConfig("nvfp4_scales", T=T, H=256, E=2, k=1, I=128, I_s=0, nvfp4=True)
    inp = moe_inputs.make_layer(cfg, seed=5)
    finite = [b for b in range(256) if b not in (0x7F, 0xFF)] + [0x38, 0xB8]   # 256 rows
    rows = torch.tensor(finite, dtype=torch.int64).to(torch.uint8)
    inp.s_down = rows[None, :, None].expand(cfg.E, cfg.H, cfg.I // 16).contiguous()
    layer = gpu_layer(inp)
    st = run_stages(layer, inp.x.cuda())
    res = oracle.moe_forward(inp, ids_override=st.ids.cpu().to(torch.int64))
    y_ref = res.y_perm * st.w_perm.cpu().double()[:, None]
    y = st.y_perm.cpu().double()
    tol = tol_for(cfg)
    for n in range(cfg.H):
        m = float(y_ref[:, n].abs().max())
        if m == 0.0:
            assert bool((y[:, n] == 0).all()), f"scale byte {finite[n]:#04x}: column not zero"
        else:
            e = float((y[:, n] - y_ref[:, n]).abs().max()) / m
            assert e <= tol, f"scale byte {finite[n]:#04x}: column error {e:.3e}"
    assert layer.device_error() == 0


@pytest.mark.parametrize("name", ["tied_router", "tied_router_rows"])
def test_tied_router_prefers_lower_id(small_inputs, name):
    inp = small_inputs[name]
    layer = gpu_layer(inp)
    st = run_stages(layer, inp.x.cuda())
    sel = oracle.select_topk(oracle.router_logits(inp.x, inp.router_w), inp.correction_bias, inp.cfg.k, 1.0,
                             False)
    # the exact ties between e and e+4 must resolve to the lower id, as the oracle does
    assert torch.equal(st.ids.cpu().long(), sel.ids)


# ------------------------------------------------------ benchmark layers ----

FULL = ["mid", "skewed", "large_prefill", "decode_w4a16", "prefill_w4a16", "decode_nvfp4"]
# layers whose every output row is compared (the oracle runs them in seconds)
ALL_ROWS = {"mid", "decode_w4a16", "decode_nvfp4"}
TILE_ROWS = 256         # routed rows per token tile of the grouped GEMMs (a CTA pair)
MIN_SAMPLE = 1024       # tokens compared on the other layers, at least


def tile_stratified_tokens(offsets, src, k, T, seed=123):
    """Tokens whose routed rows sit at the edges of every token tile of every
    expert: for each expert and each 256-row token tile of it (the last one
    ragged), the tokens of the tile's first and last row and of the two rows
    where the tile's halves meet (each CTA of a pair loads one half).  Every
    expert therefore contributes its first and its last tile, the hot expert
    of a skewed layer every tile, and, as a token's output row spans every
    weight-row tile of the down projection, every expert's last weight-row
    tile is covered too.  Random tokens fill the sample up to MIN_SAMPLE."""
    off = offsets.tolist()
    rows = set()
    for e in range(len(off) - 1):
        for r0 in range(off[e], off[e + 1], TILE_ROWS):
            n = min(TILE_ROWS, off[e + 1] - r0)
            half = (n + 15) // 16 * 8          # token columns of the first CTA (MMA N rounded to 16, halved)
            for r in (r0, r0 + n - 1, r0 + min(half, n) - 1, r0 + min(half, n - 1)):
                rows.add(r)
    src_l = src.tolist()
    toks = {src_l[r] // k for r in rows}
    if len(toks) < MIN_SAMPLE:
        g = torch.Generator().manual_seed(seed)
        for t in torch.randperm(T, generator=g).tolist():
            if len(toks) >= MIN_SAMPLE:
                break
            toks.add(t)
    return sorted(toks), sorted(rows)


@pytest.mark.parametrize("name", FULL)
def test_full_size_layer(name):
    cfg = CONFIGS[name]
    wdev = "cpu" if name == "mid" else "cuda"
    inp = moe_inputs.make_layer(cfg, seed=0, weight_device=wdev)
    layer = gpu_layer(inp)
    x = inp.x.cuda()
    st = run_stages(layer, x)

    # router ids for every token
    sel = oracle.select_topk(oracle.router_logits(inp.x, inp.router_w), inp.correction_bias, cfg.k, cfg.alpha,
                             cfg.renorm)
    n_tie, n_tie_mis = check_ids(st.ids, sel)
    ties = f"near-ties {n_tie} (gap < 1e-6), of which the GPU chose differently: {n_tie_mis}"
    gpu_ids = st.ids.cpu().to(torch.int64)
    chosen = torch.gather(sel.scores, 1, gpu_ids)
    if cfg.renorm:
        chosen = chosen / chosen.sum(1, keepdim=True)
    assert torch.allclose(st.topk_w.cpu().double(), cfg.alpha * chosen, rtol=1e-5, atol=1e-7), ties

    # permutation for every slot
    perm = oracle.permute(gpu_ids, cfg.E)
    assert torch.equal(st.offsets.cpu().long(), perm.expert_offsets), ties
    # the maps-only permute and the FFN with the gather fused into its loads
    # give the x_perm path's maps and bits at full size as well
    for got, want in zip(st.maps, (st.offsets, st.row_of, st.src, st.w_perm)):
        assert torch.equal(got, want)
    assert torch.equal(st.y_perm_g, st.y_perm)
    if cfg.I_s > 0:
        assert torch.equal(st.shared_out_g, st.shared_out)
    assert torch.equal(st.row_of.cpu().long(), perm.row_of), ties
    assert torch.equal(st.src.cpu().long(), perm.src), ties
    src_dev = st.src.long()
    assert torch.equal(st.x_perm, x[src_dev // cfg.k])
    assert torch.equal(st.w_perm, st.topk_w.reshape(-1)[src_dev])

    # layer output: every row, or the tile-stratified token sample (with the GPU's ids)
    if name in ALL_ROWS:
        toks = list(range(cfg.T))
    else:
        toks, _ = tile_stratified_tokens(perm.expert_offsets, perm.src, cfg.k, cfg.T)
    tt = torch.tensor(toks, dtype=torch.int64)
    res = oracle.moe_forward(inp, tokens=toks, ids_override=gpu_ids[tt])
    tol = tol_for(cfg)
    what = f"{name}: {len(toks)} of {cfg.T} tokens; {ties}"
    err = rel_err(st.out.cpu()[tt], res.out)
    assert err <= tol, f"{what}: output error {err:.3e}"
    if cfg.I_s > 0:
        e_sh = rel_err(st.shared_out.cpu()[tt], res.shared)
        assert e_sh <= tol, f"{what}: shared-expert error {e_sh:.3e}"
    # the routed rows of the compared tokens, one by one: y_perm[r] = w_perm[r] * FFN_e(x_t)
    k = cfg.k
    slots = (tt[:, None] * k + torch.arange(k)[None, :]).reshape(-1)          # GPU slot ids
    gpu_rows = st.row_of.cpu().long()[slots]
    loc_rows = res.perm.row_of                                                # oracle rows, same slot order
    y_ref = res.y_perm[loc_rows] * st.w_perm.cpu().double()[gpu_rows][:, None]
    e_y = rel_err(st.y_perm.cpu()[gpu_rows], y_ref)
    assert e_y <= tol, f"{what}: routed-row error {e_y:.3e}"
    out2 = layer.forward(x)
    torch.cuda.synchronize()
    assert torch.equal(out2, st.out)
    assert layer.device_error() == 0
    print(f"{what}; output error {err:.3e}, routed-row error {e_y:.3e}")
