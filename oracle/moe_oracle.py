"""CPU oracle for the routed MoE SwiGLU layer forward (fp64).

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The product path
(the CUDA library and its Python binding) never calls it, and shares no code
with it: no kernels, headers, helpers, tables or pre/post-processing.

Everything is evaluated in float64 on the CPU with plain torch ops.  Inputs
are the exact bf16 / fp32 / uint4 values widened to float64, so products are
exact and only the fp64 sums round.  No step is blocked, fused or reordered
beyond what the definition states; a matmul serves as the library primitive
for "apply this linear map to these rows", and a stable sort as the library
primitive for "order by key, keep input order among equal keys".

Sources (web pages on the method):
  [glm5next]  "Module glm5next_mlp" (metrale model-arch docs):
              §Numerics the kernels rely on; §One all-reduce for both EP and
              TP; Constants KERNEL_MAX_TOP_K, MOE_MODULE, W4A16_GEMV_MODULE;
              Modules forward / forward_prefill_gemm / build.
  [mstar]     "mstar.model.components.distributed.mlp", class
              ParallelGatedMLP (fused gate/up, SwiGLU, down).
  [beam]      "bridge.models.beam.modeling_beam", _BeamRouterGatingLinear,
              beam_router_gating_linear, BeamTopKRouter (fp32 router GEMM).

Readings where the pages are silent (each also listed in the design notes):
  * the correction bias is added to the sigmoid score (not to the logit);
  * no group-limited routing; no router linear bias (only the correction
    bias); renormalisation (when enabled) divides by the sum of the k chosen
    unbiased scores and happens before routed_scaling_factor;
  * ties in the biased score go to the lower expert id, and the k ids of a
    token are emitted in (biased score descending, id ascending) order;
  * the shared expert uses the same clamped SwiGLU and is not scaled;
  * gate rows come first in the fused gate/up weight ([0, I) gate, [I, 2I) up);
  * W4A16: two uint4 codes per byte along K, low nibble = even k, zero point
    8, one bf16 scale per (output row, 128-wide K group): w = (q - 8) * scale.
  * NVFP4 (the module summary's "routed NVFP4 MoE"; the pages give no
    layout): FP4 E2M1 codes packed as for W4A16, one FP8 E4M3 scale per
    (output row, 16-wide K block), and one fp32 scale per expert and weight
    tensor (the fused gate/up is one tensor):
    w = e2m1(code) * e4m3(block scale) * tensor scale.  The element formats
    are the OCP ones: E2M1 of the Microscaling Formats (MX) v1.0
    specification, E4M3 of the OCP 8-bit Floating Point specification.

Pins: tests/test_oracle.py checks every function here against hand-worked
closed forms (tests/golden/), brute-force enumeration, invariants and
library special cases.  The choice "bias added to the score" is a reading:
nothing on the pages can pin it (parity of that choice is unpinned).
"""

from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

f64 = torch.float64


def _cpu64(t: torch.Tensor) -> torch.Tensor:
    return t.detach().to(device="cpu").to(f64)


# ---------------------------------------------------------------- router ----

def router_logits(x: torch.Tensor, router_w: torch.Tensor) -> torch.Tensor:
    """logit[t, e] = sum_h x[t, h] * Wr[e, h]   ([beam] beam_router_gating_linear:
    inp @ weight.T in the router dtype; no linear bias here).  fp64 [T, E]."""
    return _cpu64(x) @ _cpu64(router_w).T


def sigmoid(z: torch.Tensor) -> torch.Tensor:
    """s = 1 / (1 + exp(-z))  ([glm5next] §Numerics: sigmoid score)."""
    return 1.0 / (1.0 + torch.exp(-z))


@dataclass
class Selection:
    ids: torch.Tensor        # [T, k] int64, (biased desc, id asc) order
    weights: torch.Tensor    # [T, k] fp64, emitted combine weights
    scores: torch.Tensor     # [T, E] fp64 unbiased sigmoid scores
    biased: torch.Tensor     # [T, E] fp64 scores + correction bias
    gap: torch.Tensor        # [T] fp64: k-th minus (k+1)-th biased score


def select_topk(logits: torch.Tensor, correction_bias: Optional[torch.Tensor],
                k: int, alpha: float, renorm: bool) -> Selection:
    """Biased top-k selection with unbiased emitted weights.

    [glm5next] §Numerics: the correction bias steers selection only; the
    emitted weight is the chosen expert's unbiased sigmoid score, and
    routed_scaling_factor multiplies the top-k weights.  Ties go to the lower
    expert id; optional renormalisation of the k weights to sum 1 comes before
    the scaling.
    """
    logits = _cpu64(logits)
    T, E = logits.shape
    if not (1 <= k <= E):
        raise ValueError("need 1 <= k <= E")
    s = sigmoid(logits)
    bias = torch.zeros(E, dtype=f64) if correction_bias is None else _cpu64(correction_bias)
    b = s + bias[None, :]
    # A stable descending sort keeps equal keys in ascending expert order,
    # which is exactly "ties -> lower id".
    order = torch.sort(b, dim=1, descending=True, stable=True).indices
    ids = order[:, :k]
    b_sorted = torch.gather(b, 1, order)
    if k < E:
        gap = b_sorted[:, k - 1] - b_sorted[:, k]
    else:
        gap = torch.full((T,), math.inf, dtype=f64)
    chosen = torch.gather(s, 1, ids)
    if renorm:
        chosen = chosen / chosen.sum(dim=1, keepdim=True)
    weights = alpha * chosen
    return Selection(ids, weights, s, b, gap)


def override_selection(sel: Selection, ids: torch.Tensor, alpha: float,
                       renorm: bool) -> Selection:
    """The selection with its ids replaced by ``ids`` (another valid choice,
    e.g. for a token whose k-th and (k+1)-th biased scores nearly tie).  The
    emitted weights follow the given ids exactly as for a routed selection
    ([glm5next] §Numerics): the unbiased scores of those ids, renormalised
    over them when enabled, then times routed_scaling_factor."""
    ids = ids.to(torch.int64).cpu()
    chosen = torch.gather(sel.scores, 1, ids)
    if renorm:
        chosen = chosen / chosen.sum(dim=1, keepdim=True)
    return Selection(ids, alpha * chosen, sel.scores, sel.biased, sel.gap)


# --------------------------------------------------------------- permute ----

@dataclass
class Permutation:
    expert_offsets: torch.Tensor  # [E+1] int64, offsets[E] = T*k
    row_of: torch.Tensor          # [T*k] int64: routed row of slot i = t*k + j
    src: torch.Tensor             # [T*k] int64: slot i of routed row r


def permute(ids: torch.Tensor, num_experts: int) -> Permutation:
    """Token sort by expert ([glm5next] MOE_MODULE: token sort / permute /
    unpermute).  A stable counting sort of the slots i = t*k + j by expert id:
    expert e owns rows [offsets[e], offsets[e+1]) and, inside them, its slots
    in ascending i (equivalently ascending token, as a token picks an expert
    at most once)."""
    flat = ids.reshape(-1).to(torch.int64).cpu()
    R = flat.numel()
    counts = torch.bincount(flat, minlength=num_experts)
    offsets = torch.zeros(num_experts + 1, dtype=torch.int64)
    offsets[1:] = torch.cumsum(counts, 0)
    src = torch.sort(flat, stable=True).indices
    row_of = torch.empty(R, dtype=torch.int64)
    row_of[src] = torch.arange(R, dtype=torch.int64)
    return Permutation(offsets, row_of, src)


# ------------------------------------------------------------------- FFN ----

def swiglu_clamped(gate: torch.Tensor, up: torch.Tensor, limit: float) -> torch.Tensor:
    """silu(min(gate, L)) * clamp(up, -L, L)  ([glm5next] §Numerics: the clamp
    is asymmetric, gate bounded above only, up on both sides; L = +inf means
    no clamp).  silu(g) = g / (1 + exp(-g))."""
    g = torch.clamp(gate, max=limit)
    u = torch.clamp(up, min=-limit, max=limit)
    return (g / (1.0 + torch.exp(-g))) * u


def dequant_int4_g128(q: torch.Tensor, scale: torch.Tensor) -> torch.Tensor:
    """W4A16 weight: w[n, k] = (code[n, k] - 8) * scale[n, k // 128], with the
    codes of byte q[n, c] at k = 2c (low nibble) and k = 2c + 1 (high nibble).
    q: uint8 [N, K/2], scale: bf16 [N, K/128] -> fp64 [N, K]."""
    q = q.detach().cpu()
    N, half = q.shape
    K = 2 * half
    lo = (q & 0xF).to(f64)
    hi = (q >> 4).to(f64)
    codes = torch.stack([lo, hi], dim=-1).reshape(N, K)
    sc = _cpu64(scale).repeat_interleave(128, dim=1)
    assert sc.shape == (N, K)
    return (codes - 8.0) * sc


def e2m1_value(code: torch.Tensor) -> torch.Tensor:
    """FP4 E2M1 (OCP Microscaling Formats v1.0): bit 3 sign, bits 2..1
    exponent with bias 1, bit 0 mantissa.  Exponent field 0 is subnormal,
    m * 2^-1 (0 or 0.5); otherwise (1 + m / 2) * 2^(e - 1).  The format has
    no infinity and no NaN.  code: integer tensor of 4-bit values -> fp64."""
    c = code.to(torch.int64)
    sign = (c >> 3) & 1
    e = ((c >> 1) & 3).to(f64)
    m = (c & 1).to(f64)
    mag = torch.where(e == 0, m * 0.5, (1.0 + m / 2.0) * torch.pow(2.0, e - 1.0))
    return torch.where(sign == 1, -mag, mag)


def e4m3_value(b: torch.Tensor) -> torch.Tensor:
    """FP8 E4M3 (OCP 8-bit Floating Point): bit 7 sign, bits 6..3 exponent
    with bias 7, bits 2..0 mantissa.  Exponent field 0 is subnormal,
    (m / 8) * 2^-6; otherwise (1 + m / 8) * 2^(e - 7).  No infinity; the two
    patterns S.1111.111 are NaN.  b: uint8 tensor -> fp64."""
    c = b.to(torch.int64)
    sign = (c >> 7) & 1
    e = ((c >> 3) & 15).to(f64)
    m = (c & 7).to(f64)
    mag = torch.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * torch.pow(2.0, e - 7.0))
    mag = torch.where((e == 15) & (m == 7), torch.full_like(mag, float("nan")), mag)
    return torch.where(sign == 1, -mag, mag)


def dequant_nvfp4(q: torch.Tensor, block_scale: torch.Tensor, tensor_scale) -> torch.Tensor:
    """NVFP4 weight: w[n, k] = e2m1(code[n, k]) * e4m3(block_scale[n, k // 16])
    * tensor_scale, with the codes of byte q[n, c] at k = 2c (low nibble) and
    k = 2c + 1 (high nibble).  q: uint8 [N, K/2], block_scale: uint8
    [N, K/16] (E4M3 bit patterns), tensor_scale: fp32 scalar -> fp64 [N, K]."""
    q = q.detach().cpu()
    N, half = q.shape
    K = 2 * half
    # each format's values, evaluated once by the definitions above, then looked up
    e2m1 = e2m1_value(torch.arange(16))
    e4m3 = e4m3_value(torch.arange(256, dtype=torch.int64).to(torch.uint8))
    lo = e2m1[(q & 0xF).long()]
    hi = e2m1[(q >> 4).long()]
    vals = torch.stack([lo, hi], dim=-1).reshape(N, K)
    sc = e4m3[block_scale.detach().cpu().long()].repeat_interleave(16, dim=1)
    assert sc.shape == (N, K)
    g = float(torch.as_tensor(tensor_scale, dtype=torch.float32))
    return vals * sc * g


def expert_ffn(v: torch.Tensor, w_gate_up: torch.Tensor, w_down: torch.Tensor,
               limit: float) -> torch.Tensor:
    """FFN(v) = W_down (silu(min(W_gate v, L)) * clamp(W_up v, -L, L)).

    [mstar] ParallelGatedMLP: gate and up are one fused projection, gate =
    shard 0, up = shard 1; down maps back to hidden.  w_gate_up [2I, H]
    (fp64, gate rows first), w_down [H, I]; v [n, H] -> [n, H]."""
    I = w_down.shape[1]
    gu = v @ w_gate_up.T
    h = swiglu_clamped(gu[:, :I], gu[:, I:], limit)
    return h @ w_down.T


def expert_hidden(v, w_gate_up, limit):
    """The SwiGLU activations h = silu(min(G, L)) * clamp(U, -L, L) only."""
    I = w_gate_up.shape[0] // 2
    gu = v @ w_gate_up.T
    return swiglu_clamped(gu[:, :I], gu[:, I:], limit)


def expert_weights64(layer, e: int):
    """Routed expert e's (w_gate_up [2I, H], w_down [H, I]) in fp64."""
    if getattr(layer.cfg, "nvfp4", False):
        return (dequant_nvfp4(layer.w_gate_up[e], layer.s_gate_up[e], layer.g_gate_up[e].cpu()),
                dequant_nvfp4(layer.w_down[e], layer.s_down[e], layer.g_down[e].cpu()))
    if layer.cfg.w4a16:
        return (dequant_int4_g128(layer.w_gate_up[e], layer.s_gate_up[e]),
                dequant_int4_g128(layer.w_down[e], layer.s_down[e]))
    return _cpu64(layer.w_gate_up[e]), _cpu64(layer.w_down[e])


# ----------------------------------------------------------------- layer ----

@dataclass
class LayerResult:
    out: torch.Tensor             # [T, H] fp64
    selection: Selection
    perm: Permutation
    y_perm: torch.Tensor          # [R, H] fp64 unweighted FFN_e(x_t) per routed row
    h_perm: Optional[torch.Tensor]  # [R, I] fp64 (if requested)
    shared: torch.Tensor          # [T, H] fp64 (zeros without a shared expert)
    shared_h: Optional[torch.Tensor]
    tokens: torch.Tensor          # which tokens of the layer these rows are


def moe_forward(layer, tokens: Optional[Sequence[int]] = None,
                keep_hidden: bool = False,
                ids_override: Optional[torch.Tensor] = None) -> LayerResult:
    """out[t] = FFN_shared(x[t]) + sum_j w[t, j] * FFN_{e_j}(x[t]).

    [glm5next] §One all-reduce: the shared output and the routed slots are
    added in one combine; §Numerics: routed_scaling_factor scales the routed
    weights only, the shared expert is added unscaled.  With ``tokens`` only
    those rows of x are evaluated (the layer is per-token).  ``ids_override``
    replaces the selected ids (weights recomputed from the same scores), for
    re-evaluating tokens whose selection is a near-tie."""
    cfg = layer.cfg
    if tokens is None:
        tok = torch.arange(layer.x.shape[0])
    else:
        tok = torch.as_tensor(list(tokens), dtype=torch.int64)
    x = layer.x.detach().cpu()[tok]
    x64 = x.to(f64)
    T, H, E, k, L = x.shape[0], cfg.H, cfg.E, cfg.k, cfg.swiglu_limit

    sel = select_topk(router_logits(x, layer.router_w), layer.correction_bias,
                      k, cfg.alpha, cfg.renorm)
    if ids_override is not None:
        sel = override_selection(sel, ids_override, cfg.alpha, cfg.renorm)
    perm = permute(sel.ids, E)

    R = T * k
    y_perm = torch.zeros(R, H, dtype=f64)
    h_perm = torch.zeros(R, cfg.I, dtype=f64) if keep_hidden else None
    for e in range(E):
        r0, r1 = int(perm.expert_offsets[e]), int(perm.expert_offsets[e + 1])
        if r1 == r0:
            continue
        rows_tok = perm.src[r0:r1] // k
        wgu, wd = expert_weights64(layer, e)
        h = expert_hidden(x64[rows_tok], wgu, L)
        if keep_hidden:
            h_perm[r0:r1] = h
        y_perm[r0:r1] = h @ wd.T

    if cfg.I_s > 0:
        sgu, sd = _cpu64(layer.shared_w_gate_up), _cpu64(layer.shared_w_down)
        shared_h = expert_hidden(x64, sgu, L)
        shared = shared_h @ sd.T
    else:
        shared_h = None
        shared = torch.zeros(T, H, dtype=f64)

    out = shared.clone()
    rows = perm.row_of.view(T, k)
    for j in range(k):
        out += sel.weights[:, j:j + 1] * y_perm[rows[:, j]]
    return LayerResult(out, sel, perm, y_perm, h_perm, shared,
                       shared_h if keep_hidden else None, tok)


# ------------------------------------------------- expert parallelism ----

def moe_partial(layer, expert_begin: int, expert_end: int, shared_begin: int, shared_end: int,
                tokens: Optional[Sequence[int]] = None,
                ids_override: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One rank's partial sum under expert parallelism ([glm5next] §One
    all-reduce for both EP and TP: each rank adds the shared output and its
    local routed slots in its combine; one all-reduce of the [T, H] partials
    gives the layer output).  The rank owns routed experts
    [expert_begin, expert_end) and the shared expert's intermediate features
    [shared_begin, shared_end): the clamped SwiGLU acts feature by feature, so
    the shared output is the sum over feature slices of W_down[:, slice]
    h[slice].  The router is the full one (every rank ranks all experts).
      out_r[t] = sum_{f in slice} W_sd[:, f] h_s[t, f]
                 + sum_{j : expert_begin <= e_j < expert_end} w[t, j] FFN_{e_j}(x[t])
    fp64 [T, H]."""
    res = moe_forward(layer, tokens=tokens, keep_hidden=True, ids_override=ids_override)
    T = res.out.shape[0]
    H, k = layer.cfg.H, layer.cfg.k
    out = torch.zeros(T, H, dtype=f64)
    if layer.cfg.I_s > 0 and shared_end > shared_begin:
        sd = _cpu64(layer.shared_w_down)
        out += res.shared_h[:, shared_begin:shared_end] @ sd[:, shared_begin:shared_end].T
    rows = res.perm.row_of.view(T, k)
    ids = res.selection.ids
    for j in range(k):
        local = ((ids[:, j] >= expert_begin) & (ids[:, j] < expert_end)).to(f64)[:, None]
        out += local * res.selection.weights[:, j:j + 1] * res.y_perm[rows[:, j]]
    return out
