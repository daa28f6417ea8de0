"""Pins for the CPU oracle (no GPU).

Each test ties the oracle to something other than itself: hand-worked closed
forms (tests/golden/hand_example.json), brute-force enumeration, invariants,
and special cases that reduce to textbook library routines.
"""

import itertools
import json
import math
import os
import random
from fractions import Fraction

import pytest
import torch
import torch.nn.functional as F

import moe_inputs
from moe_inputs import LayerInputs
from moe_inputs.configs import CONFIGS, LayerConfig, SKEW_BIAS_SCALE
import oracle

f64 = torch.float64


@pytest.fixture(scope="module")
def hand(golden_dir):
    with open(os.path.join(golden_dir, "hand_example.json")) as f:
        return json.load(f)


@pytest.fixture(scope="module")
def hand_nvfp4(golden_dir):
    with open(os.path.join(golden_dir, "nvfp4_hand.json")) as f:
        return json.load(f)


def _s(z):
    return 1.0 / (1.0 + math.exp(-z))


# ------------------------------------------------------------ hand example --

def test_hand_router_scores_and_selection(hand):
    x = torch.tensor([hand["x"]], dtype=torch.bfloat16)
    wr = torch.tensor(hand["router_w"], dtype=torch.float32)
    logits = oracle.router_logits(x, wr)
    assert logits[0].tolist() == hand["logits"]
    sel = oracle.select_topk(logits, torch.tensor(hand["selection"]["bias"]), 2, 1.0, False)
    assert torch.allclose(sel.scores[0], torch.tensor(hand["scores"], dtype=f64), atol=1e-15)
    # fp32 bias 0.3 is not exactly 0.3: 1e-7 slack on biased values only
    assert torch.allclose(sel.biased[0], torch.tensor(hand["selection"]["biased"], dtype=f64), atol=1e-7)
    assert sel.ids[0].tolist() == hand["selection"]["ids"]
    assert torch.allclose(sel.weights[0], torch.tensor(hand["selection"]["weights_alpha1_norenorm"], dtype=f64), atol=1e-15)
    assert abs(float(sel.gap[0]) - hand["selection"]["gap"]) < 1e-7
    sel = oracle.select_topk(logits, torch.tensor(hand["selection"]["bias"]), 2, 2.5, True)
    assert sel.ids[0].tolist() == hand["selection"]["ids"]
    assert torch.allclose(sel.weights[0], torch.tensor(hand["selection"]["weights_alpha2.5_renorm"], dtype=f64), atol=1e-14)


def test_hand_tie_goes_to_lower_id(hand):
    logits = torch.tensor([hand["logits"]], dtype=f64)
    tc = hand["tie_case"]
    sel = oracle.select_topk(logits, torch.tensor(tc["bias"]), 2, 1.0, False)
    assert sel.ids[0].tolist() == tc["ids_k2"]
    assert abs(float(sel.gap[0]) - (_s(1.0) - _s(0.0))) < 1e-15
    sel = oracle.select_topk(logits, torch.tensor(tc["bias"]), 1, 1.0, False)
    assert sel.ids[0].tolist() == tc["ids_k1"]
    assert float(sel.gap[0]) == tc["gap_k1"]


def test_hand_swiglu_clamp(hand):
    ex = hand["expert_ffn"]
    wgu = torch.tensor(ex["w_gate_up"], dtype=f64)
    wd = torch.tensor(ex["w_down"], dtype=f64)
    v = torch.tensor([[1.0, -1.0]], dtype=f64)
    y = oracle.expert_ffn(v, wgu, wd, 7.0)
    assert torch.allclose(y[0], torch.tensor(ex["limit7"]["y"], dtype=f64), atol=1e-14)
    h = oracle.expert_hidden(v, wgu, 0.5)
    assert abs(float(h[0, 0]) - ex["limit0.5"]["h"]) < 1e-15
    c = ex["gate_minus10_unclamped_below"]
    h = oracle.swiglu_clamped(torch.tensor([c["gate"]], dtype=f64), torch.tensor([c["up"]], dtype=f64), c["limit"])
    assert abs(float(h[0]) - c["h"]) < 1e-18
    c = ex["up_clamped_both_sides"]
    h = oracle.swiglu_clamped(torch.tensor([c["gate"]], dtype=f64), torch.tensor([c["up"]], dtype=f64), c["limit"])
    assert abs(float(h[0]) - c["h"]) < 1e-14


def _hand_layer(hand, alpha=1.0, renorm=False):
    lay = hand["layer"]
    cfg = LayerConfig("hand", T=1, H=2, E=4, k=2, I=1, I_s=1, alpha=alpha, renorm=renorm)
    bf = torch.bfloat16
    return LayerInputs(cfg, torch.tensor([hand["x"]], dtype=bf),
                    torch.tensor(hand["router_w"], dtype=torch.float32),
                    torch.tensor(hand["selection"]["bias"], dtype=torch.float32),
                    torch.tensor(lay["w_gate_up"], dtype=bf), torch.tensor(lay["w_down"], dtype=bf),
                    None, None,
                    torch.tensor(lay["shared_w_gate_up"], dtype=bf),
                    torch.tensor(lay["shared_w_down"], dtype=bf))


def test_hand_layer_output(hand):
    res = oracle.moe_forward(_hand_layer(hand))
    assert res.selection.ids[0].tolist() == [0, 1]
    assert torch.allclose(res.out[0], torch.tensor(hand["layer"]["out"], dtype=f64), atol=1e-14)


def test_hand_override_renormalises_the_given_ids(hand):
    """ids_override: the weights come from the unbiased scores of the given
    ids, renormalised over those ids before alpha, in the given slot order."""
    ov = hand["layer_override_renorm"]
    lay = _hand_layer(hand, alpha=ov["alpha"], renorm=True)
    res = oracle.moe_forward(lay, ids_override=torch.tensor([ov["ids"]]), keep_hidden=True)
    assert res.selection.ids[0].tolist() == ov["ids"]
    assert torch.allclose(res.selection.weights[0], torch.tensor(ov["weights"], dtype=f64), atol=1e-14)
    # expert 3's routed row holds h3 (rows of expert 0 come first in the permutation)
    assert res.perm.expert_offsets.tolist() == [0, 1, 1, 1, 2]
    assert abs(float(res.h_perm[1, 0]) - ov["h3"]) < 1e-16
    assert torch.allclose(res.out[0], torch.tensor(ov["out"], dtype=f64), atol=1e-14)


def test_hand_w4a16_dequant(hand):
    w = hand["w4a16"]
    q = torch.full((1, 64), w["q_fill_byte"], dtype=torch.uint8)
    q[0, 0], q[0, 1] = w["q_bytes_first"]
    s = torch.tensor([[w["scale"]]], dtype=torch.bfloat16)
    W = oracle.dequant_int4_g128(q, s)
    assert W.shape == (1, 128)
    assert W[0, :4].tolist() == w["w_first4"]
    assert (W[0, 4:] == 0).all()


def test_dequant_group_index():
    """Scale of group g covers k in [128g, 128g+128) only."""
    q = torch.full((2, 128), 0x99, dtype=torch.uint8)   # code 9 everywhere -> (9-8)=1
    s = torch.tensor([[1.0, 2.0], [4.0, 8.0]], dtype=torch.bfloat16)
    W = oracle.dequant_int4_g128(q, s)
    assert (W[0, :128] == 1).all() and (W[0, 128:] == 2).all()
    assert (W[1, :128] == 4).all() and (W[1, 128:] == 8).all()


# ------------------------------------------------------------------- NVFP4 --

def test_e2m1_table(hand_nvfp4):
    """Every FP4 E2M1 code against the format's value set (and its sign bit)."""
    got = oracle.e2m1_value(torch.arange(16))
    assert got.tolist() == hand_nvfp4["e2m1_by_code"]
    assert (torch.signbit(got[8:])).all() and not torch.signbit(got[:8]).any()


def test_e4m3_matches_torch_float8():
    """All 256 E4M3 bit patterns against torch's float8_e4m3fn conversion
    (a library routine), NaN exactly at S.1111.111."""
    b = torch.arange(256, dtype=torch.int64).to(torch.uint8)
    got = oracle.e4m3_value(b)
    lib = b.view(torch.float8_e4m3fn).to(f64)
    assert torch.equal(torch.isnan(got), torch.isnan(lib))
    assert torch.isnan(got).nonzero().flatten().tolist() == [0x7F, 0xFF]
    ok = ~torch.isnan(lib)
    assert torch.equal(got[ok], lib[ok])


def test_e4m3_hand_values(hand_nvfp4):
    sp = hand_nvfp4["e4m3_spot"]
    got = oracle.e4m3_value(torch.tensor(sp["bytes"], dtype=torch.int64).to(torch.uint8))
    assert got.tolist() == sp["values"]
    assert torch.isnan(oracle.e4m3_value(torch.tensor(sp["nan_bytes"], dtype=torch.int64).to(torch.uint8))).all()


def test_hand_nvfp4_dequant(hand_nvfp4):
    d = hand_nvfp4["dequant"]
    q = torch.zeros(1, 16, dtype=torch.uint8)
    for c, v in d["q_bytes"].items():
        q[0, int(c)] = v
    bs = torch.tensor([d["block_scale_bytes"]], dtype=torch.uint8)
    W = oracle.dequant_nvfp4(q, bs, torch.tensor(d["tensor_scale"], dtype=torch.float32))
    want = torch.zeros(1, 32, dtype=f64)
    for k, v in d["w_nonzero"].items():
        want[0, int(k)] = v
    assert W.shape == (1, 32)
    assert torch.equal(W, want)


def test_nvfp4_block_index():
    """Block scale b covers k in [16b, 16b + 16) of its own row only."""
    q = torch.full((2, 32), 0x22, dtype=torch.uint8)          # code 2 (= 1.0) everywhere
    bs = torch.tensor([[0x38, 0x40, 0x48, 0x50], [0x30, 0x28, 0x20, 0x18]], dtype=torch.uint8)
    W = oracle.dequant_nvfp4(q, bs, 1.0)
    want_row = [[1.0, 2.0, 4.0, 8.0], [0.5, 0.25, 0.125, 0.0625]]
    for n in range(2):
        for b in range(4):
            assert (W[n, 16 * b:16 * b + 16] == want_row[n][b]).all()


def test_nvfp4_layer_reduces_to_bf16_layer(hand_nvfp4):
    """An NVFP4 layer with power-of-two tensor scales gives the same output
    as the bf16 layer holding its weights, formed here from the E2M1 value
    table and torch's float8_e4m3fn (e2m1 x e4m3 has at most 6 significant
    bits, exact in bf16)."""
    cfg = LayerConfig("fp4", T=6, H=256, E=3, k=2, I=128, I_s=128, alpha=2.5, renorm=True,
                      nvfp4=True)
    g = torch.Generator().manual_seed(4)
    base = moe_inputs.make_layer(cfg.with_(nvfp4=False), seed=9)
    table = torch.tensor(hand_nvfp4["e2m1_by_code"], dtype=f64)

    def pack(E, N, K):
        codes = torch.randint(0, 16, (E, N, K), generator=g, dtype=torch.int64)
        sb = torch.randint(0x20, 0x48, (E, N, K // 16), generator=g, dtype=torch.int64).to(torch.uint8)
        ts = 2.0 ** (-torch.randint(3, 7, (E,), generator=g)).to(torch.float32)
        w = (table[codes] * sb.view(torch.float8_e4m3fn).to(f64).repeat_interleave(16, dim=2)
             * ts.to(f64)[:, None, None])
        q = (codes[..., 0::2] | (codes[..., 1::2] << 4)).to(torch.uint8)
        return q, sb, ts, w.to(torch.bfloat16)

    qgu, sgu, tgu, wgu = pack(cfg.E, 2 * cfg.I, cfg.H)
    qd, sd, td, wd = pack(cfg.E, cfg.H, cfg.I)
    lay4 = LayerInputs(cfg, base.x, base.router_w, base.correction_bias, qgu, qd, sgu, sd,
                       base.shared_w_gate_up, base.shared_w_down, tgu, td)
    lay16 = LayerInputs(cfg.with_(nvfp4=False), base.x, base.router_w, base.correction_bias,
                        wgu, wd, None, None, base.shared_w_gate_up, base.shared_w_down)
    a, b = oracle.moe_forward(lay4), oracle.moe_forward(lay16)
    assert (a.selection.ids == b.selection.ids).all()
    assert torch.allclose(a.out, b.out, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------- brute force --

def _brute_topk(b, k):
    """All k-subsets; max exact (rational) sum; lexicographically smallest id
    tuple among the maxima; then ordered by (b desc, id asc)."""
    E = len(b)
    fr = [Fraction(v) for v in b]
    best, best_set = None, None
    for comb in itertools.combinations(range(E), k):
        sm = sum(fr[i] for i in comb)
        if best is None or sm > best:
            best, best_set = sm, comb
    return best_set


@pytest.mark.parametrize("seed", range(40))
def test_bruteforce_topk(seed):
    rng = random.Random(seed)
    E = rng.randint(2, 10)
    k = rng.randint(1, min(4, E))
    T = 6
    if seed % 2 == 0:   # many exact ties: small integer logits, zero bias
        logits = torch.tensor([[rng.randint(-2, 2) for _ in range(E)] for _ in range(T)], dtype=f64)
        bias = torch.zeros(E)
    else:
        logits = torch.tensor([[rng.gauss(0, 1) for _ in range(E)] for _ in range(T)], dtype=f64)
        bias = torch.tensor([rng.uniform(-0.1, 0.1) for _ in range(E)], dtype=torch.float32)
    sel = oracle.select_topk(logits, bias, k, 1.0, False)
    for t in range(T):
        b = [_s(float(logits[t, e])) + float(bias[e]) for e in range(E)]
        want = _brute_topk(b, k)
        got = sel.ids[t].tolist()
        assert sorted(got) == sorted(want), (t, b, got, want)
        # emitted order: biased descending, equal values by ascending id
        for j in range(k - 1):
            a, c = got[j], got[j + 1]
            assert b[a] > b[c] or (b[a] == b[c] and a < c)
        if k < E:
            rest = sorted((v for e, v in enumerate(b) if e not in got), reverse=True)
            assert float(sel.gap[t]) == pytest.approx(b[got[-1]] - rest[0], abs=1e-15)


# -------------------------------------------------------------- invariants --

@pytest.fixture(scope="module")
def tiny_layer():
    return moe_inputs.make_layer(CONFIGS["tiny"], seed=0)


@pytest.fixture(scope="module")
def tiny_result(tiny_layer):
    return oracle.moe_forward(tiny_layer, keep_hidden=True)


def test_selection_invariants(tiny_layer, tiny_result):
    cfg = tiny_layer.cfg
    sel = tiny_result.selection
    T, E, k = cfg.T, cfg.E, cfg.k
    x = tiny_layer.x.float().tolist()
    wr = tiny_layer.router_w.tolist()
    for t in range(T):
        ids = sel.ids[t].tolist()
        assert len(set(ids)) == k and all(0 <= e < E for e in ids)
        for j, e in enumerate(ids):
            # independent scalar recomputation of the unbiased score
            logit = math.fsum(x[t][h] * wr[e][h] for h in range(cfg.H))
            assert float(sel.weights[t, j]) == pytest.approx(cfg.alpha * _s(logit), rel=1e-13)


def test_renorm_sums_to_alpha():
    cfg = CONFIGS["tiny"].with_(alpha=2.5, renorm=True)
    lay = moe_inputs.make_layer(cfg, seed=3)
    sel = oracle.moe_forward(lay).selection
    assert torch.allclose(sel.weights.sum(1), torch.full((cfg.T,), 2.5, dtype=f64), atol=1e-14)
    s = sel.scores.gather(1, sel.ids)
    assert torch.allclose(sel.weights, 2.5 * s / s.sum(1, keepdim=True), atol=1e-14)


def test_permutation_invariants(tiny_layer, tiny_result):
    cfg = tiny_layer.cfg
    p = tiny_result.perm
    ids = tiny_result.selection.ids.reshape(-1)
    R = cfg.T * cfg.k
    off = p.expert_offsets.tolist()
    assert off[0] == 0 and off[-1] == R
    assert all(off[e] <= off[e + 1] for e in range(cfg.E))
    assert sorted(p.row_of.tolist()) == list(range(R))
    assert (p.src[p.row_of] == torch.arange(R)).all()
    for e in range(cfg.E):
        slots = p.src[off[e]:off[e + 1]].tolist()
        assert all(int(ids[i]) == e for i in slots)
        toks = [i // cfg.k for i in slots]
        assert toks == sorted(toks) and len(set(toks)) == len(toks)
    counts = torch.bincount(ids, minlength=cfg.E)
    assert [off[e + 1] - off[e] for e in range(cfg.E)] == counts.tolist()


def test_expert_relabel_invariance(tiny_layer, tiny_result):
    """Relabel experts by a random permutation pi (router rows, bias and
    expert weights move together): the output is unchanged and the ids map
    through pi."""
    cfg = tiny_layer.cfg
    g = torch.Generator().manual_seed(7)
    pi = torch.randperm(cfg.E, generator=g)           # new id of old expert e
    inv = torch.argsort(pi)                           # old id of new expert e'
    lay2 = LayerInputs(cfg, tiny_layer.x, tiny_layer.router_w[inv], tiny_layer.correction_bias[inv],
                    tiny_layer.w_gate_up[inv], tiny_layer.w_down[inv], None, None,
                    tiny_layer.shared_w_gate_up, tiny_layer.shared_w_down)
    res2 = oracle.moe_forward(lay2)
    assert (res2.selection.ids == pi[tiny_result.selection.ids]).all()
    assert torch.allclose(res2.out, tiny_result.out, rtol=1e-12, atol=1e-12)


def test_combine_slot_order_invariance(tiny_layer, tiny_result):
    """Shuffling the k slots of each token (weights follow their ids) leaves
    the output unchanged."""
    ids = tiny_result.selection.ids
    g = torch.Generator().manual_seed(11)
    shuffled = torch.stack([row[torch.randperm(row.numel(), generator=g)] for row in ids])
    res2 = oracle.moe_forward(tiny_layer, ids_override=shuffled)
    assert torch.allclose(res2.out, tiny_result.out, rtol=1e-12, atol=1e-12)


def test_sampled_tokens_match_full(tiny_layer, tiny_result):
    toks = [0, 5, 17, 63]
    res = oracle.moe_forward(tiny_layer, tokens=toks)
    assert torch.allclose(res.out, tiny_result.out[toks], rtol=1e-12, atol=1e-12)
    assert (res.selection.ids == tiny_result.selection.ids[toks]).all()


# ------------------------------------------------ library special cases ----

def _textbook_swiglu_ffn(v, wgu, wd):
    I = wd.shape[1]
    return F.linear(F.silu(F.linear(v, wgu[:I])) * F.linear(v, wgu[I:]), wd)


def test_unclamped_ffn_is_textbook_swiglu():
    g = torch.Generator().manual_seed(1)
    v = torch.randn(5, 24, generator=g, dtype=f64) * 3
    wgu = torch.randn(2 * 7, 24, generator=g, dtype=f64)
    wd = torch.randn(24, 7, generator=g, dtype=f64)
    got = oracle.expert_ffn(v, wgu, wd, math.inf)
    assert torch.allclose(got, _textbook_swiglu_ffn(v, wgu, wd), rtol=1e-12, atol=1e-12)
    # a finite limit far above every pre-activation is the same map
    assert torch.allclose(oracle.expert_ffn(v, wgu, wd, 1e6), got, rtol=1e-12, atol=1e-12)


def test_single_expert_layer_is_dense_sum():
    """E = 1, k = 1 with renormalisation: every token's weight is alpha, and
    out = FFN_shared(x) + alpha * FFN_0(x) (unclamped: textbook SwiGLU)."""
    cfg = LayerConfig("one", T=9, H=16, E=1, k=1, I=8, I_s=12, swiglu_limit=math.inf,
                      alpha=2.5, renorm=True)
    lay = moe_inputs.make_layer(cfg, seed=5)
    res = oracle.moe_forward(lay)
    assert (res.selection.ids == 0).all()
    assert torch.allclose(res.selection.weights, torch.full((9, 1), 2.5, dtype=f64), atol=0)
    x = lay.x.to(f64)
    want = (_textbook_swiglu_ffn(x, lay.shared_w_gate_up.to(f64), lay.shared_w_down.to(f64))
            + 2.5 * _textbook_swiglu_ffn(x, lay.w_gate_up[0].to(f64), lay.w_down[0].to(f64)))
    assert torch.allclose(res.out, want, rtol=1e-12, atol=1e-12)


def test_w4a16_layer_reduces_to_bf16_layer():
    """A W4A16 layer whose dequantised weights are exactly representable in
    bf16 (codes * power-of-two scales) gives the same output as the bf16
    layer holding those weights.  Packing: low nibble = even k."""
    cfg = LayerConfig("w4", T=6, H=256, E=3, k=2, I=128, I_s=128, alpha=2.5, renorm=True,
                      w4a16=True)
    g = torch.Generator().manual_seed(2)
    base = moe_inputs.make_layer(cfg.with_(w4a16=False), seed=9)

    def pack(E, N, K):
        codes = torch.randint(0, 16, (E, N, K), generator=g, dtype=torch.int64)
        sc = 2.0 ** (-torch.randint(4, 9, (E, N, K // 128), generator=g)).to(torch.float64)
        w = (codes.to(f64) - 8) * sc.repeat_interleave(128, dim=2)
        q = (codes[..., 0::2] | (codes[..., 1::2] << 4)).to(torch.uint8)
        return q, sc.to(torch.bfloat16), w.to(torch.bfloat16)

    qgu, sgu, wgu = pack(cfg.E, 2 * cfg.I, cfg.H)
    qd, sd, wd = pack(cfg.E, cfg.H, cfg.I)
    lay4 = LayerInputs(cfg, base.x, base.router_w, base.correction_bias, qgu, qd, sgu, sd,
                    base.shared_w_gate_up, base.shared_w_down)
    lay16 = LayerInputs(cfg.with_(w4a16=False), base.x, base.router_w, base.correction_bias,
                     wgu, wd, None, None, base.shared_w_gate_up, base.shared_w_down)
    a, b = oracle.moe_forward(lay4), oracle.moe_forward(lay16)
    assert (a.selection.ids == b.selection.ids).all()
    assert torch.allclose(a.out, b.out, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------ input recipe --

def test_skew_calibration_matches(golden_dir):
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "make_skew_calibration", os.path.join(golden_dir, "make_skew_calibration.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    res = mod.calibrate()
    with open(os.path.join(golden_dir, "skew_calibration.json")) as f:
        stored = json.load(f)
    assert res == stored
    assert res["bias_scale"] == SKEW_BIAS_SCALE
    assert res["zero_token_experts"] >= 8
    assert res["max_load"] / res["median_nonzero_load"] > 50


def test_generator_is_deterministic():
    a = moe_inputs.make_layer(CONFIGS["tiny"], seed=0)
    b = moe_inputs.make_layer(CONFIGS["tiny"], seed=0)
    for name in ("x", "router_w", "correction_bias", "w_gate_up", "w_down",
                 "shared_w_gate_up", "shared_w_down"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
    c = moe_inputs.make_layer(CONFIGS["tiny"], seed=1)
    assert not torch.equal(a.x, c.x)


# ------------------------------------------------- expert parallelism ----

@pytest.mark.parametrize("world", [2, 3])
def test_partials_over_a_partition_add_up_to_the_layer(tiny_layer, tiny_result, world):
    """Expert ranges partitioning [0, E) and shared-feature slices partitioning
    [0, I_s): the ranks' partial sums add up to the layer output (the one
    all-reduce of glm5next §One all-reduce)."""
    cfg = tiny_layer.cfg
    # plain index arithmetic for the partition (independent of any product helper)
    e_cuts = [round(i * cfg.E / world) for i in range(world + 1)]
    s_cuts = [8 * round(i * (cfg.I_s // 8) / world) for i in range(world + 1)]
    total = torch.zeros_like(tiny_result.out)
    for r in range(world):
        total += oracle.moe_partial(tiny_layer, e_cuts[r], e_cuts[r + 1], s_cuts[r], s_cuts[r + 1])
    assert torch.allclose(total, tiny_result.out, rtol=1e-12, atol=1e-12)


def test_partial_of_everything_is_the_layer_and_of_nothing_is_zero(tiny_layer, tiny_result):
    cfg = tiny_layer.cfg
    assert torch.allclose(oracle.moe_partial(tiny_layer, 0, cfg.E, 0, cfg.I_s), tiny_result.out, rtol=1e-12,
                          atol=1e-12)
    assert torch.count_nonzero(oracle.moe_partial(tiny_layer, 3, 3, 16, 16)) == 0


def test_hand_layer_partials(hand):
    """The one-token hand layer: expert 0's rank holds 0.5*y0, expert 1's
    s1*y1, the shared slice holds [s1, s1] (closed forms of the layer's
    worked output: out = [s1, s1] + 0.5 [3 s1, -6 s1] + s1 [s1, s1])."""
    lay = _hand_layer(hand)
    s1 = _s(1.0)
    p0 = oracle.moe_partial(lay, 0, 1, 0, 0)[0].tolist()
    p1 = oracle.moe_partial(lay, 1, 4, 0, 0)[0].tolist()
    ps = oracle.moe_partial(lay, 4, 4, 0, 1)[0].tolist()
    assert p0 == pytest.approx([1.5 * s1, -3.0 * s1], abs=1e-14)
    assert p1 == pytest.approx([s1 * s1, s1 * s1], abs=1e-14)
    assert ps == pytest.approx([s1, s1], abs=1e-14)
