"""Plant plausible mistakes in the oracle (on the CPU) and check that the
pins of test_oracle.py catch each one."""

import math

import pytest
import torch

import oracle
import oracle.moe_oracle as om
import test_oracle as pins

f64 = torch.float64


def _patch(monkeypatch, name, fn):
    monkeypatch.setattr(om, name, fn)
    monkeypatch.setattr(oracle, name, fn)


def _sym_clamp(gate, up, limit):            # gate clamped on both sides
    g = torch.clamp(gate, min=-limit, max=limit)
    u = torch.clamp(up, min=-limit, max=limit)
    return (g / (1.0 + torch.exp(-g))) * u


def _no_up_clamp(gate, up, limit):
    g = torch.clamp(gate, max=limit)
    return (g / (1.0 + torch.exp(-g))) * up


def _select_bias_on_logit(logits, bias, k, alpha, renorm):
    b = torch.zeros(logits.shape[1], dtype=f64) if bias is None else bias.to(f64)
    sel = om.Selection.__new__(om.Selection)
    shifted = om._cpu64(logits) + b[None, :]
    real = _orig_select(shifted, None, k, alpha, renorm)
    s = om.sigmoid(om._cpu64(logits))
    chosen = torch.gather(s, 1, real.ids)
    if renorm:
        chosen = chosen / chosen.sum(1, keepdim=True)
    return om.Selection(real.ids, alpha * chosen, s, real.biased, real.gap)


def _select_biased_weight(logits, bias, k, alpha, renorm):
    sel = _orig_select(logits, bias, k, alpha, renorm)
    chosen = torch.gather(sel.biased, 1, sel.ids)
    if renorm:
        chosen = chosen / chosen.sum(1, keepdim=True)
    return om.Selection(sel.ids, alpha * chosen, sel.scores, sel.biased, sel.gap)


def _select_tie_high(logits, bias, k, alpha, renorm):
    E = logits.shape[1]
    flipped = _orig_select(torch.flip(om._cpu64(logits), [1]),
                           None if bias is None else torch.flip(bias, [0]), k, alpha, renorm)
    return om.Selection(E - 1 - flipped.ids, flipped.weights, torch.flip(flipped.scores, [1]),
                        torch.flip(flipped.biased, [1]), flipped.gap)


def _select_renorm_after_alpha(logits, bias, k, alpha, renorm):
    sel = _orig_select(logits, bias, k, 1.0, False)
    w = alpha * sel.weights
    if renorm:
        w = w / w.sum(1, keepdim=True)
    return om.Selection(sel.ids, w, sel.scores, sel.biased, sel.gap)


def _dequant_hi_first(q, scale):
    q = q.detach().cpu()
    N, half = q.shape
    codes = torch.stack([(q >> 4).to(f64), (q & 0xF).to(f64)], -1).reshape(N, 2 * half)
    return (codes - 8.0) * om._cpu64(scale).repeat_interleave(128, dim=1)


def _nvfp4_hi_first(q, block_scale, tensor_scale):      # high nibble taken as the even k
    q = q.detach().cpu()
    N, half = q.shape
    vals = torch.stack([om.e2m1_value(q >> 4), om.e2m1_value(q & 0xF)], -1).reshape(N, 2 * half)
    sc = om.e4m3_value(block_scale.detach().cpu()).repeat_interleave(16, dim=1)
    return vals * sc * float(tensor_scale)


def _nvfp4_block32(q, block_scale, tensor_scale):       # one scale per 32 instead of 16
    q = q.detach().cpu()
    N, half = q.shape
    vals = torch.stack([om.e2m1_value(q & 0xF), om.e2m1_value(q >> 4)], -1).reshape(N, 2 * half)
    sc = om.e4m3_value(block_scale.detach().cpu()).repeat_interleave(32, dim=1)[:, :2 * half]
    return vals * sc * float(tensor_scale)


def _nvfp4_no_tensor_scale(q, block_scale, tensor_scale):
    return _orig_nvfp4(q, block_scale, 1.0)


def _e2m1_bias0(code):                                   # exponent bias 0 instead of 1
    return 2.0 * _orig_e2m1(code)


def _e2m1_no_subnormal(code):                            # exponent field 0 read as normal
    c = code.to(torch.int64)
    v = _orig_e2m1(code)
    sub = ((c >> 1) & 3) == 0
    fixed = torch.where((c & 1) == 1, torch.full_like(v, 0.75), torch.full_like(v, 0.5))
    fixed = torch.where(((c >> 3) & 1) == 1, -fixed, fixed)
    return torch.where(sub, fixed, v)


def _e4m3_bias8(b):                                      # exponent bias 8 instead of 7
    return 0.5 * _orig_e4m3(b)


def _ffn_down_transposed(v, w_gate_up, w_down, limit):
    I = w_down.shape[1]
    gu = v @ w_gate_up.T
    h = om.swiglu_clamped(gu[:, :I], gu[:, I:], limit)
    return h @ w_down.reshape(I, -1)


_orig_select = om.select_topk
_orig_nvfp4 = om.dequant_nvfp4
_orig_e2m1 = om.e2m1_value
_orig_e4m3 = om.e4m3_value


def _expect_fail(fn, *args):
    with pytest.raises(AssertionError):
        fn(*args)


def test_symmetric_gate_clamp_is_caught(monkeypatch, hand):
    _patch(monkeypatch, "swiglu_clamped", _sym_clamp)
    _expect_fail(pins.test_hand_swiglu_clamp, hand)


def test_missing_up_clamp_is_caught(monkeypatch, hand):
    _patch(monkeypatch, "swiglu_clamped", _no_up_clamp)
    _expect_fail(pins.test_hand_swiglu_clamp, hand)


def test_bias_on_logit_is_caught(monkeypatch, hand):
    _patch(monkeypatch, "select_topk", _select_bias_on_logit)
    _expect_fail(pins.test_hand_router_scores_and_selection, hand)


def test_biased_weight_is_caught(monkeypatch, hand):
    _patch(monkeypatch, "select_topk", _select_biased_weight)
    _expect_fail(pins.test_hand_router_scores_and_selection, hand)


def test_tie_to_higher_id_is_caught(monkeypatch, hand):
    _patch(monkeypatch, "select_topk", _select_tie_high)
    _expect_fail(pins.test_hand_tie_goes_to_lower_id, hand)


def test_renorm_after_alpha_is_caught(monkeypatch, hand):
    _patch(monkeypatch, "select_topk", _select_renorm_after_alpha)
    _expect_fail(pins.test_hand_router_scores_and_selection, hand)


def test_nibble_order_is_caught(monkeypatch, hand):
    _patch(monkeypatch, "dequant_int4_g128", _dequant_hi_first)
    _expect_fail(pins.test_hand_w4a16_dequant, hand)


def test_nvfp4_nibble_order_is_caught(monkeypatch, hand_nvfp4):
    _patch(monkeypatch, "dequant_nvfp4", _nvfp4_hi_first)
    _expect_fail(pins.test_hand_nvfp4_dequant, hand_nvfp4)


def test_nvfp4_block_of_32_is_caught(monkeypatch, hand_nvfp4):
    _patch(monkeypatch, "dequant_nvfp4", _nvfp4_block32)
    _expect_fail(pins.test_nvfp4_block_index)


def test_nvfp4_dropped_tensor_scale_is_caught(monkeypatch, hand_nvfp4):
    _patch(monkeypatch, "dequant_nvfp4", _nvfp4_no_tensor_scale)
    _expect_fail(pins.test_hand_nvfp4_dequant, hand_nvfp4)


def test_nvfp4_layer_dispatch_is_caught(monkeypatch, hand_nvfp4):
    _patch(monkeypatch, "dequant_nvfp4", _nvfp4_no_tensor_scale)
    _expect_fail(pins.test_nvfp4_layer_reduces_to_bf16_layer, hand_nvfp4)


def test_e2m1_wrong_bias_is_caught(monkeypatch, hand_nvfp4):
    _patch(monkeypatch, "e2m1_value", _e2m1_bias0)
    _expect_fail(pins.test_e2m1_table, hand_nvfp4)
    _expect_fail(pins.test_hand_nvfp4_dequant, hand_nvfp4)


def test_e2m1_missing_subnormal_is_caught(monkeypatch, hand_nvfp4):
    _patch(monkeypatch, "e2m1_value", _e2m1_no_subnormal)
    _expect_fail(pins.test_e2m1_table, hand_nvfp4)


def test_e4m3_wrong_bias_is_caught(monkeypatch, hand_nvfp4):
    _patch(monkeypatch, "e4m3_value", _e4m3_bias8)
    _expect_fail(pins.test_e4m3_matches_torch_float8)
    _expect_fail(pins.test_e4m3_hand_values, hand_nvfp4)
    _expect_fail(pins.test_hand_nvfp4_dequant, hand_nvfp4)


def test_transposed_down_is_caught(monkeypatch):
    _patch(monkeypatch, "expert_ffn", _ffn_down_transposed)
    _expect_fail(pins.test_unclamped_ffn_is_textbook_swiglu)


def test_scaled_shared_expert_is_caught(monkeypatch):
    orig = om.moe_forward

    def scaled(layer, **kw):
        res = orig(layer, **kw)
        res.out = res.out + (layer.cfg.alpha - 1.0) * res.shared
        return res
    _patch(monkeypatch, "moe_forward", scaled)
    _expect_fail(pins.test_single_expert_layer_is_dense_sum)


def test_dropped_shared_expert_is_caught(monkeypatch, hand):
    orig = om.moe_forward

    def dropped(layer, **kw):
        res = orig(layer, **kw)
        res.out = res.out - res.shared
        return res
    _patch(monkeypatch, "moe_forward", dropped)
    _expect_fail(pins.test_hand_layer_output, hand)


def _override_from_biased(sel, ids, alpha, renorm):      # weights from the biased scores
    ids = ids.to(torch.int64).cpu()
    chosen = torch.gather(sel.biased, 1, ids)
    if renorm:
        chosen = chosen / chosen.sum(1, keepdim=True)
    return om.Selection(ids, alpha * chosen, sel.scores, sel.biased, sel.gap)


def _override_without_renorm(sel, ids, alpha, renorm):    # renormalisation skipped
    ids = ids.to(torch.int64).cpu()
    return om.Selection(ids, alpha * torch.gather(sel.scores, 1, ids), sel.scores, sel.biased, sel.gap)


def test_override_weights_from_biased_scores_are_caught(monkeypatch, hand):
    _patch(monkeypatch, "override_selection", _override_from_biased)
    _expect_fail(pins.test_hand_override_renormalises_the_given_ids, hand)


def test_override_without_renorm_is_caught(monkeypatch, hand):
    _patch(monkeypatch, "override_selection", _override_without_renorm)
    _expect_fail(pins.test_hand_override_renormalises_the_given_ids, hand)


hand = pins.hand
hand_nvfp4 = pins.hand_nvfp4


def test_partial_with_inclusive_range_is_caught(monkeypatch, tiny_layer, tiny_result):
    orig = om.moe_partial

    def inclusive(layer, b, e, s0, s1, **kw):        # the range's end expert counted too
        return orig(layer, b, min(e + 1, layer.cfg.E), s0, s1, **kw)
    _patch(monkeypatch, "moe_partial", inclusive)
    _expect_fail(pins.test_partials_over_a_partition_add_up_to_the_layer, tiny_layer, tiny_result, 2)


def test_partial_with_scaled_shared_slice_is_caught(monkeypatch, tiny_layer, tiny_result):
    orig = om.moe_partial

    def scaled(layer, b, e, s0, s1, **kw):           # shared slice divided by the rank count
        p = orig(layer, b, e, s0, s1, **kw)
        if s1 > s0:
            p = p - 0.5 * orig(layer, b, b, s0, s1, **kw)
        return p
    _patch(monkeypatch, "moe_partial", scaled)
    _expect_fail(pins.test_partials_over_a_partition_add_up_to_the_layer, tiny_layer, tiny_result, 2)


tiny_layer = pins.tiny_layer
tiny_result = pins.tiny_result
