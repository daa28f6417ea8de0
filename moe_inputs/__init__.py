"""Seeded synthetic inputs for the routed MoE SwiGLU layer.

This module is shared by the CUDA path (tests, bench) and by the CPU oracle.
It draws random tensors and nothing else: it holds none of the layer's
arithmetic (no router, no top-k, no SwiGLU, no combine).

Workload shapes follow the five layer configurations of the routed-MoE
benchmark (tiny, mid, large prefill, skewed load, W4A16 decode).  The value
distributions follow their statement: activations ~N(0,1) in bf16, expert
and shared weights ~N(0, 1/fan_in) in bf16 (fan_in = hidden for gate/up and
the router, intermediate for down), fp32 router weights ~N(0, 1/hidden),
correction bias ~U(-b, b), and for the W4A16 layer uint4 codes ~U{0..15}
packed two per byte (low nibble = even k) with bf16 per-group scales
~U(0.005, 0.02), group 128 along K.  NVFP4 layers (not one of the five):
e2m1 codes ~U{0..15} packed the same way, one FP8 E4M3 scale byte per 16
along K drawn uniformly from 0x30..0x3F (the E4M3 values 0.5 .. 1.875), and
one fp32 scale per expert and projection ~U(0.25, 0.35) / sqrt(fan_in) --
the bytes are drawn, never decoded, here.

Draw order (one ``torch.Generator`` per device):
  CPU generator, seed s:    x, router weight, correction bias
  weight-device generator,  seed s + 1:
                            routed gate/up, routed down, shared gate/up,
                            shared down  (W4A16: codes and scales per tensor;
                            NVFP4: codes, scale bytes and fp32 scales per
                            tensor)

The routed/shared weights come from a generator on ``weight_device`` so the
multi-GB layers can be drawn on the GPU in well under a second; their values
therefore depend on that device, and every consumer of one ``LayerInputs``
object (CUDA path and oracle alike) sees exactly the same tensors.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

from .configs import CONFIGS, LayerConfig, SKEW_BIAS_SCALE  # noqa: F401

__all__ = ["CONFIGS", "LayerConfig", "LayerInputs", "make_layer", "make_x",
           "zipf_log_bias", "SKEW_BIAS_SCALE"]


@dataclasses.dataclass
class LayerInputs:
    """All inputs of one MoE layer call.  Shapes use T, H, E, k, I, I_s."""
    cfg: LayerConfig
    x: torch.Tensor                 # [T, H] bf16
    router_w: torch.Tensor          # [E, H] fp32
    correction_bias: torch.Tensor   # [E] fp32
    w_gate_up: torch.Tensor         # bf16 [E, 2I, H]  | uint8 [E, 2I, H/2]
    w_down: torch.Tensor            # bf16 [E, H, I]   | uint8 [E, H, I/2]
    s_gate_up: Optional[torch.Tensor]  # bf16 [E, 2I, H/128] (W4A16) | uint8 [E, 2I, H/16] (NVFP4)
    s_down: Optional[torch.Tensor]     # bf16 [E, H, I/128]  (W4A16) | uint8 [E, H, I/16]  (NVFP4)
    shared_w_gate_up: Optional[torch.Tensor]  # bf16 [2I_s, H]
    shared_w_down: Optional[torch.Tensor]     # bf16 [H, I_s]
    g_gate_up: Optional[torch.Tensor] = None  # fp32 [E] (NVFP4 only)
    g_down: Optional[torch.Tensor] = None     # fp32 [E] (NVFP4 only)

    def to(self, device) -> "LayerInputs":
        def mv(t):
            return None if t is None else t.to(device)
        return dataclasses.replace(
            self, x=mv(self.x), router_w=mv(self.router_w),
            correction_bias=mv(self.correction_bias),
            w_gate_up=mv(self.w_gate_up), w_down=mv(self.w_down),
            s_gate_up=mv(self.s_gate_up), s_down=mv(self.s_down),
            shared_w_gate_up=mv(self.shared_w_gate_up),
            shared_w_down=mv(self.shared_w_down),
            g_gate_up=mv(self.g_gate_up), g_down=mv(self.g_down))


def _normal(shape, std, gen, device, dtype=torch.bfloat16):
    # Sample in fp32 then round to the storage type (bf16: round to nearest even).
    t = torch.empty(shape, dtype=torch.float32, device=device)
    t.normal_(0.0, std, generator=gen)
    return t.to(dtype)


def _uniform(shape, lo, hi, gen, device, dtype=torch.float32):
    t = torch.empty(shape, dtype=torch.float32, device=device)
    t.uniform_(lo, hi, generator=gen)
    return t.to(dtype)


def zipf_log_bias(num_experts: int, s: float, scale: float) -> torch.Tensor:
    """Skewed-load correction bias: bias_e = scale * log p_e, where p is the
    normalised Zipf(s) law p_e = (e+1)^-s / sum_j (j+1)^-s.  (Input recipe,
    not layer arithmetic.)"""
    e = torch.arange(num_experts, dtype=torch.float64)
    p = (e + 1.0) ** (-s)
    p = p / p.sum()
    return (scale * torch.log(p)).to(torch.float32)


def make_x(cfg: LayerConfig, seed: int = 0, T: Optional[int] = None):
    """Only the CPU-generator part (x, router weight, bias).  ``T`` overrides
    the token count (the draw is then a different tensor)."""
    T = cfg.T if T is None else T
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = _normal((T, cfg.H), cfg.x_scale, g, "cpu")
    router_w = _normal((cfg.E, cfg.H), 1.0 / math.sqrt(cfg.H), g, "cpu",
                       dtype=torch.float32)
    if cfg.bias_kind == "uniform":
        bias = _uniform((cfg.E,), -cfg.bias_range, cfg.bias_range, g, "cpu")
    elif cfg.bias_kind == "zipf":
        bias = zipf_log_bias(cfg.E, cfg.zipf_s, cfg.bias_scale)
    elif cfg.bias_kind == "zero":
        bias = torch.zeros(cfg.E, dtype=torch.float32)
    else:
        raise ValueError(cfg.bias_kind)
    return x, router_w, bias


def make_layer(cfg: LayerConfig, seed: int = 0, weight_device="cpu",
               T: Optional[int] = None) -> LayerInputs:
    """Draw one layer's inputs.  x / router / bias are always on the CPU;
    the expert and shared weights live on ``weight_device``."""
    x, router_w, bias = make_x(cfg, seed, T)
    dev = torch.device(weight_device)
    g = torch.Generator(device=dev).manual_seed(seed + 1)
    E, H, I, Is = cfg.E, cfg.H, cfg.I, cfg.I_s
    g_gu = g_d = None

    def codes(shape):
        # two independent U{0..15} nibbles == one uniform byte
        t = torch.empty(shape, dtype=torch.uint8, device=dev)
        return t.random_(0, 256, generator=g)

    def scale_bytes(shape):
        t = torch.empty(shape, dtype=torch.uint8, device=dev)
        return t.random_(0x30, 0x40, generator=g)

    if cfg.nvfp4:
        q_gu = codes((E, 2 * I, H // 2))
        s_gu = scale_bytes((E, 2 * I, H // 16))
        g_gu = _uniform((E,), 0.25 / math.sqrt(H), 0.35 / math.sqrt(H), g, dev)
        q_d = codes((E, H, I // 2))
        s_d = scale_bytes((E, H, I // 16))
        g_d = _uniform((E,), 0.25 / math.sqrt(I), 0.35 / math.sqrt(I), g, dev)
        w_gu, w_d = q_gu, q_d
    elif cfg.w4a16:
        q_gu = codes((E, 2 * I, H // 2))
        s_gu = _uniform((E, 2 * I, H // 128), 0.005, 0.02, g, dev, torch.bfloat16)
        q_d = codes((E, H, I // 2))
        s_d = _uniform((E, H, I // 128), 0.005, 0.02, g, dev, torch.bfloat16)
        w_gu, w_d = q_gu, q_d
    else:
        w_gu = _normal((E, 2 * I, H), 1.0 / math.sqrt(H), g, dev)
        w_d = _normal((E, H, I), 1.0 / math.sqrt(I), g, dev)
        s_gu = s_d = None
    if Is > 0:
        sgu = _normal((2 * Is, H), 1.0 / math.sqrt(H), g, dev)
        sd = _normal((H, Is), 1.0 / math.sqrt(Is), g, dev)
    else:
        sgu = sd = None
    return LayerInputs(cfg, x, router_w, bias, w_gu, w_d, s_gu, s_d, sgu, sd, g_gu, g_d)
