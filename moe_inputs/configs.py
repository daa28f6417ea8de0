"""The five layer shapes the routed-MoE benchmark is stated on.

Sizes only; nothing here computes any part of the layer.
"""

from __future__ import annotations

import dataclasses

# Scale ``a`` of the skewed-load correction bias  bias_e = a * log p_e
# (p = normalised Zipf(1.2)).  The benchmark text for this layer is garbled
# ("2.0*log(1/(e+1))-normalised Zipf"); read literally (a = 2.0) nearly every
# token goes to experts 0..7, which contradicts its own "loads span ~100x".
# ``a`` is therefore calibrated: the smallest value on the grid 0.100, 0.105,
# ... for which at least 8 of the 128 experts receive zero tokens under the
# exact (fp64) router on the seed-0 inputs.  The value is written by
# tests/golden/make_skew_calibration.py and re-checked by the CPU tests.
SKEW_BIAS_SCALE = 0.125


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int           # tokens
    H: int           # hidden
    E: int           # routed experts
    k: int           # top_k
    I: int           # expert intermediate
    I_s: int         # shared-expert intermediate (0 = none)
    swiglu_limit: float = 7.0
    alpha: float = 1.0          # routed_scaling_factor
    renorm: bool = False        # renormalise the top-k weights before alpha
    bias_kind: str = "uniform"  # uniform | zipf | zero
    bias_range: float = 0.1
    zipf_s: float = 1.2
    bias_scale: float = 0.0
    w4a16: bool = False
    nvfp4: bool = False         # NVFP4 routed experts (e2m1 codes, e4m3 scale per 16, fp32 per expert)
    x_scale: float = 1.0        # x ~ N(0, x_scale^2) (1 in every benchmark layer)

    @property
    def R(self) -> int:
        return self.T * self.k

    def with_(self, **kw) -> "LayerConfig":
        return dataclasses.replace(self, **kw)


TINY = LayerConfig("tiny", T=64, H=128, E=8, k=2, I=64, I_s=64,
                   alpha=1.0, renorm=False, bias_range=0.1)
MID = LayerConfig("mid", T=4096, H=2048, E=64, k=6, I=1408, I_s=2816,
                  alpha=2.5, renorm=True, bias_range=0.1)
LARGE = LayerConfig("large_prefill", T=16384, H=6144, E=256, k=8, I=2048,
                    I_s=2048, alpha=2.5, renorm=True, bias_range=0.05)
SKEWED = LayerConfig("skewed", T=8192, H=4096, E=128, k=8, I=1536, I_s=1536,
                     alpha=1.0, renorm=False, bias_kind="zipf", zipf_s=1.2,
                     bias_scale=SKEW_BIAS_SCALE)
DECODE_W4A16 = LayerConfig("decode_w4a16", T=32, H=6144, E=256, k=8, I=2048,
                           I_s=2048, alpha=2.5, renorm=True, bias_range=0.05,
                           w4a16=True)

# Not one of the five benchmark layers: the large prefill shape with the
# decode layer's int4 group-128 expert weights, for the grouped W4A16 GEMM.
PREFILL_W4A16 = LayerConfig("prefill_w4a16", T=16384, H=6144, E=256, k=8, I=2048,
                            I_s=2048, alpha=2.5, renorm=True, bias_range=0.05,
                            w4a16=True)

# Not benchmark layers either: the decode and the large prefill shapes with
# NVFP4 expert weights (the routed NVFP4 MoE the module summary names).
DECODE_NVFP4 = LayerConfig("decode_nvfp4", T=32, H=6144, E=256, k=8, I=2048,
                           I_s=2048, alpha=2.5, renorm=True, bias_range=0.05,
                           nvfp4=True)
PREFILL_NVFP4 = LayerConfig("prefill_nvfp4", T=16384, H=6144, E=256, k=8, I=2048,
                            I_s=2048, alpha=2.5, renorm=True, bias_range=0.05,
                            nvfp4=True)

CONFIGS = {c.name: c for c in (TINY, MID, LARGE, SKEWED, DECODE_W4A16, PREFILL_W4A16, DECODE_NVFP4,
                               PREFILL_NVFP4)}
