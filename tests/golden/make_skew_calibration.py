"""Calibrate the skewed-load correction-bias scale and write it as a golden file.

The skewed layer's bias is bias_e = a * log p_e with p the normalised
Zipf(1.2) law over the 128 experts.  ``a`` is the smallest value on the grid
0.100, 0.105, ... for which at least 8 experts receive zero tokens when the
seed-0 tokens are routed by the exact (fp64) oracle router.  This script
calls only the input generator and ``oracle/``; it writes
``skew_calibration.json`` next to itself.  ``moe_inputs.configs`` carries the
value as ``SKEW_BIAS_SCALE`` and the CPU tests re-derive it.

    python tests/golden/make_skew_calibration.py
"""

import json
import os
import sys

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import moe_inputs  # noqa: E402
from moe_inputs.configs import SKEWED  # noqa: E402
import oracle  # noqa: E402


def calibrate(seed=0, min_zero=8):
    cfg = SKEWED
    x, router_w, _ = moe_inputs.make_x(cfg, seed)
    logits = oracle.router_logits(x, router_w)
    a = 0.100
    while a < 5.0:
        bias = moe_inputs.zipf_log_bias(cfg.E, cfg.zipf_s, round(a, 3))
        sel = oracle.select_topk(logits, bias, cfg.k, cfg.alpha, cfg.renorm)
        counts = torch.bincount(sel.ids.reshape(-1), minlength=cfg.E)
        zero = int((counts == 0).sum())
        if zero >= min_zero:
            nz = counts[counts > 0].to(torch.float64)
            return {
                "bias_scale": round(a, 3),
                "zero_token_experts": zero,
                "max_load": int(counts.max()),
                "median_nonzero_load": float(nz.median()),
                "min_nonzero_load": int(nz.min()),
                "seed": seed,
                "grid": "0.100 + 0.005 n",
            }
        a += 0.005
    raise RuntimeError("no scale on the grid gives the zero-load experts")


if __name__ == "__main__":
    res = calibrate()
    with open(os.path.join(HERE, "skew_calibration.json"), "w") as f:
        json.dump(res, f, indent=1)
        f.write("\n")
    print(res)
