"""The quantities bench.py reports beside its timings, checked on the CPU
against facts fixed independently of the code that computes them: the FLOP
count of the layer from its shapes, the kernels one forward launches (as
listed by the committed ncu launch lists), the bytes a W4A16 expert holds
(from the weight format: two codes per byte, one bf16 scale per 128
weights), and the rule that a DRAM traffic figure is reported only while the
profiled kernel source is unchanged."""

import datetime
import hashlib
import json
import os
import sys

import pytest

import bench
from moe_inputs.configs import CONFIGS


def test_gemm_flops_of_the_mid_layer():
    cfg = CONFIGS["mid"]
    routed, shared = bench.gemm_flops(cfg)
    R = 4096 * 6
    # gate/up: 2 * R * H * 2I; down: 2 * R * I * H
    assert routed == 2 * R * 2048 * 2 * 1408 + 2 * R * 1408 * 2048 == 425_201_762_304
    assert shared == 2 * 4096 * 2048 * 2 * 2816 + 2 * 4096 * 2816 * 2048 == 141_733_920_768


@pytest.mark.parametrize("name,expected", [
    # router split + tensor-core logits + top-k, count/rank (+ scan) + scatter,
    # gate/up + down (shared expert as a second problem), combine
    ("mid", 8),
    ("large_prefill", 8),
    # ... + W4A16 (prep + GEMV) x 2, the shared expert inside the GEMV launches
    ("decode_w4a16", 10),
    # ... + token prep + dequantising gate/up and down + bf16 shared gate/up
    # and down launches
    ("prefill_w4a16", 11),
    # NVFP4 experts take the same two paths by the same rule
    ("decode_nvfp4", 10),
    ("prefill_nvfp4", 11),
])
def test_launches_per_step_match_the_launch_lists(name, expected):
    assert bench.launches_per_step(CONFIGS[name]) == expected


def test_launch_list_of_the_mid_layer_has_eight_kernels_per_forward():
    """The committed launch list names eight distinct kernels of one forward;
    each appears once per forward (the FFN kernel twice: gate/up and down)."""
    text = open(os.path.join(bench.ROOT, "profiles", "launches_mid.md")).read()
    kernels = {"ffn_pair_kernel<GateUp>", "ffn_pair_kernel<Down>", "combine_kernel", "perm_scatter_kernel",
               "router_topk_rows_kernel", "splitk_gemm_kernel", "perm_count_rank_kernel", "router_split_kernel"}
    for k in kernels:
        assert f"| {k}" in text, k
    assert len(kernels) == bench.launches_per_step(CONFIGS["mid"])


def test_w4a16_bytes_of_one_touched_expert():
    import torch
    cfg = CONFIGS["decode_w4a16"]
    ids = torch.tensor([[3, 3], [3, 3]])  # one touched expert
    touched, total = bench.w4a16_bytes(cfg, ids)
    H, I, Is, T, k = 6144, 2048, 2048, cfg.T, cfg.k
    codes = (2 * I * H + H * I) // 2            # two 4-bit codes per byte
    scales = 2 * (2 * I * H + H * I) // 128      # one bf16 per 128 weights
    shared = 2 * (3 * H * Is)                    # bf16 shared expert
    acts = 2 * T * H * (2 + 2 * k)
    assert touched == 1
    assert codes + scales == 19_464_192
    assert total == codes + scales + shared + acts


def test_nvfp4_bytes_of_one_touched_expert():
    import torch
    cfg = CONFIGS["decode_nvfp4"]
    touched, total = bench.w4a16_bytes(cfg, torch.tensor([[7, 7]]))
    H, I, Is, T, k = 6144, 2048, 2048, cfg.T, cfg.k
    codes = (2 * I * H + H * I) // 2            # two E2M1 codes per byte
    scales = (2 * I * H + H * I) // 16          # one E4M3 byte per 16 weights
    assert touched == 1
    assert total == codes + scales + 8 + 2 * (3 * H * Is) + 2 * T * H * (2 + 2 * k)


def test_traffic_is_reported_only_for_the_profiled_source(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cu"
    src.write_bytes(b"// kernel v1\n")
    sha = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"grouped_ffn_x": {"source": "kernel.cu", "source_sha256_16": sha, "dram_bytes_per_call": 1234}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_from_profile("grouped_ffn_x") == 1234
    assert bench.traffic_from_profile("grouped_ffn_y") is None
    src.write_bytes(b"// kernel v2\n")  # the kernel changed after the capture
    assert bench.traffic_from_profile("grouped_ffn_x") is None


def test_clock_sampler_drains_a_pipe_larger_than_its_buffer():
    """The sampler reads its nvidia-smi child's output as it comes: a run
    longer than a pipe buffer's worth of samples neither stalls the child
    nor loses the later samples, and finish() returns promptly."""
    import subprocess
    import threading
    import time

    line = "2026/12/03 10:00:00.000, 1965, 1965, Not Active, Not Active, Not Active, Active"
    n = 20000  # about 1.7 MB: far more than a 64 KB pipe buffer
    c = bench.ClockSampler.__new__(bench.ClockSampler)
    c.lines, c.windows = [], []
    c.proc = subprocess.Popen([sys.executable, "-c", f"import sys\nfor _ in range({n}): print({line!r})"],
                              stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
    c.reader = threading.Thread(target=c._drain, daemon=True)
    c.reader.start()
    assert c.proc.wait(timeout=60) == 0  # the child never blocks on a full pipe
    ts = datetime.datetime.strptime(line.split(",")[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
    c.mark(ts - 1, ts + 1)
    t0 = time.time()
    res = c.finish()
    assert time.time() - t0 < 15
    assert res["samples"] == n and res["sm_mhz"] == 1965.0 and res["reasons"] == ["sw_power_cap"]


def test_reference_arm_prints_the_contract_line(capsys):
    """`bench.py --impl reference` times the oracle on the host (no GPU) and
    prints one JSON line with the contract's keys, on a layer with fewer
    tokens than its default per-step sample."""
    import json
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3", "--workload", "tiny"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e", "gpu_launches"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["gpu_launches"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert "64 of the 64 tokens" in line["cpu_baseline"]["sample"]
