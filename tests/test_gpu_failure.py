"""Device-side failure handling, exercised without a GPU fault.

The tensor-core kernels bound every wait on another role's progress; when a
wait runs out the kernel records MOE_ERR_DEVICE_TIMEOUT in the workspace
error word, drains its own copies and MMAs, frees its tensor memory and
returns.  moe_selftest_device_timeout runs the split-K tensor-core GEMM on
one tiny tile with the "MMAs finished" signal withheld and a 20 ms limit, so
the epilogue's wait is the one that runs out; moe_selftest_pair_timeout does
the same to the grouped GEMMs that run on CTA pairs (bf16 and int4), whose
two CTAs must both leave through their cluster barrier and reset the tile
queue.  The tests check that the status reaches the host, that reading it
clears it, that the tile-queue words are back at zero, and that the context
still computes a correct layer afterwards.
"""

import time

import pytest
import torch

import moe_inputs
import oracle
from moe_inputs.configs import CONFIGS
from routed_swiglu_experts_b200 import _abi

from gpu_util import TOL_BF16, TOL_W4A16, cuda_available, gpu_layer, rel_err

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]


def test_forced_wait_timeout_is_reported_and_context_survives():
    dev = torch.device("cuda")
    scratch = torch.zeros(_abi.MOE_SELFTEST_SCRATCH_BYTES, dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    _abi.moe_selftest_device_timeout(scratch)
    code = _abi.moe_read_device_error(scratch)
    elapsed = time.perf_counter() - t0
    assert code == _abi.MOE_ERR_DEVICE_TIMEOUT
    assert elapsed < 2.0, f"the 20 ms wait limit took {elapsed:.2f} s to fire"
    assert _abi.moe_read_device_error(scratch) == 0  # reading clears it

    # the same process keeps computing correct results
    inp = moe_inputs.make_layer(CONFIGS["tiny"], seed=0)
    layer = gpu_layer(inp)
    ids = torch.empty(inp.cfg.T, inp.cfg.k, dtype=torch.int32, device=dev)
    out = layer.forward(inp.x.to(dev), topk_ids=ids)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    ref = oracle.moe_forward(inp, ids_override=ids.cpu().long())
    assert rel_err(out.cpu(), ref.out) <= TOL_BF16


@pytest.mark.parametrize("kernel", [_abi.MOE_SELFTEST_PAIR_BF16, _abi.MOE_SELFTEST_PAIR_INT4])
def test_pair_kernel_timeout_is_reported_and_context_survives(kernel):
    dev = torch.device("cuda")
    scratch = torch.zeros(_abi.MOE_SELFTEST_SCRATCH_BYTES, dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    _abi.moe_selftest_pair_timeout(scratch, kernel)
    code = _abi.moe_read_device_error(scratch)
    elapsed = time.perf_counter() - t0
    assert code == _abi.MOE_ERR_DEVICE_TIMEOUT
    assert elapsed < 2.0, f"the 20 ms wait limit took {elapsed:.2f} s to fire"
    header = scratch[:256].view(torch.int32).cpu()
    assert torch.count_nonzero(header[2:10]).item() == 0, f"tile queue words {header[2:10].tolist()}"
    assert _abi.moe_read_device_error(scratch) == 0  # reading clears it

    # the same process keeps computing correct results with the same kernel
    from moe_inputs.configs import LayerConfig
    cfg = (CONFIGS["tiny"] if kernel == _abi.MOE_SELFTEST_PAIR_BF16 else
           LayerConfig("w4a16_prefill_after_timeout", T=300, H=256, E=4, k=2, I=256, I_s=128, w4a16=True))
    inp = moe_inputs.make_layer(cfg, seed=0)
    layer = gpu_layer(inp)
    ids = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=dev)
    out = layer.forward(inp.x.to(dev), topk_ids=ids)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    ref = oracle.moe_forward(inp, ids_override=ids.cpu().long())
    assert rel_err(out.cpu(), ref.out) <= (TOL_W4A16 if cfg.w4a16 else TOL_BF16)
