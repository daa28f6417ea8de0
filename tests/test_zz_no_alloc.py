"""moe_permute_no_alloc: the permute for callers that cannot allocate device
memory on their enqueue path (plugins and serving loops that own all device
memory and only pass input/output buffers).  Its scratch is a fixed array
inside the library instead of a caller workspace.

Checked through the C ABI against moe_permute (which takes a workspace) on
three calls in a row with different shapes, so leftovers of one call in the
shared scratch would show up in the next; the last one sits exactly at the
scratch's limit (T*k == MOE_NO_ALLOC_MAX_ROWS, E == MOE_MAX_EXPERTS).  Integer and copy outputs
must match bit for bit.  This file is collected last on purpose."""

import pytest
import torch

from routed_swiglu_experts_b200 import _abi

pytestmark = pytest.mark.gpu


def _case(T, H, E, k, seed):
    g = torch.Generator().manual_seed(seed)
    ids = torch.rand(T, E, generator=g).topk(k, dim=1).indices.to(torch.int32)   # k distinct experts
    w = torch.rand(T, k, generator=g)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    cfg = _abi.make_config(H, E, k, 64, 0, 7.0, 1.0, False)
    return cfg, ids.cuda(), w.cuda(), x.cuda()


def _outputs(T, H, E, k):
    R = T * k
    i32 = dict(dtype=torch.int32, device="cuda")
    return (torch.full((E + 1,), -1, **i32), torch.full((R,), -1, **i32), torch.full((R,), -1, **i32),
            torch.full((R,), -1.0, dtype=torch.float32, device="cuda"),
            torch.zeros(R, H, dtype=torch.bfloat16, device="cuda"))


def test_no_alloc_permute_matches_workspace_permute():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    # the mid layer's shape, a ragged small one, then the scratch's limit:
    # T * k == MOE_NO_ALLOC_MAX_ROWS with E == MOE_MAX_EXPERTS uses every
    # (chunk, expert) count slot and the last per-slot rank
    limit_T = _abi.MOE_NO_ALLOC_MAX_ROWS // 8
    for (T, H, E, k, seed) in [(4096, 2048, 64, 6, 0), (333, 200, 5, 3, 1),
                               (limit_T, 64, _abi.MOE_MAX_EXPERTS, 8, 2)]:
        cfg, ids, w, x = _case(T, H, E, k, seed)
        ws = torch.empty(_abi.moe_workspace_size(cfg, T), dtype=torch.uint8, device="cuda")
        _abi.moe_workspace_init(ws)
        ref = _outputs(T, H, E, k)
        _abi.moe_permute(cfg, ids, w, x, T, *ref, ws)
        got = _outputs(T, H, E, k)
        _abi.moe_permute_no_alloc(cfg, ids, w, x, T, *got)
        torch.cuda.synchronize()
        for name, a, b in zip(("expert_offsets", "row_of", "src", "w_perm", "x_perm"), got, ref):
            assert torch.equal(a, b), f"T={T}: {name} differs from moe_permute"
        assert int(ref[0][-1]) == T * k


def test_no_alloc_permute_rejects_batches_above_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    k = 8
    T = _abi.MOE_NO_ALLOC_MAX_ROWS // k + 1
    cfg = _abi.make_config(128, 16, k, 64, 0, 7.0)
    buf = torch.empty(16, dtype=torch.int32, device="cuda")    # never touched: rejected on the host
    with pytest.raises(_abi.MoEError) as ei:
        _abi.moe_permute_no_alloc(cfg, buf, buf, buf, T, buf, buf, buf, buf, buf)
    assert ei.value.status == _abi.MOE_ERR_UNSUPPORTED
