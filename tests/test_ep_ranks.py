"""Expert parallelism's host side on CPU with gloo ranks: the rank partition
(expert ranges and shared-expert feature slices) and the one all-reduce of
the ranks' partial sums ("Module glm5next_mlp", §One all-reduce for both EP
and TP) reproduce the single-rank layer.  The partials here come from the
oracle; the CUDA path's partials are checked against the oracle's on the GPU
(tests/test_gpu_ep.py)."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from routed_swiglu_experts_b200 import ep


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("E,world", [(8, 2), (8, 3), (5, 4), (3, 4), (256, 8)])
def test_expert_ranges_partition_the_experts(E, world):
    rs = ep.expert_ranges(E, world)
    assert len(rs) == world and rs[0][0] == 0 and rs[-1][1] == E
    assert all(rs[i][1] == rs[i + 1][0] for i in range(world - 1))
    sizes = [e - b for b, e in rs]
    assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 0


@pytest.mark.parametrize("Is,world", [(64, 2), (64, 3), (2816, 8), (8, 2), (0, 2)])
def test_shared_slices_partition_the_features(Is, world):
    ss = ep.shared_slices(Is, world)
    assert ss[0][0] == 0 and ss[-1][1] == Is
    assert all(ss[i][1] == ss[i + 1][0] for i in range(world - 1))
    assert all(b % 8 == 0 and e % 8 == 0 for b, e in ss)


def test_local_tensors_slice_the_right_rows():
    E, I, H, Is = 6, 16, 8, 24
    wgu = torch.arange(E * 2 * I * H).reshape(E, 2 * I, H)
    wd = torch.arange(E * H * I).reshape(E, H, I)
    sgu = torch.arange(2 * Is * H).reshape(2 * Is, H)
    sd = torch.arange(H * Is).reshape(H, Is)
    loc = ep.local_tensors(1, 2, E, Is, w_gate_up=wgu, w_down=wd, shared_w_gate_up=sgu, shared_w_down=sd)
    assert loc["expert_range"] == (3, 6)
    assert torch.equal(loc["w_gate_up"], wgu[3:6]) and torch.equal(loc["w_down"], wd[3:6])
    s0, s1 = loc["shared_slice"]
    assert (s0, s1) == (16, 24)  # 3 units of 8 features: 2 on rank 0, 1 on rank 1
    # gate rows of the slice, then its up rows (gate = shard 0, up = shard 1 of the fused weight)
    assert torch.equal(loc["shared_w_gate_up"], torch.cat([sgu[16:24], sgu[24 + 16:24 + 24]]))
    assert torch.equal(loc["shared_w_down"], sd[:, 16:24])
    assert loc["s_gate_up"] is None and loc["g_gate_up"] is None and loc["g_down"] is None


def test_local_tensors_slice_the_4bit_scales_with_their_experts():
    """Block scales and (NVFP4) per-expert tensor scales follow the rank's
    expert range like the codes they belong to."""
    E, I, H = 5, 16, 32
    q_gu = torch.arange(E * 2 * I * H // 2).reshape(E, 2 * I, H // 2)
    q_d = torch.arange(E * H * I // 2).reshape(E, H, I // 2)
    s_gu = torch.arange(E * 2 * I * H // 16).reshape(E, 2 * I, H // 16)
    s_d = torch.arange(E * H * I // 16).reshape(E, H, I // 16)
    g_gu = torch.arange(E, dtype=torch.float32) + 0.5
    g_d = torch.arange(E, dtype=torch.float32) + 0.25
    for rank in range(2):
        loc = ep.local_tensors(rank, 2, E, 0, w_gate_up=q_gu, w_down=q_d, s_gate_up=s_gu, s_down=s_d,
                               g_gate_up=g_gu, g_down=g_d)
        b, e = loc["expert_range"]
        assert (b, e) == ((0, 3), (3, 5))[rank]
        for name, full in (("w_gate_up", q_gu), ("w_down", q_d), ("s_gate_up", s_gu), ("s_down", s_d),
                           ("g_gate_up", g_gu), ("g_down", g_d)):
            assert torch.equal(loc[name], full[b:e]), name
            assert loc[name].is_contiguous()


def _rank_main(rank, world, port, results):
    import moe_inputs
    import oracle
    from moe_inputs.configs import CONFIGS
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        layer = moe_inputs.make_layer(CONFIGS["tiny"], seed=0)
        cfg = layer.cfg
        b, e = ep.expert_ranges(cfg.E, world)[rank]
        s0, s1 = ep.shared_slices(cfg.I_s, world)[rank]
        part = oracle.moe_partial(layer, b, e, s0, s1)
        ep.all_reduce_partials(part)
        full = oracle.moe_forward(layer).out
        results[rank] = float((part - full).abs().max() / full.abs().max())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_all_reduce_of_partials_gives_the_layer(world):
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), results), nprocs=world, start_method="spawn")
    assert len(results) == world
    assert all(v < 1e-12 for v in results.values()), dict(results)
