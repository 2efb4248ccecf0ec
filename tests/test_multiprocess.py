"""Host logic of the multi-GPU path on CPU: greedy layer assignment and the
one-AllGather replication of updated weights, as world-size-2 gloo ranks.
The per-rank step is a host stand-in here; on GPUs it is BlockedShampoo."""
import os
import socket

import numpy as np
import pytest

from matrix_roots_b200 import distributed as D
from matrix_roots_b200 import workloads as W


def test_layer_cost_counts_blocks():
    assert D.layer_cost((1024, 4096), 1024) == 4 * (1024 ** 3 + 1024 ** 3)
    assert D.layer_cost((300, 100), 128) == sum(r ** 3 + 100 ** 3 for r in (128, 128, 44))


def test_assign_layers_greedy_and_balanced():
    shapes = [(2, 2), (1, 1)]
    assert D.assign_layers(shapes, 0, 1) == [0, 0]
    assert D.assign_layers(shapes, 0, 2) == [0, 1]
    shapes = [(16, 16), (8, 8), (12, 12), (12, 12), (4, 4)]
    owner = D.assign_layers(shapes, 0, 2)
    # costs (one block each, m^3 + n^3) 8192, 1024, 3456, 3456, 128; by the
    # hand schedule: 8192 -> r0; 3456 -> r1; 3456 -> r1 (6912 < 8192);
    # 1024 -> r1 (7936 < 8192); 128 -> r1 (8064 < 8192)
    assert owner == [0, 1, 1, 1, 1]
    tr = W.transformer_shapes()
    for world in (2, 4, 8):
        o = D.assign_layers(tr, 1024, world)
        loads = [sum(D.layer_cost(tr[i], 1024) for i in range(len(tr)) if o[i] == k) for k in range(world)]
        assert sorted(set(o)) == list(range(world))
        assert max(loads) <= 1.35 * (sum(loads) / world)


def test_local_config_renumbers_one_sided_layers():
    from matrix_roots_b200.optimizer import ShampooConfig
    cfg = ShampooConfig(block_size=64, one_sided=(1, 4))
    loc = D.local_config(cfg, [4, 0, 2])
    assert loc.one_sided == (0,) and loc.block_size == 64 and cfg.one_sided == (1, 4)
    assert D.local_config(ShampooConfig(), [0, 1]).one_sided == ()
    assert D.local_config(_HostCfg(), [0]) is not None


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


class _HostCfg:
    block_size = 4


def _host_step(Wl, Gl):
    for w, g in zip(Wl, Gl):
        w.sub_(0.5 * g)


def _rank_main(rank, world, port, shapes, out_dir):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(0)  # same data on every rank (data parallel)
        Wt = [torch.from_numpy(rng.standard_normal(s)).float() for s in shapes]
        Gt = [torch.from_numpy(rng.standard_normal(s)).float() for s in shapes]
        opt = D.DistributedShampoo(shapes, _HostCfg(), local_step=_host_step)
        for _ in range(2):
            opt.step(Wt, Gt)
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), *[w.numpy() for w in Wt], owner=np.asarray(opt.owner))
    finally:
        dist.destroy_process_group()


def test_distributed_step_replicates_owned_updates(tmp_path):
    import torch.multiprocessing as mp
    shapes = [(8, 4), (4, 4), (12, 8), (4, 8), (2, 2)]
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), shapes, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    rng = np.random.default_rng(0)
    W0 = [rng.standard_normal(s).astype(np.float32) for s in shapes]
    G0 = [rng.standard_normal(s).astype(np.float32) for s in shapes]
    expect = [w - np.float32(0.5) * g - np.float32(0.5) * g for w, g in zip(W0, G0)]
    outs = [np.load(tmp_path / f"r{r}.npz") for r in range(world)]
    owner = outs[0]["owner"]
    assert set(owner.tolist()) == {0, 1}
    for r in range(world):
        for i in range(len(shapes)):
            np.testing.assert_array_equal(outs[r][f"arr_{i}"], expect[i])
