"""Head partition of one forward across ranks, on CPU.

Every (b, h) is independent, so each rank computes its heads' slice with the
oracle and the gathered result must equal the unsharded oracle bit for bit
(the oracle computes every query row the same way whatever else is in the
call). Two gloo ranks, even and uneven head counts, a shared bias and one
bias per batch entry.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from diffusion_transformers_b200 import shard


def test_head_range_covers_every_head_once():
    for H in range(1, 20):
        for world in range(1, H + 1):
            ranges = [shard.head_range(H, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == H
            for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
                assert a1 == b0
            sizes = [b - a for a, b in ranges]
            assert min(sizes) >= 1 and max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard.head_range(2, 3, 0)
    with pytest.raises(ValueError):
        shard.head_range(4, 2, 2)


def test_shard_inputs_slices_the_head_axes():
    from diffusion_transformers_b200.synthetic import make_custom
    c = make_custom(2, 5, 16, 8, seed=1, with_bias=True)
    c["H"] = 5
    s = shard.shard_inputs(c, 2, 1)
    h0, h1 = s["heads"]
    assert (h0, h1) == (2, 5) and s["H"] == 3
    assert np.array_equal(s["q"], c["q"][:, 2:5]) and s["q"].flags.c_contiguous
    assert np.array_equal(s["bias"], c["bias"][2:5])
    assert shard.shard_inputs(dict(c, bias=None), 2, 0)["bias"] is None
    # one bias per batch entry [B, H, N, N]: sliced on its head axis
    from diffusion_transformers_b200.synthetic import per_sample_bias
    pb = per_sample_bias(2, 5, 16, seed=3)
    sp = shard.shard_inputs(dict(c, bias=pb), 2, 1)
    assert np.array_equal(sp["bias"], pb[:, 2:5]) and sp["bias"].flags.c_contiguous


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _oracle_forward(orc, c, bias, scale):
    """The oracle's forward; a per-sample bias [B, H, N, N] runs it per batch
    entry with that entry's bias."""
    if bias is None or bias.ndim == 3:
        return orc.forward(c["q"], c["k"], bias, c["v"], scale)
    return np.concatenate([orc.forward(c["q"][b:b + 1], c["k"][b:b + 1], bias[b], c["v"][b:b + 1], scale)
                           for b in range(bias.shape[0])])


def _worker(rank, world, port, H, per_sample, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import oracle
    from diffusion_transformers_b200.synthetic import make_custom

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        orc = oracle.get()
        orc.set_num_threads(1)
        c = make_custom(2, H, 40, 72, seed=17, with_bias=True, bias_std=0.5)
        c["H"] = H
        if per_sample:
            from diffusion_transformers_b200.synthetic import per_sample_bias
            c["bias"] = per_sample_bias(2, H, 40, seed=19)
        mine = shard.shard_inputs(c, world, rank)  # this rank holds only its slices
        o_local = _oracle_forward(orc, mine, mine["bias"], c["softmax_scale"])
        o = shard.gather_heads(torch.from_numpy(o_local), H, world, rank)
        full = _oracle_forward(orc, c, c["bias"], c["softmax_scale"])
        out[rank] = (bool(np.array_equal(o.numpy(), full)), tuple(o.shape), mine["heads"])
    finally:
        dist.destroy_process_group()


def _bwd_worker(rank, world, port, H, out):
    # the backward partitions by heads the same way: each rank's dV, ds, dt
    # [B, h1-h0, N, d] and dbias [h1-h0, N, N] (its heads' bias, summed over
    # b on the rank) gathered on the head axis equal the unsharded backward
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import oracle
    from diffusion_transformers_b200.synthetic import make_custom, upstream_grad

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        orc = oracle.get()
        orc.set_num_threads(1)
        c = make_custom(2, H, 24, 40, seed=23, with_bias=True, bias_std=0.5)
        c["H"] = H
        c["dO"] = upstream_grad(2, H, 24, 40, seed=24)
        mine = shard.shard_inputs(c, world, rank)
        dO_mine = shard.slice_heads(c["dO"], *mine["heads"], 1)
        g = orc.backward(mine["q"], mine["k"], mine["bias"], mine["v"], dO_mine, c["softmax_scale"])
        full = orc.backward(c["q"], c["k"], c["bias"], c["v"], c["dO"], c["softmax_scale"])
        same = []
        for x, w in zip(g[:3], full[:3]):
            same.append(bool(np.array_equal(shard.gather_heads(torch.from_numpy(x), H, world, rank).numpy(), w)))
        # dbias carries heads on its first axis: gather it as [1, h1-h0, N, N]
        db = shard.gather_heads(torch.from_numpy(g[3][None]), H, world, rank)[0].numpy()
        same.append(bool(np.array_equal(db, full[3])))
        out[rank] = tuple(same)
    finally:
        dist.destroy_process_group()


def test_two_ranks_backward_gather_equals_unsharded_oracle():
    world, H = 2, 5
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_bwd_worker, args=(world, _free_port(), H, out), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        assert out[r] == (True, True, True, True), f"rank {r}: gathered gradients differ {out[r]}"


@pytest.mark.parametrize("H,per_sample", [(4, False), (5, False), (5, True)])
def test_two_ranks_gather_equals_unsharded_oracle(H, per_sample):
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), H, per_sample, out), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        same, shape, heads = out[r]
        assert same, f"rank {r}: gathered O differs from the unsharded oracle"
        assert shape == (2, H, 40, 72)
        assert heads == shard.head_range(H, world, r)
