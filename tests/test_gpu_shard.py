"""The head partition of one forward, through the real kernels on one GPU.

Every (b, h) is an independent problem and no rank waits on another (there is
no collective on the data path), so the ranks of a head-sharded call can be
run one after the other on one device: each runs the library on its slices
(Q, K, V [B, H/g, N, d] and bias [H/g, N, N] only), and the concatenated O
must equal the unsharded call bit for bit (same kernels, same per-pair work;
no tail split at these sizes).
"""
import numpy as np
import pytest
import torch

from diffusion_transformers_b200 import binattn, shard
from diffusion_transformers_b200.synthetic import make_custom
from parity import dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world", [2, 3, 4])
@pytest.mark.parametrize("with_bias", [True, False])
def test_head_shards_concatenate_to_the_whole_call(world, with_bias):
    B, H, N, d = 2, 12, 512, 72
    c = make_custom(B, H, N, d, seed=world + 5, with_bias=with_bias, bias_std=0.5)
    c["H"] = H

    def run(inp):
        q, k, v = dev(inp["q"]), dev(inp["k"]), dev(inp["v"])
        qb, aq = binattn.pack(q)
        kb, ak = binattn.pack(k)
        return binattn.forward(qb, kb, aq, ak, dev(inp["bias"]) if with_bias else None, v, c["softmax_scale"])

    whole = run(c)
    parts = []
    for r in range(world):
        mine = shard.shard_inputs(c, world, r)
        assert mine["q"].shape[1] == mine["H"] and (mine["bias"] is None or mine["bias"].shape[0] == mine["H"])
        parts.append(run(mine))
    torch.cuda.synchronize()
    binattn.device_status()
    got = torch.cat(parts, dim=1)
    assert torch.equal(got.view(torch.int16), whole.view(torch.int16))
