"""The host-to-host pipelined forward (HostPipeline) on the GPU.

Its chunks are whole (b, head group) problems run by the library's own calls,
so with N % 8 == 0 (the bias read as it is) O equals binattn.forward on the
whole batch bit for bit; every case also meets the oracle. Calls back to back
reuse the buffers without a race.
"""
import numpy as np
import pytest
import torch

from diffusion_transformers_b200 import binattn
from diffusion_transformers_b200.pipeline import HostPipeline
from diffusion_transformers_b200.synthetic import make_custom
from parity import bf16_to_f64, check_o, dev

pytestmark = pytest.mark.gpu


def _pinned(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).pin_memory()


@pytest.mark.parametrize("shape,hpc", [((2, 4, 512, 72), None), ((2, 4, 512, 72), 1), ((1, 6, 300, 64), 2),
                                       ((3, 2, 197, 64), 2), ((2, 16, 1024, 72), None)])
@pytest.mark.parametrize("with_bias", [True, False])
def test_pipeline_matches(orc, shape, hpc, with_bias):
    B, H, N, d = shape
    c = make_custom(B, H, N, d, seed=B * N + H + d, with_bias=with_bias, bias_std=0.5)
    pipe = HostPipeline(B, H, N, d, heads_per_chunk=hpc, has_bias=with_bias)
    qh, kh, vh = _pinned(c["q"]), _pinned(c["k"]), _pinned(c["v"])
    oh = torch.empty((B, H, N, d), dtype=torch.bfloat16).pin_memory()
    bias = dev(c["bias"]) if with_bias else None
    outs = []
    for _ in range(2):  # twice in a row on one stream: the second reuses every buffer
        pipe.run(qh, kh, vh, bias, c["softmax_scale"], oh)
        torch.cuda.current_stream().synchronize()
        outs.append(oh.clone())
    binattn.device_status()
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    if N % 8 == 0 or not with_bias:
        qb, aq = binattn.pack(dev(c["q"]))
        kb, ak = binattn.pack(dev(c["k"]))
        want = binattn.forward(qb, kb, aq, ak, bias, dev(c["v"]), c["softmax_scale"]).cpu()
        assert torch.equal(outs[0].view(torch.int16), want.view(torch.int16))
    if B * H * N <= 40000:
        ref = orc.forward(c["q"], c["k"], c["bias"] if with_bias else None, c["v"], c["softmax_scale"])
        check_o(bf16_to_f64(outs[0]), ref, f"pipeline {shape} bias={with_bias}")
