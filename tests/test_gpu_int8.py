"""The 8-bit P.V variant on the GPU, through the C ABI, against the oracle.

V's per-channel 8-bit code and scales: exact (the same fp32 decisions on
both sides). O of binattn_forward_int8 against the oracle's 8-bit forward
(u = rint(255 exp(logit - row max)), O = s * sum u vq / sum u): max-abs 2e-2
and rel-RMS 5e-3, on small shapes and on every row of the five workloads.
"""
import numpy as np
import pytest
import torch

from diffusion_transformers_b200 import binattn
from diffusion_transformers_b200.synthetic import f32_to_bf16_bits, make_custom, make_inputs
from parity import bf16_to_f64, check_o, dev

pytestmark = pytest.mark.gpu

INT8_SHAPES = [(1, 2, 256, 64), (2, 3, 129, 72), (1, 1, 1, 64), (2, 1, 7, 32), (1, 2, 197, 64),
               (2, 2, 512, 72), (1, 1, 72, 16), (1, 3, 1000, 72), (1, 2, 130, 80)]


@pytest.mark.parametrize("shape", INT8_SHAPES + [(1, 2, 33, 128), (2, 1, 5, 8)])
def test_quantize_v_exact(orc, shape):
    B, H, N, d = shape
    c = make_custom(B, H, N, d, seed=N + 3 * d, with_bias=False)
    v = c["v"].copy()
    v[0, 0, :, 0] = 0  # an all-zero channel
    if N >= 2:  # exact ties at scale 1: 127 then 2.5, -3.5
        v[-1, -1, :, -1] = f32_to_bf16_bits(np.zeros(N, dtype=np.float32))
        v[-1, -1, 0, -1] = f32_to_bf16_bits(np.array([127.0], dtype=np.float32))[0]
        v[-1, -1, 1, -1] = f32_to_bf16_bits(np.array([2.5], dtype=np.float32))[0]
    vq, s = binattn.quantize_v(dev(v))
    ovq, os_ = orc.quantize_v(v)
    assert np.array_equal(vq.cpu().numpy(), ovq)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), os_.view(np.uint32))


@pytest.mark.parametrize("shape", INT8_SHAPES)
@pytest.mark.parametrize("with_bias", [True, False])
def test_forward_int8_small(orc, shape, with_bias):
    B, H, N, d = shape
    c = make_custom(B, H, N, d, seed=17 * N + d, with_bias=with_bias, bias_std=0.5)
    ref = orc.forward_int8(c["q"], c["k"], c["bias"], c["v"], c["softmax_scale"])
    q, k, v = dev(c["q"]), dev(c["k"]), dev(c["v"])
    bias = dev(c["bias"]) if with_bias else None
    qb, aq = binattn.pack(q)
    kb, ak = binattn.pack(k)
    out = binattn.forward_int8(qb, kb, aq, ak, bias, v, c["softmax_scale"])
    torch.cuda.synchronize()
    binattn.device_status()
    check_o(bf16_to_f64(out), ref, f"int8 {shape} bias={with_bias}")


@pytest.mark.parametrize("name,with_bias", [("dit_xl_1024", True), ("dit_xl_1024", False), ("dit_xl_512", True),
                                            ("vit_l384", True), ("deit_b", True), ("tiny", True)])
def test_forward_int8_every_row(orc, name, with_bias):
    inp = make_inputs(name, with_bias=with_bias)
    bias_np = inp["bias"] if with_bias else None
    ref = orc.forward_int8(inp["q"], inp["k"], bias_np, inp["v"], inp["softmax_scale"])
    q, k, v = dev(inp["q"]), dev(inp["k"]), dev(inp["v"])
    bias = dev(bias_np)
    qb, aq = binattn.pack(q)
    kb, ak = binattn.pack(k)
    out = binattn.forward_int8(qb, kb, aq, ak, bias, v, inp["softmax_scale"])
    torch.cuda.synchronize()
    binattn.device_status()
    check_o(bf16_to_f64(out), ref, f"int8 {name} bias={with_bias}")
    # and the 8-bit result stays near the full-precision one (the quantisation itself)
    exact = orc.forward_rows(inp["q"], inp["k"], bias_np, inp["v"], inp["softmax_scale"], np.arange(0, q.shape[0] * q.shape[1] * q.shape[2], 97))
    got = bf16_to_f64(out).reshape(-1, inp["d"])[::97]
    assert np.linalg.norm(got - exact) / np.linalg.norm(exact) < 0.05
