"""The in-build bf16 softmax attention (the speed reference the binary kernel is
compared against) against a plain fp64 numpy softmax attention of the same
bf16 inputs. It is not part of the method; these tests only make sure the
comparison is against a correct kernel."""
import numpy as np
import pytest
import torch

from diffusion_transformers_b200 import binattn
from diffusion_transformers_b200.synthetic import bf16_bits_to_f32, make_custom, make_inputs
from parity import REL_RMS, bf16_half_ulp, bf16_to_f64, dev, sample_rows

pytestmark = pytest.mark.gpu


def numpy_attention(q, k, v, bias, scale, rows=None):
    """O = softmax(scale * Q K^T + bias) V in fp64 for flat rows (all if None)."""
    f = lambda x: bf16_bits_to_f32(x).astype(np.float64)
    Q, K, V = f(q), f(k), f(v)
    B, H, N, d = Q.shape
    Bb = None if bias is None else f(bias)
    if rows is None:
        rows = np.arange(B * H * N)
    out = np.zeros((len(rows), d))
    for n, rid in enumerate(rows):
        bh, i = divmod(int(rid), N)
        b, h = divmod(bh, H)
        lg = scale * (K[b, h] @ Q[b, h, i])
        if Bb is not None:
            lg = lg + Bb[h, i]
        p = np.exp(lg - lg.max())
        out[n] = (p / p.sum()) @ V[b, h]
    return out


def check_ref(o_gpu, o_ref, vmax, what):
    """P is rounded to bf16 (relative 2^-9 per element, sum of P = 1), so each
    output element can be off by up to about 2^-9 * max|V|, plus half a bf16 ulp
    of the output. The bound used is twice the first term plus the second."""
    err = np.abs(o_gpu - o_ref)
    bound = 2.0 ** -8 * vmax + bf16_half_ulp(o_ref) + 1e-3
    assert np.all(err <= bound), f"{what}: max excess {float((err - bound).max()):.3e}"
    rel_rms = float(np.linalg.norm(o_gpu - o_ref) / np.linalg.norm(o_ref))
    assert rel_rms <= REL_RMS, f"{what}: rel-RMS {rel_rms:.3e}"


@pytest.mark.parametrize("shape", [(1, 2, 256, 64), (2, 3, 129, 72), (1, 2, 197, 64),
                                   (1, 1, 300, 128), (2, 1, 7, 32), (1, 2, 130, 96)])
@pytest.mark.parametrize("with_bias", [True, False])
def test_ref_attention_small(shape, with_bias):
    B, H, N, d = shape
    c = make_custom(B, H, N, d, seed=N + 3 * d, with_bias=with_bias, bias_std=0.5)
    out = binattn.ref_bf16_forward(dev(c["q"]), dev(c["k"]), dev(c["bias"]) if with_bias else None,
                                   dev(c["v"]), c["softmax_scale"])
    torch.cuda.synchronize()
    binattn.device_status()
    ref = numpy_attention(c["q"], c["k"], c["v"], c["bias"] if with_bias else None,
                          c["softmax_scale"]).reshape(B, H, N, d)
    vmax = float(np.abs(bf16_bits_to_f32(c["v"])).max())
    check_ref(bf16_to_f64(out), ref, vmax, f"ref {shape} bias={with_bias}")


@pytest.mark.parametrize("name,with_bias", [("dit_xl_1024", True), ("dit_xl_1024", False),
                                            ("vit_l384", True)])
def test_ref_attention_full_size_sampled(name, with_bias):
    inp = make_inputs(name, with_bias=with_bias)
    B, H, N, d = inp["B"], inp["H"], inp["N"], inp["d"]
    out = binattn.ref_bf16_forward(dev(inp["q"]), dev(inp["k"]), dev(inp["bias"]), dev(inp["v"]),
                                   inp["softmax_scale"])
    torch.cuda.synchronize()
    binattn.device_status()
    rows = sample_rows(B, H, N, 32, seed=7)
    got = out.view(B * H * N, d)[torch.from_numpy(rows).cuda()]
    ref = numpy_attention(inp["q"], inp["k"], inp["v"], inp["bias"], inp["softmax_scale"], rows)
    vmax = float(np.abs(bf16_bits_to_f32(inp["v"])).max())
    check_ref(bf16_to_f64(got), ref, vmax, f"ref {name} bias={with_bias}")


# binattn_ref_bf16_forward_ws runs the reference with the binary forward's
# launch plan: at DiT-XL/2 1024 px the pairs of heads 14 and 15 are in the
# split tail (two key halves joined by the combine kernel). Rows there, and
# elsewhere, against the fp64 attention.
@pytest.mark.parametrize("with_bias", [True, False])
def test_ref_attention_ws_split_tail(with_bias):
    inp = make_inputs("dit_xl_1024", with_bias=with_bias)
    B, H, N, d = inp["B"], inp["H"], inp["N"], inp["d"]
    bias = dev(inp["bias"]) if with_bias else None
    out = binattn.ref_bf16_forward_ws(dev(inp["q"]), dev(inp["k"]), bias, dev(inp["v"]), inp["softmax_scale"])
    torch.cuda.synchronize()
    binattn.device_status()
    rng = np.random.default_rng(11)
    tail = [(b * H + h) * N + i for b, h, i in zip(rng.integers(0, B, 24), rng.integers(14, 16, 24),
                                                  rng.integers(0, N, 24))]
    rows = np.concatenate([np.array(tail, dtype=np.int64), sample_rows(B, H, N, 16, seed=5)])
    got = out.view(B * H * N, d)[torch.from_numpy(rows).cuda()]
    ref = numpy_attention(inp["q"], inp["k"], inp["v"], inp["bias"] if with_bias else None,
                          inp["softmax_scale"], rows)
    vmax = float(np.abs(bf16_bits_to_f32(inp["v"])).max())
    check_ref(bf16_to_f64(got), ref, vmax, f"ref_ws dit_xl_1024 bias={with_bias}")
