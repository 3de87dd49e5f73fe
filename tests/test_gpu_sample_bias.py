"""The context-aware form of the bias on the GPU: one dense bias per batch
entry, through binattn_forward_sample_bias_ws.

A bias computed from each sample's content differs per sample; the forward
takes it as bf16 [B, H, N, ld]. Batch entry b then computes exactly what the
shared-bias forward computes for a batch of one with bias[b], so the oracle is
run per batch entry (oracle_forward with B = 1 and that entry's bias). Three
checks:
- every output row against the oracle, within the stated bar, for ragged and
  whole tiles, padded and unpadded rows, and a split tail;
- with the same bias in every entry, the result equals binattn_forward_ws
  bit for bit (the same kernel arithmetic on the same values);
- reversing the batch order of every input reverses the output, bit for bit
  (entry b reads bias row block b * H + h, not h * B + b).
"""
import numpy as np
import pytest
import torch

from diffusion_transformers_b200 import binattn
from diffusion_transformers_b200.synthetic import make_custom, make_inputs, per_sample_bias
from parity import bf16_to_f64, check_o, dev

pytestmark = pytest.mark.gpu

# (B, H, N, d): whole and ragged key tiles, N % 8 != 0 (padded into the
# workspace), several pairs per CTA, and a split tail (19 heads of 2048 rows)
CASES = [(2, 3, 256, 64), (3, 2, 197, 72), (2, 2, 129, 40), (4, 40, 96, 32), (2, 19, 1024, 72),
         (1, 19, 2048, 72)]


def _oracle_per_sample(orc, c, bias_b):
    """O and its spread E [B, H, N, d]: the oracle's forward of each batch entry
    alone, with that entry's bias."""
    parts = [orc.forward_spread(c["q"][b:b + 1], c["k"][b:b + 1], bias_b[b], c["v"][b:b + 1], c["softmax_scale"])
             for b in range(c["B"])]
    return np.concatenate([o for o, _ in parts]), np.concatenate([e for _, e in parts])


def _stored(bias: torch.Tensor, ld: int) -> torch.Tensor:
    B, H, N, _ = bias.shape
    out = torch.full((B, H, N, ld), 7.0, dtype=torch.bfloat16, device=bias.device)  # never read beyond N
    out[..., :N] = bias
    return out


@pytest.mark.parametrize("shape", CASES)
def test_sample_bias_every_row(orc, shape):
    B, H, N, d = shape
    c = make_custom(B, H, N, d, seed=31 * N + d, with_bias=False)
    bias_b = per_sample_bias(B, H, N, seed=N + 3 * d)
    q, k, v, bias = dev(c["q"]), dev(c["k"]), dev(c["v"]), dev(bias_b)
    qb, aq = binattn.pack(q)
    kb, ak = binattn.pack(k)
    ref, spread = _oracle_per_sample(orc, c, bias_b)
    ld8 = binattn.padded_bias_ld(N)
    first = None
    for ld in sorted({N, ld8, ld8 + 3}):
        got = binattn.forward_sample_bias_ws(qb, kb, aq, ak, bias if ld == N else _stored(bias, ld), v,
                                             c["softmax_scale"])
        torch.cuda.synchronize()
        binattn.device_status()
        if first is None:
            first = got
            check_o(bf16_to_f64(got), ref, f"sample bias {shape}", spread)
        else:  # the row stride changes where the bias is read, not the result
            assert torch.equal(got.view(torch.int16), first.view(torch.int16)), f"{shape} ld={ld}"


@pytest.mark.parametrize("shape", [(2, 3, 256, 64), (3, 2, 197, 72), (1, 19, 2048, 72)])
def test_sample_bias_shared_equals_forward_ws(shape):
    B, H, N, d = shape
    c = make_custom(B, H, N, d, seed=5 * N + d, with_bias=True, bias_std=0.5)
    q, k, v, bias = dev(c["q"]), dev(c["k"]), dev(c["v"]), dev(c["bias"])
    qb, aq = binattn.pack(q)
    kb, ak = binattn.pack(k)
    want = binattn.forward_ws(qb, kb, aq, ak, bias, v, c["softmax_scale"])
    same = bias.unsqueeze(0).expand(B, H, N, N).contiguous()
    got = binattn.forward_sample_bias_ws(qb, kb, aq, ak, same, v, c["softmax_scale"])
    torch.cuda.synchronize()
    binattn.device_status()
    assert torch.equal(got.view(torch.int16), want.view(torch.int16)), f"{shape}"


@pytest.mark.parametrize("shape", [(3, 2, 197, 72), (4, 40, 96, 32)])
def test_sample_bias_batch_order(shape):
    B, H, N, d = shape
    c = make_custom(B, H, N, d, seed=11 * N + d, with_bias=False)
    q, k, v = dev(c["q"]), dev(c["k"]), dev(c["v"])
    bias = dev(per_sample_bias(B, H, N, seed=7 * N + d))
    qb, aq = binattn.pack(q)
    kb, ak = binattn.pack(k)
    got = binattn.forward_sample_bias_ws(qb, kb, aq, ak, bias, v, c["softmax_scale"])
    r = torch.arange(B - 1, -1, -1, device="cuda")
    qr, kr = binattn.pack(q[r].contiguous()), binattn.pack(k[r].contiguous())
    rev = binattn.forward_sample_bias_ws(qr[0], kr[0], qr[1], kr[1], bias[r].contiguous(), v[r].contiguous(),
                                         c["softmax_scale"])
    torch.cuda.synchronize()
    binattn.device_status()
    assert torch.equal(rev.view(torch.int16), got[r].view(torch.int16)), f"{shape}"


def test_sample_bias_dit_xl_1024_every_row(orc):
    # DiT-XL/2 at 1024 px: 2 x 16 x 4096 x 4096 bias values (1.07 GB), entry b
    # the workload's bias with its heads rotated by b; the call runs the
    # persistent waves, the split tail and the combine, as the bench times it.
    inp = make_inputs("dit_xl_1024", with_bias=True)
    B, H, N, d = inp["B"], inp["H"], inp["N"], inp["d"]
    bias_b = per_sample_bias(B, H, N, seed=0, base=inp["bias"])
    assert binattn.lib().binattn_forward_sample_bias_workspace_bytes(B, H, N, d, N) > 0  # split partials
    q, k, v, bias = dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), dev(bias_b)
    qb, aq = binattn.pack(q)
    kb, ak = binattn.pack(k)
    got = binattn.forward_sample_bias_ws(qb, kb, aq, ak, bias, v, inp["softmax_scale"])
    torch.cuda.synchronize()
    binattn.device_status()
    del bias
    ref, spread = _oracle_per_sample(orc, inp, bias_b)
    check_o(bf16_to_f64(got), ref, "sample bias dit_xl_1024", spread)
