"""The position-sensitive bias on the GPU, through the C ABI.

binattn_forward_relpos gathers the bias from a relative-position table in
shared memory. The oracle expands the same table to the dense bias
(oracle_expand_relpos_bias, pinned on CPU): the table call must equal
binattn_forward_ws on that dense bias bit for bit (same kernel arithmetic,
the bias values are the same bf16 numbers), and meet the oracle's forward
within the stated bar.
"""
import numpy as np
import pytest
import torch

from diffusion_transformers_b200 import binattn
from diffusion_transformers_b200.synthetic import f32_to_bf16_bits, make_custom, make_inputs
from parity import bf16_to_f64, check_o, dev, sample_rows

pytestmark = pytest.mark.gpu

# (B, H, gh, gw, n_cls, d): square and oblong grids, with and without a class
# token (DeiT-B's 14 x 14 + 1), ragged and whole key tiles, a split tail
RELPOS_CASES = [(1, 2, 8, 8, 0, 64), (2, 3, 14, 14, 1, 64), (1, 2, 16, 16, 0, 72), (1, 1, 32, 33, 1, 72),
                (2, 2, 20, 24, 1, 40), (1, 1, 3, 5, 1, 16), (1, 19, 32, 64, 0, 72)]


def _table(rng, H, gh, gw, n_cls, std=0.5):
    R = binattn.relpos_table_entries(gh, gw, n_cls)
    return f32_to_bf16_bits((rng.standard_normal((H, R)) * std).astype(np.float32))


@pytest.mark.parametrize("case", RELPOS_CASES)
def test_relpos_equals_dense_expansion(orc, case):
    B, H, gh, gw, n_cls, d = case
    N = n_cls + gh * gw
    rng = np.random.default_rng(gh * 100 + gw + n_cls)
    table = _table(rng, H, gh, gw, n_cls)
    dense = orc.expand_relpos_bias(table, gh, gw, n_cls)
    c = make_custom(B, H, N, d, seed=N + d, with_bias=False)
    q, k, v = dev(c["q"]), dev(c["k"]), dev(c["v"])
    qb, aq = binattn.pack(q)
    kb, ak = binattn.pack(k)
    got = binattn.forward_relpos(qb, kb, aq, ak, dev(table), (gh, gw), n_cls, v, c["softmax_scale"])
    want = binattn.forward_ws(qb, kb, aq, ak, dev(dense), v, c["softmax_scale"])
    torch.cuda.synchronize()
    binattn.device_status()
    assert torch.equal(got.view(torch.int16), want.view(torch.int16)), f"relpos {case}"
    rows = sample_rows(B, H, N, 256, seed=1) if B * H * N > 20000 else np.arange(B * H * N)
    ref = orc.forward_rows(c["q"], c["k"], dense, c["v"], c["softmax_scale"], rows)
    check_o(bf16_to_f64(got.view(B * H * N, d)[torch.from_numpy(rows).cuda()]), ref, f"relpos {case}")


def test_relpos_dit_xl_1024_sampled(orc):
    # DiT-XL/2 1024 px: a 64 x 64 latent patch grid, no class token
    inp = make_inputs("dit_xl_1024", with_bias=False)
    B, H, N, d = inp["B"], inp["H"], inp["N"], inp["d"]
    table = _table(np.random.default_rng(4), H, 64, 64, 0, std=0.05)
    q, k, v = dev(inp["q"]), dev(inp["k"]), dev(inp["v"])
    qb, aq = binattn.pack(q)
    kb, ak = binattn.pack(k)
    got = binattn.forward_relpos(qb, kb, aq, ak, dev(table), (64, 64), 0, v, inp["softmax_scale"])
    torch.cuda.synchronize()
    binattn.device_status()
    dense = orc.expand_relpos_bias(table, 64, 64, 0)
    rows = sample_rows(B, H, N, 512, seed=9)
    ref = orc.forward_rows(inp["q"], inp["k"], dense, inp["v"], inp["softmax_scale"], rows)
    check_o(bf16_to_f64(got.view(B * H * N, d)[torch.from_numpy(rows).cuda()]), ref, "relpos dit_xl_1024")
