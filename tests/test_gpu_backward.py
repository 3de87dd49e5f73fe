"""The backward on the GPU, through the C ABI (binattn_backward).

The oracle's backward (oracle_backward, pinned on CPU against automatic
differentiation, invariants and finite differences) gives dV, ds, dt and dbias
in fp64. The kernels compute in fp32 with exact softmax weights, so the bar is
the accumulation error of fp32 sums over at most N terms: relative RMS error
<= 2e-4 and every element within 1e-3 of the tensor's largest magnitude (plus
1e-7 absolute, for tensors that are exactly zero).
"""
import numpy as np
import pytest
import torch

from diffusion_transformers_b200 import binattn
from diffusion_transformers_b200.synthetic import make_custom, make_inputs, upstream_grad
from parity import dev

pytestmark = pytest.mark.gpu

REL_RMS = 2e-4
MAX_REL = 1e-3


def check_grad(got: torch.Tensor, ref: np.ndarray, what: str):
    g = got.cpu().numpy().astype(np.float64)
    assert g.shape == ref.shape, what
    scale = float(np.abs(ref).max())
    err = np.abs(g - ref)
    rel_rms = float(np.linalg.norm(g - ref) / max(np.linalg.norm(ref), 1e-30))
    assert err.max() <= MAX_REL * scale + 1e-7, f"{what}: max error {err.max():.3e} against scale {scale:.3e}"
    assert rel_rms <= REL_RMS or np.linalg.norm(ref) == 0, f"{what}: rel-RMS {rel_rms:.3e}"


def _run(c, dO, with_bias=True, with_dbias=True, scale=None):
    q, k, v = dev(c["q"]), dev(c["k"]), dev(c["v"])
    bias = dev(c["bias"]) if with_bias else None
    qb, aq = binattn.pack(q)
    kb, ak = binattn.pack(k)
    out = binattn.backward(qb, kb, aq, ak, bias, v, dev(dO), c["softmax_scale"] if scale is None else scale,
                           with_dbias=with_dbias)
    torch.cuda.synchronize()
    binattn.device_status()
    return out


# (B, H, N, d): one key, a few keys, one whole tile, ragged tiles, every count
# of sign words (d = 1 ... 128), several batch entries summed into dbias, and a
# DiT-XL/2 head shape
CASES = [(1, 1, 1, 1), (2, 2, 3, 5), (2, 3, 64, 64), (1, 2, 197, 72), (3, 2, 129, 40), (2, 2, 100, 128),
         (1, 1, 257, 33), (2, 1, 70, 1), (2, 2, 1024, 72)]


@pytest.mark.parametrize("with_bias", [True, False])
@pytest.mark.parametrize("shape", CASES)
def test_backward_matches_oracle(orc, shape, with_bias):
    B, H, N, d = shape
    c = make_custom(B, H, N, d, seed=3 * N + d, with_bias=with_bias, bias_std=0.5, zeros_frac=0.05)
    dO = upstream_grad(B, H, N, d, seed=N + d)
    dV, ds, dt, db = _run(c, dO, with_bias)
    rV, rs, rt, rb = orc.backward(c["q"], c["k"], c["bias"] if with_bias else None, c["v"], dO, c["softmax_scale"])
    tag = f"{shape} bias={with_bias}"
    check_grad(dV, rV, f"dV {tag}")
    check_grad(ds, rs, f"ds {tag}")
    check_grad(dt, rt, f"dt {tag}")
    check_grad(db, rb, f"dbias {tag}")


def test_backward_deterministic_and_dbias_optional():
    # no atomics: a second call gives the same bits; without dbias the other
    # gradients are unchanged
    B, H, N, d = 3, 2, 129, 40
    c = make_custom(B, H, N, d, seed=9, with_bias=True, bias_std=0.5)
    dO = upstream_grad(B, H, N, d, seed=10)
    first = _run(c, dO)
    second = _run(c, dO)
    for a, b_ in zip(first, second):
        assert torch.equal(a.view(torch.int32), b_.view(torch.int32))
    nodb = _run(c, dO, with_dbias=False)
    assert nodb[3] is None
    for a, b_ in zip(first[:3], nodb[:3]):
        assert torch.equal(a.view(torch.int32), b_.view(torch.int32))


def test_backward_scale_zero():
    # softmax_scale 0: the scaled binary Q and K get no gradient
    B, H, N, d = 2, 2, 97, 64
    c = make_custom(B, H, N, d, seed=4, with_bias=True, bias_std=0.5)
    dV, ds, dt, db = _run(c, upstream_grad(B, H, N, d, seed=5), scale=0.0)
    assert not ds.any() and not dt.any()


def test_backward_dit_xl_1024_properties():
    # DiT-XL/2 at 1024 px (2 x 16 x 4096 x 72, dense bias): properties that
    # hold at any size, on every (b, h): sum_j dV_j = sum_i dO_i (softmax rows
    # sum to 1) and every row of dbias sums to 0 (rows of dlogit do)
    inp = make_inputs("dit_xl_1024", with_bias=True)
    B, H, N, d = inp["B"], inp["H"], inp["N"], inp["d"]
    dO = upstream_grad(B, H, N, d, seed=12)
    dV, ds, dt, db = _run(inp, dO)
    for x in (dV, ds, dt, db):
        assert torch.isfinite(x).all()
    want = dev(dO).float().double().sum(2)
    got = dV.double().sum(2)
    assert torch.allclose(got, want, rtol=1e-3, atol=1e-3 * float(want.abs().max()))
    rows = db.double().sum(-1)
    l1 = db.double().abs().sum(-1)
    assert float((rows.abs() / l1.clamp_min(1e-30)).max()) <= 1e-4
