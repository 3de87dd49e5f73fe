"""binattn_forward_static_ws: the padded-bias forward on the library's static
device workspace. Same result as the oracle, and the call allocates no device
memory (free device memory and torch's allocator unchanged across it)."""
import ctypes

import pytest
import torch

from diffusion_transformers_b200 import binattn
from diffusion_transformers_b200.synthetic import make_custom
from parity import bf16_to_f64, check_o, dev

pytestmark = pytest.mark.gpu


def test_static_workspace_forward_matches_oracle_and_allocates_nothing(orc):
    c = make_custom(2, 3, 197, 64, seed=23, with_bias=True, bias_std=0.5)
    ref = orc.forward(c["q"], c["k"], c["bias"], c["v"], c["softmax_scale"])
    q, k, v, bias = dev(c["q"]), dev(c["k"]), dev(c["v"]), dev(c["bias"])
    qb, aq = binattn.pack(q)
    kb, ak = binattn.pack(k)
    assert binattn.workspace_bytes(2, 3, 197, 64, True) > 0  # the padded-bias path runs
    out = torch.empty_like(v)
    binattn.forward_static_ws(qb, kb, aq, ak, bias, v, c["softmax_scale"], out=out)  # module loaded
    torch.cuda.synchronize()
    out2 = torch.empty_like(v)
    free0, _ = torch.cuda.mem_get_info()
    held0 = torch.cuda.memory_allocated()
    binattn.forward_static_ws(qb, kb, aq, ak, bias, v, c["softmax_scale"], out=out2)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == held0
    assert free1 == free0
    binattn.device_status()
    check_o(bf16_to_f64(out2), ref, "static workspace")
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))


def test_static_workspace_too_small_is_reported():
    L = binattn.lib()
    A, P = 0x10000, ctypes.c_void_p  # checked on the host before any device access
    H, N = 2, 4095  # [2][4095][4096] bf16 = 67 MB of padded bias: above the static 32 MiB
    assert binattn.workspace_bytes(1, H, N, 64, True) > 32 << 20
    rc = L.binattn_forward_static_ws(P(A), P(A), P(A), P(A), P(A), P(A), ctypes.c_float(0.125), 1, H, N, 64,
                                     P(A), None)
    assert rc == 5
    assert b"static" in L.binattn_last_error_message()
