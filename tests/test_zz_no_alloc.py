"""binattn_forward_static_ws: the forward for callers that cannot allocate
device memory (a plug-in handed its buffers by a framework that owns the
allocator, or a loop where cudaMalloc's possible device synchronisation is not
allowed). Its scratch is a fixed 32 MiB array inside the library.

Checked here through the C ABI: two calls in a row give the same result as
binattn_forward_ws with a caller-owned workspace (within the parity tolerance),
on a shape that pads the bias into the scratch and on one that splits the last
wave of row pairs into key halves whose partials live in the scratch; the calls
allocate nothing; a shape that needs more scratch is refused on the host.

This file is collected last, so a run that stops at its first failure has run
every other test before it.
"""
import ctypes

import pytest
import torch

from diffusion_transformers_b200 import binattn
from diffusion_transformers_b200.synthetic import make_custom
from parity import bf16_to_f64, check_o, dev

pytestmark = pytest.mark.gpu


def _split_heads(N: int) -> int:
    """Smallest H (B = 1) whose 256-row pairs leave a last wave at most half full."""
    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    per_head = (N + 255) // 256
    for H in range(1, 4 * nsm):
        P = H * per_head
        if P >= nsm and 0 < P % nsm <= nsm // 2:
            return H
    raise AssertionError("no head count gives a split tail")


def _inputs(B, H, N, d, seed, bias_std):
    c = make_custom(B, H, N, d, seed=seed, with_bias=True, bias_std=bias_std)
    q, k, v, bias = dev(c["q"]), dev(c["k"]), dev(c["v"]), dev(c["bias"])
    qb, aq = binattn.pack(q)
    kb, ak = binattn.pack(k)
    torch.cuda.synchronize()
    return c, (qb, kb, aq, ak, bias, v)


def _static_call(args, scale, out):
    qb, kb, aq, ak, bias, v = args
    B, H, N, d = v.shape
    P = ctypes.c_void_p
    rc = binattn.lib().binattn_forward_static_ws(
        P(qb.data_ptr()), P(kb.data_ptr()), P(aq.data_ptr()), P(ak.data_ptr()), P(bias.data_ptr()),
        P(v.data_ptr()), ctypes.c_float(scale), B, H, N, d, P(out.data_ptr()),
        P(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, binattn.lib().binattn_last_error_message()


def test_static_workspace_matches_caller_workspace_twice(orc):
    cases = []
    # bias with N % 8 != 0: the bias rows are padded into the scratch
    c, args = _inputs(2, 3, 197, 64, seed=23, bias_std=0.5)
    assert binattn.workspace_bytes(2, 3, 197, 64, True) > 0
    cases.append(("padded bias", c, args))
    # a short last wave: split partials in the scratch (N % 8 == 0, no padding)
    H = _split_heads(2048)
    c2, args2 = _inputs(1, H, 2048, 64, seed=29, bias_std=0.1)
    assert 0 < binattn.workspace_bytes(1, H, 2048, 64, True) <= 32 << 20
    cases.append(("split tail", c2, args2))

    for what, c, args in cases:
        qb, kb, aq, ak, bias, v = args
        ref = binattn.forward_ws(qb, kb, aq, ak, bias, v, c["softmax_scale"])  # existing entry point
        torch.cuda.synchronize()
        binattn.device_status()
        ref64 = bf16_to_f64(ref)
        for call in range(2):
            out = torch.full_like(v, float("nan"))
            torch.cuda.synchronize()
            free0, _ = torch.cuda.mem_get_info()
            held0 = torch.cuda.memory_allocated()
            _static_call(args, c["softmax_scale"], out)
            torch.cuda.synchronize()
            free1, _ = torch.cuda.mem_get_info()
            binattn.device_status()
            if call == 1:  # the first call may load the module; the second must allocate nothing
                assert free1 == free0, f"{what}: device memory changed across the call"
                assert torch.cuda.memory_allocated() == held0
            check_o(bf16_to_f64(out), ref64, f"{what}, static call {call}")
        if what == "padded bias":  # small enough for the oracle as well
            o_ref = orc.forward(c["q"], c["k"], c["bias"], c["v"], c["softmax_scale"])
            check_o(bf16_to_f64(out), o_ref, f"{what} vs oracle")


def test_static_workspace_too_small_is_reported():
    L = binattn.lib()
    A, P = 0x10000, ctypes.c_void_p  # refused on the host before any device access
    H, N = 2, 4095  # [2][4095][4096] bf16 = 67 MB of padded bias: above the static 32 MiB
    assert binattn.workspace_bytes(1, H, N, 64, True) > 32 << 20
    rc = L.binattn_forward_static_ws(P(A), P(A), P(A), P(A), P(A), P(A), ctypes.c_float(0.125), 1, H, N, 64,
                                     P(A), None)
    assert rc == 5
    assert b"static" in L.binattn_last_error_message()
