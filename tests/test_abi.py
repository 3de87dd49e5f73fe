"""The C-ABI library without a GPU: it loads, exports every symbol the header
declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import math
import os
import re

import pytest

from diffusion_transformers_b200 import binattn

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "binattn.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(binattn_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    return binattn.lib()


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 9
    assert set(names) == set(binattn.EXPORTS)
    for n in names:
        assert hasattr(L, n), f"{n} not exported by {binattn.library_path()}"


def test_abi_version_and_strerror(L):
    assert L.binattn_abi_version() == 1
    for code in range(0, 9):
        s = L.binattn_strerror(code)
        assert s and isinstance(s, bytes)
    assert L.binattn_strerror(99) == b"unknown status"


A = 0x10000  # aligned fake device addresses: never dereferenced by these calls
P = ctypes.c_void_p


def _fwd(L, q=A, k=A, aq=A, ak=A, bias=None, v=A, scale=0.125, B=1, H=1, N=16, d=64, out=A,
         engine=0):
    return L.binattn_forward_engine(P(q), P(k), P(aq), P(ak), P(bias) if bias else None, P(v),
                                    ctypes.c_float(scale), B, H, N, d, P(out), engine, None)


def test_forward_host_validation(L):
    assert _fwd(L, q=0) == 1
    assert _fwd(L, out=0) == 1
    assert _fwd(L, v=A + 8) == 4
    assert _fwd(L, bias=A + 2) == 4
    assert _fwd(L, N=0) == 2
    assert _fwd(L, d=129) == 2
    assert _fwd(L, B=300, H=300) == 2
    assert _fwd(L, N=70000) == 2
    assert _fwd(L, scale=math.inf) == 8
    assert _fwd(L, scale=math.nan) == 8
    assert _fwd(L, engine=17) == 8
    assert _fwd(L, d=33, engine=binattn.ENGINE_TC) == 5
    assert _fwd(L, d=33, engine=binattn.ENGINE_POPC_TC) == 5
    assert b"NULL" in L.binattn_last_error_message() or True


def test_bias_ld_host_validation(L):
    def fwd(bias=A, ld=24, d=64, N=16, ws=A, wsb=1 << 20):
        return L.binattn_forward_bias_ld_ws(P(A), P(A), P(A), P(A), P(bias) if bias else None, ld, P(A),
                                            ctypes.c_float(0.125), 1, 1, N, d, P(A), P(ws) if ws else None,
                                            ctypes.c_size_t(wsb), None)
    assert fwd(bias=0) == 1                 # the bias is required
    assert fwd(ld=15) == 8                  # rows closer than N
    assert fwd(d=33, ld=40) == 5            # a strided bias needs the TMA-fed pipeline
    assert fwd(bias=A + 2) == 4
    assert L.binattn_padded_bias_ld(197) == 200 and L.binattn_padded_bias_ld(200) == 200
    assert L.binattn_padded_bias_ld(0) == 0
    assert L.binattn_forward_bias_ld_workspace_bytes(1, 2, 197, 64, 150) == 0  # ld < N


def test_sample_bias_host_validation(L):
    def fwd(bias=A, ld=16, d=64, N=16, ws=A, wsb=1 << 20, B=2, H=3):
        return L.binattn_forward_sample_bias_ws(P(A), P(A), P(A), P(A), P(bias) if bias else None, ld, P(A),
                                                ctypes.c_float(0.125), B, H, N, d, P(A), P(ws) if ws else None,
                                                ctypes.c_size_t(wsb), None)
    assert fwd(bias=0) == 1                 # the bias is required
    assert fwd(ld=15) == 8                  # rows closer than N
    assert fwd(d=33) == 5                   # only the TMA-fed pipeline takes it
    assert fwd(d=96) == 5
    assert fwd(bias=A + 2) == 4
    assert fwd(ws=0, N=197, ld=197) == 1    # the padded copy needs a workspace
    assert fwd(N=197, ld=197, wsb=100) == 8
    assert b"workspace" in L.binattn_last_error_message()
    assert L.binattn_forward_sample_bias_workspace_bytes(2, 3, 197, 64, 150) == 0  # ld < N
    # the padded copy holds B * H bias matrices, not H
    for B, H, N, d, ld in [(64, 12, 197, 64, 197), (2, 16, 4096, 72, 4096), (3, 2, 300, 8, 301), (1, 19, 2048, 72, 2048)]:
        pad = 0 if ld % 8 == 0 else (B * H * N * ((N + 7) // 8 * 8) * 2 + 255) // 256 * 256
        shared = L.binattn_forward_bias_ld_workspace_bytes(B, H, N, d, ld)
        shared_pad = 0 if ld % 8 == 0 else (H * N * ((N + 7) // 8 * 8) * 2 + 255) // 256 * 256
        assert L.binattn_forward_sample_bias_workspace_bytes(B, H, N, d, ld) == pad + shared - shared_pad


def test_backward_host_validation(L):
    def bwd(q=A, dO=A, dV=A, ds=A, dt=A, dbias=A, bias=None, ws=A, wsb=1 << 20, B=1, H=2, N=16, d=64,
            scale=0.125):
        return L.binattn_backward(P(q), P(A), P(A), P(A), P(bias) if bias else None, P(A), P(dO) if dO else None,
                                  ctypes.c_float(scale), B, H, N, d, P(dV) if dV else None, P(ds) if ds else None,
                                  P(dt) if dt else None, P(dbias) if dbias else None, P(ws) if ws else None,
                                  ctypes.c_size_t(wsb), None)
    assert bwd(q=0) == 1
    assert bwd(dO=0) == 1
    assert bwd(dV=0) == 1 and bwd(ds=0) == 1 and bwd(dt=0) == 1
    assert bwd(ws=0) == 1                      # the workspace holds LSE and D
    assert bwd(dbias=A + 4) == 4
    assert bwd(bias=A + 2) == 4
    assert bwd(dV=A + 8) == 4
    assert bwd(N=0) == 2 and bwd(d=129) == 2 and bwd(B=300, H=300) == 2
    assert bwd(scale=math.nan) == 8
    assert bwd(wsb=255) == 8
    assert b"workspace" in L.binattn_last_error_message()
    # one float of LSE and one of D per query row, rounded up to 256 bytes
    assert L.binattn_backward_workspace_bytes(1, 2, 16, 64) == 256
    assert L.binattn_backward_workspace_bytes(2, 16, 4096, 72) == 2 * 2 * 16 * 4096 * 4
    assert L.binattn_backward_workspace_bytes(3, 5, 7, 1) == (2 * 3 * 5 * 7 * 4 + 255) // 256 * 256
    assert L.binattn_backward_workspace_bytes(1, 1, 16, 129) == 0


def test_relpos_host_validation(L):
    def fwd(table=A, gh=4, gw=4, ncls=0, N=16, d=64, ws=A):
        return L.binattn_forward_relpos(P(A), P(A), P(A), P(A), P(table) if table else None, gh, gw, ncls, P(A),
                                        ctypes.c_float(0.125), 1, 1, N, d, P(A), P(ws) if ws else None,
                                        ctypes.c_size_t(1 << 20), None)
    assert fwd(table=0) == 1
    assert fwd(N=17) == 2                      # N must be n_cls + gh * gw
    assert fwd(ncls=2, N=18) == 2              # at most one class token
    assert fwd(gh=80, gw=80, N=6400) == 5      # 159^2 entries do not fit
    assert fwd(d=33, N=16) == 5
    assert fwd(table=A + 2) == 4


def test_pack_host_validation(L):
    def pack(x=A, dt=1, B=1, H=1, N=4, d=64, bits=A, alpha=A):
        return L.binattn_pack(P(x), dt, B, H, N, d, P(bits), P(alpha), None)
    assert pack(x=0) == 1
    assert pack(alpha=0) == 1
    assert pack(bits=A + 4) == 4
    assert pack(dt=7) == 3
    assert pack(d=0) == 2
    assert pack(N=-1) == 2


def test_scores_and_ref_host_validation(L):
    assert L.binattn_scores_debug(P(A), P(0), 1, 1, 4, 64, P(A), 0, None) == 1
    assert L.binattn_scores_debug(P(A), P(A), 1, 1, 4, 200, P(A), 0, None) == 2
    assert L.binattn_scores_debug(P(A), P(A), 1, 1, 4, 64, P(A), 9, None) == 8
    # both TC score kernels need d % 8 == 0; TC_BIASED is not a forward engine
    assert L.binattn_scores_debug(P(A), P(A), 1, 1, 4, 33, P(A), binattn.ENGINE_TC_BIASED, None) == 5
    assert L.binattn_scores_debug(P(A), P(A), 1, 1, 4, 33, P(A), binattn.ENGINE_TC, None) == 5
    assert _fwd(L, engine=binattn.ENGINE_TC_BIASED) == 8
    assert L.binattn_ref_bf16_forward(P(A), P(A), None, P(A), ctypes.c_float(1.0), 1, 1, 4, 33,
                                      P(A), None) == 5
    assert L.binattn_ref_bf16_forward(P(A), P(A), None, P(A + 2), ctypes.c_float(1.0), 1, 1, 4, 64,
                                      P(A), None) == 4
    assert L.binattn_ref_bf16_forward(P(A), P(A), None, P(A), ctypes.c_float(math.inf), 1, 1, 4, 64,
                                      P(A), None) == 8


def test_ref_ws_host_validation(L):
    def rws(ws=A, size=1 << 30, N=4096, d=72, bias=A):
        return L.binattn_ref_bf16_forward_ws(P(A), P(A), P(bias) if bias else None, P(A), ctypes.c_float(0.125),
                                             2, 16, N, d, P(A), P(ws) if ws else None, ctypes.c_size_t(size), None)
    # the reference's workspace is the split partials of the binary forward's
    # plan (none on a shape the TMA-fed reference does not take)
    assert L.binattn_ref_bf16_forward_workspace_bytes(2, 16, 4096, 72, 1) == _expected_ws(2, 16, 4096, 72, False)
    assert L.binattn_ref_bf16_forward_workspace_bytes(2, 16, 4096, 80, 1) == 0
    assert L.binattn_ref_bf16_forward_workspace_bytes(0, 16, 4096, 72, 1) == 0
    assert rws(d=33) == 5
    assert rws(bias=A + 2) == 4
    assert rws(N=0) == 2
    need = L.binattn_ref_bf16_forward_workspace_bytes(2, 16, 4096, 72, 1)
    if need:  # only with a device to ask for the SM count
        assert rws(ws=0) == 1
        assert rws(ws=A + 8) == 4
        assert rws(size=need - 1) == 8


def test_last_error_message_is_specific(L):
    assert _fwd(L, v=A + 8) == 4
    assert b"v is not 16-byte aligned" in L.binattn_last_error_message()


def _expected_ws(B, H, N, d, has_bias):
    """Padded bias (rounded to 256 bytes) + split-tail partials (only with a device to ask)."""
    pad = 0
    if has_bias and N % 8:
        pad = -(-H * N * (-(-N // 8) * 8) * 2 // 256) * 256
    split = 0
    import torch
    if torch.cuda.is_available():
        nsm = torch.cuda.get_device_properties(0).multi_processor_count
        P = B * H * (-(-N // 256))
        tail = P - P // nsm * nsm
        if P // nsm and tail and 2 * tail <= nsm and -(-N // 64) >= 32:
            split = tail * 512 * 2 * (d + 2) * 4
    return pad + split


def test_workspace_bytes(L):
    # a bias whose rows are not a multiple of 8 elements: [H][N][roundup(N, 8)] bf16
    for shape in [(64, 12, 197, 64), (32, 16, 577, 64), (2, 16, 4096, 72), (1, 2, 300, 8)]:
        assert L.binattn_forward_workspace_bytes(*shape, 1) == _expected_ws(*shape, True), shape
    assert L.binattn_forward_workspace_bytes(64, 12, 197, 64, 1) >= 12 * 197 * 200 * 2
    # no bias, or a shape the TMA-fed pipeline does not take
    assert L.binattn_forward_workspace_bytes(64, 12, 197, 64, 0) == _expected_ws(64, 12, 197, 64, False)
    assert L.binattn_forward_workspace_bytes(1, 1, 197, 128, 1) == 0
    assert L.binattn_forward_workspace_bytes(1, 1, 197, 33, 1) == 0
    assert L.binattn_forward_workspace_bytes(0, 1, 197, 64, 1) == 0


def test_forward_ws_host_validation(L):
    def fws(ws=A, size=1 << 30, bias=A, N=197, d=64):
        return L.binattn_forward_ws(P(A), P(A), P(A), P(A), P(bias) if bias else None, P(A),
                                    ctypes.c_float(0.125), 1, 2, N, d, P(A),
                                    P(ws) if ws else None, ctypes.c_size_t(size), None)
    need = L.binattn_forward_workspace_bytes(1, 2, 197, 64, 1)
    assert fws(ws=0) == 1
    assert fws(ws=A + 8) == 4
    assert fws(size=need - 1) == 8
    assert b"workspace" in L.binattn_last_error_message()
    assert fws(bias=A + 2) == 4
    assert fws(N=0) == 2


def test_fused_workspace_bytes(L):
    # bf16 Q on the TMA-fed pipeline: the forward's own workspace only
    for shape in [(64, 12, 197, 64), (2, 16, 4096, 72), (1, 2, 300, 8)]:
        assert L.binattn_forward_fused_workspace_bytes(*shape, 1, 1) == L.binattn_forward_workspace_bytes(*shape, 1)
    # fp32 Q or a shape the TMA-fed pipeline does not take: room for Q's sign words and alpha_q
    B, H, N, d = 1, 2, 197, 33
    tok = B * H * N
    r256 = lambda x: -(-x // 256) * 256
    assert L.binattn_forward_fused_workspace_bytes(B, H, N, d, 1, 1) == r256(tok * 2 * 4) + r256(tok * 4)
    fw = L.binattn_forward_workspace_bytes(1, 2, 197, 64, 1)
    assert L.binattn_forward_fused_workspace_bytes(1, 2, 197, 64, 0, 1) == r256(fw) + r256(394 * 2 * 4) + r256(394 * 4)
    assert L.binattn_forward_fused_workspace_bytes(0, 2, 197, 64, 1, 1) == 0


def test_forward_fused_host_validation(L):
    def ffs(q=A, dt=1, ws=A, size=1 << 30, bias=A, N=197, d=64, out=A):
        return L.binattn_forward_fused_ws(P(q) if q else None, dt, P(A), P(A), P(bias) if bias else None, P(A),
                                          ctypes.c_float(0.125), 1, 2, N, d, P(out) if out else None,
                                          P(ws) if ws else None, ctypes.c_size_t(size), None)
    need = L.binattn_forward_fused_workspace_bytes(1, 2, 197, 64, 1, 1)
    assert need > 0
    assert ffs(q=0) == 1
    assert ffs(q=A + 4) == 4
    assert ffs(dt=5) == 3
    assert ffs(out=0) == 1
    assert ffs(ws=0) == 1
    assert ffs(size=need - 1) == 8
    assert ffs(N=0) == 2
    assert ffs(bias=A + 2) == 4


def test_binding_checks_shapes_dtypes_and_device():
    # The binding checks sizes, dtypes and the device before any call into the
    # library: the ABI sees bare pointers and would read a short tensor out of
    # bounds. CPU tensors of the right shapes reach the device check.
    import torch

    B, H, N, d = 2, 3, 37, 72
    W = 3
    bf = dict(dtype=torch.bfloat16)
    q, k, v = torch.zeros(B, H, N, d, **bf), torch.zeros(B, H, N, d, **bf), torch.zeros(B, H, N, d, **bf)
    bias = torch.zeros(H, N, N, **bf)
    qb, kb = torch.zeros(B, H, N, W, dtype=torch.int32), torch.zeros(B, H, N, W, dtype=torch.int32)
    aq, ak = torch.zeros(B, H, N), torch.zeros(B, H, N)
    cpu = "libbinattn takes CUDA tensors"

    def raises(exc, match, fn, *a, **kw):
        with pytest.raises(exc, match=match):
            fn(*a, **kw)

    # valid shapes: only the device is wrong
    raises(ValueError, cpu, binattn.pack, q)
    raises(ValueError, cpu, binattn.pack, q, qb, aq)
    raises(ValueError, cpu, binattn.forward, qb, kb, aq, ak, bias, v, 0.1)
    raises(ValueError, cpu, binattn.forward, qb, kb, aq, ak, None, v, 0.1, out=torch.zeros_like(v))
    raises(ValueError, cpu, binattn.forward_static_ws, qb, kb, aq, ak, bias, v, 0.1)
    raises(ValueError, cpu, binattn.scores_debug, qb, kb, d)
    raises(ValueError, cpu, binattn.ref_bf16_forward, q, k, bias, v, 0.1)
    raises(ValueError, cpu, binattn.forward_ws, qb, kb, aq, ak, bias, v, 0.1,
           workspace=torch.zeros(64, dtype=torch.uint8))
    raises(ValueError, cpu, binattn.forward_fused_ws, q.float(), kb, ak, None, v, 0.1)
    # wrong shapes and dtypes
    raises(ValueError, "bits has shape", binattn.pack, q, qb[..., :2], aq)
    raises(ValueError, "alpha has shape", binattn.pack, q, qb, aq[:, :, :5])
    raises(TypeError, "bits has dtype", binattn.pack, q, qb.float(), aq)
    raises(ValueError, "k_bits has shape", binattn.forward, qb, kb[:, :, :5], aq, ak, bias, v, 0.1)
    raises(ValueError, "q_bits has shape", binattn.forward, qb[..., :2], kb, aq, ak, bias, v, 0.1)
    raises(ValueError, "bias has shape", binattn.forward, qb, kb, aq, ak, bias[:, :5], v, 0.1)
    raises(ValueError, "bias has shape", binattn.forward_ws, qb, kb, aq, ak, bias[:1], v, 0.1)
    raises(TypeError, "bias has dtype", binattn.forward, qb, kb, aq, ak, bias.float(), v, 0.1)
    raises(TypeError, "v has dtype", binattn.forward, qb, kb, aq, ak, bias, v.float(), 0.1)
    raises(ValueError, "alpha_q has shape", binattn.forward_static_ws, qb, kb, aq[:1], ak, bias, v, 0.1)
    raises(ValueError, "out has shape", binattn.forward, qb, kb, aq, ak, bias, v, 0.1, out=v[:1])
    raises(ValueError, "alpha_k has shape", binattn.forward_fused_ws, q, kb, ak[:1], bias, v, 0.1)
    raises(ValueError, "q has shape", binattn.forward_fused_ws, q[:1], kb, ak, bias, v, 0.1)
    raises(ValueError, "S has shape", binattn.scores_debug, qb, kb, d, S=torch.zeros(1, dtype=torch.int32))
    raises(ValueError, "k has shape", binattn.ref_bf16_forward, q, k[:1], bias, v, 0.1)
    # the words per token follow d
    raises(ValueError, "q_bits has shape", binattn.scores_debug, qb, kb, 64)


def test_binding_marshals_every_call(monkeypatch):
    # Each binding function, with its device handling stubbed out, hands the
    # library exactly the arguments the ABI declares: the count of the real
    # argtypes, the sizes of the tensors and the pointers of the tensors.
    import contextlib
    import types

    import torch

    real = binattn.lib()
    calls = []

    class FakeLib:
        def __getattr__(self, name):
            fn = getattr(real, name)

            def call(*args):
                if fn.argtypes is not None:
                    assert len(args) == len(fn.argtypes), name
                calls.append((name, args))
                return 0 if name != "binattn_forward_workspace_bytes" else 4096
            return call

    cpu = torch.device("cpu")
    monkeypatch.setattr(binattn, "lib", lambda: FakeLib())
    monkeypatch.setattr(binattn, "_device", lambda *t: cpu)
    monkeypatch.setattr(torch.cuda, "device", lambda dev: contextlib.nullcontext())
    monkeypatch.setattr(torch.cuda, "current_stream", lambda dev=None: types.SimpleNamespace(cuda_stream=0, device=cpu))

    B, H, N, d = 1, 2, 33, 40
    bf = dict(dtype=torch.bfloat16)
    q, v = torch.zeros(B, H, N, d, **bf), torch.zeros(B, H, N, d, **bf)
    bias = torch.zeros(H, N, N, **bf)
    qb, aq = binattn.pack(q)
    assert qb.shape == (B, H, N, 2) and qb.dtype == torch.int32 and aq.shape == (B, H, N)
    name, args = calls[-1]
    assert name == "binattn_pack" and args[1:6] == (binattn.BF16, B, H, N, d)
    assert args[0].value == q.data_ptr() and args[6].value == qb.data_ptr()
    out = binattn.forward(qb, qb, aq, aq, bias, v, 0.25, engine="tc")
    name, args = calls[-1]
    assert name == "binattn_forward_engine" and args[7:11] == (B, H, N, d) and args[12] == binattn.ENGINE_TC
    assert args[4].value == bias.data_ptr() and args[11].value == out.data_ptr() and args[6] == 0.25
    binattn.forward(qb, qb, aq, aq, None, v, 0.25)
    assert calls[-1][1][4] is None
    binattn.forward_ws(qb, qb, aq, aq, bias, v, 0.25)
    name, args = calls[-1]
    assert name == "binattn_forward_ws" and args[13].value == 4096
    binattn.forward_static_ws(qb, qb, aq, aq, bias, v, 0.25)
    assert calls[-1][0] == "binattn_forward_static_ws"
    binattn.forward_fused_ws(q, qb, aq, bias, v, 0.25)
    name, args = calls[-1]
    assert name == "binattn_forward_fused_ws" and args[1] == binattn.BF16 and args[7:11] == (B, H, N, d)
    S = binattn.scores_debug(qb, qb, d)
    assert S.shape == (B, H, N, N) and calls[-1][1][2:6] == (B, H, N, d)
    binattn.ref_bf16_forward(q, q, None, v, 0.25)
    assert calls[-1][0] == "binattn_ref_bf16_forward" and calls[-1][1][5:9] == (B, H, N, d)
    binattn.ref_bf16_forward_ws(q, q, bias, v, 0.25, workspace=torch.zeros(64, dtype=torch.uint8))
    name, args = calls[-1]
    assert name == "binattn_ref_bf16_forward_ws" and args[5:9] == (B, H, N, d) and args[11].value == 64
    assert args[2].value == bias.data_ptr()
    sbias = torch.zeros(B, H, N, N + 7, **bf)
    binattn.forward_sample_bias_ws(qb, qb, aq, aq, sbias, v, 0.25, workspace=torch.zeros(32, dtype=torch.uint8))
    name, args = calls[-1]
    assert name == "binattn_forward_sample_bias_ws" and args[5] == N + 7 and args[8:12] == (B, H, N, d)
    assert args[4].value == sbias.data_ptr() and args[14].value == 32
    with pytest.raises(ValueError, match="bias must be"):
        binattn.forward_sample_bias_ws(qb, qb, aq, aq, bias, v, 0.25)
    dV, ds, dt, db = binattn.backward(qb, qb, aq, aq, bias, v, q, 0.25)
    name, args = calls[-1]
    assert name == "binattn_backward" and args[8:12] == (B, H, N, d) and args[7] == 0.25
    assert args[6].value == q.data_ptr() and args[12].value == dV.data_ptr() and args[15].value == db.data_ptr()
    assert dV.dtype == torch.float32 and dV.shape == (B, H, N, d) and db.shape == (H, N, N)
    binattn.backward(qb, qb, aq, aq, None, v, q, 0.25, with_dbias=False)
    assert calls[-1][1][4] is None and calls[-1][1][15] is None


@pytest.mark.parametrize("lang,std", [("c", "c99"), ("c++", "c++11")])
def test_header_is_plain_c(tmp_path, lang, std):
    # The boundary header needs no CUDA or torch include: it compiles as plain
    # C99 and C++11, and a C program can take the address of every entry point.
    import shutil
    import subprocess

    cc = shutil.which("gcc" if lang == "c" else "g++")
    if cc is None:
        pytest.skip("no host compiler")
    inc = os.path.dirname(HEADER)
    src = tmp_path / ("use.c" if lang == "c" else "use.cpp")
    names = declared_functions()
    src.write_text('#include "binattn.h"\nvoid* const table[] = {\n' +
                   ",\n".join(f"  (void*){n}" for n in names) + "\n};\n")
    subprocess.run([cc, f"-std={std}", "-Wall", "-Werror", "-fsyntax-only", "-I", inc, str(src)], check=True)
