"""Thin Python binding of libbinattn (the C ABI in include/binattn.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libbinattn.so. torch is used for device memory and streams. There is
no CPU fallback: if the library is missing, importing a function raises.
Each call first checks the shapes, dtypes and device of its tensors, which the
ABI cannot see behind its pointers, and runs with that device current.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

OK = 0
F32, BF16 = 0, 1
ENGINE_AUTO, ENGINE_SIMT, ENGINE_POPC_TC, ENGINE_TC, ENGINE_TC_BIASED = 0, 1, 2, 3, 4
ENGINES = {"auto": ENGINE_AUTO, "simt": ENGINE_SIMT, "popc_tc": ENGINE_POPC_TC, "tc": ENGINE_TC,
           "tc_biased": ENGINE_TC_BIASED}

# Every symbol include/binattn.h declares.
EXPORTS = (
    "binattn_pack", "binattn_forward", "binattn_forward_engine", "binattn_forward_workspace_bytes",
    "binattn_forward_ws", "binattn_forward_static_ws", "binattn_forward_fused_workspace_bytes",
    "binattn_forward_fused_ws", "binattn_scores_debug",
    "binattn_ref_bf16_forward", "binattn_device_status", "binattn_strerror",
    "binattn_last_error_message", "binattn_abi_version", "binattn_test_wait_timeout",
    "binattn_forward_bias_ld_workspace_bytes", "binattn_padded_bias_ld", "binattn_forward_bias_ld_ws",
    "binattn_quantize_v", "binattn_forward_int8_workspace_bytes", "binattn_forward_int8",
    "binattn_forward_relpos_workspace_bytes", "binattn_forward_relpos",
    "binattn_ref_bf16_forward_workspace_bytes", "binattn_ref_bf16_forward_ws",
    "binattn_forward_sample_bias_workspace_bytes", "binattn_forward_sample_bias_ws",
    "binattn_backward_workspace_bytes", "binattn_backward",
)


class BinattnError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__(f"{where}: status {status} ({detail})")


_lib = None


def library_path() -> str:
    return _build.LIBRARY


def lib() -> ctypes.CDLL:
    """Load libbinattn.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m diffusion_transformers_b200.build`")
    L = ctypes.CDLL(path)
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    L.binattn_pack.argtypes = [P, I, I, I, I, I, P, P, P]
    L.binattn_forward.argtypes = [P, P, P, P, P, P, F, I, I, I, I, P, P]
    L.binattn_forward_engine.argtypes = [P, P, P, P, P, P, F, I, I, I, I, P, I, P]
    L.binattn_forward_workspace_bytes.argtypes = [I, I, I, I, I]
    L.binattn_forward_workspace_bytes.restype = ctypes.c_size_t
    L.binattn_forward_ws.argtypes = [P, P, P, P, P, P, F, I, I, I, I, P, P, ctypes.c_size_t, P]
    L.binattn_forward_static_ws.argtypes = [P, P, P, P, P, P, F, I, I, I, I, P, P]
    L.binattn_forward_bias_ld_workspace_bytes.argtypes = [I, I, I, I, I]
    L.binattn_forward_bias_ld_workspace_bytes.restype = ctypes.c_size_t
    L.binattn_padded_bias_ld.argtypes = [I]
    L.binattn_padded_bias_ld.restype = I
    L.binattn_forward_bias_ld_ws.argtypes = [P, P, P, P, P, I, P, F, I, I, I, I, P, P, ctypes.c_size_t, P]
    L.binattn_forward_bias_ld_ws.restype = I
    L.binattn_forward_sample_bias_workspace_bytes.argtypes = [I, I, I, I, I]
    L.binattn_forward_sample_bias_workspace_bytes.restype = ctypes.c_size_t
    L.binattn_forward_sample_bias_ws.argtypes = [P, P, P, P, P, I, P, F, I, I, I, I, P, P, ctypes.c_size_t, P]
    L.binattn_forward_sample_bias_ws.restype = I
    L.binattn_backward_workspace_bytes.argtypes = [I, I, I, I]
    L.binattn_backward_workspace_bytes.restype = ctypes.c_size_t
    L.binattn_backward.argtypes = [P, P, P, P, P, P, P, F, I, I, I, I, P, P, P, P, P, ctypes.c_size_t, P]
    L.binattn_backward.restype = I
    L.binattn_quantize_v.argtypes = [P, I, I, I, I, P, P, P]
    L.binattn_quantize_v.restype = I
    L.binattn_forward_int8_workspace_bytes.argtypes = [I, I, I, I, I]
    L.binattn_forward_int8_workspace_bytes.restype = ctypes.c_size_t
    L.binattn_forward_int8.argtypes = [P, P, P, P, P, P, F, I, I, I, I, P, P, ctypes.c_size_t, P]
    L.binattn_forward_int8.restype = I
    L.binattn_forward_relpos_workspace_bytes.argtypes = [I, I, I, I]
    L.binattn_forward_relpos_workspace_bytes.restype = ctypes.c_size_t
    L.binattn_forward_relpos.argtypes = [P, P, P, P, P, I, I, I, P, F, I, I, I, I, P, P, ctypes.c_size_t, P]
    L.binattn_forward_relpos.restype = I
    L.binattn_forward_fused_workspace_bytes.argtypes = [I, I, I, I, I, I]
    L.binattn_forward_fused_workspace_bytes.restype = ctypes.c_size_t
    L.binattn_forward_fused_ws.argtypes = [P, I, P, P, P, P, F, I, I, I, I, P, P, ctypes.c_size_t, P]
    L.binattn_scores_debug.argtypes = [P, P, I, I, I, I, P, I, P]
    L.binattn_ref_bf16_forward.argtypes = [P, P, P, P, F, I, I, I, I, P, P]
    L.binattn_ref_bf16_forward_workspace_bytes.argtypes = [I, I, I, I, I]
    L.binattn_ref_bf16_forward_workspace_bytes.restype = ctypes.c_size_t
    L.binattn_ref_bf16_forward_ws.argtypes = [P, P, P, P, F, I, I, I, I, P, P, ctypes.c_size_t, P]
    L.binattn_ref_bf16_forward_ws.restype = I
    L.binattn_test_wait_timeout.argtypes = [P, P, P, P, P, P, F, I, I, I, I, P, I, P]
    L.binattn_device_status.argtypes = [P]
    L.binattn_strerror.argtypes = [I]
    L.binattn_strerror.restype = ctypes.c_char_p
    L.binattn_last_error_message.restype = ctypes.c_char_p
    for name in ("binattn_pack", "binattn_forward", "binattn_forward_engine", "binattn_forward_ws",
                 "binattn_forward_static_ws", "binattn_forward_fused_ws",
                 "binattn_scores_debug",
                 "binattn_ref_bf16_forward", "binattn_device_status", "binattn_abi_version",
                 "binattn_test_wait_timeout"):
        getattr(L, name).restype = I
    _lib = L
    return L


def _check(rc: int, where: str) -> None:
    if rc != OK:
        L = lib()
        detail = L.binattn_last_error_message().decode() or L.binattn_strerror(rc).decode()
        raise BinattnError(rc, where, detail)


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libbinattn must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


_BITS = (torch.int32, getattr(torch, "uint32", torch.int32))


def _expect(t: torch.Tensor | None, name: str, shape, dtypes) -> None:
    """Shape and dtype of one argument; the C ABI sees only pointers, so a
    tensor smaller than the sizes passed with it would be read out of bounds."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} has dtype {t.dtype}, expected one of {tuple(str(d) for d in dtypes)}")


def _device(*tensors: torch.Tensor | None) -> torch.device:
    """The one CUDA device that holds every given tensor."""
    devs = {t.device for t in tensors if t is not None}
    if len(devs) != 1:
        raise ValueError(f"all tensors must be on one CUDA device, got {sorted(str(d) for d in devs)}")
    dev = devs.pop()
    if dev.type != "cuda":
        raise ValueError(f"libbinattn takes CUDA tensors, got {dev}")
    return dev


def _stream(stream, dev: torch.device) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    elif stream.device != dev:
        raise ValueError(f"stream is on {stream.device}, the tensors on {dev}")
    return ctypes.c_void_p(stream.cuda_stream)


def _words(d: int) -> int:
    return (d + 31) // 32


def pack(x: torch.Tensor, bits: torch.Tensor | None = None, alpha: torch.Tensor | None = None,
         stream=None):
    """x [B,H,N,d] (float32 or bfloat16, CUDA) -> (bits uint32-as-int32 [B,H,N,W], alpha fp32 [B,H,N])."""
    B, H, N, d = x.shape
    dt = {torch.float32: F32, torch.bfloat16: BF16}.get(x.dtype)
    if dt is None:
        raise TypeError(f"pack takes float32 or bfloat16, got {x.dtype}")
    _expect(bits, "bits", (B, H, N, _words(d)), _BITS)
    _expect(alpha, "alpha", (B, H, N), (torch.float32,))
    dev = _device(x, bits, alpha)
    if bits is None:
        bits = torch.empty((B, H, N, _words(d)), dtype=torch.int32, device=dev)
    if alpha is None:
        alpha = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _check(lib().binattn_pack(_ptr(x), dt, B, H, N, d, _ptr(bits), _ptr(alpha), _stream(stream, dev)),
               "binattn_pack")
    return bits, alpha


def _forward_args(q_bits, k_bits, alpha_q, alpha_k, bias, v, out) -> torch.device:
    """Checks shared by the forward calls; V [B,H,N,d] fixes the sizes."""
    B, H, N, d = v.shape
    _expect(v, "v", (B, H, N, d), (torch.bfloat16,))
    _expect(q_bits, "q_bits", (B, H, N, _words(d)), _BITS)
    _expect(k_bits, "k_bits", (B, H, N, _words(d)), _BITS)
    _expect(alpha_q, "alpha_q", (B, H, N), (torch.float32,))
    _expect(alpha_k, "alpha_k", (B, H, N), (torch.float32,))
    _expect(bias, "bias", (H, N, N), (torch.bfloat16,))
    _expect(out, "out", (B, H, N, d), (torch.bfloat16,))
    return _device(q_bits, k_bits, alpha_q, alpha_k, bias, v, out)


def forward(q_bits: torch.Tensor, k_bits: torch.Tensor, alpha_q: torch.Tensor,
            alpha_k: torch.Tensor, bias: torch.Tensor | None, v: torch.Tensor,
            softmax_scale: float, out: torch.Tensor | None = None, engine: int | str = ENGINE_AUTO,
            stream=None) -> torch.Tensor:
    """O [B,H,N,d] bfloat16 = softmax(scale * a_q a_k^T * S + bias) V."""
    B, H, N, d = v.shape
    if isinstance(engine, str):
        engine = ENGINES[engine]
    dev = _forward_args(q_bits, k_bits, alpha_q, alpha_k, bias, v, out)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
    with torch.cuda.device(dev):
        _check(lib().binattn_forward_engine(_ptr(q_bits), _ptr(k_bits), _ptr(alpha_q), _ptr(alpha_k),
                                            _ptr(bias), _ptr(v), float(softmax_scale), B, H, N, d,
                                            _ptr(out), int(engine), _stream(stream, dev)),
               "binattn_forward_engine")
    return out


def scores_debug(q_bits: torch.Tensor, k_bits: torch.Tensor, d: int,
                 engine: int | str = ENGINE_AUTO, S: torch.Tensor | None = None,
                 stream=None) -> torch.Tensor:
    """Integer scores S [B,H,N,N] int32 as the given engine computes them."""
    B, H, N, _ = q_bits.shape
    if isinstance(engine, str):
        engine = ENGINES[engine]
    _expect(q_bits, "q_bits", (B, H, N, _words(d)), _BITS)
    _expect(k_bits, "k_bits", (B, H, N, _words(d)), _BITS)
    _expect(S, "S", (B, H, N, N), (torch.int32,))
    dev = _device(q_bits, k_bits, S)
    if S is None:
        S = torch.empty((B, H, N, N), dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        _check(lib().binattn_scores_debug(_ptr(q_bits), _ptr(k_bits), B, H, N, d, _ptr(S), int(engine),
                                          _stream(stream, dev)), "binattn_scores_debug")
    return S


def workspace_bytes(B: int, H: int, N: int, d: int, has_bias: bool) -> int:
    """Device workspace bytes forward_ws needs (0: forward already takes the fast path)."""
    return int(lib().binattn_forward_workspace_bytes(B, H, N, d, int(bool(has_bias))))


def forward_ws(q_bits: torch.Tensor, k_bits: torch.Tensor, alpha_q: torch.Tensor,
               alpha_k: torch.Tensor, bias: torch.Tensor | None, v: torch.Tensor,
               softmax_scale: float, workspace: torch.Tensor | None = None,
               out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """forward (engine AUTO) with a caller-owned workspace (uint8 CUDA tensor of at
    least workspace_bytes(...) bytes; allocated here when None)."""
    B, H, N, d = v.shape
    dev = _forward_args(q_bits, k_bits, alpha_q, alpha_k, bias, v, out)
    if workspace is not None:
        _device(workspace, v)
    need = workspace_bytes(B, H, N, d, bias is not None)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
    size = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        _check(lib().binattn_forward_ws(_ptr(q_bits), _ptr(k_bits), _ptr(alpha_q), _ptr(alpha_k), _ptr(bias),
                                        _ptr(v), float(softmax_scale), B, H, N, d, _ptr(out), _ptr(workspace),
                                        ctypes.c_size_t(size), _stream(stream, dev)),
               "binattn_forward_ws")
    return out


def padded_bias_ld(N: int) -> int:
    """Row stride (elements) at which a stored bias is read by the TMA-fed
    pipeline as it is: N rounded up to a multiple of 8."""
    return int(lib().binattn_padded_bias_ld(int(N)))


def pad_bias(bias: torch.Tensor) -> torch.Tensor:
    """A learned bias [H, N, N] stored once as [H, N, padded_bias_ld(N)] (zero
    pad), for forward_bias_ld_ws. Plain torch copy: it is done once, not per call."""
    H, N, _ = bias.shape
    out = torch.zeros((H, N, padded_bias_ld(N)), dtype=bias.dtype, device=bias.device)
    out[:, :, :N] = bias
    return out


def forward_bias_ld_ws(q_bits: torch.Tensor, k_bits: torch.Tensor, alpha_q: torch.Tensor,
                       alpha_k: torch.Tensor, bias: torch.Tensor, v: torch.Tensor, softmax_scale: float,
                       workspace: torch.Tensor | None = None, out: torch.Tensor | None = None,
                       stream=None) -> torch.Tensor:
    """forward_ws with a bias [H, N, ld] whose rows are ld >= N elements apart
    (only its first N columns are read), e.g. from pad_bias()."""
    B, H, N, d = v.shape
    if bias.dim() != 3 or bias.shape[0] != H or bias.shape[1] != N or bias.shape[2] < N:
        raise ValueError(f"bias must be [H={H}, N={N}, ld >= N], got {tuple(bias.shape)}")
    if bias.dtype != torch.bfloat16 or not bias.is_contiguous():
        raise TypeError("bias must be a contiguous bfloat16 tensor")
    ld = bias.shape[2]
    dev = _forward_args(q_bits, k_bits, alpha_q, alpha_k, None, v, out)
    _device(bias, v)
    if workspace is not None:
        _device(workspace, v)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
    need = int(lib().binattn_forward_bias_ld_workspace_bytes(B, H, N, d, ld))
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    size = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        _check(lib().binattn_forward_bias_ld_ws(_ptr(q_bits), _ptr(k_bits), _ptr(alpha_q), _ptr(alpha_k), _ptr(bias),
                                                ld, _ptr(v), float(softmax_scale), B, H, N, d, _ptr(out),
                                                _ptr(workspace), ctypes.c_size_t(size), _stream(stream, dev)),
               "binattn_forward_bias_ld_ws")
    return out


def forward_sample_bias_ws(q_bits: torch.Tensor, k_bits: torch.Tensor, alpha_q: torch.Tensor,
                           alpha_k: torch.Tensor, bias: torch.Tensor, v: torch.Tensor, softmax_scale: float,
                           workspace: torch.Tensor | None = None, out: torch.Tensor | None = None,
                           stream=None) -> torch.Tensor:
    """forward_ws with one bias per batch entry (a context-aware bias, computed
    per sample): bias [B, H, N, ld], ld >= N (only its first N columns are read)."""
    B, H, N, d = v.shape
    if bias.dim() != 4 or tuple(bias.shape[:3]) != (B, H, N) or bias.shape[3] < N:
        raise ValueError(f"bias must be [B={B}, H={H}, N={N}, ld >= N], got {tuple(bias.shape)}")
    if bias.dtype != torch.bfloat16 or not bias.is_contiguous():
        raise TypeError("bias must be a contiguous bfloat16 tensor")
    ld = bias.shape[3]
    dev = _forward_args(q_bits, k_bits, alpha_q, alpha_k, None, v, out)
    _device(bias, v)
    if workspace is not None:
        _device(workspace, v)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
    need = int(lib().binattn_forward_sample_bias_workspace_bytes(B, H, N, d, ld))
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    size = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        _check(lib().binattn_forward_sample_bias_ws(_ptr(q_bits), _ptr(k_bits), _ptr(alpha_q), _ptr(alpha_k),
                                                    _ptr(bias), ld, _ptr(v), float(softmax_scale), B, H, N, d,
                                                    _ptr(out), _ptr(workspace), ctypes.c_size_t(size),
                                                    _stream(stream, dev)),
               "binattn_forward_sample_bias_ws")
    return out


def backward(q_bits: torch.Tensor, k_bits: torch.Tensor, alpha_q: torch.Tensor, alpha_k: torch.Tensor,
             bias: torch.Tensor | None, v: torch.Tensor, dO: torch.Tensor, softmax_scale: float,
             with_dbias: bool = True, workspace: torch.Tensor | None = None, stream=None):
    """Gradients of the forward for an upstream gradient dO (bf16 [B,H,N,d]):
    (dV, ds, dt, dbias), dV/ds/dt fp32 [B,H,N,d] (ds, dt with respect to the
    scaled binary Q and K, alpha * sign), dbias fp32 [H,N,N] summed over the
    batch, or None without with_dbias."""
    B, H, N, d = v.shape
    dev = _forward_args(q_bits, k_bits, alpha_q, alpha_k, bias, v, None)
    _expect(dO, "dO", (B, H, N, d), (torch.bfloat16,))
    _device(dO, v)
    if workspace is not None:
        _device(workspace, v)
    f32 = dict(dtype=torch.float32, device=dev)
    dV, ds, dt = (torch.empty((B, H, N, d), **f32) for _ in range(3))
    dbias = torch.empty((H, N, N), **f32) if with_dbias else None
    need = int(lib().binattn_backward_workspace_bytes(B, H, N, d))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    size = workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        _check(lib().binattn_backward(_ptr(q_bits), _ptr(k_bits), _ptr(alpha_q), _ptr(alpha_k), _ptr(bias), _ptr(v),
                                      _ptr(dO), float(softmax_scale), B, H, N, d, _ptr(dV), _ptr(ds), _ptr(dt),
                                      _ptr(dbias), _ptr(workspace), ctypes.c_size_t(size), _stream(stream, dev)),
               "binattn_backward")
    return dV, ds, dt, dbias


def quantize_v(v: torch.Tensor, stream=None):
    """V's per-channel 8-bit code: vq int8 [B,H,N,d] and scale fp32 [B,H,d]."""
    B, H, N, d = v.shape
    _expect(v, "v", (B, H, N, d), (torch.bfloat16,))
    dev = _device(v)
    vq = torch.empty((B, H, N, d), dtype=torch.int8, device=dev)
    scale = torch.empty((B, H, d), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _check(lib().binattn_quantize_v(_ptr(v), B, H, N, d, _ptr(vq), _ptr(scale), _stream(stream, dev)),
               "binattn_quantize_v")
    return vq, scale


def int8_workspace_bytes(B: int, H: int, N: int, d: int, has_bias: bool) -> int:
    return int(lib().binattn_forward_int8_workspace_bytes(B, H, N, d, int(has_bias)))


def forward_int8(q_bits: torch.Tensor, k_bits: torch.Tensor, alpha_q: torch.Tensor, alpha_k: torch.Tensor,
                 bias: torch.Tensor | None, v: torch.Tensor, softmax_scale: float,
                 workspace: torch.Tensor | None = None, out: torch.Tensor | None = None,
                 stream=None) -> torch.Tensor:
    """O [B,H,N,d] bfloat16 of the 8-bit P.V forward (binattn_forward_int8)."""
    B, H, N, d = v.shape
    dev = _forward_args(q_bits, k_bits, alpha_q, alpha_k, bias, v, out)
    if workspace is not None:
        _device(workspace, v)
    need = int8_workspace_bytes(B, H, N, d, bias is not None)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
    size = workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        _check(lib().binattn_forward_int8(_ptr(q_bits), _ptr(k_bits), _ptr(alpha_q), _ptr(alpha_k), _ptr(bias),
                                          _ptr(v), float(softmax_scale), B, H, N, d, _ptr(out), _ptr(workspace),
                                          ctypes.c_size_t(size), _stream(stream, dev)), "binattn_forward_int8")
    return out


def relpos_table_entries(gh: int, gw: int, n_cls: int) -> int:
    """Entries per head of a relative-position table: (2gh-1)(2gw-1) + 3 n_cls."""
    return (2 * gh - 1) * (2 * gw - 1) + 3 * n_cls


def forward_relpos(q_bits: torch.Tensor, k_bits: torch.Tensor, alpha_q: torch.Tensor, alpha_k: torch.Tensor,
                   table: torch.Tensor, grid: tuple[int, int], n_cls: int, v: torch.Tensor, softmax_scale: float,
                   workspace: torch.Tensor | None = None, out: torch.Tensor | None = None,
                   stream=None) -> torch.Tensor:
    """forward with the position-sensitive bias: a relative-position table
    [H, relpos_table_entries(gh, gw, n_cls)] (bf16) of a gh x gw patch grid
    after n_cls class tokens (binattn_forward_relpos)."""
    B, H, N, d = v.shape
    gh, gw = grid
    _expect(table, "table", (H, relpos_table_entries(gh, gw, n_cls)), (torch.bfloat16,))
    dev = _forward_args(q_bits, k_bits, alpha_q, alpha_k, None, v, out)
    _device(table, v)
    if workspace is not None:
        _device(workspace, v)
    need = int(lib().binattn_forward_relpos_workspace_bytes(B, H, N, d))
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
    size = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        _check(lib().binattn_forward_relpos(_ptr(q_bits), _ptr(k_bits), _ptr(alpha_q), _ptr(alpha_k), _ptr(table),
                                            int(gh), int(gw), int(n_cls), _ptr(v), float(softmax_scale), B, H, N, d,
                                            _ptr(out), _ptr(workspace), ctypes.c_size_t(size), _stream(stream, dev)),
               "binattn_forward_relpos")
    return out


def forward_static_ws(q_bits: torch.Tensor, k_bits: torch.Tensor, alpha_q: torch.Tensor,
                      alpha_k: torch.Tensor, bias: torch.Tensor | None, v: torch.Tensor,
                      softmax_scale: float, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """forward_ws on the library's static workspace: the call allocates no device memory."""
    B, H, N, d = v.shape
    dev = _forward_args(q_bits, k_bits, alpha_q, alpha_k, bias, v, out)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
    with torch.cuda.device(dev):
        _check(lib().binattn_forward_static_ws(_ptr(q_bits), _ptr(k_bits), _ptr(alpha_q), _ptr(alpha_k),
                                               _ptr(bias), _ptr(v), float(softmax_scale), B, H, N, d, _ptr(out),
                                               _stream(stream, dev)),
               "binattn_forward_static_ws")
    return out


def fused_workspace_bytes(B: int, H: int, N: int, d: int, q_dtype: torch.dtype, has_bias: bool) -> int:
    """Device workspace bytes forward_fused_ws needs."""
    dt = {torch.float32: F32, torch.bfloat16: BF16}[q_dtype]
    return int(lib().binattn_forward_fused_workspace_bytes(B, H, N, d, dt, int(bool(has_bias))))


def forward_fused_ws(q: torch.Tensor, k_bits: torch.Tensor, alpha_k: torch.Tensor, bias: torch.Tensor | None,
                     v: torch.Tensor, softmax_scale: float, workspace: torch.Tensor | None = None,
                     out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """pack(Q) + forward_ws in one call; the forward kernel binarises bf16 Q itself
    where the shape allows (same result as pack followed by forward_ws)."""
    B, H, N, d = v.shape
    dt = {torch.float32: F32, torch.bfloat16: BF16}.get(q.dtype)
    if dt is None:
        raise TypeError(f"q must be float32 or bfloat16, got {q.dtype}")
    _expect(q, "q", (B, H, N, d), (q.dtype,))
    dev = _forward_args(None, k_bits, None, alpha_k, bias, v, out)
    _device(q, v, workspace)
    need = fused_workspace_bytes(B, H, N, d, q.dtype, bias is not None)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
    size = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        _check(lib().binattn_forward_fused_ws(_ptr(q), dt, _ptr(k_bits), _ptr(alpha_k), _ptr(bias), _ptr(v),
                                              float(softmax_scale), B, H, N, d, _ptr(out), _ptr(workspace),
                                              ctypes.c_size_t(size), _stream(stream, dev)),
               "binattn_forward_fused_ws")
    return out


def ref_bf16_forward(q: torch.Tensor, k: torch.Tensor, bias: torch.Tensor | None, v: torch.Tensor,
                     softmax_scale: float, out: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
    """Full-precision bf16 softmax attention on the same shapes (speed reference)."""
    B, H, N, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out)):
        _expect(t, name, (B, H, N, d), (torch.bfloat16,))
    _expect(bias, "bias", (H, N, N), (torch.bfloat16,))
    dev = _device(q, k, bias, v, out)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
    with torch.cuda.device(dev):
        _check(lib().binattn_ref_bf16_forward(_ptr(q), _ptr(k), _ptr(bias), _ptr(v), float(softmax_scale),
                                              B, H, N, d, _ptr(out), _stream(stream, dev)),
               "binattn_ref_bf16_forward")
    return out


def ref_bf16_forward_ws(q: torch.Tensor, k: torch.Tensor, bias: torch.Tensor | None, v: torch.Tensor,
                        softmax_scale: float, workspace: torch.Tensor | None = None,
                        out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """ref_bf16_forward with the long-sequence launch plan of forward_ws (a
    short last wave split by key halves); workspace of
    binattn_ref_bf16_forward_workspace_bytes, allocated here when None."""
    B, H, N, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out)):
        _expect(t, name, (B, H, N, d), (torch.bfloat16,))
    _expect(bias, "bias", (H, N, N), (torch.bfloat16,))
    dev = _device(q, k, bias, v, out)
    if workspace is not None:
        _device(workspace, v)
    need = int(lib().binattn_ref_bf16_forward_workspace_bytes(B, H, N, d, bias is not None))
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
    size = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        _check(lib().binattn_ref_bf16_forward_ws(_ptr(q), _ptr(k), _ptr(bias), _ptr(v), float(softmax_scale),
                                                 B, H, N, d, _ptr(out), _ptr(workspace), ctypes.c_size_t(size),
                                                 _stream(stream, dev)),
               "binattn_ref_bf16_forward_ws")
    return out


def test_wait_timeout(q_bits: torch.Tensor, k_bits: torch.Tensor, alpha_q: torch.Tensor,
                      alpha_k: torch.Tensor, bias: torch.Tensor | None, v: torch.Tensor,
                      softmax_scale: float, stall_after: int, out: torch.Tensor | None = None,
                      stream=None) -> torch.Tensor:
    """Test only: the 64-key forward with its TMA producer stopped at key tile
    stall_after, so that its bounded waits run out (binattn_test_wait_timeout).
    `out` is undefined afterwards; the timeout shows in device_status()."""
    B, H, N, d = v.shape
    dev = _forward_args(q_bits, k_bits, alpha_q, alpha_k, bias, v, out)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
    with torch.cuda.device(dev):
        _check(lib().binattn_test_wait_timeout(_ptr(q_bits), _ptr(k_bits), _ptr(alpha_q), _ptr(alpha_k),
                                               _ptr(bias), _ptr(v), float(softmax_scale), B, H, N, d,
                                               _ptr(out), int(stall_after), _stream(stream, dev)),
               "binattn_test_wait_timeout")
    return out


def device_status(stream=None) -> None:
    """Synchronize and raise if a kernel abandoned a bounded wait (current device,
    or the device of `stream`)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if stream is None else stream.device
    with torch.cuda.device(dev):
        _check(lib().binattn_device_status(_stream(stream, dev)), "binattn_device_status")


def abi_version() -> int:
    return int(lib().binattn_abi_version())
