"""CPU oracle for the BinaryAttention forward pass (ctypes wrapper).

TEST INFRASTRUCTURE, NOT PRODUCT CODE. Only the tests, the smoke check and the
benchmark's CPU-baseline / reference arm import this module; the GPU library
never does, and this module imports nothing from the GPU package.

The arithmetic lives in ``binattn_oracle.c`` (plain C, fp64, OpenMP over query
rows). This file only marshals numpy arrays. See the C file's header for the
steps and the passages of "BinaryAttention: One-Bit QK-Attention for Vision and
Diffusion Transformers" that each step follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "binattn_oracle.c")
LIBRARY = os.path.join(_HERE, "liboracle.so")

F32 = 0
BF16 = 1

_i64p = ctypes.POINTER(ctypes.c_int64)


def build(source: str = SOURCE, out: str = LIBRARY, extra_flags=()) -> str:
    """Compile the oracle with gcc (-O2, no fast-math, OpenMP). Returns the path."""
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
           *extra_flags, "-o", out, source, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _needs_build(src: str, lib: str) -> bool:
    return (not os.path.exists(lib)) or os.path.getmtime(lib) < os.path.getmtime(src)


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return ctypes.c_void_p(a.ctypes.data)


class Oracle:
    """One loaded copy of the oracle library."""

    def __init__(self, lib_path: str = LIBRARY):
        if lib_path == LIBRARY and _needs_build(SOURCE, LIBRARY):
            build()
        self.path = lib_path
        lib = ctypes.CDLL(lib_path)
        L, I, D, V = ctypes.c_long, ctypes.c_int, ctypes.c_double, ctypes.c_void_p
        lib.oracle_pack.argtypes = [V, I, L, L, L, L, V, V]
        lib.oracle_scores_rows.argtypes = [V, V, I, L, L, L, L, L, _i64p, V]
        lib.oracle_probs_rows.argtypes = [V, V, I, V, D, L, L, L, L, L, _i64p, V]
        lib.oracle_forward_rows.argtypes = [V, V, I, V, V, D, L, L, L, L, L, _i64p, V]
        lib.oracle_forward.argtypes = [V, V, I, V, V, D, L, L, L, L, V]
        lib.oracle_forward_spread.argtypes = [V, V, I, V, V, D, L, L, L, L, V, V]
        lib.oracle_quantize_v.argtypes = [V, L, L, L, L, V, V]
        lib.oracle_forward_int8_rows.argtypes = [V, V, I, V, V, D, L, L, L, L, L, _i64p, V]
        lib.oracle_forward_int8.argtypes = [V, V, I, V, V, D, L, L, L, L, V]
        lib.oracle_expand_relpos_bias.argtypes = [V, L, L, L, L, V]
        lib.oracle_backward.argtypes = [V, V, I, V, V, V, D, L, L, L, L, V, V, V, V]
        lib.oracle_num_threads.restype = I
        lib.oracle_set_num_threads.argtypes = [I]
        for f in ("oracle_pack", "oracle_scores_rows", "oracle_probs_rows",
                  "oracle_forward_rows", "oracle_forward", "oracle_forward_spread",
                  "oracle_quantize_v", "oracle_forward_int8_rows", "oracle_forward_int8",
                  "oracle_expand_relpos_bias", "oracle_backward"):
            getattr(lib, f).restype = I
        self.lib = lib

    # ---------------------------------------------------------------- helpers
    @staticmethod
    def _dtype_code(x: np.ndarray) -> int:
        if x.dtype == np.float32:
            return F32
        if x.dtype == np.uint16:  # bf16 bit patterns
            return BF16
        raise TypeError(f"oracle takes float32 or bf16-as-uint16, got {x.dtype}")

    @staticmethod
    def _bf16(a, name: str, shape) -> np.ndarray | None:
        """bf16 bit patterns (uint16) of the given shape, C-contiguous; None stays None."""
        if a is None:
            return None
        if a.dtype != np.uint16:
            raise TypeError(f"{name} must hold bf16 bit patterns (uint16), got {a.dtype}")
        if tuple(a.shape) != tuple(shape):
            raise ValueError(f"{name} has shape {tuple(a.shape)}, expected {tuple(shape)}")
        return np.ascontiguousarray(a)

    @staticmethod
    def _qk(q, k) -> tuple[np.ndarray, np.ndarray]:
        """Q and K of one shape and one dtype, C-contiguous."""
        if q.shape != k.shape or q.dtype != k.dtype:
            raise ValueError(f"q {q.shape} {q.dtype} and k {k.shape} {k.dtype} differ")
        return np.ascontiguousarray(q), np.ascontiguousarray(k)

    @staticmethod
    def _rows(rows) -> np.ndarray:
        r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))
        return r

    def num_threads(self) -> int:
        return int(self.lib.oracle_num_threads())

    def set_num_threads(self, n: int) -> None:
        self.lib.oracle_set_num_threads(int(n))

    # -------------------------------------------------------------- functions
    def pack(self, x: np.ndarray):
        """Sign bits uint32 [B,H,N,ceil(d/32)] and alpha fp64 [B,H,N]."""
        B, H, N, d = x.shape
        W = (d + 31) // 32
        bits = np.zeros((B, H, N, W), dtype=np.uint32)
        alpha = np.zeros((B, H, N), dtype=np.float64)
        x = np.ascontiguousarray(x)
        rc = self.lib.oracle_pack(_ptr(x), self._dtype_code(x), B, H, N, d,
                                  _ptr(bits), _ptr(alpha))
        if rc:
            raise RuntimeError(f"oracle_pack failed ({rc})")
        return bits, alpha

    def scores_rows(self, q: np.ndarray, k: np.ndarray, rows) -> np.ndarray:
        """Integer scores S[r, j] for flat query-row ids rows[r] = (b*H+h)*N+i."""
        B, H, N, d = q.shape
        r = self._rows(rows)
        S = np.zeros((r.size, N), dtype=np.int32)
        q, k = self._qk(q, k)
        rc = self.lib.oracle_scores_rows(_ptr(q), _ptr(k), self._dtype_code(q), B, H, N, d,
                                         r.size, r.ctypes.data_as(_i64p), _ptr(S))
        if rc:
            raise RuntimeError(f"oracle_scores_rows failed ({rc})")
        return S

    def scores(self, q: np.ndarray, k: np.ndarray) -> np.ndarray:
        """All integer scores int32 [B,H,N,N]."""
        B, H, N, _ = q.shape
        return self.scores_rows(q, k, np.arange(B * H * N)).reshape(B, H, N, N)

    def probs_rows(self, q, k, bias, softmax_scale, rows) -> np.ndarray:
        B, H, N, d = q.shape
        r = self._rows(rows)
        P = np.zeros((r.size, N), dtype=np.float64)
        q, k = self._qk(q, k)
        b = self._bf16(bias, "bias", (H, N, N))
        rc = self.lib.oracle_probs_rows(_ptr(q), _ptr(k), self._dtype_code(q), _ptr(b),
                                        float(softmax_scale), B, H, N, d,
                                        r.size, r.ctypes.data_as(_i64p), _ptr(P))
        if rc:
            raise RuntimeError(f"oracle_probs_rows failed ({rc})")
        return P

    def forward_rows(self, q, k, bias, v, softmax_scale, rows) -> np.ndarray:
        """O rows (fp64, unrounded) for flat query-row ids."""
        B, H, N, d = q.shape
        r = self._rows(rows)
        O = np.zeros((r.size, d), dtype=np.float64)
        q, k = self._qk(q, k)
        v = self._bf16(v, "v", (B, H, N, d))
        b = self._bf16(bias, "bias", (H, N, N))
        rc = self.lib.oracle_forward_rows(_ptr(q), _ptr(k), self._dtype_code(q), _ptr(b),
                                          _ptr(v), float(softmax_scale), B, H, N, d,
                                          r.size, r.ctypes.data_as(_i64p), _ptr(O))
        if rc:
            raise RuntimeError(f"oracle_forward_rows failed ({rc})")
        return O

    def forward(self, q, k, bias, v, softmax_scale) -> np.ndarray:
        """O fp64 [B,H,N,d] for every row."""
        B, H, N, d = q.shape
        O = np.zeros((B, H, N, d), dtype=np.float64)
        q, k = self._qk(q, k)
        v = self._bf16(v, "v", (B, H, N, d))
        b = self._bf16(bias, "bias", (H, N, N))
        rc = self.lib.oracle_forward(_ptr(q), _ptr(k), self._dtype_code(q), _ptr(b), _ptr(v),
                                     float(softmax_scale), B, H, N, d, _ptr(O))
        if rc:
            raise RuntimeError(f"oracle_forward failed ({rc})")
        return O

    def forward_spread(self, q, k, bias, v, softmax_scale):
        """O and its spread E, both fp64 [B,H,N,d], for every row:
        E[b,h,i,c] = sum_j P_ij |V_jc - O_ic| (the bf16-P error scale)."""
        B, H, N, d = q.shape
        O = np.zeros((B, H, N, d), dtype=np.float64)
        E = np.zeros((B, H, N, d), dtype=np.float64)
        q, k = self._qk(q, k)
        v = self._bf16(v, "v", (B, H, N, d))
        b = self._bf16(bias, "bias", (H, N, N))
        rc = self.lib.oracle_forward_spread(_ptr(q), _ptr(k), self._dtype_code(q), _ptr(b), _ptr(v),
                                            float(softmax_scale), B, H, N, d, _ptr(O), _ptr(E))
        if rc:
            raise RuntimeError(f"oracle_forward_spread failed ({rc})")
        return O, E

    # ------------------------------------------------- the 8-bit P.V variant
    def quantize_v(self, v):
        """Per-channel 8-bit code of V (bf16 bits [B,H,N,d]): vq int8 [B,H,N,d]
        and the scale s fp32 [B,H,d], V ~ s * vq."""
        B, H, N, d = v.shape
        v = self._bf16(v, "v", (B, H, N, d))
        vq = np.zeros((B, H, N, d), dtype=np.int8)
        s = np.zeros((B, H, d), dtype=np.float32)
        rc = self.lib.oracle_quantize_v(_ptr(v), B, H, N, d, _ptr(vq), _ptr(s))
        if rc:
            raise RuntimeError(f"oracle_quantize_v failed ({rc})")
        return vq, s

    def forward_int8_rows(self, q, k, bias, v, softmax_scale, rows) -> np.ndarray:
        """O rows (fp64, unrounded) of the 8-bit P.V forward for flat query-row ids."""
        B, H, N, d = q.shape
        r = self._rows(rows)
        O = np.zeros((r.size, d), dtype=np.float64)
        q, k = self._qk(q, k)
        v = self._bf16(v, "v", (B, H, N, d))
        b = self._bf16(bias, "bias", (H, N, N))
        rc = self.lib.oracle_forward_int8_rows(_ptr(q), _ptr(k), self._dtype_code(q), _ptr(b), _ptr(v),
                                               float(softmax_scale), B, H, N, d,
                                               r.size, r.ctypes.data_as(_i64p), _ptr(O))
        if rc:
            raise RuntimeError(f"oracle_forward_int8_rows failed ({rc})")
        return O

    def forward_int8(self, q, k, bias, v, softmax_scale) -> np.ndarray:
        """O fp64 [B,H,N,d] of the 8-bit P.V forward, every row."""
        B, H, N, d = q.shape
        O = np.zeros((B, H, N, d), dtype=np.float64)
        q, k = self._qk(q, k)
        v = self._bf16(v, "v", (B, H, N, d))
        b = self._bf16(bias, "bias", (H, N, N))
        rc = self.lib.oracle_forward_int8(_ptr(q), _ptr(k), self._dtype_code(q), _ptr(b), _ptr(v),
                                          float(softmax_scale), B, H, N, d, _ptr(O))
        if rc:
            raise RuntimeError(f"oracle_forward_int8 failed ({rc})")
        return O

    # ----------------------------------------- the position-sensitive bias
    def expand_relpos_bias(self, table, gh: int, gw: int, n_cls: int) -> np.ndarray:
        """The dense bias [H, N, N] (bf16 bits), N = n_cls + gh * gw, of a
        relative-position table [H, (2gh-1)(2gw-1) + 3 n_cls] (bf16 bits)."""
        H, R = table.shape
        if R != (2 * gh - 1) * (2 * gw - 1) + 3 * n_cls:
            raise ValueError(f"table has {R} entries per head, expected {(2 * gh - 1) * (2 * gw - 1) + 3 * n_cls}")
        t = self._bf16(table, "table", (H, R))
        N = n_cls + gh * gw
        out = np.zeros((H, N, N), dtype=np.uint16)
        rc = self.lib.oracle_expand_relpos_bias(_ptr(t), H, gh, gw, n_cls, _ptr(out))
        if rc:
            raise RuntimeError(f"oracle_expand_relpos_bias failed ({rc})")
        return out


    # ------------------------------------------------------------ backward
    def backward(self, q, k, bias, v, dO, softmax_scale, with_dbias: bool = True):
        """Gradients for an upstream gradient dO (bf16 bits [B,H,N,d]): dV, ds,
        dt fp64 [B,H,N,d] (ds, dt with respect to the scaled binary Q and K,
        s = alpha_q sign(q), t = alpha_k sign(k)) and dbias fp64 [H,N,N] summed
        over the batch (None unless with_dbias)."""
        B, H, N, d = q.shape
        q, k = self._qk(q, k)
        v = self._bf16(v, "v", (B, H, N, d))
        g = self._bf16(dO, "dO", (B, H, N, d))
        b = self._bf16(bias, "bias", (H, N, N))
        dV = np.zeros((B, H, N, d), dtype=np.float64)
        ds = np.zeros((B, H, N, d), dtype=np.float64)
        dt = np.zeros((B, H, N, d), dtype=np.float64)
        db = np.zeros((H, N, N), dtype=np.float64) if with_dbias else None
        rc = self.lib.oracle_backward(_ptr(q), _ptr(k), self._dtype_code(q), _ptr(b), _ptr(v), _ptr(g),
                                      float(softmax_scale), B, H, N, d, _ptr(dV), _ptr(ds), _ptr(dt), _ptr(db))
        if rc:
            raise RuntimeError(f"oracle_backward failed ({rc})")
        return dV, ds, dt, db


_default: Oracle | None = None


def get() -> Oracle:
    """The oracle built from this directory's source (compiled on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default
