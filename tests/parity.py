"""Helpers shared by the GPU parity tests: moving seeded numpy inputs to the
device, running the whole path through the C ABI, and the tolerance check.

Tolerance on O (bf16 output, fp32 accumulation): max |O_gpu - O_ref| <= 2e-2
and ||O_gpu - O_ref||_2 / ||O_ref||_2 <= 5e-3, with O_ref the oracle's
unrounded fp64 result. Where |O_ref| >= 8 the bf16 half-ulp alone (>= 2^-5)
exceeds 2e-2; there the element bound becomes 2e-2 + half an ulp of bf16 at
|O_ref|. Where the values a row averages are spread widely (outlier V
channels), rounding P to bf16 alone can move O by more than 2e-2; tests that
pass the oracle's spread E use 2^-8 E + half an ulp + 1e-3 as the element
bound there. A warning names every case that needed either.
"""
from __future__ import annotations

import warnings

import numpy as np
import torch

from diffusion_transformers_b200 import binattn

MAX_ABS = 2e-2
REL_RMS = 5e-3


def dev(x: np.ndarray | None) -> torch.Tensor | None:
    """numpy float32 or bf16-bits (uint16) array -> CUDA tensor of the same bytes."""
    if x is None:
        return None
    if x.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def run_path(inp: dict, engine="auto", with_bias=True):
    """pack(Q), pack(K), forward through the C ABI. Returns device tensors."""
    q, k, v = dev(inp["q"]), dev(inp["k"]), dev(inp["v"])
    bias = dev(inp["bias"]) if with_bias else None
    qb, aq = binattn.pack(q)
    kb, ak = binattn.pack(k)
    out = binattn.forward(qb, kb, aq, ak, bias, v, inp["softmax_scale"], engine=engine)
    torch.cuda.synchronize()
    binattn.device_status()
    return dict(q=q, k=k, v=v, bias=bias, qb=qb, kb=kb, aq=aq, ak=ak, out=out)


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 numbers at |x| (8 significant bits)."""
    ax = np.maximum(np.abs(x), np.finfo(np.float32).tiny)
    return np.ldexp(1.0, np.floor(np.log2(ax)).astype(np.int64) - 8)


# Unit roundoff of a bf16 significand (8 bits): P is rounded to bf16 before P.V.
U_BF16 = 2.0 ** -9


def spread_bound(o_ref: np.ndarray, spread: np.ndarray) -> np.ndarray:
    """Per-element bound from the arithmetic the path is specified to do: each
    P_ij rounded to bf16 (relative U_BF16), with the row sum l taken from the
    same rounded values, moves O_ic by at most 2 U_BF16 sum_j P_ij |V_jc - O_ic|
    = 2^-8 E_ic to first order; the bf16 output adds half an ulp of O_ic; 1e-3
    covers the fp32 logits, exps and accumulation."""
    return 2 * U_BF16 * spread + bf16_half_ulp(o_ref) + 1e-3


def check_o(o_gpu: np.ndarray, o_ref: np.ndarray, what: str = "", spread: np.ndarray | None = None) -> dict:
    """The stated bar (max-abs 2e-2, rel-RMS 5e-3). Where |O_ref| >= 8 an
    element may also pass under 2e-2 + half an ulp; with `spread` (the oracle's
    E = sum_j P_ij |V_jc - O_ic|) an element may also pass under
    spread_bound(). Either fallback raises a warning that names the case."""
    err = np.abs(o_gpu - o_ref)
    rel_rms = float(np.linalg.norm(o_gpu - o_ref) / max(np.linalg.norm(o_ref), 1e-30))
    bound = np.full(err.shape, MAX_ABS)
    big = np.abs(o_ref) >= 8.0
    bound[big] += bf16_half_ulp(o_ref[big])
    if spread is not None:
        bound = np.maximum(bound, spread_bound(o_ref, spread))
    bad = err > bound
    if bad.any():
        worst = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} elements beyond their bound; worst error "
                             f"{float(err[worst]):.3e} against {float(bound[worst]):.3e} at {tuple(int(x) for x in worst)}"
                             f" (|O_ref| {abs(float(o_ref[worst])):.3f})")
    over = err > MAX_ABS
    fallback = bool(over.any())
    if fallback:  # flagged, not silent: the plain 2e-2 bar did not hold there
        kinds = "2e-2 + half a bf16 ulp (|O_ref| >= 8)" if spread is None else "the bf16-P spread bound"
        warnings.warn(f"{what}: {int(over.sum())} elements passed only under {kinds} "
                      f"(max-abs {float(err.max()):.3e})")
    assert rel_rms <= REL_RMS, f"{what}: rel-RMS {rel_rms:.3e} > {REL_RMS}"
    return dict(max_abs=float(err.max()), rel_rms=rel_rms, half_ulp_fallback=fallback)


def sample_rows(B: int, H: int, N: int, n: int, seed: int = 0) -> np.ndarray:
    """Flat row ids (b*H+h)*N+i: corners, the ragged last query tile, and random rows."""
    rng = np.random.default_rng(seed)
    T = B * H * N
    fixed = [0, N - 1, T - 1, T - N, (B * H // 2) * N + N // 2]
    tail0 = (N // 128) * 128
    fixed += [(b * H + h) * N + i for b, h in [(0, 0), (B - 1, H - 1)]
              for i in range(tail0, N, max(1, (N - tail0) // 4 or 1))]
    rnd = rng.integers(0, T, size=max(0, n - len(fixed)))
    return np.unique(np.concatenate([np.array(fixed, dtype=np.int64), rnd]))
