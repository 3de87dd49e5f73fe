"""Seeded synthetic inputs shaped like ViT / DiT attention layers.

This module only draws random numbers and rounds them to storage types. It
holds none of the method's arithmetic, imports nothing else from this package,
and is the one piece shared by the GPU tests, the CPU oracle tests and the
benchmark.

The workloads stand in for the attention layers of the models evaluated in
"BinaryAttention: One-Bit QK-Attention for Vision and Diffusion Transformers"
(§4 results: DeiT / ViT classifiers on ImageNet-1K, DiT-XL/2 generation at
256-1024 px). No dataset or trained weight is used; only the layer shapes and
simple value distributions are reproduced.

Draw order for each workload (``numpy.random.default_rng(seed)``): optional
outlier-channel choice, then Q, K, V, then the bias. Every draw is float32;
bf16 tensors are rounded to nearest-even from those draws and returned as their
uint16 bit patterns (numpy has no bf16 dtype).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    qk_dtype: str          # "f32" or "bf16" storage of Q and K
    value_kind: str        # "normal" | "token_std" | "outlier_channels"
    bias_std: float        # 0 means no bias
    seed: int
    note: str = ""

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def W(self) -> int:
        return (self.d + 31) // 32


# The five workloads. Seeds 0..4 in this order.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 256, 64, "f32", "normal", 0.1, 0,
                     "fp32 Q,K,V; V and bias rounded to bf16 for the forward call"),
    "deit_b": Workload("deit_b", 64, 12, 197, 64, "bf16", "token_std", 0.1, 1,
                       "DeiT-B: 196 patches + cls token; per-token std ~ U(0.5, 2)"),
    "vit_l384": Workload("vit_l384", 32, 16, 577, 64, "bf16", "outlier_channels", 0.1, 2,
                         "ViT-L/16 at 384 px: 576 patches + cls; 3 of 64 channels x8"),
    "dit_xl_512": Workload("dit_xl_512", 8, 16, 1024, 72, "bf16", "normal", 0.05, 3,
                           "DiT-XL/2 at 512 px: 32x32 latent patches, head dim 72"),
    "dit_xl_1024": Workload("dit_xl_1024", 2, 16, 4096, 72, "bf16", "normal", 0.05, 4,
                            "DiT-XL/2 at 1024 px: 64x64 latent patches, head dim 72"),
}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _draw_values(rng: np.random.Generator, w: Workload, shape, outlier_ch):
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if w.value_kind == "token_std":
        std = rng.uniform(0.5, 2.0, size=shape[:-1] + (1,)).astype(np.float32)
        x = x * std
    elif w.value_kind == "outlier_channels":
        x = x * outlier_ch[None, :, None, :]
    return x


def make_inputs(w: Workload | str, with_bias: bool = True, seed: int | None = None,
                B: int | None = None) -> dict:
    """Draw one workload's inputs.

    Returns a dict with ``q``, ``k`` (float32 for ``qk_dtype == "f32"``, else
    bf16 bits as uint16), ``v`` (bf16 bits, [B,H,N,d]), ``bias`` (bf16 bits
    [H,N,N] or None), and the sizes. ``B`` overrides the batch size (the draw is
    then a different stream; used for bounded samples).
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    Bn = w.B if B is None else B
    rng = np.random.default_rng(w.seed if seed is None else seed)
    shape = (Bn, w.H, w.N, w.d)
    outlier = None
    if w.value_kind == "outlier_channels":
        n_out = round(0.05 * w.d)
        outlier = np.ones((w.H, w.d), dtype=np.float32)
        for h in range(w.H):
            outlier[h, rng.choice(w.d, size=n_out, replace=False)] = 8.0
    q = _draw_values(rng, w, shape, outlier)
    k = _draw_values(rng, w, shape, outlier)
    v = _draw_values(rng, w, shape, outlier)
    bias = None
    if with_bias and w.bias_std > 0:
        bias = f32_to_bf16_bits(
            rng.standard_normal(size=(w.H, w.N, w.N), dtype=np.float32) * np.float32(w.bias_std))
    if w.qk_dtype == "bf16":
        q = f32_to_bf16_bits(q)
        k = f32_to_bf16_bits(k)
    return dict(q=q, k=k, v=f32_to_bf16_bits(v), bias=bias, B=Bn, H=w.H, N=w.N, d=w.d,
                softmax_scale=w.softmax_scale, qk_dtype=w.qk_dtype, name=w.name)


def make_custom(B: int, H: int, N: int, d: int, seed: int, qk_dtype: str = "bf16",
                with_bias: bool = True, bias_std: float = 0.1, zeros_frac: float = 0.0,
                value_scale: float = 1.0) -> dict:
    """Arbitrary-size inputs for edge-case tests (ragged N, odd d, injected zeros).

    ``zeros_frac`` replaces that fraction of Q and K entries with +0.0 or -0.0
    (half each), so the sign predicate at zero is exercised.
    """
    rng = np.random.default_rng(seed)
    shape = (B, H, N, d)
    q = rng.standard_normal(size=shape, dtype=np.float32) * np.float32(value_scale)
    k = rng.standard_normal(size=shape, dtype=np.float32) * np.float32(value_scale)
    v = rng.standard_normal(size=shape, dtype=np.float32)
    if zeros_frac > 0:
        for x in (q, k):
            m = rng.random(size=shape) < zeros_frac
            neg = rng.random(size=shape) < 0.5
            x[m & neg] = np.float32(-0.0)
            x[m & ~neg] = np.float32(0.0)
    bias = None
    if with_bias:
        bias = f32_to_bf16_bits(
            rng.standard_normal(size=(H, N, N), dtype=np.float32) * np.float32(bias_std))
    if qk_dtype == "bf16":
        q = f32_to_bf16_bits(q)
        k = f32_to_bf16_bits(k)
    return dict(q=q, k=k, v=f32_to_bf16_bits(v), bias=bias, B=B, H=H, N=N, d=d,
                softmax_scale=1.0 / math.sqrt(d), qk_dtype=qk_dtype, name=f"custom{B}x{H}x{N}x{d}")


def per_sample_bias(B: int, H: int, N: int, seed: int, bias_std: float = 0.5,
                    base: np.ndarray | None = None) -> np.ndarray:
    """One dense bias per batch entry, bf16 bits [B, H, N, N]: the stand-in for a
    context-aware bias, which differs from sample to sample.

    Without ``base``: B independent N(0, bias_std^2) draws. With ``base`` (bf16
    bits [H, N, N], e.g. a workload's shared bias): entry b is ``base`` with its
    heads rotated by b, distinct per sample without a second draw of N^2 values
    per head (used at full size).
    """
    if base is not None:
        assert base.shape == (H, N, N)
        return np.stack([np.roll(base, -b, axis=0) for b in range(B)])
    rng = np.random.default_rng(seed)
    return f32_to_bf16_bits(rng.standard_normal(size=(B, H, N, N), dtype=np.float32) * np.float32(bias_std))


def upstream_grad(B: int, H: int, N: int, d: int, seed: int) -> np.ndarray:
    """An upstream gradient dLoss/dO for the backward, bf16 bits [B, H, N, d]:
    N(0, 1) draws from default_rng(seed)."""
    rng = np.random.default_rng(seed)
    return f32_to_bf16_bits(rng.standard_normal(size=(B, H, N, d), dtype=np.float32))
