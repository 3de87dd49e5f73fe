"""Checks that pin the CPU oracle to facts outside itself.

Each ``pin_*`` function takes a loaded ``oracle.Oracle`` and raises
AssertionError when the oracle disagrees with what "BinaryAttention: One-Bit
QK-Attention for Vision and Diffusion Transformers" fixes or with textbook
mathematics: an exhaustive sign predicate, numpy's packbits layout, the
Hamming identity behind XNOR/popcount, closed forms, invariants, special cases
that reduce to scipy's softmax, a hand-worked example, and an independent
matrix-form formulation on tiny inputs.

They are run against the real oracle (test_oracle_pins.py) and against
deliberately broken copies of it (test_oracle_mutants.py), where at least one
of them must fail.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
from scipy.special import softmax as scipy_softmax

from diffusion_transformers_b200.synthetic import (bf16_bits_to_f32, f32_to_bf16_bits,
                                                  make_custom)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f64(x: np.ndarray) -> np.ndarray:
    """Exact float64 view of a float32 or bf16-bits array."""
    if x.dtype == np.uint16:
        return bf16_bits_to_f32(x).astype(np.float64)
    return x.astype(np.float64)


# ----------------------------------------------------------------- a1: bits
def pin_sign_predicate_exhaustive(orc):
    """Every non-NaN bf16 pattern (one channel per token): bit == (x >= 0) as
    evaluated by numpy; +0.0 and -0.0 both give 1 (sign of the stored value,
    'sign' of the scaled binary representation)."""
    pats = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    f = bf16_bits_to_f32(pats)
    keep = ~np.isnan(f)
    x = pats[keep].reshape(1, 1, -1, 1)
    bits, _ = orc.pack(x)
    want = (f[keep] >= np.float32(0)).astype(np.uint32)
    assert np.array_equal(bits.reshape(-1), want), "sign predicate differs from x >= 0"
    # the same for fp32 special values
    specials = np.array([0.0, -0.0, 1e-45, -1e-45, 1.17e-38, -1.17e-38, np.inf, -np.inf,
                         3.4e38, -3.4e38, 1.0, -1.0], dtype=np.float32)
    b2, _ = orc.pack(specials.reshape(1, 1, -1, 1))
    assert np.array_equal(b2.reshape(-1), (specials >= 0).astype(np.uint32))


def pin_pack_layout_packbits(orc):
    """Word c//32, bit c%32, LSB first, pad bits zero: equal to numpy's
    little-endian packbits of (x >= 0) read back as little-endian uint32."""
    rng = np.random.default_rng(11)
    for d in (1, 5, 31, 32, 33, 64, 72, 96, 100, 128, 200):
        x = rng.standard_normal((2, 3, 7, d)).astype(np.float32)
        bits, _ = orc.pack(x)
        W = (d + 31) // 32
        pb = np.packbits(x >= 0, axis=-1, bitorder="little")
        pad = np.zeros(pb.shape[:-1] + (W * 4 - pb.shape[-1],), dtype=np.uint8)
        want = np.concatenate([pb, pad], axis=-1).copy().view("<u4")
        assert bits.shape == (2, 3, 7, W)
        assert np.array_equal(bits, want), f"bit layout differs at d={d}"


# ---------------------------------------------------------------- a2: alpha
def pin_alpha_mean_abs(orc):
    """alpha = mean |x| over the d real channels: numpy's fp64 mean of |x|,
    exact closed form |c| for x = c * (+-1), and exact scaling by powers of 2
    (bits unchanged)."""
    rng = np.random.default_rng(12)
    for d in (1, 7, 64, 72, 128):
        x = rng.standard_normal((2, 2, 9, d)).astype(np.float32)
        _, a = orc.pack(x)
        want = np.mean(np.abs(x.astype(np.float64)), axis=-1)
        assert np.allclose(a, want, rtol=1e-14, atol=0), f"alpha != mean|x| at d={d}"
        # closed form: x = c * s with s in {+1,-1}
        c = rng.uniform(0.1, 4.0, size=(2, 2, 9, 1)).astype(np.float32)
        s = np.where(rng.random((2, 2, 9, d)) < 0.5, -1.0, 1.0).astype(np.float32)
        _, a2 = orc.pack(c * s)
        assert np.array_equal(a2, np.broadcast_to(c[..., 0].astype(np.float64), a2.shape)), \
            "alpha of c*(+-1) is not |c|"
        # power-of-two scaling: alpha scales exactly, bits do not change
        b1, a1 = orc.pack(x)
        b4, a4 = orc.pack(x * np.float32(4.0))
        assert np.array_equal(b1, b4) and np.array_equal(a4, 4.0 * a1)
    # bf16 storage path gives the same as the exactly widened fp32 values
    xb = f32_to_bf16_bits(rng.standard_normal((1, 2, 5, 72)).astype(np.float32))
    _, ab = orc.pack(xb)
    _, af = orc.pack(bf16_bits_to_f32(xb))
    assert np.array_equal(ab, af)


# --------------------------------------------------------------- a3: scores
def pin_hamming_identity_exhaustive(orc):
    """<sign q, sign k> = d - 2 * Hamming(q, k) (XNOR/popcount similarity) for
    every pair of sign vectors at d = 1..10."""
    for d in range(1, 11):
        n = 1 << d
        idx = np.arange(n)
        signs = np.where((idx[:, None] >> np.arange(d)[None, :]) & 1, 1.0, -1.0)
        x = signs.astype(np.float32).reshape(1, 1, n, d)
        S = orc.scores(x, x)[0, 0].astype(np.int64)
        ham = np.array([[bin(a ^ b).count("1") for b in range(n)] for a in range(n)]) \
            if d <= 6 else _popcount_table(idx[:, None] ^ idx[None, :])
        assert np.array_equal(S, d - 2 * ham), f"Hamming identity fails at d={d}"


def _popcount_table(z: np.ndarray) -> np.ndarray:
    z = z.astype(np.uint32)
    return np.unpackbits(z.view(np.uint8).reshape(z.shape + (4,)), axis=-1).sum(-1).astype(np.int64)


def pin_scores_matmul(orc):
    """S equals an int64 matrix product of the +-1 sign matrices (numpy), per
    (b, h), for several d including padded ones."""
    rng = np.random.default_rng(13)
    for d in (33, 64, 72, 128):
        q = f32_to_bf16_bits(rng.standard_normal((2, 3, 17, d)).astype(np.float32))
        k = f32_to_bf16_bits(rng.standard_normal((2, 3, 17, d)).astype(np.float32))
        S = orc.scores(q, k).astype(np.int64)
        sq = np.where(_f64(q) >= 0, 1, -1).astype(np.int64)
        sk = np.where(_f64(k) >= 0, 1, -1).astype(np.int64)
        want = np.einsum("bhic,bhjc->bhij", sq, sk)
        assert np.array_equal(S, want), f"scores differ from +-1 matmul at d={d}"


def pin_scores_special_cases(orc):
    """All-equal signs give S == d; K = -Q (no zeros) gives S_ii = -d; negating
    Q negates S; +0.0 and -0.0 both count as +1."""
    rng = np.random.default_rng(14)
    d = 72
    pos = np.abs(rng.standard_normal((1, 2, 9, d))).astype(np.float32) + 0.1
    S = orc.scores(pos, pos * np.float32(3.0))
    assert np.all(S == d)
    q = rng.standard_normal((1, 2, 9, d)).astype(np.float32)
    q[q == 0] = 1.0
    S2 = orc.scores(q, -q)
    assert np.all(np.diagonal(S2, axis1=2, axis2=3) == -d)
    k = rng.standard_normal((1, 2, 9, d)).astype(np.float32)
    k[k == 0] = 1.0
    assert np.array_equal(orc.scores(-q, k), -orc.scores(q, k))
    z = np.zeros((1, 1, 2, d), dtype=np.float32)
    z[0, 0, 1] = -0.0
    assert np.all(orc.scores(z, np.ones_like(z)) == d)


# -------------------------------------------------------------- a4/a5: softmax
def pin_softmax_rows_sum_to_one(orc):
    c = make_custom(2, 3, 37, 72, seed=15, bias_std=0.5)
    rows = np.arange(2 * 3 * 37)
    P = orc.probs_rows(c["q"], c["k"], c["bias"], c["softmax_scale"], rows)
    assert np.all(P >= 0)
    assert np.allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-12)


def pin_softmax_bias_only(orc):
    """softmax_scale = 0 leaves only the bias: each row of P is scipy's softmax
    of bias[h, i, :], the same for every b (bias broadcast over the batch)."""
    B, H, N = 2, 3, 23
    c = make_custom(B, H, N, 40, seed=16, bias_std=1.0)
    rows = np.arange(B * H * N)
    P = orc.probs_rows(c["q"], c["k"], c["bias"], 0.0, rows).reshape(B, H, N, N)
    bias = _f64(c["bias"])
    want = scipy_softmax(bias, axis=-1)
    for b in range(B):
        assert np.allclose(P[b], want, rtol=1e-12, atol=1e-15), "P != softmax(bias)"


def pin_softmax_shift_invariance(orc):
    """Adding a per-row constant to the logits (through the bias, exactly
    representable in bf16) leaves P unchanged."""
    B, H, N, d = 1, 2, 19, 64
    c = make_custom(B, H, N, d, seed=17, with_bias=False)
    rng = np.random.default_rng(18)
    k8 = rng.integers(-16, 17, size=(H, N, N)).astype(np.float32) / 8.0
    shift = (np.arange(N) % 4).astype(np.float32)[None, :, None] * 8.0
    b0 = f32_to_bf16_bits(k8)
    b1 = f32_to_bf16_bits(k8 + shift)
    assert np.array_equal(_f64(b1) - _f64(b0), np.broadcast_to(shift, (H, N, N)).astype(np.float64))
    rows = np.arange(B * H * N)
    P0 = orc.probs_rows(c["q"], c["k"], b0, c["softmax_scale"], rows)
    P1 = orc.probs_rows(c["q"], c["k"], b1, c["softmax_scale"], rows)
    assert np.allclose(P0, P1, rtol=1e-12, atol=1e-15)


def pin_scale_invariances(orc):
    """Scaling Q (or K) by 2 multiplies alpha_q (alpha_k) by 2 and leaves the
    signs alone, so halving softmax_scale gives the same O; the bias is not
    scaled, so this holds with a bias present."""
    c = make_custom(2, 2, 21, 72, seed=19, qk_dtype="f32", bias_std=0.3)
    rows = np.arange(2 * 2 * 21)
    s = c["softmax_scale"] * 4.0
    O = orc.forward_rows(c["q"], c["k"], c["bias"], c["v"], s, rows)
    Oq = orc.forward_rows(c["q"] * np.float32(2), c["k"], c["bias"], c["v"], s / 2, rows)
    Ok = orc.forward_rows(c["q"], c["k"] * np.float32(2), c["bias"], c["v"], s / 2, rows)
    assert np.allclose(O, Oq, rtol=1e-12, atol=1e-13), "alpha_q does not enter the logit"
    assert np.allclose(O, Ok, rtol=1e-12, atol=1e-13), "alpha_k does not enter the logit"
    # and the logits do depend on the scale (guards against a constant result)
    O2 = orc.forward_rows(c["q"], c["k"], c["bias"], c["v"], s * 3, rows)
    assert not np.allclose(O, O2, rtol=1e-6, atol=1e-8)


# ------------------------------------------------------------ a6: P.V and O
def pin_uniform_scores_mean_v(orc):
    """Every key row identical within a head (different across heads) and no
    bias: scores are constant along j, P is uniform, and O_i = mean_j V_j."""
    B, H, N, d = 2, 3, 13, 72
    rng = np.random.default_rng(20)
    q = rng.standard_normal((B, H, N, d)).astype(np.float32)
    krow = rng.standard_normal((B, H, 1, d)).astype(np.float32)
    k = np.ascontiguousarray(np.broadcast_to(krow, (B, H, N, d)))
    v = f32_to_bf16_bits(rng.standard_normal((B, H, N, d)).astype(np.float32))
    O = orc.forward(q, k, None, v, 0.7)
    want = np.broadcast_to(_f64(v).mean(axis=2, keepdims=True), O.shape)
    assert np.allclose(O, want, rtol=1e-12, atol=1e-14)


def pin_onehot_bias_gather(orc):
    """softmax_scale = 0 and bias[h, i, pi(i)] = 40 (others 0): P puts all but
    (N-1)e^-40 of its mass on key pi(i), so O_i = V[pi(i)] (a permutation
    gather, different per head and batch index)."""
    B, H, N, d = 2, 2, 11, 33
    rng = np.random.default_rng(21)
    c = make_custom(B, H, N, d, seed=22, with_bias=False)
    bias = np.zeros((H, N, N), dtype=np.float32)
    perms = [rng.permutation(N) for _ in range(H)]
    for h in range(H):
        bias[h, np.arange(N), perms[h]] = 40.0
    O = orc.forward(c["q"], c["k"], f32_to_bf16_bits(bias), c["v"], 0.0)
    v = _f64(c["v"])
    tol = N * math.exp(-40) * np.abs(v).max() * 2
    for b in range(B):
        for h in range(H):
            assert np.allclose(O[b, h], v[b, h, perms[h]], rtol=0, atol=tol)


def pin_convex_hull(orc):
    """Each O_i[c] lies between min_j V_jc and max_j V_jc (P is a probability
    vector)."""
    c = make_custom(2, 2, 31, 72, seed=23, bias_std=1.0)
    O = orc.forward(c["q"], c["k"], c["bias"], c["v"], c["softmax_scale"])
    v = _f64(c["v"])
    lo = v.min(axis=2, keepdims=True) - 1e-12
    hi = v.max(axis=2, keepdims=True) + 1e-12
    assert np.all(O >= lo) and np.all(O <= hi)


def pin_bruteforce_matrix_form(orc):
    """Tiny cases (N <= 8) against a second, matrix-form fp64 formulation:
    S = sign(Q) sign(K)^T, L = scale * a_q a_k^T * S + bias, P = scipy softmax,
    O = P V."""
    rng = np.random.default_rng(24)
    for (B, H, N, d) in [(1, 1, 1, 1), (2, 2, 3, 5), (1, 3, 8, 72), (2, 1, 8, 33), (1, 2, 7, 64)]:
        for with_bias in (False, True):
            c = make_custom(B, H, N, d, seed=int(rng.integers(1 << 30)), qk_dtype="bf16",
                            with_bias=with_bias, bias_std=0.7, zeros_frac=0.1)
            q, k, v = _f64(c["q"]), _f64(c["k"]), _f64(c["v"])
            sq, sk = np.where(q >= 0, 1.0, -1.0), np.where(k >= 0, 1.0, -1.0)
            aq, ak = np.abs(q).mean(-1), np.abs(k).mean(-1)
            S = sq @ np.swapaxes(sk, -1, -2)
            L = c["softmax_scale"] * aq[..., :, None] * ak[..., None, :] * S
            if with_bias:
                L = L + _f64(c["bias"])[None]
            want = scipy_softmax(L, axis=-1) @ v
            O = orc.forward(c["q"], c["k"], c["bias"], c["v"], c["softmax_scale"])
            assert np.allclose(O, want, rtol=1e-12, atol=1e-14), f"brute force fails at {B,H,N,d}"


def pin_worked_example(orc):
    """Hand-worked example (tests/golden/worked_example.json): sign bits,
    alphas, integer scores and logits derived by hand as rationals; O from the
    closed-form two-key softmax."""
    with open(os.path.join(GOLDEN, "worked_example.json")) as f:
        g = json.load(f)
    q = np.array(g["Q"], dtype=np.float32).reshape(1, 1, 2, 3)
    k = np.array(g["K"], dtype=np.float32).reshape(1, 1, 2, 3)
    v = f32_to_bf16_bits(np.array(g["V"], dtype=np.float32).reshape(1, 1, 2, 3))
    bias = f32_to_bf16_bits(np.array(g["bias"], dtype=np.float32).reshape(1, 2, 2))
    bits, aq = orc.pack(q)
    assert bits.reshape(-1).tolist() == g["q_bits"]
    assert np.allclose(aq.reshape(-1), [eval(a) for a in g["alpha_q"]], rtol=1e-15)
    S = orc.scores(q, k)[0, 0]
    assert S.tolist() == g["S"]
    logits = np.array([[eval(x) for x in row] for row in g["logits"]])
    # two keys: P_i0 = 1 / (1 + exp(l_i1 - l_i0))
    p0 = 1.0 / (1.0 + np.exp(logits[:, 1] - logits[:, 0]))
    V = np.array(g["V"], dtype=np.float64)
    want = p0[:, None] * V[0][None, :] + (1 - p0)[:, None] * V[1][None, :]
    O = orc.forward(q, k, bias, v, g["softmax_scale"])[0, 0]
    assert np.allclose(O, want, rtol=1e-14, atol=1e-15)


# ------------------------------------------------- statistics of the inputs
def pin_alpha_half_normal_mean(orc):
    """For x ~ N(0, sigma^2) the mean of |x| is sqrt(2/pi) * sigma (the
    half-normal mean), so the average alpha over many tokens of each synthetic
    workload is sqrt(2/pi) times its mean channel scale: 1 for N(0,1), E[U(0.5,2)]
    = 1.25 for per-token stds, (61 + 3 * 8) / 64 with three x8 outlier channels.
    Checks the generators' recipes together with the oracle's alpha (5 standard
    errors)."""
    from diffusion_transformers_b200.synthetic import make_inputs

    c = math.sqrt(2.0 / math.pi)
    for name, scale in (("dit_xl_512", 1.0), ("deit_b", 1.25), ("vit_l384", (61 + 3 * 8) / 64)):
        inp = make_inputs(name, with_bias=False, B=1)
        for key in ("q", "k"):
            _, a = orc.pack(inp[key])
            a = a.reshape(-1)
            se = a.std() / math.sqrt(a.size)
            assert abs(a.mean() - c * scale) <= 5 * se + 2e-3 * c * scale, \
                f"{name} {key}: mean alpha {a.mean():.5f} vs sqrt(2/pi)*{scale:.4f} = {c * scale:.5f}"


def pin_sign_correlation_arcsin(orc):
    """For a bivariate normal pair with correlation rho, E[sign x * sign y] =
    (2/pi) * arcsin(rho) (the orthant-probability identity). Q and K drawn
    with channel-wise correlation rho give mean S_ii / d at that value; pairs of
    independent tokens give 0. d = 72 also exercises the pad bits."""
    rng = np.random.default_rng(21)
    H, N, d = 4, 256, 72
    for rho in (-0.7, 0.0, 0.3, 0.9):
        q = rng.standard_normal((1, H, N, d))
        k = rho * q + math.sqrt(1.0 - rho * rho) * rng.standard_normal((1, H, N, d))
        S = orc.scores(q.astype(np.float32), k.astype(np.float32)).astype(np.float64) / d
        diag = np.diagonal(S, axis1=2, axis2=3)
        want = 2.0 / math.pi * math.asin(rho)
        se = math.sqrt(max(1.0 - want * want, 1e-3) / (diag.size * d))
        assert abs(diag.mean() - want) <= 5 * se, f"rho={rho}: mean S/d {diag.mean():.4f} vs {want:.4f}"
        off = S.sum(axis=(2, 3)) - diag.sum(axis=2)
        n_off = H * N * (N - 1)
        assert abs(off.sum() / n_off) <= 5 / math.sqrt(n_off * d), f"rho={rho}: independent tokens correlate"


# ------------------------------------- spread of an output (tolerance scale)
def pin_spread_uniform_is_mean_abs_deviation(orc):
    """Uniform P (every key row of a head identical, no bias): O_i = mean_j V_j
    and E_ic = mean_j |V_jc - mean V_c|, the mean absolute deviation."""
    B, H, N, d = 2, 2, 9, 40
    rng = np.random.default_rng(41)
    q = rng.standard_normal((B, H, N, d)).astype(np.float32)
    k = np.ascontiguousarray(np.broadcast_to(rng.standard_normal((B, H, 1, d)).astype(np.float32), (B, H, N, d)))
    v = f32_to_bf16_bits(rng.standard_normal((B, H, N, d)).astype(np.float32) * 3)
    O, E = orc.forward_spread(q, k, None, v, 0.9)
    vf = _f64(v)
    mad = np.abs(vf - vf.mean(axis=2, keepdims=True)).mean(axis=2, keepdims=True)
    assert np.array_equal(O, orc.forward(q, k, None, v, 0.9))
    assert np.allclose(E, np.broadcast_to(mad, E.shape), rtol=1e-12, atol=1e-14)


def pin_spread_two_keys_closed_form(orc):
    """N = 2, scale 0, bias row (b1, b2): P = (p, 1 - p) with
    p = 1 / (1 + e^(b2 - b1)), and E_ic = 2 p (1 - p) |V_0c - V_1c|; a one-hot
    bias (+40) gives E ~ 0 (at most 2 e^-40 max|V|)."""
    B, H, N, d = 1, 3, 2, 16
    rng = np.random.default_rng(42)
    c = make_custom(B, H, N, d, seed=43, with_bias=False)
    bias = f32_to_bf16_bits(rng.uniform(-2, 2, size=(H, N, N)).astype(np.float32))
    O, E = orc.forward_spread(c["q"], c["k"], bias, c["v"], 0.0)
    b, v = _f64(bias), _f64(c["v"])
    for h in range(H):
        for i in range(N):
            p = 1.0 / (1.0 + math.exp(b[h, i, 1] - b[h, i, 0]))
            assert np.allclose(E[0, h, i], 2 * p * (1 - p) * np.abs(v[0, h, 0] - v[0, h, 1]), rtol=1e-12, atol=1e-15)
    onehot = np.zeros((H, N, N), dtype=np.float32)
    onehot[:, :, 0] = 40.0
    _, E1 = orc.forward_spread(c["q"], c["k"], f32_to_bf16_bits(onehot), c["v"], 0.0)
    assert np.all(E1 <= 2 * math.exp(-40) * np.abs(v).max() * 2)


# ------------------------------------------------- the 8-bit P.V variant
def _exact_v(rng, B, H, N, d):
    """bf16 V whose every channel of every (b, h) holds k * 2^-3 with integers
    |k| <= 127 and some |k| = 127: the per-channel scale is exactly 2^-3 and
    the 8-bit code is k itself."""
    kk = rng.integers(-127, 128, size=(B, H, N, d))
    kk[:, :, 0, :] = 127 * np.where(rng.random((B, H, d)) < 0.5, 1, -1)
    return f32_to_bf16_bits((kk * 0.125).astype(np.float32)), kk


def pin_quantize_v_closed_form(orc):
    """Per-channel code: V = k * 2^-3 with max |k| = 127 gives s = 2^-3 and
    vq = k exactly; an all-zero channel gives s = 0, vq = 0; ties round to
    even (2.5 -> 2, 3.5 -> 4, -2.5 -> -2 at s = 1)."""
    rng = np.random.default_rng(51)
    v, kk = _exact_v(rng, 2, 3, 17, 12)
    vb = v.copy()
    vb[1, 2, :, 5] = 0  # an all-zero channel
    vq, s = orc.quantize_v(vb)
    want = kk.copy()
    want[1, 2, :, 5] = 0
    assert np.array_equal(vq, want.astype(np.int8))
    ws = np.full(s.shape, 0.125, dtype=np.float32)
    ws[1, 2, 5] = 0.0
    assert np.array_equal(s, ws)
    t = np.zeros((1, 1, 5, 1), dtype=np.float32)
    t[0, 0, :, 0] = [127.0, 2.5, 3.5, -2.5, -126.5]
    vq, s = orc.quantize_v(f32_to_bf16_bits(t))
    assert s[0, 0, 0] == 1.0 and list(vq[0, 0, :, 0]) == [127, 2, 4, -2, -126]


def pin_int8_uniform_scores(orc):
    """Every key row of a head identical, no bias: every u is 255, and
    O = s * mean_j vq_j = 2^-3 * mean_j k_j for the exact V above."""
    B, H, N, d = 2, 2, 11, 24
    rng = np.random.default_rng(52)
    q = rng.standard_normal((B, H, N, d)).astype(np.float32)
    k = np.ascontiguousarray(np.broadcast_to(rng.standard_normal((B, H, 1, d)).astype(np.float32), (B, H, N, d)))
    v, kk = _exact_v(rng, B, H, N, d)
    O = orc.forward_int8(q, k, None, v, 0.8)
    want = np.broadcast_to(0.125 * kk.mean(axis=2, keepdims=True), O.shape)
    assert np.allclose(O, want, rtol=1e-13, atol=1e-15)


def pin_int8_two_keys_closed_form(orc):
    """N = 2, scale 0, bias row (b0, b1): the larger logit gets u = 255, the
    other u = rint(255 e^-|b0 - b1|), and O = 2^-3 (u0 k0 + u1 k1) / (u0 + u1);
    a one-hot bias of 40 gives O = 2^-3 k of that key (u = 0 elsewhere)."""
    B, H, N, d = 1, 4, 2, 8
    rng = np.random.default_rng(53)
    c = make_custom(B, H, N, d, seed=54, with_bias=False)
    v, kk = _exact_v(rng, B, H, N, d)
    bias = f32_to_bf16_bits(rng.uniform(-3, 3, size=(H, N, N)).astype(np.float32))
    O = orc.forward_int8(c["q"], c["k"], bias, v, 0.0)
    b = _f64(bias)
    for h in range(H):
        for i in range(N):
            e = np.exp(b[h, i] - b[h, i].max())
            u = np.array([255.0 if x == 1.0 else float(np.rint(255.0 * x)) for x in e])
            want = 0.125 * (u[:, None] * kk[0, h]).sum(axis=0) / u.sum()
            assert np.allclose(O[0, h, i], want, rtol=1e-13, atol=1e-15), (h, i)
    onehot = np.zeros((H, N, N), dtype=np.float32)
    onehot[:, 0, 1] = 40.0
    onehot[:, 1, 0] = 40.0
    O1 = orc.forward_int8(c["q"], c["k"], f32_to_bf16_bits(onehot), v, 0.0)
    assert np.array_equal(O1[0, :, 0], 0.125 * kk[0, :, 1]) and np.array_equal(O1[0, :, 1], 0.125 * kk[0, :, 0])


# ------------------------------------------------ position-sensitive bias
def pin_relpos_one_hot_counts(orc):
    """A table that is 1 at one displacement (dy, dx) and 0 elsewhere expands
    to a bias whose 1s are exactly the patch pairs at that displacement:
    (gh - |dy|)(gw - |dx|) of them per head, each with y_i - y_j = dy and
    x_i - x_j = dx; the class entries land on the class row and column."""
    for gh, gw, n_cls in [(3, 4, 0), (4, 3, 1), (1, 5, 1), (5, 5, 0)]:
        R0 = (2 * gh - 1) * (2 * gw - 1)
        N = n_cls + gh * gw
        for dy in range(-(gh - 1), gh):
            for dx in range(-(gw - 1), gw):
                t = np.zeros((1, R0 + 3 * n_cls), dtype=np.float32)
                t[0, (dy + gh - 1) * (2 * gw - 1) + dx + gw - 1] = 1.0
                b = _f64(orc.expand_relpos_bias(f32_to_bf16_bits(t), gh, gw, n_cls))[0]
                ii, jj = np.nonzero(b)
                assert len(ii) == (gh - abs(dy)) * (gw - abs(dx)), (gh, gw, dy, dx)
                assert np.all(ii >= n_cls) and np.all(jj >= n_cls)
                pi, pj = ii - n_cls, jj - n_cls
                assert np.all(pi // gw - pj // gw == dy) and np.all(pi % gw - pj % gw == dx)
        if n_cls:
            for e, (i, j) in enumerate([(0, 5 % N or 1), (min(2, N - 1), 0), (0, 0)]):
                t = np.zeros((1, R0 + 3), dtype=np.float32)
                t[0, R0 + e] = 2.0
                b = _f64(orc.expand_relpos_bias(f32_to_bf16_bits(t), gh, gw, 1))[0]
                assert b[i, j] == 2.0
                assert np.count_nonzero(b) == [N - 1, N - 1, 1][e]


def pin_relpos_translation_invariance(orc):
    """A random table: pairs of patches with the same displacement get the same
    value, and every table entry of a head is reached (the map from
    displacements to entries is onto), also per head."""
    rng = np.random.default_rng(61)
    gh, gw = 4, 6
    R0 = (2 * gh - 1) * (2 * gw - 1)
    t = f32_to_bf16_bits(rng.standard_normal((2, R0)).astype(np.float32))
    b = _f64(orc.expand_relpos_bias(t, gh, gw, 0))
    y, x = np.divmod(np.arange(gh * gw), gw)
    dy, dx = y[:, None] - y[None, :], x[:, None] - x[None, :]
    for h in range(2):
        seen = {}
        for a, c, v in zip(dy.ravel(), dx.ravel(), b[h].ravel()):
            assert seen.setdefault((a, c), v) == v
        assert len(seen) == R0
        assert sorted(seen.values()) == sorted(_f64(t)[h].tolist())


# ---------------------------------------------------- the backward (row f4)
def _loss(orc, q, k, bias, v, dO, scale) -> float:
    """The scalar loss sum(dO * O) whose gradients the backward returns."""
    return float((orc.forward(q, k, bias, v, scale) * _f64(dO)).sum())


def _grad_of_definition(q, k, bias, v, dO, scale, H, N):
    """Gradients of sum(dO * O) by torch's automatic differentiation (fp64) of
    the forward's matrix form, with s = alpha_q sign(q), t = alpha_k sign(k),
    V and the bias as the leaves."""
    import torch
    qf, kf = _f64(q), _f64(k)
    s = torch.tensor(np.abs(qf).mean(-1)[..., None] * np.where(qf >= 0, 1.0, -1.0), requires_grad=True)
    t = torch.tensor(np.abs(kf).mean(-1)[..., None] * np.where(kf >= 0, 1.0, -1.0), requires_grad=True)
    V = torch.tensor(_f64(v), requires_grad=True)
    b = torch.tensor(_f64(bias) if bias is not None else np.zeros((H, N, N)), requires_grad=True)
    L = scale * (s @ t.transpose(-1, -2)) + b
    O = torch.softmax(L, dim=-1) @ V
    (O * torch.tensor(_f64(dO))).sum().backward()
    return V.grad.numpy(), s.grad.numpy(), t.grad.numpy(), b.grad.numpy()


def pin_backward_autograd(orc):
    """dV, ds, dt and dbias (summed over the batch) equal what automatic
    differentiation of the forward's definition gives, on small shapes with
    and without a bias (a zero bias still has a gradient)."""
    rng = np.random.default_rng(41)
    for (B, H, N, d) in [(1, 1, 1, 1), (2, 2, 3, 5), (1, 3, 8, 72), (2, 1, 8, 33), (3, 2, 7, 64)]:
        for with_bias in (False, True):
            c = make_custom(B, H, N, d, seed=int(rng.integers(1 << 30)), qk_dtype="bf16",
                            with_bias=with_bias, bias_std=0.7, zeros_frac=0.1)
            dO = f32_to_bf16_bits(rng.standard_normal((B, H, N, d)).astype(np.float32))
            got = orc.backward(c["q"], c["k"], c["bias"], c["v"], dO, c["softmax_scale"])
            want = _grad_of_definition(c["q"], c["k"], c["bias"], c["v"], dO, c["softmax_scale"], H, N)
            for name, g, w in zip(("dV", "ds", "dt", "dbias"), got, want):
                assert g.shape == w.shape, name
                assert np.allclose(g, w, rtol=1e-10, atol=1e-13), f"{name} differs from autograd at {B,H,N,d}"


def pin_backward_invariants(orc):
    """Rows of dlogit (so of dbias) sum to 0, because softmax rows sum to 1;
    sum_j dV_j = sum_i dO_i; at softmax_scale 0 the scaled binary Q and K get
    no gradient, and with no bias the attention is uniform, so dV_j is the
    mean of dO over the rows; doubling dO doubles every gradient."""
    B, H, N, d = 2, 2, 37, 40
    c = make_custom(B, H, N, d, seed=5, with_bias=True, bias_std=0.8)
    rng = np.random.default_rng(6)
    dO = f32_to_bf16_bits(rng.standard_normal((B, H, N, d)).astype(np.float32))
    dV, ds, dt, db = orc.backward(c["q"], c["k"], c["bias"], c["v"], dO, c["softmax_scale"])
    assert np.abs(db.sum(-1)).max() <= 1e-13 * max(1.0, np.abs(db).max()) * N, "dbias rows do not sum to 0"
    assert np.allclose(dV.sum(2), _f64(dO).sum(2), rtol=1e-12, atol=1e-12), "sum_j dV_j != sum_i dO_i"
    _, ds0, dt0, _ = orc.backward(c["q"], c["k"], c["bias"], c["v"], dO, 0.0)
    assert not ds0.any() and not dt0.any(), "scale 0 must give ds = dt = 0"
    dV0, _, _, _ = orc.backward(c["q"], c["k"], None, c["v"], dO, 0.0)
    want = np.broadcast_to(_f64(dO).mean(2, keepdims=True), dV0.shape)
    assert np.allclose(dV0, want, rtol=1e-13, atol=1e-15), "uniform attention: dV_j != mean_i dO_i"
    dO2 = f32_to_bf16_bits(2 * bf16_bits_to_f32(dO))  # exact in bf16
    for g1, g2 in zip(orc.backward(c["q"], c["k"], c["bias"], c["v"], dO, c["softmax_scale"]),
                      orc.backward(c["q"], c["k"], c["bias"], c["v"], dO2, c["softmax_scale"])):
        assert np.allclose(g2, 2 * g1, rtol=1e-13, atol=1e-15), "not linear in dO"


def pin_backward_finite_differences(orc):
    """Differences of the forward oracle's loss sum(dO * O), on inputs with
    few significant bits so that every perturbed input below is exact:
    - the loss is linear in V, so one step of V_jc gives dV_jc exactly;
    - scaling query row i by lambda scales alpha_q_i (its signs stay), so
      dloss/dlambda = <ds_i, s_i>; likewise key row j gives <dt_j, t_j>;
    - adding delta to the bias column of key j in every row of head h gives
      sum_i dbias[h, i, j].
    The last three use Richardson extrapolation of central differences."""
    B, H, N, d = 1, 2, 12, 24
    rng = np.random.default_rng(77)
    q = (rng.integers(-120, 121, size=(B, H, N, d)) / 64).astype(np.float32)
    k = (rng.integers(-120, 121, size=(B, H, N, d)) / 64).astype(np.float32)
    v = f32_to_bf16_bits((rng.integers(-60, 61, size=(B, H, N, d)) / 16).astype(np.float32))
    bias = f32_to_bf16_bits((rng.integers(-200, 201, size=(H, N, N)) / 256).astype(np.float32))
    dO = f32_to_bf16_bits(rng.standard_normal((B, H, N, d)).astype(np.float32))
    scale = 0.3
    dV, ds, dt, db = orc.backward(q, k, bias, v, dO, scale)
    base = _loss(orc, q, k, bias, v, dO, scale)

    def richardson(f, e):
        d1 = (f(e) - f(-e)) / (2 * e)
        d2 = (f(2 * e) - f(-2 * e)) / (4 * e)
        return (4 * d1 - d2) / 3

    for (h, j, c_) in [(0, 0, 0), (1, 11, 23), (1, 5, 7)]:
        v2 = bf16_bits_to_f32(v).copy()
        v2[0, h, j, c_] += np.float32(1 / 16)
        fd = (_loss(orc, q, k, bias, f32_to_bf16_bits(v2), dO, scale) - base) * 16
        assert abs(fd - dV[0, h, j, c_]) <= 1e-9 * (1 + abs(fd)), f"dV[{h},{j},{c_}]"
    s = np.abs(q.astype(np.float64)).mean(-1)[..., None] * np.where(q >= 0, 1.0, -1.0)
    t = np.abs(k.astype(np.float64)).mean(-1)[..., None] * np.where(k >= 0, 1.0, -1.0)
    e = 2.0 ** -12
    for (h, i) in [(0, 0), (1, 7), (0, 11)]:
        def fq(x, h=h, i=i):
            q2 = q.copy()
            q2[0, h, i] = q[0, h, i] * np.float32(1 + x)
            return _loss(orc, q2, k, bias, v, dO, scale)

        def fk(x, h=h, i=i):
            k2 = k.copy()
            k2[0, h, i] = k[0, h, i] * np.float32(1 + x)
            return _loss(orc, q, k2, bias, v, dO, scale)
        want_q = float((ds[0, h, i] * s[0, h, i]).sum())
        want_k = float((dt[0, h, i] * t[0, h, i]).sum())
        assert abs(richardson(fq, e) - want_q) <= 1e-8 * (1 + abs(want_q)), f"<ds, s> at row {h},{i}"
        assert abs(richardson(fk, e) - want_k) <= 1e-8 * (1 + abs(want_k)), f"<dt, t> at row {h},{i}"
    delta = 2.0 ** -8
    for (h, j) in [(0, 0), (1, 6), (1, 11)]:
        def fb(x, h=h, j=j):
            b2 = bf16_bits_to_f32(bias).copy()
            b2[h, :, j] += np.float32(x)
            return _loss(orc, q, k, f32_to_bf16_bits(b2), v, dO, scale)
        want_b = float(db[h, :, j].sum())
        assert abs(richardson(fb, delta) - want_b) <= 1e-7 * (1 + abs(want_b)), f"dbias column {h},{j}"


ALL_PINS = [
    pin_sign_predicate_exhaustive,
    pin_pack_layout_packbits,
    pin_alpha_mean_abs,
    pin_hamming_identity_exhaustive,
    pin_scores_matmul,
    pin_scores_special_cases,
    pin_softmax_rows_sum_to_one,
    pin_softmax_bias_only,
    pin_softmax_shift_invariance,
    pin_scale_invariances,
    pin_uniform_scores_mean_v,
    pin_onehot_bias_gather,
    pin_convex_hull,
    pin_bruteforce_matrix_form,
    pin_worked_example,
    pin_alpha_half_normal_mean,
    pin_sign_correlation_arcsin,
    pin_spread_uniform_is_mean_abs_deviation,
    pin_spread_two_keys_closed_form,
    pin_quantize_v_closed_form,
    pin_int8_uniform_scores,
    pin_int8_two_keys_closed_form,
    pin_relpos_one_hot_counts,
    pin_relpos_translation_invariance,
    pin_backward_autograd,
    pin_backward_invariants,
    pin_backward_finite_differences,
]
