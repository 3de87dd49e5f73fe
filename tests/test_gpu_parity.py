"""GPU path (through the C ABI) against the CPU oracle, on the same seeded inputs.

Bits: exact. alpha: relative 1e-6 (fp32 tree sum of depth <= W + 6, each step
rounding by at most 2^-24). Integer scores: exact. O: max-abs 2e-2 and
rel-RMS 5e-3 against the oracle's unrounded fp64 result.
"""
import numpy as np
import pytest
import torch

from diffusion_transformers_b200 import binattn
from diffusion_transformers_b200.synthetic import WORKLOADS, make_custom, make_inputs
from parity import bf16_to_f64, check_o, dev, run_path, sample_rows

pytestmark = pytest.mark.gpu

ENGINES = ["simt", "popc_tc", "tc"]

SMALL_SHAPES = [  # (B, H, N, d): several tiles and a ragged tail
    (1, 2, 256, 64), (2, 3, 129, 72), (1, 2, 197, 64), (1, 1, 1, 64), (2, 1, 7, 32),
    (1, 2, 127, 96), (1, 1, 300, 128), (2, 2, 257, 8), (1, 1, 130, 72),
    # N % 8 == 0 with d <= 80 runs the TMA-fed pipeline: with and without a
    # ragged last key tile, several query tiles, two key tiles in flight
    (1, 2, 304, 64), (2, 2, 512, 72), (1, 1, 72, 16), (1, 3, 1000, 72),
]
ODD_D_SHAPES = [(1, 2, 65, 33), (1, 1, 40, 1), (2, 1, 33, 100), (1, 1, 31, 127)]


def _engines_for(d):
    return [e for e in ENGINES if e == "simt" or d % 8 == 0]


# ------------------------------------------------------------------ pack (a1, a2)
@pytest.mark.parametrize("shape", SMALL_SHAPES + ODD_D_SHAPES)
@pytest.mark.parametrize("qk_dtype", ["bf16", "f32"])
def test_pack_exact(orc, shape, qk_dtype):
    B, H, N, d = shape
    c = make_custom(B, H, N, d, seed=N * 7 + d, qk_dtype=qk_dtype, zeros_frac=0.05)
    bits, alpha = binattn.pack(dev(c["q"]))
    ob, oa = orc.pack(c["q"])
    assert np.array_equal(bits.cpu().numpy().view(np.uint32), ob)
    np.testing.assert_allclose(alpha.cpu().numpy().astype(np.float64), oa, rtol=1e-6, atol=0)


# bf16 tokens of whole 16-byte chunks (one thread per token, the arithmetic
# of the forward's own binarisation of Q): every d % 8 == 0 up to 128, with
# ragged last blocks; bits exact, alpha within 1e-6.
@pytest.mark.parametrize("d", [8, 16, 24, 40, 56, 64, 72, 80, 88, 104, 120, 128])
def test_pack_rows_every_chunk_count(orc, d):
    for N in (1, 193, 1000):
        c = make_custom(2, 3, N, d, seed=N + d, zeros_frac=0.05)
        bits, alpha = binattn.pack(dev(c["q"]))
        ob, oa = orc.pack(c["q"])
        assert np.array_equal(bits.cpu().numpy().view(np.uint32), ob), (N, d)
        np.testing.assert_allclose(alpha.cpu().numpy().astype(np.float64), oa, rtol=1e-6, atol=0)


@pytest.mark.parametrize("name", ["tiny", "deit_b", "vit_l384", "dit_xl_512", "dit_xl_1024"])
def test_pack_exact_full_size(orc, name):
    inp = make_inputs(name, with_bias=False)
    for key in ("q", "k"):
        bits, alpha = binattn.pack(dev(inp[key]))
        ob, oa = orc.pack(inp[key])
        assert np.array_equal(bits.cpu().numpy().view(np.uint32), ob), f"{name} {key} bits"
        np.testing.assert_allclose(alpha.cpu().numpy().astype(np.float64), oa, rtol=1e-6, atol=0)


# --------------------------------------------------------------- scores (a3, a8)
# The POPC_TC forward uses the same __popc routine as SIMT (one debug kernel);
# the TC engine has its own tensor-core score routines and needs d % 8 == 0:
# "tc" and "tc_biased" dump the scores of the kernel the TC forward runs (the
# TMA-fed 64-key pipeline where it applies, with or without a bias).
TC_SCORE_ENGINES = ["tc", "tc_biased"]
SCORE_CASES = [(s, e) for s in SMALL_SHAPES + ODD_D_SHAPES for e in ["simt"] + TC_SCORE_ENGINES
               if e == "simt" or s[3] % 8 == 0]


@pytest.mark.parametrize("shape,engine", SCORE_CASES)
def test_scores_exact(orc, shape, engine):
    B, H, N, d = shape
    c = make_custom(B, H, N, d, seed=N + d, zeros_frac=0.05)
    qb, _ = binattn.pack(dev(c["q"]))
    kb, _ = binattn.pack(dev(c["k"]))
    S = binattn.scores_debug(qb, kb, d, engine=engine).cpu().numpy()
    assert np.array_equal(S, orc.scores(c["q"], c["k"]))


@pytest.mark.parametrize("name", ["deit_b", "vit_l384", "dit_xl_512", "dit_xl_1024"])
def test_scores_exact_full_size_sampled(orc, name):
    inp = make_inputs(name, with_bias=False)
    B, H, N, d = inp["B"], inp["H"], inp["N"], inp["d"]
    qb, _ = binattn.pack(dev(inp["q"]))
    kb, _ = binattn.pack(dev(inp["k"]))
    rows = sample_rows(B, H, N, 48)
    for engine in ["simt", "popc_tc"] + TC_SCORE_ENGINES:
        S = binattn.scores_debug(qb, kb, d, engine=engine)
        got = S.view(B * H * N, N)[torch.from_numpy(rows).cuda()].cpu().numpy()
        del S
        assert np.array_equal(got, orc.scores_rows(inp["q"], inp["k"], rows)), f"{name} {engine}"


# ------------------------------------------------------------ forward (a1-a8)
@pytest.mark.parametrize("shape", SMALL_SHAPES + ODD_D_SHAPES)
@pytest.mark.parametrize("with_bias", [True, False])
def test_forward_small(orc, shape, with_bias):
    B, H, N, d = shape
    c = make_custom(B, H, N, d, seed=3 * N + d, with_bias=with_bias, bias_std=0.5)
    ref = orc.forward(c["q"], c["k"], c["bias"], c["v"], c["softmax_scale"])
    for engine in _engines_for(d):
        r = run_path(c, engine=engine, with_bias=with_bias)
        check_o(bf16_to_f64(r["out"]), ref, f"{shape} bias={with_bias} {engine}")


@pytest.mark.parametrize("with_bias", [True, False])
def test_forward_tiny_config(orc, with_bias):
    inp = make_inputs("tiny", with_bias=with_bias)
    ref = orc.forward(inp["q"], inp["k"], inp["bias"], inp["v"], inp["softmax_scale"])
    for engine in ENGINES:
        r = run_path(inp, engine=engine, with_bias=with_bias)
        check_o(bf16_to_f64(r["out"]), ref, f"tiny {engine}")


@pytest.mark.parametrize("name,with_bias", [
    ("deit_b", True), ("vit_l384", True), ("dit_xl_512", True),
    ("dit_xl_1024", True), ("dit_xl_1024", False)])
def test_forward_full_size_sampled(orc, name, with_bias):
    inp = make_inputs(name, with_bias=with_bias)
    B, H, N, d = inp["B"], inp["H"], inp["N"], inp["d"]
    rows = sample_rows(B, H, N, 96, seed=5)
    ref = orc.forward_rows(inp["q"], inp["k"], inp["bias"], inp["v"], inp["softmax_scale"], rows)
    engines = [e for e in ENGINES if e != "simt"] or ["simt"]
    for engine in engines:
        r = run_path(inp, engine=engine, with_bias=with_bias)
        got = r["out"].view(B * H * N, d)[torch.from_numpy(rows).cuda()]
        check_o(bf16_to_f64(got), ref, f"{name} bias={with_bias} {engine}")


# -------------------------------------------------------------- edge cases
@pytest.mark.parametrize("engine", ENGINES)
def test_forward_special_cases(orc, engine):
    B, H, N, d = 1, 2, 130, 72
    # softmax_scale = 0: P = softmax(bias); large scale: very peaked rows;
    # negative scale; value scale 1e3 (alpha large) and 1e-3 (alpha small).
    for kw in [dict(scale=0.0), dict(scale=8.0), dict(scale=-0.5), dict(vs=1e3, scale=1e-3),
               dict(vs=1e-3, scale=1e3)]:
        c = make_custom(B, H, N, d, seed=77, bias_std=0.5, value_scale=kw.get("vs", 1.0))
        c["softmax_scale"] = kw["scale"]
        ref = orc.forward(c["q"], c["k"], c["bias"], c["v"], c["softmax_scale"])
        r = run_path(c, engine=engine)
        check_o(bf16_to_f64(r["out"]), ref, f"{kw} {engine}")


# Keys whose scale alpha_k grows with the key index: every later key tile has
# larger logits, so the running max grows tile after tile and O (with l) is
# rescaled again and again, with and without a bias, on a ragged N.
@pytest.mark.parametrize("with_bias", [False, True])
@pytest.mark.parametrize("d", [64, 72])
def test_forward_growing_max(orc, with_bias, d):
    from diffusion_transformers_b200.synthetic import f32_to_bf16_bits
    B, H, N = 1, 2, 700
    c = make_custom(B, H, N, d, seed=91 + d, with_bias=with_bias, bias_std=0.5)
    grow = (1.0 + np.arange(N, dtype=np.float32) / 24.0)[None, None, :, None]
    c["k"] = f32_to_bf16_bits(bf16_to_f64_np(c["k"]) * grow)
    ref = orc.forward(c["q"], c["k"], c["bias"] if with_bias else None, c["v"], c["softmax_scale"])
    r = run_path(c, with_bias=with_bias)
    check_o(bf16_to_f64(r["out"]), ref, f"growing max d={d} bias={with_bias}")


def bf16_to_f64_np(bits):
    from diffusion_transformers_b200.synthetic import bf16_bits_to_f32
    return bf16_bits_to_f32(bits).astype(np.float32)


@pytest.mark.parametrize("engine", ENGINES)
def test_forward_deterministic(engine):
    c = make_custom(2, 2, 300, 72, seed=9)
    a = run_path(c, engine=engine)["out"].clone()
    b = run_path(c, engine=engine)["out"]
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_device_errors_are_reported():
    x = torch.zeros(1, 1, 4, 64, dtype=torch.bfloat16, device="cuda")
    bits = torch.empty(1, 1, 4, 2, dtype=torch.int32, device="cuda")
    alpha = torch.empty(1, 1, 4, dtype=torch.float32, device="cuda")
    L = binattn.lib()
    import ctypes
    rc = L.binattn_pack(ctypes.c_void_p(x.data_ptr() + 2), 1, 1, 1, 4, 64,
                        ctypes.c_void_p(bits.data_ptr()), ctypes.c_void_p(alpha.data_ptr()), None)
    assert rc == 4
    binattn.device_status()


# ------------------------------------------- forward with a workspace
# Bias rows of N % 8 != 0 elements are not TMA rows; binattn_forward_ws pads
# them into the workspace and runs the TMA-fed pipeline, and splits a short
# last wave of row pairs by key halves (partials joined by a combine kernel).
# Same bar as forward.
WS_SHAPES = [(2, 3, 129, 72), (1, 2, 197, 64), (1, 1, 130, 72), (2, 2, 65, 16), (1, 1, 1, 64),
             (1, 3, 1001, 40), (1, 2, 300, 8)]


def _run_ws(inp, with_bias=True):
    q, k, v = dev(inp["q"]), dev(inp["k"]), dev(inp["v"])
    bias = dev(inp["bias"]) if with_bias else None
    qb, aq = binattn.pack(q)
    kb, ak = binattn.pack(k)
    B, H, N, d = v.shape
    need = binattn.workspace_bytes(B, H, N, d, with_bias)
    ws = torch.full((max(need, 16),), 0xA5, dtype=torch.uint8, device="cuda")  # stale bytes on purpose
    out = binattn.forward_ws(qb, kb, aq, ak, bias, v, inp["softmax_scale"], workspace=ws)
    torch.cuda.synchronize()
    binattn.device_status()
    return out, need


@pytest.mark.parametrize("shape", WS_SHAPES)
def test_forward_ws_small(orc, shape):
    B, H, N, d = shape
    c = make_custom(B, H, N, d, seed=5 * N + d, with_bias=True, bias_std=0.5)
    ref = orc.forward(c["q"], c["k"], c["bias"], c["v"], c["softmax_scale"])
    out, need = _run_ws(c)
    if N % 8:
        assert need >= H * N * ((N + 7) // 8 * 8) * 2
    check_o(bf16_to_f64(out), ref, f"ws {shape}")


@pytest.mark.parametrize("name", ["deit_b", "vit_l384"])
def test_forward_ws_full_size_sampled(orc, name):
    inp = make_inputs(name, with_bias=True)
    B, H, N, d = inp["B"], inp["H"], inp["N"], inp["d"]
    rows = sample_rows(B, H, N, 96, seed=7)
    ref = orc.forward_rows(inp["q"], inp["k"], inp["bias"], inp["v"], inp["softmax_scale"], rows)
    out, need = _run_ws(inp)
    assert need > 0
    got = out.view(B * H * N, d)[torch.from_numpy(rows).cuda()]
    check_o(bf16_to_f64(got), ref, f"ws {name}")


# Shapes whose 256-row pairs leave a short last wave behind at least one full
# wave, with >= 32 key tiles: the tail pairs run split by key halves. Checked on
# every row of the split pairs (the last pairs in launch order) plus random rows.
SPLIT_SHAPES = [(1, 19, 2048, 72, True), (2, 10, 2100, 40, False)]


@pytest.mark.parametrize("shape", SPLIT_SHAPES)
def test_forward_ws_split_tail(orc, shape):
    B, H, N, d, with_bias = shape
    c = make_custom(B, H, N, d, seed=7 * N + d, with_bias=with_bias, bias_std=0.5)
    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    nq = (N + 255) // 256
    pairs = B * H * nq
    tail = pairs % nsm
    assert pairs // nsm and tail and 2 * tail <= nsm  # the split runs
    rows = []
    for pidx in range(pairs - tail, pairs):  # pair -> (b, query tile, h), b fastest
        b, qt, h = pidx % B, (pidx // B) % nq, pidx // (B * nq)
        rows += [(b * H + h) * N + i for i in range(qt * 256, min(N, qt * 256 + 256))]
    rows = np.unique(np.concatenate([np.array(rows, dtype=np.int64), sample_rows(B, H, N, 64, seed=3)]))
    ref = orc.forward_rows(c["q"], c["k"], c["bias"] if with_bias else None, c["v"], c["softmax_scale"], rows)
    out, need = _run_ws(c, with_bias=with_bias)
    assert need > 0
    got = out.view(B * H * N, d)[torch.from_numpy(rows).cuda()]
    check_o(bf16_to_f64(got), ref, f"split {shape}")


# ------------------------------- forward that binarises Q itself (fused a1/a2)
# bf16 Q on the TMA-fed pipelines is binarised inside the forward kernel with
# the same device code as binattn_pack, so O must equal pack + forward_ws bit
# for bit; fp32 Q and other shapes go through pack into the workspace.
FUSED_SHAPES = [(2, 3, 129, 72, True), (1, 2, 197, 64, True), (2, 2, 300, 64, False), (1, 2, 256, 40, False),
                (1, 1, 65, 16, True), (1, 2, 100, 36, True), (1, 19, 2048, 72, True), (2, 10, 2100, 40, False)]


@pytest.mark.parametrize("shape", FUSED_SHAPES)
def test_forward_fused_equals_pack_then_forward(orc, shape):
    B, H, N, d, with_bias = shape
    c = make_custom(B, H, N, d, seed=11 * N + d, with_bias=with_bias, bias_std=0.5)
    q, k, v = dev(c["q"]), dev(c["k"]), dev(c["v"])
    bias = dev(c["bias"]) if with_bias else None
    qb, aq = binattn.pack(q)
    kb, ak = binattn.pack(k)
    want = binattn.forward_ws(qb, kb, aq, ak, bias, v, c["softmax_scale"])
    got = binattn.forward_fused_ws(q, kb, ak, bias, v, c["softmax_scale"])
    torch.cuda.synchronize()
    binattn.device_status()
    assert torch.equal(got.view(torch.int16), want.view(torch.int16)), f"fused {shape}"
    if B * H * N <= 4096:
        ref = orc.forward(c["q"], c["k"], c["bias"] if with_bias else None, c["v"], c["softmax_scale"])
        check_o(bf16_to_f64(got), ref, f"fused {shape}")


def test_forward_fused_fp32_q_and_full_size():
    # fp32 Q (the tiny config) takes the pack-into-workspace route
    inp = make_inputs("tiny", with_bias=True)
    q, k, v, bias = dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), dev(inp["bias"])
    qb, aq = binattn.pack(q)
    kb, ak = binattn.pack(k)
    want = binattn.forward_ws(qb, kb, aq, ak, bias, v, inp["softmax_scale"])
    got = binattn.forward_fused_ws(q, kb, ak, bias, v, inp["softmax_scale"])
    torch.cuda.synchronize()
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))
    # DiT-XL/2 1024 px, both bias cases, whole output
    for with_bias in (True, False):
        inp = make_inputs("dit_xl_1024", with_bias=with_bias)
        q, k, v = dev(inp["q"]), dev(inp["k"]), dev(inp["v"])
        bias = dev(inp["bias"]) if with_bias else None
        qb, aq = binattn.pack(q)
        kb, ak = binattn.pack(k)
        want = binattn.forward_ws(qb, kb, aq, ak, bias, v, inp["softmax_scale"])
        got = binattn.forward_fused_ws(q, kb, ak, bias, v, inp["softmax_scale"])
        torch.cuda.synchronize()
        binattn.device_status()
        assert torch.equal(got.view(torch.int16), want.view(torch.int16)), f"dit_xl_1024 bias={with_bias}"
        del q, k, v, bias, qb, kb, aq, ak, want, got


# ------------------------------------------- the benchmarked calls, every row
# bench.py times binattn_forward_ws with a workspace of
# binattn_forward_workspace_bytes: at DiT-XL/2 1024 px that is the full waves
# of 256-row pairs, the key-split tail pairs and the combine kernel, with and
# without the bias; on the other workloads the padded-bias route or the plain
# forward. Each call is compared here with the oracle on every output row, at
# the workload's own size and seed, together with binattn_forward (no
# workspace) and binattn_forward_fused_ws on the same inputs.
BENCHMARKED = [("dit_xl_1024", True), ("dit_xl_1024", False), ("dit_xl_512", True),
               ("vit_l384", True), ("deit_b", True), ("tiny", True)]


@pytest.mark.parametrize("name,with_bias", BENCHMARKED)
def test_benchmarked_calls_every_row(orc, name, with_bias):
    inp = make_inputs(name, with_bias=with_bias)
    B, H, N, d = inp["B"], inp["H"], inp["N"], inp["d"]
    ref, spread = orc.forward_spread(inp["q"], inp["k"], inp["bias"] if with_bias else None, inp["v"],
                                     inp["softmax_scale"])
    out, need = _run_ws(inp, with_bias=with_bias)
    if name == "dit_xl_1024":
        assert need > 0  # the split tail runs, as in the bench
    check_o(bf16_to_f64(out), ref, f"forward_ws {name} bias={with_bias}", spread)
    del out
    r = run_path(inp, engine="auto", with_bias=with_bias)
    check_o(bf16_to_f64(r["out"]), ref, f"forward {name} bias={with_bias}", spread)
    if inp["q"].dtype == np.uint16:
        got = binattn.forward_fused_ws(r["q"], r["kb"], r["ak"], r["bias"], r["v"], inp["softmax_scale"])
        torch.cuda.synchronize()
        binattn.device_status()
        check_o(bf16_to_f64(got), ref, f"forward_fused_ws {name} bias={with_bias}", spread)


# ------------------------------------------------- a bounded wait runs out
# The TMA producer stops after two key tiles: every CTA's consumers give up
# once their bounded waits run out (about 2 s), the CTA drains its own
# tensor-core work, frees its tensor memory and returns, and the device status
# reports the timeout. The context stays usable: the next call on it meets the
# oracle.
@pytest.mark.parametrize("with_bias", [True, False])
def test_bounded_wait_runs_out_and_context_survives(orc, with_bias):
    c = make_custom(1, 2, 512, 72, seed=123, with_bias=with_bias, bias_std=0.5)
    q, k, v = dev(c["q"]), dev(c["k"]), dev(c["v"])
    bias = dev(c["bias"]) if with_bias else None
    qb, aq = binattn.pack(q)
    kb, ak = binattn.pack(k)
    binattn.device_status()
    binattn.test_wait_timeout(qb, kb, aq, ak, bias, v, c["softmax_scale"], stall_after=2)
    with pytest.raises(binattn.BinattnError) as exc:
        binattn.device_status()
    assert exc.value.status == 7  # BINATTN_ERR_TIMEOUT
    binattn.device_status()  # read and cleared
    ref = orc.forward(c["q"], c["k"], c["bias"] if with_bias else None, c["v"], c["softmax_scale"])
    r = run_path(c, engine="tc", with_bias=with_bias)
    check_o(bf16_to_f64(r["out"]), ref, f"after timeout bias={with_bias}")


# ------------------------------------------ bias stored once with padded rows
# A learned bias stored with rows bias_ld apart: with bias_ld % 8 == 0 the
# TMA-fed pipeline reads it as it is (no padding kernel on the call), with any
# other bias_ld the call pads it as binattn_forward_ws does. Either way O is
# bit-identical to binattn_forward_ws on the same values, and meets the oracle.
@pytest.mark.parametrize("shape", [(1, 2, 197, 64), (2, 3, 129, 72), (1, 2, 1001, 40), (2, 2, 256, 64)])
def test_forward_bias_ld(orc, shape):
    B, H, N, d = shape
    c = make_custom(B, H, N, d, seed=13 * N + d, with_bias=True, bias_std=0.5)
    q, k, v, bias = dev(c["q"]), dev(c["k"]), dev(c["v"]), dev(c["bias"])
    qb, aq = binattn.pack(q)
    kb, ak = binattn.pack(k)
    want = binattn.forward_ws(qb, kb, aq, ak, bias, v, c["softmax_scale"])
    ld8 = binattn.padded_bias_ld(N)
    assert ld8 % 8 == 0 and N <= ld8 < N + 8
    for ld in (ld8, ld8 + 3, ld8 + 8):
        stored = torch.zeros((H, N, ld), dtype=torch.bfloat16, device="cuda")
        stored[:, :, :N] = bias
        stored[:, :, N:] = 7.0  # columns beyond N are never read
        got = binattn.forward_bias_ld_ws(qb, kb, aq, ak, stored, v, c["softmax_scale"])
        torch.cuda.synchronize()
        binattn.device_status()
        assert torch.equal(got.view(torch.int16), want.view(torch.int16)), f"{shape} ld={ld}"
        if ld % 8 == 0:  # no padded copy: only the split partials, as without a bias
            assert binattn.lib().binattn_forward_bias_ld_workspace_bytes(B, H, N, d, ld) == \
                binattn.workspace_bytes(B, H, N, d, False)
    ref = orc.forward(c["q"], c["k"], c["bias"], c["v"], c["softmax_scale"])
    check_o(bf16_to_f64(binattn.forward_bias_ld_ws(qb, kb, aq, ak, binattn.pad_bias(bias), v, c["softmax_scale"])),
            ref, f"bias_ld {shape}")


# ------------------------------------- persistent launches: several pairs per CTA
# With more 256-row pairs than SMs, the 64-key pipeline runs one CTA per SM,
# each taking pairs c, c + S, ... in turn with its rings running on across
# them. One, two and three key tiles per pair (with one, the pairs alternate
# between the two P.V completion barriers), 320 pairs: every output row, the
# dense-bias forward, both 8-bit P.V passes and the score dump of that pipeline.
@pytest.mark.parametrize("shape", [(16, 20, 56, 64), (8, 40, 96, 72), (4, 80, 136, 32)])
def test_persistent_many_pairs(orc, shape):
    B, H, N, d = shape
    c = make_custom(B, H, N, d, seed=7 * N + d, with_bias=True, bias_std=0.5, zeros_frac=0.05)
    q, k, v, bias = dev(c["q"]), dev(c["k"]), dev(c["v"]), dev(c["bias"])
    qb, aq = binattn.pack(q)
    kb, ak = binattn.pack(k)
    S = binattn.scores_debug(qb, kb, d, engine="tc_biased").cpu().numpy()
    assert np.array_equal(S, orc.scores(c["q"], c["k"])), f"scores {shape}"
    o = binattn.forward(qb, kb, aq, ak, bias, v, c["softmax_scale"], engine="tc")
    o_ws = binattn.forward_ws(qb, kb, aq, ak, bias, v, c["softmax_scale"])
    o8 = binattn.forward_int8(qb, kb, aq, ak, bias, v, c["softmax_scale"])
    o8n = binattn.forward_int8(qb, kb, aq, ak, None, v, c["softmax_scale"])
    torch.cuda.synchronize()
    binattn.device_status()
    ref, spread = orc.forward_spread(c["q"], c["k"], c["bias"], c["v"], c["softmax_scale"])
    check_o(bf16_to_f64(o), ref, f"persistent {shape}", spread=spread)
    assert torch.equal(o.view(torch.int16), o_ws.view(torch.int16)), f"forward_ws {shape}"
    check_o(bf16_to_f64(o8), orc.forward_int8(c["q"], c["k"], c["bias"], c["v"], c["softmax_scale"]),
            f"persistent int8 {shape}")
    check_o(bf16_to_f64(o8n), orc.forward_int8(c["q"], c["k"], None, c["v"], c["softmax_scale"]),
            f"persistent int8 no bias {shape}")


# ------------------------------------------------------------- maximum sizes
# The host accepts N <= 65535 and B * H <= 65535. At N = 65535 (1024 key
# tiles of 64, a ragged last tile of 63 keys, on a persistent grid of 256
# pairs) sampled rows of the tensor-core and CUDA-core forwards meet the
# oracle. At B * H = 65535 with N = 8, the forward runs 65535 pairs on a
# persistent grid (about 443 pairs per CTA, one key tile each), with and
# without a bias: every row against the oracle.
def test_max_sequence_length(orc):
    B, H, N, d = 1, 1, 65535, 64
    c = make_custom(B, H, N, d, seed=65535, with_bias=False, zeros_frac=0.01)
    q, k, v = dev(c["q"]), dev(c["k"]), dev(c["v"])
    qb, aq = binattn.pack(q)
    kb, ak = binattn.pack(k)
    rows = np.concatenate([np.arange(4), np.arange(N - 4, N), sample_rows(B, H, N, 24, seed=3)])
    ref = orc.forward_rows(c["q"], c["k"], None, c["v"], c["softmax_scale"], rows)
    for engine in ("tc", "simt"):
        out = binattn.forward(qb, kb, aq, ak, None, v, c["softmax_scale"], engine=engine)
        torch.cuda.synchronize()
        binattn.device_status()
        got = out.view(B * H * N, d)[torch.from_numpy(rows).cuda()]
        check_o(bf16_to_f64(got), ref, f"N = 65535 {engine}")


@pytest.mark.parametrize("B,H,with_bias", [(65535, 1, False), (1, 65535, True), (65535, 1, True)])
def test_max_batch_heads(orc, B, H, with_bias):
    N, d = 8, 64
    c = make_custom(B, H, N, d, seed=B + 2 * H, with_bias=with_bias, bias_std=0.5)
    q, k, v = dev(c["q"]), dev(c["k"]), dev(c["v"])
    bias = dev(c["bias"]) if with_bias else None
    qb, aq = binattn.pack(q)
    kb, ak = binattn.pack(k)
    out = binattn.forward(qb, kb, aq, ak, bias, v, c["softmax_scale"], engine="tc")
    torch.cuda.synchronize()
    binattn.device_status()
    ref = orc.forward(c["q"], c["k"], c["bias"] if with_bias else None, c["v"], c["softmax_scale"])
    check_o(bf16_to_f64(out), ref, f"B={B} H={H} bias={with_bias}")
