"""Host logic of bench.py, on CPU.

- The multi-rank path with gloo, world size 2: each rank draws its own batch
  (weak scaling) and the reported time is the max over ranks; no collective
  touches the data path.
- The source digest that keeps the ncu traffic figure tied to the kernels.
- The percentiles of the timed steps.
- The algorithmic bytes and work behind the roofline.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import bench
    from diffusion_transformers_b200.synthetic import WORKLOADS, make_inputs

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = WORKLOADS["tiny"]
        # per-rank time: the job's time is the slowest rank's
        t = bench.max_over_ranks_of(1.0 + rank * 0.25, world, torch.device("cpu"))
        # and the same call order on every rank keeps the collectives matched
        t2 = bench.max_over_ranks_of(5.0 - rank, world, torch.device("cpu"))
        seed = bench.rank_seed(w, rank)
        q = make_inputs(w, with_bias=False, seed=seed)["q"]
        out[rank] = (t, t2, seed, float(abs(q).sum()), bench.job_units(10, world))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_distinct_batches():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    r0, r1 = out[0], out[1]
    assert r0[0] == r1[0] == 1.25
    assert r0[1] == r1[1] == 5.0
    assert r0[2] != r1[2]          # every rank its own batch
    assert r0[3] != r1[3]
    assert r0[4] == r1[4] == 20    # units of the whole job


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks_of(3.5, 1, None) == 3.5
    assert bench.job_units(7, 1) == 7


def test_reference_arm_other_ranks_do_no_work(capsys):
    import argparse

    import bench
    from diffusion_transformers_b200.synthetic import WORKLOADS
    args = argparse.Namespace(steps=1, warmup=0, gpus=2, cpu_seconds=0.1, workload="tiny")
    bench.run_reference(args, WORKLOADS["tiny"], rank=1)
    assert capsys.readouterr().out == ""


def test_traffic_digest_ignores_comments_only():
    import bench

    src = 'int f(int x) { // doubles\n  return 2 * x; /* multi\n line */ }\nconst char* s = "a//b /*c*/";\n'
    same = '/* header */ int f(int x) {\n\n return 2*x; }   const char* s = "a//b /*c*/";'
    assert bench.code_only(src) == bench.code_only(same.replace("2*x", "2 * x"))
    assert '"a//b /*c*/"' in bench.code_only(src)
    assert bench.code_only(src) != bench.code_only(src.replace("2 * x", "3 * x"))


def test_percentile_matches_numpy():
    import numpy as np

    import bench

    rng = np.random.default_rng(4)
    for n in (1, 2, 5, 20, 101):
        xs = rng.random(n).tolist()
        for q in (0.0, 0.1, 0.5, 0.9, 1.0):
            assert abs(bench.percentile(xs, q) - float(np.percentile(xs, 100 * q))) < 1e-12


def test_algorithmic_work_matches_the_hand_figures():
    # Bytes (bits + alphas + V + O + bias once) and work per forward call,
    # against the figures worked out by hand for the five workloads:
    # MB to 0.1, pairs to 3 digits, P.V GFLOP to 3 digits.
    import bench
    from diffusion_transformers_b200.synthetic import WORKLOADS

    want = {  # name: (MB with bias, pairs, P.V GFLOP)
        "tiny": (0.41, 1.31e5, 0.0168),
        "deit_b": (43.3, 2.98e7, 3.81),
        "vit_l384": (93.4, 1.70e8, 21.8),
        "dit_xl_512": (75.5, 1.34e8, 19.3),
        "dit_xl_1024": (578.8, 5.37e8, 77.3),
    }
    for name, (mb, pairs, gflop) in want.items():
        a = bench.algorithmic(WORKLOADS[name], True)
        assert round(a["bytes"] / 1e6, 1 if mb >= 1 else 2) == mb, name
        assert abs(a["pairs"] / pairs - 1) < 5e-3, name
        assert abs(a["pv_flops"] / 1e9 / gflop - 1) < 5e-3, name
        assert a["eff_flops"] == 2 * a["pv_flops"] == a["pv_flops"] + a["qk_ops"]
    assert round(bench.algorithmic(WORKLOADS["dit_xl_1024"], False)["bytes"] / 1e6, 1) == 41.9
    # one bias per batch entry: 2 x 16 x 4096^2 bf16 values (1073.7 MB) in place of 536.9 MB
    assert round(bench.algorithmic(WORKLOADS["dit_xl_1024"], True, bias_per_sample=True)["bytes"] / 1e6, 1) == 1115.7
    # the backward at DiT-1024: bits 3.1 MB + alphas 1.0 MB + V and dO 37.7 MB + bias 536.9 MB read,
    # dV, ds, dt 113.2 MB + dbias (fp32) 1073.7 MB written; 4 products of 2d flops per pair
    ab = bench.algorithmic_backward(WORKLOADS["dit_xl_1024"])
    assert round(ab["bytes"] / 1e6, 1) == 1765.8
    assert ab["pv_like_flops"] == 4 * 77_309_411_328 and ab["qk_ops"] == 77_309_411_328


def test_rank_inputs_heads_shard_one_batch():
    # --shard heads: every rank slices the same batch (the workload's seed) and
    # holds only its heads; replicas: every rank its own seed, all heads
    import bench
    from diffusion_transformers_b200.synthetic import WORKLOADS, make_inputs

    w = WORKLOADS["tiny"]
    full = make_inputs(w, with_bias=True, seed=w.seed)
    parts = [bench.rank_inputs(w, r, 2, "heads") for r in range(2)]
    assert [p[0].H for p in parts] == [1, 1]
    q = np.concatenate([p[1]["q"] for p in parts], axis=1)
    b = np.concatenate([p[1]["bias"] for p in parts], axis=0)
    assert np.array_equal(q, full["q"]) and np.array_equal(b, full["bias"])
    w1, inp1 = bench.rank_inputs(w, 1, 2, "none")
    assert w1.H == w.H and not np.array_equal(inp1["q"], full["q"])
    assert bench.rank_inputs(w, 0, 1, "heads")[0].H == w.H


def test_roofline_prices_qk_at_the_e4m3_pipe():
    # T_roof = max(T_mem, T_QK + T_PV), T_QK at twice the bf16 rate (the e4m3
    # pipe the binary scores run on); frac = T_roof / time
    import bench
    from diffusion_transformers_b200.synthetic import WORKLOADS

    peaks = dict(hbm_gbs=6540.8, bf16_tflops=1622.9, sm_max_mhz=1965.0)
    w = WORKLOADS["dit_xl_1024"]
    r = bench.roofline_terms(w, True, peaks)
    assert abs(r["t_qk"] * 2 - r["t_pv"]) < 1e-15
    assert abs(r["t_mem"] * 1e6 - 88.49) < 0.01 and abs(r["t_tensor"] * 1e6 - 71.45) < 0.01
    assert r["bound"] == "hbm" and r["t_roof"] == r["t_mem"]
    assert abs(r["t_mufu"] * 1e6 - 115.38) < 0.01
    line = bench.roofline_line(w, True, peaks, 309e-6)
    assert abs(line["frac"] - 0.2864) < 1e-4 and line["unit"] == "GB/s"
    r0 = bench.roofline_terms(w, False, peaks)
    assert r0["bound"] == "tensor"
    line0 = bench.roofline_line(w, False, peaks, 2 * r0["t_tensor"])
    assert line0["frac"] == 0.5 and abs(line0["achieved"] * 2 - line0["peak"]) < 0.02
