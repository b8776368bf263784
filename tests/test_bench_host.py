"""Host logic of bench.py on the CPU: the max-over-ranks reduction across two gloo ranks,
the output-channel sharding of one layer (each rank its own rows of one weight; two gloo
ranks running the oracle on their shards reproduce the unsharded layer bit for bit), and
the JSON contract of the reference arm (the CPU oracle timed on this host)."""
import json
import os
import re
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from bit_matmul_decomposition_b200 import synth  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks([rank + 1.0, 10.0 - rank, 0.5 * rank])
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        assert out[r] == [2.0, 10.0, 0.5]


def test_max_over_ranks_without_process_group_is_identity():
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]


def test_shard_rows_partition_the_output_channels():
    for N in (1, 7, 101, 49152):
        for world in (1, 2, 3, 8):
            if world > N:
                continue
            blocks = [synth.shard_rows(N, r, world) for r in range(world)]
            assert blocks[0][0] == 0 and blocks[-1][1] == N
            assert all(blocks[i][1] == blocks[i + 1][0] for i in range(world - 1))
            sizes = [b - a for a, b in blocks]
            assert max(sizes) - min(sizes) <= 1


def test_each_rank_holds_rows_of_one_weight():
    w = synth.Workload("t", 8, 64, 2500, seed=7)
    for world in (1, 2, 3):
        layer, _ = bench.rank_workload(w, 0, world)
        assert layer.N == world * w.N and layer.seed == w.seed
        W = synth.make_w(layer)
        b = synth.make_bias(layer)
        parts = []
        for r in range(world):
            lay_r, rows = bench.rank_workload(w, r, world)
            assert lay_r == layer and rows[1] - rows[0] == w.N   # weak scaling: N per rank
            parts.append(synth.make_w(layer, rows))
            assert np.array_equal(synth.make_bias(layer, rows), b[rows[0]:rows[1]])
        # the ranks' blocks are the rows of the one weight, in order
        assert np.array_equal(np.concatenate(parts), W)
        # the hidden states are the same on every rank
        assert np.array_equal(synth.make_x(layer), synth.make_x(w))
    layer1, rows1 = bench.rank_workload(w, 0, 1)
    assert layer1 == w and rows1 == (0, w.N)     # one GPU: the workload itself


def _shard_worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        from oracle import oracle as O
        w = synth.Workload("shard", 24, 128, 101, seed=5, fixed_cols=(3, 77))
        rows = synth.shard_rows(w.N, rank, world)
        X = synth.make_x(w)                      # replicated
        W_r = synth.make_w(w, rows)
        b_r = synth.make_bias(w, rows)
        CB_r, SCB_r = O.quantize_weight(W_r)
        r = O.linear_forward(X, CB_r, SCB_r, b_r, w.threshold)
        mine = dict(rows=rows, mask=r["mask_words"], SCx=r["SCx"], Xq=r["Xq"], CB=CB_r,
                    SCB=SCB_r, C=r["C"])
        got = [None] * world
        dist.all_gather_object(got, mine)
        if rank == 0:
            full_W, full_b = synth.make_w(w), synth.make_bias(w)
            CB, SCB = O.quantize_weight(full_W)
            ref = O.linear_forward(X, CB, SCB, full_b, w.threshold)
            ok = [got[i]["rows"] == synth.shard_rows(w.N, i, world) for i in range(world)]
            for g in got:   # every rank found the same outlier columns and row scales
                ok.append(np.array_equal(g["mask"], ref["mask_words"]))
                ok.append(np.array_equal(g["SCx"].view(np.uint32), ref["SCx"].view(np.uint32)))
                ok.append(np.array_equal(g["Xq"], ref["Xq"]))
            ok.append(np.array_equal(np.concatenate([g["CB"] for g in got]), CB))
            ok.append(np.array_equal(np.concatenate([g["SCB"] for g in got]).view(np.uint32),
                                     SCB.view(np.uint32)))
            C = np.concatenate([g["C"] for g in got], axis=1)
            ok.append(C.shape == ref["C"].shape
                      and np.array_equal(C.view(np.uint64), ref["C"].view(np.uint64)))
            out["ok"] = ok
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_one_layer_like_one_gpu():
    """N = 101 over two ranks (blocks of 50 and 51 channels): each rank runs the oracle on
    its rows of the one weight; the gathered blocks equal the unsharded layer bit for bit
    (mask, row scales, codes, CB/SCB and the fp64 output)."""
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_shard_worker, args=(world, port, out), nprocs=world, join=True)
    assert out["ok"] and all(out["ok"]), out["ok"]


REQUIRED = ["metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
            "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config"]


def _run_ref(extra_env=None, *args):
    env = dict(os.environ, **(extra_env or {}))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--workload", "tiny", "--steps", "2", "--warmup", "3", *args],
                          capture_output=True, text=True, env=env, timeout=600)


def test_reference_arm_prints_one_contract_line():
    r = _run_ref()
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in REQUIRED:
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "TOPS"
    assert d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "TOPS", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["workload"].startswith("tiny")


def test_reference_arm_other_ranks_exit_quietly():
    r = _run_ref({"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_l2_policy_flushes_only_inputs_that_fit_twice_in_l2():
    import bench
    assert bench.l2_policy("auto", 2048, 16384, 4096)[0]            # 84 MB of inputs
    no, desc = bench.l2_policy("auto", 16, 57344, 14336)             # CB 822 MB
    assert not no and "no flush" in desc
    assert bench.l2_policy("always", 16, 57344, 14336)[0]


def test_work_counts_split_the_product_at_the_outlier_columns():
    T, N, K = 2048, 16384, 4096
    i8, f16, eff, nbytes = bench.work_counts(T, N, K, 0)
    assert i8 == eff == 2.0 * T * N * K and f16 == 0.0
    i8, f16, eff, _ = bench.work_counts(T, N, K, 6)
    assert i8 + f16 == eff and f16 == 2.0 * T * N * 6
    # the bytes include at least CB once, X once and C once
    assert nbytes >= N * K + 2 * T * K + 2 * T * N


def test_traffic_is_reported_only_for_the_sources_it_was_measured_on(monkeypatch):
    rec = bench.traffic_record("i8_gemm_tcgen05_kernel", "opt6.7b_ffn_up_prefill_2048x4096x16384")
    if rec is not None:   # the committed capture matches the current CUDA sources
        assert rec["dram_bytes_per_launch"] > 0
    monkeypatch.setattr(bench, "source_hash", lambda kernel=None: "0" * 64)
    assert bench.traffic_record("i8_gemm_tcgen05_kernel",
                                "opt6.7b_ffn_up_prefill_2048x4096x16384") is None
    assert bench.traffic_record("decode_kernel", "no_such_workload") is None


def test_kernel_source_hash_covers_its_headers_and_the_launch_code():
    # every kernel's hash reads api.cu (launch sizing) and common.cuh, and its own header
    for k, files in bench.KERNEL_SOURCES.items():
        assert {"api.cu", "common.cuh"} <= set(files), k
        assert set(files) <= set(bench.CUDA_SOURCES), k
    assert "gemv.cuh" in bench.KERNEL_SOURCES["decode_kernel"]
    assert "gemm_wide.cuh" in bench.KERNEL_SOURCES["i8_gemm_wide_kernel"]
    # headers a kernel's header includes are in its list
    csrc = os.path.join(bench.ROOT, "bit_matmul_decomposition_b200", "csrc")
    own = {"decode_kernel": "gemv.cuh", "prepare_kernel": "quant.cuh",
           "i8_gemm_tcgen05_kernel": "gemm.cuh", "i8_gemm_wide_kernel": "gemm_wide.cuh"}
    for k, hdr in own.items():
        todo, seen = [hdr], set()
        while todo:
            f = todo.pop()
            if f in seen:
                continue
            seen.add(f)
            with open(os.path.join(csrc, f)) as fh:
                todo += re.findall(r'#include "([a-z_]+\.cuh)"', fh.read())
        assert seen <= set(bench.KERNEL_SOURCES[k]), (k, seen)
    assert bench.source_hash("decode_kernel") != bench.source_hash("i8_gemm_tcgen05_kernel")
    assert bench.source_hash("no_such_kernel") == bench.source_hash()


def test_tensor_peak_follows_the_power_cap_seen_while_timing():
    pk = dict(hbm=6459.3, bf16=1679.9, bf16_sus=1418.9, source="measured")
    burst, why = bench.tensor_peak(pk, {"sm_mhz": 1965.0, "reasons": []})
    assert burst == 2 * 1679.9 and "burst" in why
    capped, why = bench.tensor_peak(pk, {"sm_mhz": 1380.0, "reasons": ["sw_power_cap"]})
    assert capped == 2 * 1418.9 and "sustained" in why
    unknown, why = bench.tensor_peak(pk, None, e4m3=True)
    assert unknown == 2 * 1679.9 and "fp8" in why and "no clock record" in why


def test_clock_record_keeps_only_samples_inside_the_timed_region():
    # (time, sm_mhz, max_mhz, NVML reason bits, power_w): idle samples before and after,
    # power-capped samples at 1620 MHz inside
    samples = [(0.00, 1965.0, 1965.0, 0x1, 120.0), (0.10, 1965.0, 1965.0, 0x0, 130.0),
               (0.20, 1620.0, 1965.0, 0x4, 990.0), (0.21, 1605.0, 1965.0, 0x4, 1001.0),
               (0.22, 1650.0, 1965.0, 0x0, 950.0), (0.50, 1965.0, 1965.0, 0x1, 140.0)]
    rec = bench.summarise_clock_samples(samples, 0.15, 0.30)
    assert rec["samples"] == 3
    assert rec["sm_mhz"] == 1620.0
    assert rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["sw_power_cap"]
    assert rec["power_w_max"] == 1001.0
    hot = [(0.2, 1400.0, 1965.0, 0x8 | 0x40 | 0x20, 700.0)]
    assert bench.summarise_clock_samples(hot, 0.0, 1.0)["reasons"] == [
        "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]
    assert bench.summarise_clock_samples(samples, 0.6, 0.7) is None


def test_clock_sampler_without_a_gpu_reports_nothing():
    c = bench.ClockSampler()
    c.start()
    c.begin()
    c.end()
    assert c.stop() is None
