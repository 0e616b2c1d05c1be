"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2).

The scoring path partitions into independent problems, so N GPUs run N
replicas with no data-path collective; what crosses ranks is only the timing
(max over ranks) and the whole-job throughput.  These tests run that logic on
two gloo ranks with the fp64 oracle standing in for the per-rank work.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle
from kv_cache_eviction_scores_b200 import workloads as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        spec = W.config_spec(0)
        wl = W.generate(spec, bench.rank_seed(rank))
        s = oracle.scores(wl.q, wl.k, wl.v, wl.lengths, spec.window, spec.pool)
        ms_local = 10.0 + 5.0 * rank  # rank 1 is the slow one
        ms = bench.max_over_ranks(ms_local, dist, torch.device("cpu"))
        value = bench.whole_job_value(world, sum(wl.lengths), ms)
        # gather every rank's first scores to check the shards are independent
        t = torch.from_numpy(np.nan_to_num(s[0, 0], posinf=0.0)).to(torch.float64)
        allt = [torch.zeros_like(t) for _ in range(world)]
        dist.all_gather(allt, t)
        out[rank] = (ms, value, [x.numpy().tolist() for x in allt])
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_time_is_the_max_and_value_counts_all_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert set(out.keys()) == {0, 1}
    for r in range(world):
        ms, value, allt = out[r]
        assert ms == 15.0  # max over ranks, seen identically by every rank
        assert value == pytest.approx(world * 22 / 15e-3)
        assert allt[0] != allt[1]  # independent inputs per rank (seeds 42, 43)


def test_rank_seeds_are_distinct_and_single_rank_is_identity():
    assert bench.rank_seed(0) != bench.rank_seed(1)
    assert bench.max_over_ranks(3.5, None, torch.device("cpu")) == 3.5
    assert bench.whole_job_value(1, 1000, 2.0) == pytest.approx(5e5)


def test_sequence_override_keeps_the_shape_and_budget_fraction():
    import argparse

    spec = bench.bench_spec(argparse.Namespace(config=3, seq=32768))
    full = W.config_spec(3)
    assert (spec.Hq, spec.Hkv, spec.d, spec.window, spec.pool) == \
        (full.Hq, full.Hkv, full.d, full.window, full.pool)
    assert spec.lengths == [32768] and spec.n_max == 32768 and spec.B == 1
    assert spec.keep[0] == int(full.keep[0] / full.lengths[0] * 32768)
    assert spec.outlier_channels == full.outlier_channels
    assert bench.bench_spec(argparse.Namespace(config=3, seq=None)) == full
    assert bench.NOMINAL_HBM_GBS == 8000.0


def test_visible_elements_counts_the_causal_window():
    # brute force: query t of a head sees keys 0 .. L - w + t
    spec = W.small_spec(4)
    brute = sum(sum(L - spec.window + t + 1 for t in range(spec.window)) for L in spec.lengths)
    assert bench.visible_elements(spec) == brute * spec.Hq


def test_roofline_arithmetic_of_the_passes():
    spec = W.config_spec(3)
    us = 200.0
    kv = sum(spec.lengths) * spec.Hkv * spec.d * 2  # one read of K (or V), bf16
    r = bench.roofline("k_tc_pass2", spec, us, 6554.6, 1657.0, 1965.0)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(2 * kv / (us * 1e-6) / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / 6554.6)
    flops = 4 * spec.d * bench.visible_elements(spec)
    assert r["tensor"]["achieved"] == pytest.approx(flops / (us * 1e-6) / 1e12)
    # the attention-only second pass streams K alone and runs one contraction
    ra = bench.roofline("k_tc_pass2", spec, us, 6554.6, 1657.0, 1965.0, "attention")
    assert ra["achieved"] == pytest.approx(kv / (us * 1e-6) / 1e9)
    assert ra["tensor"]["achieved"] == pytest.approx(flops / 2 / (us * 1e-6) / 1e12)
