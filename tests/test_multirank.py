"""Host logic of multi-GPU runs, exercised with two gloo ranks on CPU: every
rank prefills its own sequence (independent seeds, no collective on the data
path), the step time is the max over ranks, and the job throughput counts
every rank's tokens.  Also pins the benchmark's work accounting."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from token_level_sparse_causal_b200 import inputs


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=__import__("datetime").timedelta(seconds=60))
    try:
        wl = bench.rank_workload(inputs.WORKLOADS["c1"], rank, world)
        mine = 10.0 + 5.0 * rank                       # rank 1 is the slow one
        got = bench.reduce_max(mine, dist)
        x = inputs.make_inputs(wl.scaled(L=256), with_needles=False)
        out[rank] = (wl.seed, got, float(x["q_layers"][0].float().sum()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_independent_sequences():
    world = 2
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    (s0, t0, q0), (s1, t1, q1) = res[0], res[1]
    assert t0 == t1 == 15.0                       # every rank reports the slowest rank's time
    assert s0 != s1 and q0 != q1                   # distinct sequences per rank
    assert bench.job_throughput(2048, world, 15.0) == pytest.approx(2 * 2048 / 0.015)


def test_single_rank_needs_no_group():
    wl = inputs.WORKLOADS["c3"]
    assert bench.rank_workload(wl, 0, 1) is wl
    assert bench.reduce_max(3.5, None) == 3.5


def test_work_accounting_matches_the_exact_causal_counts():
    """Exact causal counts for the 128k workload (FLOP and bytes per the
    formulas FA = Hq*4d*L(L+1)/2, importance = Hq*64*2d*sum|C_b|)."""
    w = bench.algorithmic_work(inputs.WORKLOADS["c3"])
    L, Hq, d = 131072, 64, 128
    assert w["fa_flop"] == Hq * 4 * d * L * (L + 1) / 2
    nc = sum(max(0, 64 * (b + 1) - 128) for b in range(L // 64))
    assert w["imp_flop"] == Hq * 64 * 2 * d * nc
    assert abs(w["fa_flop"] / 2.82e14 - 1) < 0.005 and abs(w["imp_flop"] / 1.41e14 - 1) < 0.005
    assert abs(w["select_bytes"] / 4.29e9 - 1) < 0.005 and abs(w["sparse_flop"] / 4.79e12 - 1) < 0.005
    assert abs(w["gather_bytes"] / 9.62e9 - 1) < 0.005
