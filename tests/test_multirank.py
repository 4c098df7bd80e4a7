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
from oracle import hs2_oracle as orc
from token_level_sparse_causal_b200 import inputs, shard


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


def _head_split_worker(rank, world, port, out):
    """Rank `rank` takes its KV heads of one small sequence (the oracle stands
    in for the kernels on CPU), then the ranks all-gather O and the LSE."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=__import__("datetime").timedelta(seconds=60))
    try:
        L, Hq, Hkv = 96, 6, 3
        x = inputs.make_inputs(inputs.Workload("split", L, Hq, Hkv, 0, seed=5), with_needles=False)
        sh = shard.kv_head_range(Hq, Hkv, rank, world)
        part = shard.shard_inputs(sh, x["q_layers"], x["k"], x["v"])
        Q = orc.decode_bf16(inputs.as_u16(part["q_layers"][0].contiguous()))
        K = orc.decode_bf16(inputs.as_u16(part["k"].contiguous()))
        V = orc.decode_bf16(inputs.as_u16(part["v"].contiguous()))
        O, lse = orc.dense_attn(Q, K, V)
        sizes = [shard.kv_head_range(Hq, Hkv, r, world).h1 - shard.kv_head_range(Hq, Hkv, r, world).h0
                 for r in range(world)]
        O_all = shard.gather_heads(dist, torch.from_numpy(O), sizes, head_dim=1)
        lse_all = shard.gather_heads(dist, torch.from_numpy(lse), sizes, head_dim=0)
        out[rank] = (sh, O_all.numpy(), lse_all.numpy())
    finally:
        dist.destroy_process_group()


def test_kv_head_split_over_two_gloo_ranks_reassembles_the_whole():
    world = 2
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_head_split_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    x = inputs.make_inputs(inputs.Workload("split", 96, 6, 3, 0, seed=5), with_needles=False)
    O, lse = orc.dense_attn(orc.decode_bf16(inputs.as_u16(x["q_layers"][0])), orc.decode_bf16(inputs.as_u16(x["k"])),
                            orc.decode_bf16(inputs.as_u16(x["v"])))
    assert (res[0][0].g0, res[0][0].g1, res[1][0].g0, res[1][0].g1) == (0, 2, 2, 3)   # uneven: 3 KV heads on 2
    for r in range(world):
        assert abs(res[r][1] - O).max() < 1e-12 and abs(res[r][2] - lse).max() < 1e-12


def test_kv_head_ranges_partition_the_heads():
    for Hq, Hkv in ((64, 8), (32, 4), (16, 4), (24, 3)):
        for world in range(1, Hkv + 1):
            got = [shard.kv_head_range(Hq, Hkv, r, world) for r in range(world)]
            assert got[0].g0 == 0 and got[-1].g1 == Hkv
            assert all(a.g1 == b.g0 for a, b in zip(got, got[1:]))
            sizes = [s.g1 - s.g0 for s in got]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
            assert all(s.h0 == s.g0 * (Hq // Hkv) and s.h1 == s.g1 * (Hq // Hkv) for s in got)
    with pytest.raises(ValueError):
        shard.kv_head_range(64, 8, 0, 9)


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
