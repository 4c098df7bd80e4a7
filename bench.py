#!/usr/bin/env python
"""Prefill throughput of the token-level sparse attention path on B200.

One step = one prefill of the workload through the C ABI: the full-attention
layer with selection (hs2_full_attn_select) followed by every sparse layer
(hs2_sparse_attn), on inputs already resident in HBM.  The default workload is
L = 131072 tokens, 64 query / 8 KV heads, head dim 128, full layer + 3 sparse
layers (its Q/K/V/O tensors are far larger than the 126 MB L2, so no flush is
needed between steps).

  python bench.py [--gpus N --steps K --warmup W] [--impl cuda|reference]
                  [--workload c1..c5] [--stage fa|importance|select|sparse --heads HQ/HKV]

Defaults: 10 warm-up and 20 timed steps (median and P99 reported).  Under
torchrun every rank runs its own independent sequence (weak scaling, no
collective on the data path); the step time is the max over ranks.
`--impl reference` times the fp64 CPU oracle on a bounded sample instead.
`--stage` times one kernel alone (fa: kernel (1); importance: kernel (2);
select: kernel (3); sparse: kernel (4), one layer) on a reduced-head copy of
the workload (the case its ncu capture runs on).  Prints one JSON line on
rank 0.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "prefill tok/s (full-attn+select+sparse-attn) at 128k on 1 B200; % of roofline"


# ------------------------------------------------------------ accounting --

SWA_WINDOW = 128   # sliding window of the self-decoder layers in the measurements


def algorithmic_work(wl) -> dict:
    """Exact causal counts of what the method must compute or move."""
    L, Hq, Hkv, d, B, k, w = wl.L, wl.Hq, wl.Hkv, wl.d, wl.block, wl.topk, wl.recent
    fa = Hq * 4.0 * d * L * (L + 1) / 2
    nb = L // B
    e = np.minimum(L, B * (np.arange(nb) + 1)).astype(np.float64)
    nc = np.maximum(0.0, e - w)
    imp = Hq * 2.0 * d * B * nc.sum()
    sel_rows = nc > k
    select_bytes = Hkv * 4.0 * nc[sel_rows].sum()
    glob = np.minimum(nc, k)
    rec = np.minimum(w, e)
    # visible pairs per block: every query sees the global part; query i sees
    # recent positions [e_b - rec, i]
    vis = B * glob + B * (B + 1) / 2.0 + B * (rec - B)   # rec >= B since recent >= block
    sparse = Hq * 4.0 * d * vis.sum()
    kv_row = 2 * 128 + 8 if getattr(wl, "kv_dtype", "bf16") == "e4m3" else 2 * 256  # K + V row (+ scales)
    gather = Hkv * (glob + rec).sum() * kv_row
    qo = 2.0 * L * Hq * d * 2
    # sliding-window attention: query i sees min(i + 1, W) keys; Q, K, V read
    # once and O written once
    W = SWA_WINDOW
    swa_pairs = W * (W + 1) / 2.0 + max(0, L - W) * float(W) if L >= W else L * (L + 1) / 2.0
    swa = Hq * 4.0 * d * swa_pairs
    swa_bytes = qo + 2.0 * L * Hkv * d * 2
    return {"fa_flop": fa, "imp_flop": imp, "select_bytes": select_bytes, "sparse_flop": sparse,
            "gather_bytes": gather, "sparse_qo_bytes": qo, "swa_flop": swa, "swa_bytes": swa_bytes}


FA_SOURCES = ("token_level_sparse_causal_b200/csrc/flash.cuh", "token_level_sparse_causal_b200/csrc/common.cuh")
FA_TRAFFIC_PROFILE = os.path.join(ROOT, "profiles", "flash_fwd_dram_c3.json")


def kernel_source_hash(paths=FA_SOURCES) -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in paths:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, profile=FA_TRAFFIC_PROFILE):
    """DRAM bytes per full-size launch of kernel (1), from the committed record
    of an ncu capture (a JSON sidecar), or None when the kernel sources changed
    since those counters were taken or the record covers another workload."""
    if not os.path.exists(profile):
        return None
    try:
        rec = json.load(open(profile))
    except (OSError, ValueError):
        return None
    if rec.get("kernel_source_sha256_16") != kernel_source_hash() or rec.get("workload") != workload:
        return None
    try:
        return float(rec["dram_bytes_per_launch"])
    except (KeyError, TypeError, ValueError):
        return None


def arm_config(wl, world: int) -> dict:
    """The `config` object of both arms' JSON lines (the same workload)."""
    q_gb = wl.L * wl.Hq * wl.d * 2 / 1e9
    return {"workload": wl.name, "L": wl.L, "Hq": wl.Hq, "Hkv": wl.Hkv, "head_dim": wl.d,
            "layers": f"1 full + {wl.n_sparse} sparse", "topk": wl.topk, "recent": wl.recent,
            "block": wl.block, "batch_per_gpu": 1, "parallelism": f"independent sequence per GPU x{world}",
            "l2": "inputs larger than L2 (Q alone is %.1f GB); no flush" % q_gb}


def data_recipe(wl) -> str:
    """One line naming the synthetic input recipe of a workload."""
    k = "K from a 64-component Gaussian mixture, std 0.3" if wl.k_dist == "gmm64" else "Q/K/V ~ N(0,1)"
    n = wl.needles
    if n and n[0] == "total":
        k += f", {n[1]} planted needle keys"
    elif n and n[0] == "per_kv_head":
        k += f", {n[1]} planted needle keys per KV head"
    elif n and n[0] == "chains":
        k += f", {n[1]} multi-hop needle chains of {n[2]} keys"
    if wl.kv_dtype == "e4m3":
        k += ", K/V as e4m3 codes + per-token fp32 scale"
    return f"synthetic (seeded {wl.seed}; {k})"


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------ multi-rank --

def rank_workload(wl, rank: int, world: int):
    """Each rank prefills its own independent sequence (a batch of `world`
    sequences, one per GPU): same shapes, its own seed."""
    return wl.scaled(seed=wl.seed + 101 * rank) if world > 1 else wl


def reduce_max(value: float, dist, device=None) -> float:
    """Max of a per-rank timing over all ranks (identity without a group)."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], device=device if device is not None else "cpu", dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(L: int, world: int, ms: float) -> float:
    """Whole-job tokens/s: every rank processed L tokens in at most `ms`."""
    return world * L / (ms / 1e3)


# ---------------------------------------------------------------- clocks --

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.lines = []
        self.dev = device_index

    def __enter__(self):
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            target = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
            self.proc = subprocess.Popen(["nvidia-smi", "-i", target, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.t.join(timeout=2)

    def summary(self) -> dict:
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------ oracle baseline --

class _Rows:
    """Rows [s, e) of a [L][H][d] array addressed by absolute row index, so the
    oracle can run one query block of a long sequence."""

    def __init__(self, data, s, L):
        self.data, self.s, self.shape = data, s, (L,) + data.shape[1:]

    def __getitem__(self, key):
        r, rest = key[0], tuple(key[1:])
        if r == slice(None):
            return _Rows(self.data[(slice(None),) + rest], self.s, self.shape[0])
        return self.data[(slice(r.start - self.s, r.stop - self.s),) + rest]


def _unit_flop(wl, b) -> float:
    d, G, B = wl.d, wl.G, wl.block
    e_b = min(wl.L, B * (b + 1))
    n_c = max(0, e_b - wl.recent)
    lst = min(n_c, wl.topk) + min(wl.recent, e_b)
    return G * (4.0 * d * B * e_b + 2.0 * d * B * n_c + wl.n_sparse * 4.0 * d * B * lst)


def oracle_units(wl, x, units):
    """Run the fp64 oracle over (block, KV head) units of the workload whose
    tensors live in `x` (torch, any device); returns elapsed seconds."""
    from oracle import hs2_oracle as orc
    from token_level_sparse_causal_b200 import inputs
    G = wl.G
    t = 0.0
    for b, g in units:
        s_b, e_b = b * wl.block, min(wl.L, (b + 1) * wl.block)
        hs = slice(g * G, (g + 1) * G)
        Qs = [_Rows(orc.decode_bf16(inputs.as_u16(q[s_b:e_b, hs])), s_b, wl.L) for q in x["q_layers"]]
        K = orc.decode_bf16(inputs.as_u16(x["k"][:e_b, g:g + 1]))
        V = orc.decode_bf16(inputs.as_u16(x["v"][:e_b, g:g + 1]))
        t0 = time.perf_counter()
        O, lse = orc.dense_attn(Qs[0], K, V, s_b, e_b)
        I = orc.importance(Qs[0], K, lse, b, 0, wl.block, wl.recent)
        idx, cnt = orc.select(I, wl.topk, wl.recent, e_b)
        for Ql in Qs[1:]:
            orc.sparse_attn(Ql, K, V, idx, cnt, b, 0, wl.block)
        t += time.perf_counter() - t0
    return t


def sample_units(wl, seconds_target: float, rng_seed: int = 0, per_unit_s: float | None = None):
    rng = np.random.default_rng(rng_seed)
    first = max(0, -(-(wl.topk + wl.recent) // wl.block))
    units = [(wl.nb - 1, 0)]
    est_rate = 2.0e10  # fp64 flop/s guess, refined by the caller
    budget = seconds_target * est_rate
    used = _unit_flop(wl, wl.nb - 1)
    while used < budget and len(units) < 64:
        b = int(rng.integers(first, wl.nb))
        g = int(rng.integers(0, wl.Hkv))
        units.append((b, g))
        used += _unit_flop(wl, b)
    return units


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_baseline(wl, x, seconds_target: float) -> dict:
    work = algorithmic_work(wl)
    total = work["fa_flop"] + work["imp_flop"] + wl.n_sparse * work["sparse_flop"]
    units = sample_units(wl, seconds_target)
    t = oracle_units(wl, x, units)
    sample = sum(_unit_flop(wl, b) for b, _ in units)
    t_full = t * total / sample
    return {"value": wl.L / t_full, "unit": "tok/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{len(units)} (query block, KV head) units of the {wl.name} workload "
                      f"({t:.1f} s of fp64 NumPy), extrapolated to the whole prefill by the exact FLOP ratio"}


# ------------------------------------------------------------- cuda arm --

def select_alone(hs2, torch, shape, q0, k, ks, out, dev, timed, nblk=256):
    """Kernel (3) by itself on the importance rows of the last `nblk` query
    blocks (the longest rows; at 128k a 1.07 GB strip of 2048 rows, larger
    than L2 and several waves of resident CTAs, so it streams from HBM):
    device time and the row bytes it must read."""
    nb = shape.L // shape.block
    b0 = max(0, nb - nblk)
    n_c = lambda b: max(0, min(shape.L, shape.block * (b + 1)) - shape.recent)
    stride = max(4, (n_c(nb - 1) + 3) // 4 * 4)
    imp = torch.empty((shape.Hkv, nb - b0, stride), dtype=torch.float32, device=dev)
    hs2.hs2_importance(shape, q0, k, ks, out["lse"], b0, nb, imp, stride)
    ms = timed(lambda: hs2.hs2_topk_select(shape, imp, stride, b0, nb, out["idx"], out["cnt"]), 5)
    moved = shape.Hkv * 4.0 * sum(n_c(b) for b in range(b0, nb) if n_c(b) > shape.topk)
    hs2.hs2_sync()
    del imp
    return {"blocks": [b0, nb], "ms": ms, "bytes": moved, "gbs": moved / (ms / 1e3) / 1e9,
            "frac_of_hbm": moved / (ms / 1e3) / 1e9 / measured_peaks()["hbm_gbs"]}


def importance_alone(hs2, torch, shape, q0, k, ks, out, dev, timed, nblk=256):
    """Kernel (2) by itself on the last `nblk` query blocks (the longest rows,
    one launch): device time and the importance FLOP it computes."""
    nb = shape.L // shape.block
    b0 = max(0, nb - nblk)
    G = shape.Hq // shape.Hkv
    n_c = lambda b: max(0, min(shape.L, shape.block * (b + 1)) - shape.recent)
    stride = max(4, (n_c(nb - 1) + 3) // 4 * 4)
    imp = torch.empty((shape.Hkv, nb - b0, stride), dtype=torch.float32, device=dev)
    ms = timed(lambda: hs2.hs2_importance(shape, q0, k, ks, out["lse"], b0, nb, imp, stride), 3)
    flop = 2.0 * shape.d * shape.block * G * shape.Hkv * sum(n_c(b) for b in range(b0, nb))
    hs2.hs2_sync()
    del imp
    return {"blocks": [b0, nb], "ms": ms, "flop": flop, "tflops": flop / (ms / 1e3) / 1e12,
            "frac_of_sustained_bf16": flop / (ms / 1e3) / 1e12 / measured_peaks()["bf16_tflops_sustained"]}


def needle_recall(needles, idx, cnt, block: int = 64):
    """Share of planted needle keys that appear in the index list of their
    target query's block and KV head (a diagnostic of the selection on the
    workload's retrieval structure, not a parity check)."""
    if not needles:
        return None
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    hit = 0
    for n in needles:
        b = n["t"] // block
        hit += int(n["p"] in set(idx_h[n["g"], b, :cnt_h[n["g"], b]].tolist()))
    return hit / len(needles)


DECODE_BATCHES = (1, 128)   # decode queries per call: one token, and a batch at random positions


def decode_rows(hs2, torch, shape, x, k, v, ks, vs, out, dev, timed):
    """Decode-step sparse attention on the prefill's lists: device time per
    call and the listed K/V rows the queries must read (plus Q and O)."""
    res = {}
    rng = np.random.default_rng(5)
    peaks = measured_peaks()
    G = shape.Hq // shape.Hkv
    for n in DECODE_BATCHES:
        pos_h = np.array([shape.L - 1] if n == 1 else rng.integers(0, shape.L, n), dtype=np.int64)
        pos = torch.as_tensor(pos_h, dtype=torch.int32, device=dev)
        q = x["q_layers"][1][pos.long()].contiguous()
        sh = hs2.Hs2Shape(**{f: getattr(shape, f) for f, _ in hs2.Hs2Shape._fields_})
        sh.q_tok_stride, sh.q_head_stride = q.stride(0), q.stride(1)
        o = torch.empty_like(q)
        nbytes = hs2.sparse_decode_workspace_bytes(sh, n)
        ws = torch.empty(nbytes // 4 + 4, dtype=torch.float32, device=dev) if nbytes else None
        call = lambda: hs2.hs2_sparse_decode(sh, q, pos, k, v, ks, vs, out["idx"], out["cnt"], o, ws)
        us_eager = 1e3 * timed(call, 50)
        # the same calls replayed from a CUDA graph: device time without the
        # host's per-call cost
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for _ in range(20):
                call()
        us = 1e3 * timed(graph.replay, 5) / 20
        del graph
        b = pos.long() // shape.block
        lists = out["idx"][:, b, :]                       # [Hkv][n][list]
        cnts = out["cnt"][:, b]                           # [Hkv][n]
        col = torch.arange(lists.shape[-1], device=dev)
        vis = (col[None, None, :] < cnts[..., None]) & (lists >= 0) & (lists <= pos[None, :, None])
        rows = int(vis.sum())
        row_bytes = 2 * shape.d * k.element_size() + (8 if k.element_size() == 1 else 0)  # K + V (+ two scales)
        moved = rows * row_bytes + 2 * q.numel() * 2
        res[f"n{n}"] = {"us_per_call": us, "us_per_call_eager": us_eager, "queries": n, "kv_rows_read": rows, "bytes": moved,
                        "gbs": moved / (us / 1e6) / 1e9, "frac_of_hbm": moved / (us / 1e6) / 1e9 / peaks["hbm_gbs"],
                        "splits_workspace_bytes": nbytes}
        del o, ws
    return res


def run_cuda(args, wl, rank, world, dist):
    import torch
    from token_level_sparse_causal_b200 import build, hs2, inputs

    build.build()
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    my = rank_workload(wl, rank, world)
    x = inputs.make_inputs(my, device=dev, with_needles=bool(my.needles))
    q0, k, v = x["q_layers"][0], x["k"], x["v"]
    ks, vs = x.get("k_scale"), x.get("v_scale")  # e4m3 cache: codes + per-token scales
    fp8_cache = k.dtype == torch.uint8
    shape = hs2.make_shape(q0, k, wl.topk, wl.recent, kv_dtype=hs2.HS2_KV_E4M3 if fp8_cache else hs2.HS2_KV_BF16)
    out = hs2.alloc_outputs(shape, q0)
    o_sp = [torch.empty_like(q) for q in x["q_layers"][1:]]
    stream = torch.cuda.current_stream()

    def step():
        hs2.hs2_full_attn_select(shape, q0, k, v, ks, vs, out["o"], out["lse"], out["idx"], out["cnt"],
                                 out["workspace"], stream)
        for ql, ol in zip(x["q_layers"][1:], o_sp):
            hs2.hs2_sparse_attn(shape, ql, k, v, ks, vs, out["idx"], out["cnt"], ol, stream)

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    hs2.hs2_sync(stream)
    torch.cuda.synchronize()
    barrier()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    n0 = hs2.hs2_launch_count()
    with ClockSampler(dev.index) as clk:
        barrier()
        torch.cuda.synchronize()
        ev[0].record(stream)
        for i in range(args.steps):
            step()
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
        barrier()
    launches = hs2.hs2_launch_count() - n0
    hs2.hs2_sync(stream)
    per = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    total_ms = reduce_max(ev[0].elapsed_time(ev[-1]), dist, dev)
    ms = total_ms / args.steps

    # ---- per-stage device times (same stream, CUDA events), full kernel (1)
    def timed(fn, n):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        fn()
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    n_stage = max(2, min(args.steps, 5))
    # FP8 KV write (the step producing an e4m3 cache) on this workload's K
    fp8 = None
    if k.dtype == torch.bfloat16:
        codes = torch.empty(k.shape, dtype=torch.uint8, device=dev)
        kscale = torch.empty(k.shape[:2], dtype=torch.float32, device=dev)
        qk_ms = timed(lambda: hs2.hs2_quantize_kv(k, codes, kscale, stream), n_stage)
        moved = k.numel() * 2 + codes.numel() + kscale.numel() * 4
        fp8 = {"ms": qk_ms, "gbs": moved / (qk_ms / 1e3) / 1e9, "frac_of_hbm": moved / (qk_ms / 1e3) / 1e9 /
               measured_peaks()["hbm_gbs"], "bytes": moved}
        del codes, kscale
    # kernel (1) as the full layer runs it (an e4m3 cache: after the layer's
    # one f16 conversion, which is included)
    fa_ws = None
    if fp8_cache:
        fa_ws = torch.empty(hs2.attn_fwd_workspace_bytes(shape) // 4 + 4, dtype=torch.float32, device=dev)
    fa_ms = timed(lambda: hs2.hs2_attn_fwd_ws(shape, q0, k, v, ks, vs, out["o"], out["lse"], fa_ws, stream), n_stage)
    del fa_ws
    sp_ms = timed(lambda: hs2.hs2_sparse_attn(shape, x["q_layers"][1], k, v, ks, vs, out["idx"], out["cnt"],
                                              o_sp[0], stream), n_stage) if o_sp else 0.0
    fs_ms = timed(lambda: hs2.hs2_full_attn_select(shape, q0, k, v, ks, vs, out["o"], out["lse"], out["idx"],
                                                   out["cnt"], out["workspace"], stream), n_stage)
    recall_tok = needle_recall(x.get("needles"), out["idx"], out["cnt"])
    blk_ms = timed(lambda: hs2.hs2_full_attn_select_blocks(shape, q0, k, v, None, None, out["o"], out["lse"],
                                                           out["idx"], out["cnt"], out["workspace"], stream),
                   n_stage) if wl.topk % 64 == 0 and k.dtype == torch.bfloat16 else None
    recall_blk = needle_recall(x.get("needles"), out["idx"], out["cnt"]) if blk_ms is not None else None
    swa_ms = timed(lambda: hs2.hs2_swa_attn(shape, q0, k, v, SWA_WINDOW, out["o"], None, stream),
                   n_stage) if k.dtype == torch.bfloat16 else None
    decode = decode_rows(hs2, torch, shape, x, k, v, ks, vs, out, dev, timed) if o_sp else None
    select = select_alone(hs2, torch, shape, q0, k, ks, out, dev, timed)
    hs2.hs2_sync(stream)

    # ---- end to end from pinned host buffers: every step copies its inputs in
    # and every output back, through the same C ABI calls, with the copies
    # overlapped with compute on separate streams (PrefillPipeline)
    e2e = None
    if not args.no_e2e and not fp8_cache:  # the end-to-end runner takes a bf16 cache
        from token_level_sparse_causal_b200.pipeline import PrefillPipeline
        h_q = [t.cpu().pin_memory() for t in x["q_layers"]]
        h_k, h_v = k.cpu().pin_memory(), v.cpu().pin_memory()
        h_o = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in x["q_layers"]]
        h_idx = torch.empty(out["idx"].shape, dtype=torch.int32, pin_memory=True)
        h_cnt = torch.empty(out["cnt"].shape, dtype=torch.int32, pin_memory=True)
        del o_sp, out
        torch.cuda.empty_cache()
        pipe = PrefillPipeline(shape, wl.n_sparse, dev)
        n_e2e = max(12, args.steps)  # the pipeline's fill and drain are paid once per run
        for _ in range(2):  # warm-up: both buffer sets once
            pipe.submit(h_q, h_k, h_v, h_o, h_idx, h_cnt)
        pipe.synchronize()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(pipe.s_in)
        for _ in range(n_e2e):
            pipe.submit(h_q, h_k, h_v, h_o, h_idx, h_cnt)
        b.record(pipe.s_out)
        pipe.synchronize()
        e_ms = reduce_max(a.elapsed_time(b) / n_e2e, dist, dev)
        h2d = sum(t.numel() * t.element_size() for t in h_q + [h_k, h_v])
        d2h = sum(t.numel() * t.element_size() for t in h_o + [h_idx, h_cnt])
        e2e = {"value": job_throughput(wl.L, world, e_ms), "unit": "tok/s", "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "ms_per_step": e_ms, "steps": n_e2e,
               "overlap": "double-buffered; copy-in, compute and copy-out on separate streams"}
        del h_q, h_k, h_v, h_o, h_idx, h_cnt, pipe

    work = algorithmic_work(wl)
    peaks = measured_peaks()
    fa_tflops = work["fa_flop"] / (fa_ms / 1e3) / 1e12
    peak = peaks["bf16_tflops_sustained"]
    res = {
        "metric": METRIC, "value": job_throughput(wl.L, world, ms), "unit": "tok/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "p50_ms": float(np.percentile(per, 50)), "p99_ms": float(np.percentile(per, 99)),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 Q, e4m3 K/V (f16 MMA)" if fp8_cache else "bf16",
        "data": data_recipe(wl),
        "config": arm_config(wl, world),
        "roofline": {"kernel": "fa_fwd (kernel 1, dense causal attention + LSE)", "bound": "tensor",
                     "achieved": fa_tflops, "peak": peak, "unit": "TFLOP/s", "frac": fa_tflops / peak,
                     "traffic": recorded_traffic(wl.name) if not fp8_cache else None, "traffic_unit": "bytes per launch (dram read + write, ncu)",
                     "peak_note": f"{peaks['source']} sustained bf16 (the kernel runs ~{fa_ms:.0f} ms per launch)"},
        "stages_ms": {"fa_fwd": fa_ms, "importance+select": fs_ms - fa_ms, "sparse_attn_per_layer": sp_ms,
                      "full_attn_select": fs_ms},
        "stage_roofline": {
            "fa_fwd_tflops": fa_tflops,
            "importance_select_tflops": work["imp_flop"] / ((fs_ms - fa_ms) / 1e3) / 1e12 if fs_ms > fa_ms else None,
            "select_alone": select,
            "sparse_tflops": work["sparse_flop"] / (sp_ms / 1e3) / 1e12 if sp_ms else None,
            "sparse_gather_gbs": (work["gather_bytes"] + work["sparse_qo_bytes"]) / (sp_ms / 1e3) / 1e9 if sp_ms else None,
            "path_roofline_ms": 1e3 * ((work["fa_flop"] + work["imp_flop"] + wl.n_sparse * work["sparse_flop"]) /
                                       (peaks["bf16_tflops_sustained"] * 1e12) +
                                       2 * work["select_bytes"] / (peaks["hbm_gbs"] * 1e9)),
        },
        "next_rows": {"fp8_kv_write_K": fp8,
                      "block_level_full_attn_select_ms": blk_ms,
                      "token_level_full_attn_select_ms": fs_ms,
                      "needle_recall": None if recall_tok is None else {
                          "token_level": recall_tok, "block_level": recall_blk,
                          "note": "share of planted needle keys listed for their target block (diagnostic)"},
                      "swa_attn": None if swa_ms is None else {
                          "window": SWA_WINDOW, "ms": swa_ms,
                          "tflops": work["swa_flop"] / (swa_ms / 1e3) / 1e12,
                          "gbs": work["swa_bytes"] / (swa_ms / 1e3) / 1e9,
                          "roofline_ms": 1e3 * max(work["swa_flop"] / (peaks["bf16_tflops"] * 1e12),
                                                   work["swa_bytes"] / (peaks["hbm_gbs"] * 1e9)),
                          "frac_of_roofline": 1e3 * max(work["swa_flop"] / (peaks["bf16_tflops"] * 1e12),
                                                        work["swa_bytes"] / (peaks["hbm_gbs"] * 1e9)) / swa_ms,
                      },
                      "sparse_decode": decode},
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
        "e2e": e2e,
    }
    res["stage_roofline"]["path_frac"] = res["stage_roofline"]["path_roofline_ms"] / ms
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(wl, x, args.cpu_seconds)
    return res


def run_reference(args, wl, rank, world):
    """The fp64 oracle on the host cores, each step a bounded sample."""
    import torch
    from token_level_sparse_causal_b200 import inputs
    if rank != 0:
        return None
    x = inputs.make_inputs(wl, device="cuda" if torch.cuda.is_available() else "cpu",
                           with_needles=bool(wl.needles))
    work = algorithmic_work(wl)
    total = work["fa_flop"] + work["imp_flop"] + wl.n_sparse * work["sparse_flop"]
    vals = []
    for i in range(args.warmup + args.steps):
        units = sample_units(wl, args.cpu_seconds / 3, rng_seed=i)
        t = oracle_units(wl, x, units)
        if i >= args.warmup:
            vals.append(wl.L / (t * total / sum(_unit_flop(wl, b) for b, _ in units)))
    v = float(np.median(vals))
    return {"metric": METRIC, "value": v, "unit": "tok/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * wl.L / v, "extrapolated": True,
            "ms_per_step_note": "whole-prefill time extrapolated from the timed sample by the exact FLOP ratio; "
                                "the run itself takes about (warmup + steps) x cpu_seconds / 3",
            "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": data_recipe(wl), "impl": "reference",
            "config": arm_config(wl, world),
            "cpu_baseline": {"value": v, "unit": "tok/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": "per step: seeded (query block, KV head) units, extrapolated by FLOP ratio"},
            "e2e": {"value": v, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_stage(args, wl):
    """One stage alone on a reduced-footprint copy of the workload (same L and
    input recipe, the heads given by --heads, no sparse layers) -- the case
    an ncu capture of that stage's kernel runs on.  Kernel (1) for the LSE,
    then kernel (1) again (fa), kernel (2) (importance) or kernel (3)
    (select) alone on the strip of the longest rows, or one sparse layer
    (sparse) on the full layer's lists."""
    import torch
    from token_level_sparse_causal_b200 import build, hs2, inputs

    build.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    hq, hkv = (int(t) for t in args.heads.split("/")) if args.heads else (wl.Hq, wl.Hkv)
    L = args.seq or wl.L
    my = wl.scaled(name=f"{wl.name}_stage_h{hq}x{hkv}" + (f"_L{L}" if args.seq else ""), Hq=hq, Hkv=hkv, n_sparse=0,
                   L=L)
    x = inputs.make_inputs(my, device=dev, with_needles=bool(my.needles))
    q0, k, v = x["q_layers"][0], x["k"], x["v"]
    ks, vs = x.get("k_scale"), x.get("v_scale")
    fp8_cache = k.dtype == torch.uint8
    shape = hs2.make_shape(q0, k, my.topk, my.recent, kv_dtype=hs2.HS2_KV_E4M3 if fp8_cache else hs2.HS2_KV_BF16)
    out = hs2.alloc_outputs(shape, q0)
    stream = torch.cuda.current_stream()
    hs2.hs2_attn_fwd(shape, q0, k, v, ks, vs, out["o"], out["lse"], stream)

    def timed(fn, n):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        fn()
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    work = algorithmic_work(my)
    peaks = measured_peaks()
    if args.stage == "importance":
        res = importance_alone(hs2, torch, shape, q0, k, ks, out, dev, timed)
    elif args.stage == "fa":
        # kernel (1) alone, as the full layer runs it
        fa_ws = None
        if fp8_cache:
            fa_ws = torch.empty(hs2.attn_fwd_workspace_bytes(shape) // 4 + 4, dtype=torch.float32, device=dev)
        ms = timed(lambda: hs2.hs2_attn_fwd_ws(shape, q0, k, v, ks, vs, out["o"], out["lse"], fa_ws, stream), 3)
        tf = work["fa_flop"] / (ms / 1e3) / 1e12
        res = {"ms": ms, "flop": work["fa_flop"], "tflops": tf, "frac_of_sustained_bf16": tf / peaks["bf16_tflops_sustained"],
               "algorithmic_bytes": 2 * my.L * hq * my.d * 2 + 2 * my.L * hkv * my.d * k.element_size() + my.L * hq * 4}
    elif args.stage == "sparse":
        # kernel (4) alone: one sparse layer on the full layer's lists
        hs2.hs2_full_attn_select(shape, q0, k, v, ks, vs, out["o"], out["lse"], out["idx"], out["cnt"],
                                 out["workspace"], stream)
        q1 = torch.randn(q0.shape, device=dev, generator=torch.Generator(device=dev).manual_seed(my.seed * 1000 + 1)
                         ).to(torch.bfloat16)
        o1 = torch.empty_like(q1)
        ms = timed(lambda: hs2.hs2_sparse_attn(shape, q1, k, v, ks, vs, out["idx"], out["cnt"], o1, stream), 3)
        tf = work["sparse_flop"] / (ms / 1e3) / 1e12
        moved = work["gather_bytes"] + work["sparse_qo_bytes"]
        res = {"ms": ms, "flop": work["sparse_flop"], "tflops": tf,
               "frac_of_sustained_bf16": tf / peaks["bf16_tflops_sustained"], "gather_bytes": work["gather_bytes"],
               "qo_bytes": work["sparse_qo_bytes"], "gbs": moved / (ms / 1e3) / 1e9,
               "frac_of_hbm": moved / (ms / 1e3) / 1e9 / peaks["hbm_gbs"]}
    else:
        res = select_alone(hs2, torch, shape, q0, k, ks, out, dev, timed)
    hs2.hs2_sync(stream)
    return {"stage": f"{args.stage}_alone", "workload": my.name, "L": my.L, "Hq": hq, "Hkv": hkv, **res}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    # defaults: 10 warm-up and 20 timed steps, median and P99 reported (the MiMo-V3
    # prefill blog's measurement procedure, section 3.3)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--workload", default="c3", help="c1..c5 (default c3, the 128k workload)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="oracle sample size for cpu_baseline")
    ap.add_argument("--stage", choices=["select", "importance", "fa", "sparse"],
                    help="time one stage alone (1 GPU) and print its line")
    ap.add_argument("--heads", help="with --stage: query/KV heads of the reduced copy, e.g. 16/8")
    ap.add_argument("--seq", type=int, help="with --stage: sequence length of the reduced copy (default: the workload's)")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "cuda":
        ap.error("--warmup must be >= 3")

    from token_level_sparse_causal_b200 import inputs
    wl = inputs.WORKLOADS[args.workload]
    if args.stage:
        print(json.dumps(run_stage(args, wl)), flush=True)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch
        import torch.distributed as tdist
        if args.impl == "cuda":
            torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
            tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
            dist = tdist
    try:
        if args.impl == "reference":
            res = run_reference(args, wl, rank, world)
        else:
            res = run_cuda(args, wl, rank, world, dist)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
