"""Seeded synthetic inputs for token-level sparse causal attention.

This module only *draws* inputs: Q for the full-attention layer and for each
sparse layer, the shared K/V cache, planted "needle" keys and (for the FP8
cache) the e4m3 codes with their per-token scales.  It holds none of the
method's arithmetic (no scores, softmax, importance or selection), so both the
CUDA path and the fp64 oracle may consume what it produces.

Workloads (HySparse2 news summary, "token-level selection" paragraph: 1024
global tokens + 128 most recent, reused by the sparse layers; the sizes below
are the five prefill workloads this library is measured on):

  name     L        Hq/Hkv  sparse layers  values / structure
  c1       2048     4/1     1              N(0,1), 16 needles
  c2       32768    32/8    3              N(0,1), 256 needles per KV head
  c3       131072   64/8    3              K from a 64-component Gaussian mixture
  c4       262144   64/8    3              N(0,1), 8 chains x 4 multi-hop needles
  c5       1048576  32/4    1              N(0,1), 1024 needles per KV head, FP8 K/V

All tensors are batch 1, token-major: Q [L][Hq][128], K/V [L][Hkv][128].
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

HEAD_DIM = 128
E4M3_MAX = 448.0


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    L: int
    Hq: int
    Hkv: int
    n_sparse: int
    seed: int
    k_dist: str = "normal"          # "normal" | "gmm64"
    needles: tuple = ()             # ("total", n) | ("per_kv_head", n) | ("chains", n_chains, hops)
    kv_dtype: str = "bf16"          # "bf16" | "e4m3"
    block: int = 64
    topk: int = 1024
    recent: int = 128
    d: int = HEAD_DIM

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def nb(self) -> int:
        return (self.L + self.block - 1) // self.block

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "c1": Workload("c1_L2048_h4x1", 2048, 4, 1, 1, seed=0, needles=("total", 16)),
    "c2": Workload("c2_L32768_h32x8", 32768, 32, 8, 3, seed=1, needles=("per_kv_head", 256)),
    "c3": Workload("c3_L131072_h64x8_gmm", 131072, 64, 8, 3, seed=2, k_dist="gmm64"),
    "c4": Workload("c4_L262144_h64x8_chains", 262144, 64, 8, 3, seed=3, needles=("chains", 8, 4)),
    "c5": Workload("c5_L1048576_h32x4_fp8", 1048576, 32, 4, 1, seed=4,
                   needles=("per_kv_head", 1024), kv_dtype="e4m3"),
}


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _randn(shape, gen, device) -> torch.Tensor:
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32)


def _unit(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm()


def _needle_target(rng: np.random.Generator, wl: Workload, heads) -> tuple:
    """Pick a query (t, h) whose block has earlier candidates, and a key slot p
    strictly before the block's recent window."""
    B, w = wl.block, wl.recent
    t_min = min(wl.L - 1, (w // B) * B)   # first query whose block has a non-empty candidate range
    t = int(rng.integers(t_min, wl.L))
    e_b = min(wl.L, (t // B + 1) * B)
    hi = max(1, e_b - w)
    p = int(rng.integers(0, hi))
    h = int(rng.choice(heads))
    return t, h, p


def plant_needles(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, wl: Workload) -> list:
    """Overwrite some K rows with 4 * Q_target / ||Q_target|| (or, for multi-hop
    chains, with 4 * V_prev / ||V_prev||).  Positions come from
    numpy.default_rng(seed); the planted (t, h, p) list is returned."""
    if not wl.needles:
        return []
    rng = np.random.default_rng(wl.seed)
    kind = wl.needles[0]
    out = []
    G = wl.G
    if kind in ("total", "per_kv_head"):
        groups = [list(range(wl.Hq))] if kind == "total" else \
                 [list(range(g * G, (g + 1) * G)) for g in range(wl.Hkv)]
        n = wl.needles[1]
        for heads in groups:
            for _ in range(n):
                t, h, p = _needle_target(rng, wl, heads)
                g = h // G
                k[p, g] = (4.0 * _unit(q[t, h].float())).to(k.dtype)
                out.append({"t": t, "h": h, "p": p, "g": g})
    elif kind == "chains":
        n_chains, hops = wl.needles[1], wl.needles[2]
        for c in range(n_chains):
            t, h, _ = _needle_target(rng, wl, list(range(wl.Hq)))
            g = h // G
            e_b = min(wl.L, (t // wl.block + 1) * wl.block)
            hi = max(hops, e_b - wl.recent)
            ps = np.sort(rng.choice(hi, size=hops, replace=False))
            prev = q[t, h].float()
            for m, p in enumerate(ps):
                p = int(p)
                k[p, g] = (4.0 * _unit(prev)).to(k.dtype)
                out.append({"t": t, "h": h, "p": p, "g": g, "chain": c, "hop": m})
                prev = v[p, g].float()
    else:
        raise ValueError(f"unknown needle kind {kind!r}")
    return out


def quantize_e4m3(x: torch.Tensor) -> tuple:
    """Encode a [L][Hkv][d] tensor as OCP e4m3fn codes with one fp32 scale per
    (token, head): scale = amax(row) / 448, code = RNE(x / scale), clamped to
    +-448 so nothing overflows to NaN.  Returns (uint8 codes, fp32 scales)."""
    xf = x.float()
    amax = xf.abs().amax(dim=-1)
    # tensor / tensor: an IEEE fp32 division (torch turns division by a Python
    # scalar into a multiply by its reciprocal, which can differ in the last bit)
    scale = torch.where(amax > 0, amax / torch.full_like(amax, E4M3_MAX), torch.ones_like(amax))
    y = (xf / scale[..., None]).clamp_(-E4M3_MAX, E4M3_MAX)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), scale.contiguous()


def make_inputs(wl: Workload, device="cpu", with_needles: bool = True) -> dict:
    """Draw one workload's tensors on `device`.

    Returns a dict with
      q_layers: list of 1 + n_sparse bf16 tensors [L][Hq][d]
      k, v:     bf16 [L][Hkv][d]  (kv_dtype "bf16")
                uint8 e4m3 codes [L][Hkv][d] (kv_dtype "e4m3")
      k_scale, v_scale: fp32 [L][Hkv] or None
      needles:  list of planted (t, h, p, g) records
    Sparse layer l (1-based) draws its Q from seed * 1000 + l.
    """
    dev = torch.device(device)
    L, Hq, Hkv, d = wl.L, wl.Hq, wl.Hkv, wl.d
    gen = _gen(dev, wl.seed)
    q0 = _randn((L, Hq, d), gen, dev).to(torch.bfloat16)
    if wl.k_dist == "normal":
        k = _randn((L, Hkv, d), gen, dev).to(torch.bfloat16)
    elif wl.k_dist == "gmm64":
        centres = _randn((Hkv, 64, d), gen, dev)
        comp = torch.randint(0, 64, (L, Hkv), generator=gen, device=dev)
        k = torch.empty((L, Hkv, d), device=dev, dtype=torch.bfloat16)
        chunk = 1 << 15
        for s in range(0, L, chunk):
            e = min(L, s + chunk)
            c = centres[torch.arange(Hkv, device=dev)[None, :], comp[s:e]]
            k[s:e] = (c + 0.3 * _randn((e - s, Hkv, d), gen, dev)).to(torch.bfloat16)
        del centres, comp
    else:
        raise ValueError(f"unknown k_dist {wl.k_dist!r}")
    v = _randn((L, Hkv, d), gen, dev).to(torch.bfloat16)
    needles = plant_needles(q0, k, v, wl) if with_needles else []
    q_layers = [q0]
    for layer in range(1, wl.n_sparse + 1):
        gl = _gen(dev, wl.seed * 1000 + layer)
        q_layers.append(_randn((L, Hq, d), gl, dev).to(torch.bfloat16))
    out = {"q_layers": q_layers, "needles": needles, "k_scale": None, "v_scale": None}
    if wl.kv_dtype == "e4m3":
        out["k"], out["k_scale"] = quantize_e4m3(k)
        out["v"], out["v_scale"] = quantize_e4m3(v)
        del k, v
    else:
        out["k"], out["v"] = k, v
    return out


def as_u16(t: torch.Tensor) -> np.ndarray:
    """Raw bf16 bit patterns of a tensor as a numpy uint16 array (host copy)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def as_u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.uint8).cpu().numpy()
