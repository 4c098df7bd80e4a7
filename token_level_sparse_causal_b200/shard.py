"""Splitting one sequence's prefill over GPUs by KV head.

The lists are per (query block, KV head) and every KV head's group of G query
heads reads only its own K/V (HySparse2 architecture summary, KV-sharing
paragraph: the full layer's selection and KV cache serve the sparse layers
of the same group).  So the full layer, the selection and every sparse layer
of a contiguous range of KV heads and their query heads need nothing from the
other ranks: a rank passes head-strided views of the same Q/K/V to the C ABI
and gets its heads' O, LSE and lists.  The data path has no collective; a
caller that wants the whole O on one GPU gathers it afterwards.

Only argument marshalling lives here: views, the rank's hs2_shape, and the
e4m3 scale columns, which the ABI takes as a contiguous [L][Hkv] array and
which are therefore copied per rank.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import hs2


@dataclass(frozen=True)
class HeadShard:
    g0: int   # first KV head of the rank
    g1: int   # one past its last KV head
    h0: int   # first query head (g0 * G)
    h1: int   # one past the last query head


def kv_head_range(Hq: int, Hkv: int, rank: int, world: int) -> HeadShard:
    """Contiguous KV heads of `rank` out of `world`; the first Hkv % world
    ranks take one head more.  Every rank gets at least one KV head."""
    if not 0 <= rank < world or world > Hkv or Hq % Hkv:
        raise ValueError(f"cannot split {Hkv} KV heads over {world} ranks (rank {rank})")
    G = Hq // Hkv
    base, extra = divmod(Hkv, world)
    g0 = rank * base + min(rank, extra)
    g1 = g0 + base + (1 if rank < extra else 0)
    return HeadShard(g0, g1, g0 * G, g1 * G)


def shard_inputs(sh: HeadShard, q_layers, k, v, k_scale=None, v_scale=None) -> dict:
    """Head-strided views of every layer's Q and of K/V for the rank's heads;
    an e4m3 cache's per-token scales are copied to contiguous [L][g1 - g0]."""
    out = {"q_layers": [q[:, sh.h0:sh.h1] for q in q_layers], "k": k[:, sh.g0:sh.g1], "v": v[:, sh.g0:sh.g1],
           "k_scale": None, "v_scale": None}
    if k_scale is not None:
        out["k_scale"] = k_scale[:, sh.g0:sh.g1].contiguous()
        out["v_scale"] = v_scale[:, sh.g0:sh.g1].contiguous()
    return out


def prefill_shard(sh: HeadShard, q_layers, k, v, k_scale, v_scale, o_layers, topk: int = 1024, recent: int = 128,
                  stream=None) -> dict:
    """The rank's part of one prefill through the C ABI: the full layer with
    selection, then every sparse layer, for KV heads [g0, g1).  o_layers are
    whole-size [L][Hq][d] outputs; the rank writes only its heads' columns.
    Returns the rank's lse [h1 - h0][L], idx [g1 - g0][nb][topk + recent] and
    cnt [g1 - g0][nb]."""
    x = shard_inputs(sh, q_layers, k, v, k_scale, v_scale)
    q0 = x["q_layers"][0]
    kvd = hs2.HS2_KV_E4M3 if k.dtype == torch.uint8 else hs2.HS2_KV_BF16
    shape = hs2.make_shape(q0, x["k"], topk, recent, kv_dtype=kvd)
    out = hs2.alloc_outputs(shape, q0)
    o_views = [o[:, sh.h0:sh.h1] for o in o_layers]
    hs2.hs2_full_attn_select(shape, q0, x["k"], x["v"], x["k_scale"], x["v_scale"], o_views[0], out["lse"],
                             out["idx"], out["cnt"], out["workspace"], stream)
    for ql, ol in zip(x["q_layers"][1:], o_views[1:]):
        hs2.hs2_sparse_attn(shape, ql, x["k"], x["v"], x["k_scale"], x["v_scale"], out["idx"], out["cnt"], ol,
                            stream)
    return {"shape": shape, "lse": out["lse"], "idx": out["idx"], "cnt": out["cnt"]}


def gather_heads(dist, part: torch.Tensor, sizes, head_dim: int = 1) -> torch.Tensor:
    """All-gathers every rank's head slice (`part`, that rank's heads along
    `head_dim`; sizes[r] = rank r's head count) and concatenates them in head
    order.  Uneven shards are padded to the largest for the collective."""
    world = dist.get_world_size()
    assert len(sizes) == world and part.shape[head_dim] == sizes[dist.get_rank()]
    width = max(sizes)
    pad = list(part.shape)
    pad[head_dim] = width
    buf = part.new_zeros(pad)
    buf.narrow(head_dim, 0, part.shape[head_dim]).copy_(part)
    got = [torch.empty_like(buf) for _ in range(world)]
    dist.all_gather(got, buf)
    return torch.cat([g.narrow(head_dim, 0, n) for g, n in zip(got, sizes)], dim=head_dim)
