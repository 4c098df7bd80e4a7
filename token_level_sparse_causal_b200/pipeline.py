"""End-to-end prefill from pinned host memory with the copies overlapped.

Each step takes one sequence's inputs from pinned host buffers (the full
layer's Q, every sparse layer's Q, the shared K and V cache) and returns every
layer's output and the index lists to pinned host buffers.  Three CUDA streams
carry the work:

  copy-in   host -> device of a step's inputs (K, V and the full layer's Q
            first, then the sparse layers' Q in layer order);
  compute   hs2_full_attn_select, then hs2_sparse_attn per layer, each
            starting as soon as its own inputs have landed;
  copy-out  device -> host of each layer's output as soon as it is written.

Device buffers are double-buffered, so step i+1's inputs load while step i
computes and step i-1's outputs drain.  Every step still moves all of its own
bytes; only their timing overlaps.  The library calls are the C ABI's, through
the ctypes binding; this module only orders them on streams.
"""
from __future__ import annotations

import torch

from . import hs2


class PrefillPipeline:
    """Double-buffered prefill over three streams (see the module docstring).

    shape: the hs2_shape of one sequence; n_sparse: sparse layers per step.
    Q tensors are [L][Hq][d] bf16, K / V [L][Hkv][d] bf16 (contiguous)."""

    def __init__(self, shape: hs2.Hs2Shape, n_sparse: int, device: torch.device):
        self.shape, self.n_sparse, self.dev = shape, n_sparse, device
        L, Hq, Hkv, d = shape.L, shape.Hq, shape.Hkv, shape.d
        nb = L // shape.block
        lst = shape.topk + shape.recent
        bf = torch.bfloat16

        def buffers():
            return {
                "q": [torch.empty((L, Hq, d), dtype=bf, device=device) for _ in range(1 + n_sparse)],
                "k": torch.empty((L, Hkv, d), dtype=bf, device=device),
                "v": torch.empty((L, Hkv, d), dtype=bf, device=device),
                "o": [torch.empty((L, Hq, d), dtype=bf, device=device) for _ in range(1 + n_sparse)],
                "idx": torch.empty((Hkv, nb, lst), dtype=torch.int32, device=device),
                "cnt": torch.empty((Hkv, nb), dtype=torch.int32, device=device),
            }

        self.buf = [buffers(), buffers()]
        self.lse = torch.empty((Hq, L), dtype=torch.float32, device=device)
        self.ws = torch.empty(hs2.workspace_bytes(shape) // 4 + 4, dtype=torch.float32, device=device)
        self.s_in, self.s_comp, self.s_out = torch.cuda.Stream(device), torch.cuda.Stream(device), torch.cuda.Stream(device)
        ev = lambda: torch.cuda.Event()
        self.in_ready = [[ev() for _ in range(1 + n_sparse)] for _ in range(2)]  # per buffer, per layer
        self.out_ready = [[ev() for _ in range(1 + n_sparse)] for _ in range(2)]
        self.in_free = [ev(), ev()]
        self.out_free = [ev(), ev()]
        self.step = 0

    def submit(self, h_q, h_k, h_v, h_o, h_idx, h_cnt) -> None:
        """Queue one step.  h_q: 1 + n_sparse pinned host Q tensors; h_k, h_v
        pinned K / V; h_o: 1 + n_sparse pinned host outputs; h_idx / h_cnt:
        pinned host index lists and counts.  Returns at once."""
        b = self.step & 1
        B = self.buf[b]
        first_use = self.step < 2
        # ---- inputs (the buffer's previous step has finished computing)
        with torch.cuda.stream(self.s_in):
            if not first_use:
                self.s_in.wait_event(self.in_free[b])
            B["k"].copy_(h_k, non_blocking=True)
            B["v"].copy_(h_v, non_blocking=True)
            for layer in range(1 + self.n_sparse):
                B["q"][layer].copy_(h_q[layer], non_blocking=True)
                self.in_ready[b][layer].record(self.s_in)
        # ---- compute (the buffer's previous outputs have been copied out)
        with torch.cuda.stream(self.s_comp):
            if not first_use:
                self.s_comp.wait_event(self.out_free[b])
            self.s_comp.wait_event(self.in_ready[b][0])
            hs2.hs2_full_attn_select(self.shape, B["q"][0], B["k"], B["v"], None, None, B["o"][0], self.lse,
                                     B["idx"], B["cnt"], self.ws, self.s_comp)
            self.out_ready[b][0].record(self.s_comp)
            for layer in range(1, 1 + self.n_sparse):
                self.s_comp.wait_event(self.in_ready[b][layer])
                hs2.hs2_sparse_attn(self.shape, B["q"][layer], B["k"], B["v"], None, None, B["idx"], B["cnt"],
                                    B["o"][layer], self.s_comp)
                self.out_ready[b][layer].record(self.s_comp)
            self.in_free[b].record(self.s_comp)
        # ---- outputs, each as soon as it is written
        with torch.cuda.stream(self.s_out):
            self.s_out.wait_event(self.out_ready[b][0])
            h_o[0].copy_(B["o"][0], non_blocking=True)
            h_idx.copy_(B["idx"], non_blocking=True)
            h_cnt.copy_(B["cnt"], non_blocking=True)
            for layer in range(1, 1 + self.n_sparse):
                self.s_out.wait_event(self.out_ready[b][layer])
                h_o[layer].copy_(B["o"][layer], non_blocking=True)
            self.out_free[b].record(self.s_out)
        self.step += 1

    def synchronize(self) -> None:
        for s in (self.s_in, self.s_comp, self.s_out):
            s.synchronize()
        hs2.hs2_sync(self.s_comp)
