"""hs2_full_attn_select_static: the full-layer entry point for callers that
cannot allocate device memory where they call it (e.g. a plugin whose host
framework owns the device pool and passes only tensor pointers).  Its
importance scratch is a fixed 16 MiB device array inside the library.

The GPU test calls it through the C ABI twice in a row and compares each
result with hs2_full_attn_select given a caller workspace; the CPU test checks
that a shape needing more than the 16 MiB is refused before any launch.  This
file is collected last so that a run stopping at its first failure has
already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

from token_level_sparse_causal_b200 import build, hs2, inputs


def test_oversize_shape_rejected_before_launch():
    build.build()
    L, Hq, Hkv = 1 << 20, 16, 8      # one-block strip: 8 * (1M - 128) * 4 B > 16 MiB
    shape = hs2.Hs2Shape(L=L, Hq=Hq, Hkv=Hkv, d=128, block=64, topk=1024, recent=128, kv_dtype=0,
                         q_tok_stride=Hq * 128, q_head_stride=128, kv_tok_stride=Hkv * 128, kv_head_stride=128)
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: the size check comes first
    rc = hs2.lib().hs2_full_attn_select_static(ctypes.byref(shape), fake, fake, fake, None, None, fake, fake,
                                               fake, fake, ctypes.c_void_p(0))
    assert rc == hs2.HS2_ERR_WORKSPACE


def test_static_limit_accepts_the_1m_fp8_shape():
    """The 16 MiB array holds the one-block strip of the 1M-token workload with
    4 KV heads (4 * (2^20 - 128) * 4 B = 16,775,168 B) but not with 8: the
    first passes the size check and stops at the null pointers, the second is
    refused for its size.  Neither reaches a CUDA call."""
    build.build()
    for Hkv, code in ((4, hs2.HS2_ERR_INVALID_ARG), (8, hs2.HS2_ERR_WORKSPACE)):
        L, Hq = 1 << 20, 8 * Hkv
        shape = hs2.Hs2Shape(L=L, Hq=Hq, Hkv=Hkv, d=128, block=64, topk=1024, recent=128, kv_dtype=1,
                             q_tok_stride=Hq * 128, q_head_stride=128, kv_tok_stride=Hkv * 128, kv_head_stride=128)
        rc = hs2.lib().hs2_full_attn_select_static(ctypes.byref(shape), None, None, None, None, None, None, None,
                                                   None, None, ctypes.c_void_p(0))
        assert rc == code, (Hkv, rc)


@pytest.mark.gpu
@pytest.mark.parametrize("wl_name,L", [("c2", 32768), ("c1", 2048)])
def test_static_scratch_matches_workspace_path_twice(wl_name, L):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    hs2.hs2_debug_set(500_000_000, 0)
    dev = torch.device("cuda:0")
    wl = inputs.WORKLOADS[wl_name].scaled(L=L)
    x = inputs.make_inputs(wl, device=dev)
    q0, k, v = x["q_layers"][0], x["k"], x["v"]
    shape = hs2.make_shape(q0, k, wl.topk, wl.recent)
    ref = hs2.alloc_outputs(shape, q0)
    hs2.hs2_full_attn_select(shape, q0, k, v, None, None, ref["o"], ref["lse"], ref["idx"], ref["cnt"],
                             ref["workspace"])
    hs2.hs2_sync()
    for call in range(2):
        got = hs2.alloc_outputs(shape, q0, with_workspace=False)
        for t in got.values():
            t.fill_(0)
        hs2.hs2_full_attn_select_static(shape, q0, k, v, None, None, got["o"], got["lse"], got["idx"], got["cnt"])
        hs2.hs2_sync()
        assert torch.equal(got["idx"], ref["idx"]) and torch.equal(got["cnt"], ref["cnt"]), call
        d = (got["o"].float() - ref["o"].float()).abs()
        assert d.max().item() <= 1.5e-2 and d.mean().item() <= 2e-3, call
        assert (got["lse"] - ref["lse"]).abs().max().item() <= 2e-3, call


@pytest.mark.gpu
def test_static_scratch_matches_workspace_path_with_an_fp8_cache():
    """With an e4m3 cache the static entry always converts the codes inside
    kernels (1) and (2) (no room for the layer's f16 copy), while the
    workspace path converts the cache once into its workspace: the lists must
    still agree bit for bit, twice in a row."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    hs2.hs2_debug_set(500_000_000, 0)
    dev = torch.device("cuda:0")
    L, Hq, Hkv = 2048, 16, 2
    x = inputs.make_inputs(inputs.Workload("nf8", L, Hq, Hkv, 0, seed=61), device=dev)
    q0, kb, vb = x["q_layers"][0], x["k"], x["v"]
    k8 = torch.empty(kb.shape, dtype=torch.uint8, device=dev)
    v8 = torch.empty(vb.shape, dtype=torch.uint8, device=dev)
    ks = torch.empty(kb.shape[:2], dtype=torch.float32, device=dev)
    vs = torch.empty(vb.shape[:2], dtype=torch.float32, device=dev)
    hs2.hs2_quantize_kv(kb, k8, ks)
    hs2.hs2_quantize_kv(vb, v8, vs)
    shape = hs2.make_shape(q0, k8, 1024, 128, kv_dtype=hs2.HS2_KV_E4M3)
    ref = hs2.alloc_outputs(shape, q0)
    hs2.hs2_full_attn_select(shape, q0, k8, v8, ks, vs, ref["o"], ref["lse"], ref["idx"], ref["cnt"],
                             ref["workspace"])
    hs2.hs2_sync()
    for call in range(2):
        got = hs2.alloc_outputs(shape, q0, with_workspace=False)
        for t in got.values():
            t.fill_(0)
        hs2.hs2_full_attn_select_static(shape, q0, k8, v8, ks, vs, got["o"], got["lse"], got["idx"], got["cnt"])
        hs2.hs2_sync()
        assert torch.equal(got["idx"], ref["idx"]) and torch.equal(got["cnt"], ref["cnt"]), call
        d = (got["o"].float() - ref["o"].float()).abs()
        assert d.max().item() <= 1.5e-2 and d.mean().item() <= 2e-3, call
