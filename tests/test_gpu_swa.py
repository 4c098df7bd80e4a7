"""Parity of the sliding-window attention kernel (hs2_swa_attn, through the C
ABI) with the fp64 oracle's swa_attn on the same seeded input bytes.

Bars as for every bf16 attention output: max|d| <= 1.5e-2, mean|d| <= 2e-3;
LSE within 2e-3.  Small shapes are checked on every element (several tiles,
ragged tails, windows narrower than, equal to and wider than a 128-key tile);
the 128k shape of the benchmark is checked on sampled row ranges."""
import numpy as np
import pytest
import torch

from oracle import hs2_oracle as orc
from tests import gpu_harness as H
from token_level_sparse_causal_b200 import hs2, inputs

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    H.ensure_built()
    hs2.hs2_debug_set(H.WAIT_LIMIT_NS, 0)


def _inputs(L, Hq, Hkv, seed):
    wl = inputs.Workload(f"w{L}_{Hq}x{Hkv}", L, Hq, Hkv, 0, seed)
    x = inputs.make_inputs(wl)
    return x, H.to_dev(x, DEV)


def _run(xd, W, with_lse=True):
    q, k, v = xd["q_layers"][0], xd["k"], xd["v"]
    L, Hq, _ = q.shape
    shape = hs2.make_shape(q, k)
    o, ob = H.guarded((L, Hq, 128), torch.bfloat16, DEV)
    lse, lb = H.guarded((Hq, L), torch.float32, DEV) if with_lse else (None, None)
    hs2.hs2_swa_attn(shape, q, k, v, W, o, lse)
    hs2.hs2_sync()
    assert H.guards_intact(ob) and (lb is None or H.guards_intact(lb))
    return o, lse


@pytest.mark.parametrize("L,Hq,Hkv,W", [
    (1088, 8, 4, 128),    # the window of the measurements; ragged last tile
    (1088, 8, 4, 1),      # each query sees only itself
    (640, 16, 2, 200),    # window spans two key tiles, not tile-aligned
    (1088, 4, 1, 300),
    (2048, 8, 2, 129),
    (704, 8, 2, 704),     # W = L: plain causal attention
])
def test_swa_matches_oracle(L, Hq, Hkv, W):
    x, xd = _inputs(L, Hq, Hkv, seed=11 + W)
    o, lse = _run(xd, W)
    D = H.decode(x)
    O, LSE = orc.swa_attn(D["Q"][0], D["K"], D["V"], W)
    H.bf16_close(o.float().cpu().numpy(), O, f"O W={W}")
    assert np.abs(lse.cpu().numpy() - LSE).max() <= H.LSE_ATOL


def test_swa_without_lse_writes_the_same_output():
    x, xd = _inputs(1024, 8, 2, seed=5)
    o1, _ = _run(xd, 128)
    o2, _ = _run(xd, 128, with_lse=False)
    assert torch.equal(o1, o2)


@pytest.mark.parametrize("L", [1024, 1088])
def test_full_window_is_bitwise_the_dense_kernel(L):
    """With W = L no key is outside the window, so the window mode must do
    exactly the dense causal kernel's arithmetic."""
    x, xd = _inputs(L, 8, 2, seed=9)
    o, lse = _run(xd, L)
    shape = hs2.make_shape(xd["q_layers"][0], xd["k"])
    od = torch.empty_like(o)
    lsed = torch.empty_like(lse)
    hs2.hs2_attn_fwd(shape, xd["q_layers"][0], xd["k"], xd["v"], None, None, od, lsed)
    hs2.hs2_sync()
    assert torch.equal(o, od) and torch.equal(lse, lsed)


def test_swa_128k_sampled():
    """L = 131072, 64 query heads over 8 KV heads, W = 128: sampled row
    ranges against the oracle on the key segment those rows can see (the
    window's mask is shift-invariant, so the segment is exact)."""
    L, Hq, Hkv, W = 131072, 64, 8, 128
    wl = inputs.WORKLOADS["c3"]
    assert (wl.L, wl.Hq, wl.Hkv) == (L, Hq, Hkv)
    xd = inputs.make_inputs(wl, device=DEV)
    o, lse = _run(xd, W)
    G = Hq // Hkv
    rng = np.random.default_rng(8)
    starts = [0, L - 192] + [int(s) * 64 for s in rng.integers(2, L // 64 - 4, 3)]
    for s in starts:
        e = s + 192
        k0 = max(0, s - W + 1)
        for g in (1, 6):
            hs = slice(g * G, (g + 1) * G)
            Q = orc.decode_bf16(inputs.as_u16(xd["q_layers"][0][k0:e, hs]))
            K = H.decode_kv(xd["k"][k0:e, g:g + 1], None)
            V = H.decode_kv(xd["v"][k0:e, g:g + 1], None)
            O, LSE = orc.swa_attn(Q, K, V, W)
            H.bf16_close(o[s:e, hs].float().cpu().numpy(), O[s - k0:], f"O rows {s} g{g}")
            assert np.abs(lse[hs, s:e].cpu().numpy() - LSE[:, s - k0:]).max() <= H.LSE_ATOL
    del xd, o, lse
    torch.cuda.empty_cache()
