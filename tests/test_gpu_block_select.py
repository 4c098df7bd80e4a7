"""Block-level selection (HySparse v1) on the GPU against the oracle's
select_blocks, bit-exact on the same exported fp32 importance; and the needle
recall of both granularities on the 32k workload (reported, not a pin)."""
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


def _path_blocks(wl, xd):
    q0, k, v = xd["q_layers"][0], xd["k"], xd["v"]
    shape = H.shape_of(wl, xd)
    out = hs2.alloc_outputs(shape, q0)
    hs2.hs2_full_attn_select_blocks(shape, q0, k, v, xd.get("k_scale"), xd.get("v_scale"), out["o"], out["lse"],
                                    out["idx"], out["cnt"], out["workspace"])
    hs2.hs2_sync()
    return shape, out


@pytest.mark.parametrize("L,Hq,Hkv", [(4096, 8, 2), (2304, 8, 1)])
def test_block_path_bit_exact_on_exported_importance(L, Hq, Hkv):
    wl = inputs.Workload(f"b{L}", L, Hq, Hkv, 1, seed=41)
    x = inputs.make_inputs(wl)
    xd = H.to_dev(x, DEV)
    shape, out = _path_blocks(wl, xd)
    nb = L // 64
    imp = H.gpu_importance(shape, xd, out["lse"], 0, nb).cpu().numpy()
    idx, cnt = out["idx"].cpu().numpy(), out["cnt"].cpu().numpy()
    for b in range(nb):
        _, e_b = orc.block_rows(b, L, 64)
        n_c = orc.n_candidates(e_b, 128)
        for g in range(Hkv):
            want, wc = orc.select_blocks(imp[g, b, :n_c], 1024, 128, e_b)
            assert cnt[g, b] == wc and np.array_equal(idx[g, b], want), (g, b)


def test_block_select_crafted_rows():
    L, Hkv = 8192, 4
    shape = hs2.Hs2Shape(L=L, Hq=8, Hkv=Hkv, d=128, block=64, topk=1024, recent=128, kv_dtype=0,
                         q_tok_stride=8 * 128, q_head_stride=128, kv_tok_stride=Hkv * 128, kv_head_stride=128)
    nb = L // 64
    rng = np.random.default_rng(6)
    b0, b1 = nb - 6, nb
    stride = orc.n_candidates(64 * b1, 128)
    rows = np.zeros((Hkv, b1 - b0, stride), np.float32)
    for bi, b in enumerate(range(b0, b1)):
        n = orc.n_candidates(64 * (b + 1), 128)
        rows[0, bi, :n] = (rng.integers(0, 3, n) / 4).astype(np.float32)       # heavy ties between blocks
        rows[1, bi, :n] = 1.0                                                  # all blocks equal
        rows[2, bi, :n] = rng.random(n).astype(np.float32)
        rows[3, bi, :n] = np.exp(-rng.random(n) * 60).astype(np.float32)
    imp = torch.from_numpy(rows).to(DEV)
    idx = torch.full((Hkv, nb, 1152), -9, dtype=torch.int32, device=DEV)
    cnt = torch.full((Hkv, nb), -9, dtype=torch.int32, device=DEV)
    hs2.hs2_block_select(shape, imp, stride, b0, b1, idx, cnt)
    hs2.hs2_sync()
    for bi, b in enumerate(range(b0, b1)):
        e_b = 64 * (b + 1)
        n = orc.n_candidates(e_b, 128)
        for g in range(Hkv):
            want, wc = orc.select_blocks(rows[g, bi, :n], 1024, 128, e_b)
            assert int(cnt[g, b]) == wc and np.array_equal(idx[g, b].cpu().numpy(), want), (g, b)


def test_needle_recall_token_vs_block_on_32k():
    wl = inputs.WORKLOADS["c2"]
    xd = inputs.make_inputs(wl, device=DEV)
    r_tok = H.run_path(wl.scaled(n_sparse=0), {**xd, "q_layers": xd["q_layers"][:1]})
    _, r_blk = _path_blocks(wl, xd)

    def recall(idx, cnt):
        hit = 0
        for n in xd["needles"]:
            b = n["t"] // 64
            lst = idx[n["g"], b, :cnt[n["g"], b]]
            hit += int(n["p"] in set(lst.tolist()))
        return hit / len(xd["needles"])
    rt = recall(r_tok["idx"].cpu().numpy(), r_tok["cnt"].cpu().numpy())
    rb = recall(r_blk["idx"].cpu().numpy(), r_blk["cnt"].cpu().numpy())
    print(f"needle recall on the 32k workload: token-level {rt:.4f}, block-level {rb:.4f}")
    assert 0.0 <= rb <= 1.0 and 0.0 <= rt <= 1.0
