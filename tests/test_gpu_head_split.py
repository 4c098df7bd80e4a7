"""The KV-head split of one sequence (one GPU stands in for the ranks, which
run one after another: no rank waits on another).  Each rank's half of the
heads, passed as head-strided views of the same Q/K/V, must give bit for bit
the O, LSE, index lists and sparse-layer O of the matching heads of the
whole-tensor call: the heads share nothing but the shape."""
import pytest
import torch

from tests import gpu_harness as H
from token_level_sparse_causal_b200 import hs2, inputs, shard

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    H.ensure_built()
    hs2.hs2_debug_set(H.WAIT_LIMIT_NS, 0)


@pytest.mark.parametrize("L,Hq,Hkv,world,kv", [(4096, 16, 4, 2, "bf16"), (2560, 32, 4, 2, "bf16"),
                                                  (4096, 16, 4, 4, "bf16"), (3072, 16, 4, 2, "e4m3")])
def test_head_shards_equal_the_whole_call(L, Hq, Hkv, world, kv):
    wl = inputs.Workload(f"hs{L}", L, Hq, Hkv, 2, seed=53, kv_dtype=kv)
    xd = H.to_dev(inputs.make_inputs(wl), DEV)
    whole = H.run_path(wl, xd)
    o_layers = [torch.full_like(q, float("nan")) for q in xd["q_layers"]]
    for rank in range(world):
        sh = shard.kv_head_range(Hq, Hkv, rank, world)
        part = shard.prefill_shard(sh, xd["q_layers"], xd["k"], xd["v"], xd.get("k_scale"), xd.get("v_scale"),
                                   o_layers)
        hs2.hs2_sync()
        assert torch.equal(part["lse"], whole["lse"][sh.h0:sh.h1])
        assert torch.equal(part["idx"], whole["idx"][sh.g0:sh.g1])
        assert torch.equal(part["cnt"], whole["cnt"][sh.g0:sh.g1])
    assert torch.equal(o_layers[0], whole["o"])
    for got, want in zip(o_layers[1:], whole["sparse"]):
        assert torch.equal(got, want)
