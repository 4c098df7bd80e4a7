"""The double-buffered end-to-end runner (PrefillPipeline): outputs copied back
to the host must equal, bit for bit, those of the same C ABI calls made one
after another on one stream, for interleaved sequences (so that the two device
buffer sets never leak into each other)."""
import pytest
import torch

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


def _host_set(x):
    pin = lambda t: t.cpu().pin_memory()
    return [pin(q) for q in x["q_layers"]], pin(x["k"]), pin(x["v"])


def _outs(wl):
    L, Hq, Hkv, nb = wl.L, wl.Hq, wl.Hkv, wl.L // 64
    o = [torch.empty((L, Hq, 128), dtype=torch.bfloat16, pin_memory=True) for _ in range(1 + wl.n_sparse)]
    idx = torch.empty((Hkv, nb, wl.topk + wl.recent), dtype=torch.int32, pin_memory=True)
    cnt = torch.empty((Hkv, nb), dtype=torch.int32, pin_memory=True)
    return o, idx, cnt


def test_pipeline_matches_serial_calls():
    from token_level_sparse_causal_b200.pipeline import PrefillPipeline
    wls = [inputs.Workload(f"p{s}", 2048, 8, 2, 2, s) for s in (71, 72)]
    xs = [inputs.make_inputs(wl) for wl in wls]
    refs = [H.run_path(wl, H.to_dev(x, DEV)) for wl, x in zip(wls, xs)]
    shape = refs[0]["shape"]
    pipe = PrefillPipeline(shape, 2, DEV)
    order = [0, 1, 0, 1, 0]
    outs = []
    for i in order:
        h_q, h_k, h_v = _host_set(xs[i])
        o, idx, cnt = _outs(wls[i])
        pipe.submit(h_q, h_k, h_v, o, idx, cnt)
        outs.append((i, o, idx, cnt, h_q, h_k, h_v))
    pipe.synchronize()
    for i, o, idx, cnt, *_ in outs:
        r = refs[i]
        assert torch.equal(idx, r["idx"].cpu()) and torch.equal(cnt, r["cnt"].cpu())
        assert torch.equal(o[0], r["o"].cpu())
        for layer in range(2):
            assert torch.equal(o[1 + layer], r["sparse"][layer].cpu())
