"""Parity of decode-step sparse attention (hs2_sparse_decode, through the C
ABI) with the fp64 oracle's sparse_decode, on the lists the GPU full layer
selected for the same seeded inputs.

Bars as for every bf16 attention output: max|d| <= 1.5e-2, mean|d| <= 2e-3.
Query counts cover both launch shapes: few queries (each list split over
many CTAs whose partials are merged) and many (one CTA per query and KV
head)."""
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


def _decode(r, xd, q_rows, positions):
    shape = r["shape"]
    qd = q_rows.contiguous()
    sh = hs2.Hs2Shape(**{f: getattr(shape, f) for f, _ in hs2.Hs2Shape._fields_})
    sh.q_tok_stride, sh.q_head_stride = qd.stride(0), qd.stride(1)
    pos = torch.as_tensor(positions, dtype=torch.int32, device=DEV)
    nbytes = hs2.sparse_decode_workspace_bytes(sh, pos.numel())
    ws = torch.empty(max(1, nbytes // 4 + 4), dtype=torch.float32, device=DEV) if nbytes else None
    o, ob = H.guarded(tuple(qd.shape), torch.bfloat16, DEV)
    hs2.hs2_sparse_decode(sh, qd, pos, xd["k"], xd["v"], xd.get("k_scale"), xd.get("v_scale"), r["idx"], r["cnt"],
                          o, ws)
    hs2.hs2_sync()
    assert H.guards_intact(ob)
    return o, nbytes


def _positions(L, n, seed):
    rng = np.random.default_rng(seed)
    edge = [0, 1, 63, 64, 127, L - 65, L - 64, L - 1]
    pos = edge + [int(p) for p in rng.integers(0, L, max(0, n - len(edge)))]
    return np.array(pos[:n], dtype=np.int64)


@pytest.mark.parametrize("L,Hq,Hkv,n", [
    (2048, 8, 2, 1), (2048, 8, 2, 8), (4096, 16, 2, 5), (4096, 8, 1, 40), (2560, 4, 2, 300),
])
def test_decode_matches_oracle_on_gpu_lists(L, Hq, Hkv, n):
    wl = inputs.Workload(f"d{L}_{Hq}x{Hkv}", L, Hq, Hkv, 1, 41 + n, topk=1000)
    x = inputs.make_inputs(wl)
    xd = H.to_dev(x, DEV)
    r = H.run_path(wl, xd)
    pos = _positions(L, n, seed=n)
    q_rows = xd["q_layers"][1][torch.as_tensor(pos, device=DEV)]
    o, nbytes = _decode(r, xd, q_rows, pos)
    assert (nbytes > 0) == (n * Hkv < 444)
    D = H.decode(x)
    ref = orc.sparse_decode(D["Q"][1][pos], pos, D["K"], D["V"], r["idx"].cpu().numpy(), r["cnt"].cpu().numpy(), 64)
    H.bf16_close(o.float().cpu().numpy(), ref, f"decode n={n}")
    # the same rows of the prefill sparse layer (same list, other kernel):
    # both are within the bar of one reference, so within twice it of each other
    pre = r["sparse"][0][torch.as_tensor(pos, device=DEV)].float().cpu().numpy()
    d = np.abs(o.float().cpu().numpy() - pre)
    assert d.max() <= 2 * H.O_MAX and d.mean() <= 2 * H.O_MEAN


def test_decode_fp8_cache_matches_oracle():
    wl = inputs.Workload("d_fp8", 2304, 8, 2, 1, 53, kv_dtype="e4m3", topk=1000)
    x = inputs.make_inputs(wl)
    xd = H.to_dev(x, DEV)
    r = H.run_path(wl, xd)
    D = H.decode(x)
    for n in (3, 260):
        pos = _positions(wl.L, n, seed=100 + n)
        q_rows = xd["q_layers"][1][torch.as_tensor(pos, device=DEV)]
        o, _ = _decode(r, xd, q_rows, pos)
        ref = orc.sparse_decode(D["Q"][1][pos], pos, D["K"], D["V"], r["idx"].cpu().numpy(),
                                r["cnt"].cpu().numpy(), 64)
        H.bf16_close(o.float().cpu().numpy(), ref, f"decode fp8 n={n}")


def test_decode_is_deterministic_across_launch_orders():
    """Partials are merged in split order, whichever CTA finishes last."""
    wl = inputs.Workload("d_det", 4096, 8, 2, 1, 61)
    x = inputs.make_inputs(wl)
    xd = H.to_dev(x, DEV)
    r = H.run_path(wl, xd)
    pos = _positions(wl.L, 4, seed=7)
    q_rows = xd["q_layers"][1][torch.as_tensor(pos, device=DEV)]
    outs = [_decode(r, xd, q_rows, pos)[0] for _ in range(5)]
    assert all(torch.equal(outs[0], o) for o in outs[1:])


def test_decode_bad_position_is_reported_and_zero():
    wl = inputs.Workload("d_bad", 1024, 4, 2, 1, 67)
    x = inputs.make_inputs(wl)
    xd = H.to_dev(x, DEV)
    r = H.run_path(wl, xd)
    pos = np.array([5, 1024, 700])
    q_rows = xd["q_layers"][1][torch.as_tensor([5, 0, 700], device=DEV)]
    shape = r["shape"]
    qd = q_rows.contiguous()
    posd = torch.as_tensor(pos, dtype=torch.int32, device=DEV)
    nbytes = hs2.sparse_decode_workspace_bytes(shape, 3)
    ws = torch.empty(nbytes // 4 + 4, dtype=torch.float32, device=DEV)
    o = torch.full_like(qd, 7.0)
    hs2.hs2_sparse_decode(shape, qd, posd, xd["k"], xd["v"], None, None, r["idx"], r["cnt"], o, ws)
    with pytest.raises(hs2.Hs2Error) as e:
        hs2.hs2_sync()
    assert e.value.code == hs2.HS2_ERR_INDEX
    assert torch.all(o[1] == 0)
    D = H.decode(x)
    ok = np.array([5, 700])
    ref = orc.sparse_decode(D["Q"][1][ok], ok, D["K"], D["V"], r["idx"].cpu().numpy(), r["cnt"].cpu().numpy(), 64)
    H.bf16_close(o[[0, 2]].float().cpu().numpy(), ref, "good rows beside a bad one")
    hs2.hs2_sync()


def test_decode_128k_sampled():
    """The benchmark's 128k workload: decode queries at sampled positions
    against the lists of the GPU full layer, checked one KV group at a time."""
    wl = inputs.WORKLOADS["c3"]
    xd = inputs.make_inputs(wl, device=DEV)
    r = H.run_path(wl, xd)
    for n in (1, 64):
        pos = _positions(wl.L, n, seed=200 + n)
        q_rows = xd["q_layers"][1][torch.as_tensor(pos, device=DEV)]
        o, _ = _decode(r, xd, q_rows, pos)
        G = wl.G
        for g in (0, 5):
            hs = slice(g * G, (g + 1) * G)
            K = H.decode_kv(xd["k"][:, g:g + 1], None)
            V = H.decode_kv(xd["v"][:, g:g + 1], None)
            Q = orc.decode_bf16(inputs.as_u16(q_rows[:, hs]))
            ref = orc.sparse_decode(Q, pos, K, V, r["idx"][g:g + 1].cpu().numpy(), r["cnt"][g:g + 1].cpu().numpy(), 64)
            H.bf16_close(o[:, hs].float().cpu().numpy(), ref, f"decode 128k n={n} g{g}")
    del xd, r
    torch.cuda.empty_cache()
