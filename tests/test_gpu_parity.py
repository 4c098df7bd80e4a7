"""Parity of the CUDA path (through the C ABI) with the fp64 oracle on the same
seeded input bytes.

Bars: indices bit-exact when both sides select from the same exported fp32
importance; importance within rtol 1e-3; bf16 attention outputs within
max|d| <= 1.5e-2 and mean|d| <= 2e-3.  Small shapes are checked on every
output element and span several tiles with ragged tails; the 32k and 128k
workloads (the latter in the launch configuration the benchmark times) are
checked on sampled query blocks."""
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


def _wl(L, Hq, Hkv, n_sparse=1, seed=7, topk=1024, recent=128, needles=()):
    return inputs.Workload(f"t{L}_{Hq}x{Hkv}", L, Hq, Hkv, n_sparse, seed, needles=needles, topk=topk, recent=recent)


# ------------------------------------------------------------ kernel (1) --

@pytest.mark.parametrize("L,Hq,Hkv", [(1088, 8, 4), (2048, 4, 1), (640, 16, 2)])
def test_attn_fwd_matches_oracle(L, Hq, Hkv):
    wl = _wl(L, Hq, Hkv)
    x = inputs.make_inputs(wl)
    xd = H.to_dev(x, DEV)
    shape = hs2.make_shape(xd["q_layers"][0], xd["k"])
    o, ob = H.guarded((L, Hq, 128), torch.bfloat16, DEV)
    lse, lb = H.guarded((Hq, L), torch.float32, DEV)
    hs2.hs2_attn_fwd(shape, xd["q_layers"][0], xd["k"], xd["v"], None, None, o, lse)
    hs2.hs2_sync()
    D = H.decode(x)
    O, LSE = orc.dense_attn(D["Q"][0], D["K"], D["V"])
    H.bf16_close(o.float().cpu().numpy(), O, "O")
    assert np.abs(lse.cpu().numpy() - LSE).max() <= H.LSE_ATOL
    assert H.guards_intact(ob) and H.guards_intact(lb)


def test_attn_fwd_on_a_side_stream_with_padded_strides():
    """Non-default stream; Q/O with a padded head stride and K/V with a padded
    token stride (strides are honoured, nothing outside the rows is read)."""
    L, Hq, Hkv = 512, 8, 2
    wl = _wl(L, Hq, Hkv, seed=3)
    x = inputs.make_inputs(wl)
    qpad = torch.zeros((L, Hq, 136), dtype=torch.bfloat16)
    qpad[:, :, :128] = x["q_layers"][0]
    kpad = torch.zeros((L, Hkv + 1, 128), dtype=torch.bfloat16)
    vpad = torch.zeros((L, Hkv + 1, 128), dtype=torch.bfloat16)
    kpad[:, :Hkv], vpad[:, :Hkv] = x["k"], x["v"]
    q = qpad.to(DEV)[:, :, :128]
    k, v = kpad.to(DEV)[:, :Hkv], vpad.to(DEV)[:, :Hkv]
    shape = hs2.make_shape(q, k)
    assert shape.q_head_stride == 136 and shape.kv_tok_stride == (Hkv + 1) * 128
    o = torch.zeros((L, Hq, 136), dtype=torch.bfloat16, device=DEV)[:, :, :128]
    lse = torch.empty((Hq, L), device=DEV)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        hs2.hs2_attn_fwd(shape, q, k, v, None, None, o, lse, stream=s)
        hs2.hs2_sync(s)
    D = H.decode(x)
    O, LSE = orc.dense_attn(D["Q"][0], D["K"], D["V"])
    H.bf16_close(o.float().cpu().numpy(), O, "O")
    assert np.abs(lse.cpu().numpy() - LSE).max() <= H.LSE_ATOL


# ------------------------------------------------------------ kernel (2) --

@pytest.mark.parametrize("L,Hq,Hkv", [(2304, 8, 1), (1536, 8, 2), (1024, 4, 2)])
def test_importance_matches_oracle(L, Hq, Hkv):
    wl = _wl(L, Hq, Hkv, seed=11)
    x = inputs.make_inputs(wl)
    xd = H.to_dev(x, DEV)
    shape = hs2.make_shape(xd["q_layers"][0], xd["k"])
    o = torch.empty_like(xd["q_layers"][0])
    lse = torch.empty((Hq, L), device=DEV)
    hs2.hs2_attn_fwd(shape, xd["q_layers"][0], xd["k"], xd["v"], None, None, o, lse)
    nb = L // 64
    imp = H.gpu_importance(shape, xd, lse, 0, nb).cpu().numpy()
    D = H.decode(x)
    _, LSE = orc.dense_attn(D["Q"][0], D["K"], D["V"])
    worst = 0.0
    for b in range(nb):
        s_b, e_b = orc.block_rows(b, L, 64)
        for g in range(Hkv):
            ref = orc.importance(D["Q"][0], D["K"], LSE[:, s_b:e_b], b, g, 64, 128)
            got = imp[g, b, :ref.size]
            assert np.all(np.isfinite(got))
            rel = np.abs(got - ref) / np.maximum(np.abs(ref), 1e-30)
            worst = max(worst, rel.max() if ref.size else 0.0)
    assert worst <= H.IMP_RTOL, worst


@pytest.mark.parametrize("L,Hq,Hkv,kv", [(2304, 8, 1, "bf16"), (1536, 16, 2, "bf16"), (1088, 8, 2, "e4m3")])
def test_importance_mass_conservation_on_gpu(L, Hq, Hkv, kv):
    """Checking mode (debug flag bit 1): kernel (2) over every visible key
    j < e_b with the causal mask.  A row then holds, for each key, the
    probabilities the block's 64 queries of the group's G heads give it, so
    it sums to 64 * G when the GPU's own LSE normalises every query; the
    candidate part must equal the normal row bit for bit."""
    wl = inputs.Workload(f"m{L}", L, Hq, Hkv, 0, seed=19, kv_dtype=kv)
    xd = H.to_dev(inputs.make_inputs(wl), DEV)
    shape = H.shape_of(wl, xd)
    q0, k, v, ks, vs = xd["q_layers"][0], xd["k"], xd["v"], xd.get("k_scale"), xd.get("v_scale")
    o = torch.empty_like(q0)
    lse = torch.empty((Hq, L), device=DEV)
    hs2.hs2_attn_fwd(shape, q0, k, v, ks, vs, o, lse)
    nb = L // 64
    full = torch.full((Hkv, nb, L), float("nan"), device=DEV)
    hs2.hs2_debug_set(H.WAIT_LIMIT_NS, 2)
    try:
        hs2.hs2_importance(shape, q0, k, ks, lse, 0, nb, full, L)
        hs2.hs2_sync()
    finally:
        hs2.hs2_debug_set(H.WAIT_LIMIT_NS, 0)
    normal = H.gpu_importance(shape, xd, lse, 0, nb).cpu().numpy()
    full = full.cpu().numpy()
    G = Hq // Hkv
    worst = 0.0
    for b in range(nb):
        _, e_b = orc.block_rows(b, L, 64)
        n_c = orc.n_candidates(e_b, 128)
        for g in range(Hkv):
            row = full[g, b, :e_b].astype(np.float64)
            assert np.all(np.isfinite(row)) and np.all(row >= 0)
            worst = max(worst, abs(row.sum() - 64 * G) / (64 * G))
            assert np.array_equal(full[g, b, :n_c].view(np.uint32), normal[g, b, :n_c].view(np.uint32)), (g, b)
    assert worst <= 1e-4, worst


# ------------------------------------------------------------ kernel (3) --

@pytest.mark.parametrize("L,Hq,Hkv", [(2304, 8, 1), (1536, 8, 2)])
def test_select_bit_exact_on_exported_importance(L, Hq, Hkv):
    wl = _wl(L, Hq, Hkv, seed=13)
    x = inputs.make_inputs(wl)
    xd = H.to_dev(x, DEV)
    r = H.run_path(wl, xd, guards=True)
    nb = L // 64
    imp = H.gpu_importance(r["shape"], xd, r["lse"], 0, nb).cpu().numpy().astype(np.float64)
    idx, cnt = r["idx"].cpu().numpy(), r["cnt"].cpu().numpy()
    for b in range(nb):
        _, e_b = orc.block_rows(b, L, 64)
        n_c = orc.n_candidates(e_b, 128)
        for g in range(Hkv):
            want, wc = orc.select(imp[g, b, :n_c], 1024, 128, e_b)
            assert cnt[g, b] == wc
            assert np.array_equal(idx[g, b], want), (g, b)
    assert all(H.guards_intact(bb) for bb in r["bases"])


@pytest.mark.parametrize("L,Hq,Hkv,strips", [(4096, 8, 2, 5), (2560, 16, 2, 1)])
def test_select_bit_exact_on_the_rows_the_selection_consumed(L, Hq, Hkv, strips):
    """hs2_full_attn_select's own export of the importance rows it selected
    from (a small workspace, so the export spans several strips): the oracle's
    select on those rows gives the GPU's lists bit for bit, and the rows equal
    hs2_importance's recompute bit for bit."""
    wl = _wl(L, Hq, Hkv, n_sparse=0, seed=17)
    xd = H.to_dev(inputs.make_inputs(wl), DEV)
    shape = H.shape_of(wl, xd)
    q0, k, v = xd["q_layers"][0], xd["k"], xd["v"]
    nb = L // 64
    b0, b1 = 10, nb - 3
    S = hs2.importance_row_stride(shape, b1)
    exp_t = torch.full((Hkv, b1 - b0, S), float("nan"), device=DEV, dtype=torch.float32)
    row = (L - 128 + 63) // 64 * 64 * 4
    ws = torch.empty(strips * Hkv * row // 4 + 16, device=DEV, dtype=torch.float32)
    out = hs2.alloc_outputs(shape, q0, with_workspace=False)
    hs2.hs2_full_attn_select(shape, q0, k, v, None, None, out["o"], out["lse"], out["idx"], out["cnt"], ws,
                             importance_out=exp_t, strip=(b0, b1))
    hs2.hs2_sync()
    rows = exp_t.cpu().numpy()
    re = H.gpu_importance(shape, xd, out["lse"], b0, b1).cpu().numpy()
    idx, cnt = out["idx"].cpu().numpy(), out["cnt"].cpu().numpy()
    checked = 0
    for bi, b in enumerate(range(b0, b1)):
        _, e_b = orc.block_rows(b, L, 64)
        n_c = orc.n_candidates(e_b, 128)
        for g in range(Hkv):
            if n_c <= wl.topk:
                assert np.isnan(rows[g, bi]).all()       # no importance is computed there
                continue
            r_row = rows[g, bi, :n_c]
            assert np.array_equal(r_row.view(np.uint32), re[g, bi, :n_c].view(np.uint32)), (g, b)
            want, wc = orc.select(r_row.astype(np.float64), 1024, 128, e_b)
            assert cnt[g, b] == wc and np.array_equal(idx[g, b], want), (g, b)
            checked += 1
    assert checked > 0


def _crafted_rows(n, rng):
    kinds = [
        rng.random(n).astype(np.float32),                                   # distinct
        (rng.integers(0, 4, n) / 4.0).astype(np.float32),                   # 4 levels: huge ties
        np.ones(n, np.float32),                                             # all equal
        np.where(rng.random(n) < 0.5, -0.0, 0.0).astype(np.float32),        # +-0 only
        np.exp(-rng.random(n) * 80).astype(np.float32),                     # wide dynamic range
        np.concatenate([np.zeros(n - 1100, np.float32), np.full(1100, 1e-3, np.float32)]),  # tail-heavy
        rng.standard_normal(n).astype(np.float32),                          # signed: a positive threshold
        # with negative values, -0.0 and huge magnitudes beneath it
        np.where(rng.random(n) < 0.1, -3.0e38, rng.standard_normal(n) * 1e-20).astype(np.float32),
        -rng.random(n).astype(np.float32) - 1.0,                            # all negative
    ]
    return kinds


def test_select_crafted_rows_bit_exact():
    L, Hkv, topk, recent = 8192, 9, 1024, 128
    shape = hs2.Hs2Shape(L=L, Hq=18, Hkv=Hkv, d=128, block=64, topk=topk, recent=recent, kv_dtype=0,
                         q_tok_stride=18 * 128, q_head_stride=128, kv_tok_stride=Hkv * 128, kv_head_stride=128)
    nb = L // 64
    rng = np.random.default_rng(5)
    for b0, b1 in [(0, 24), (100, 104), (nb - 3, nb)]:
        stride = ((orc.n_candidates(64 * b1, recent) + 3) // 4) * 4
        rows = np.full((Hkv, b1 - b0, max(stride, 4)), np.nan, np.float32)
        for bi, b in enumerate(range(b0, b1)):
            n_c = orc.n_candidates(64 * (b + 1), recent)
            if n_c == 0:
                continue
            for g, row in enumerate(_crafted_rows(max(n_c, 1100), rng)):
                rows[g, bi, :n_c] = row[:n_c]
        imp = torch.from_numpy(rows).to(DEV)
        idx = torch.full((Hkv, nb, topk + recent), -9, dtype=torch.int32, device=DEV)
        cnt = torch.full((Hkv, nb), -9, dtype=torch.int32, device=DEV)
        hs2.hs2_topk_select(shape, imp, rows.shape[2], b0, b1, idx, cnt)
        hs2.hs2_sync()
        idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
        for bi, b in enumerate(range(b0, b1)):
            e_b = 64 * (b + 1)
            n_c = orc.n_candidates(e_b, recent)
            for g in range(Hkv):
                want, wc = orc.select(rows[g, bi, :n_c].astype(np.float64), topk, recent, e_b)
                assert cnt_h[g, b] == wc and np.array_equal(idx_h[g, b], want), (b, g)
        untouched = [bb for bb in range(nb) if not b0 <= bb < b1]
        assert np.all(idx_h[:, untouched] == -9) and np.all(cnt_h[:, untouched] == -9)


def _threshold_sample_positions(n_c):
    """Where kernel (3)'s threshold sample reads a row of n_c > 4096
    candidates: 2^(lg-3) groups of 8 consecutive values, group t starting at
    (t * n_c >> (lg - 3)) rounded down to a multiple of 8."""
    lg = 12 if n_c >= 8 * 4096 else 11 if n_c >= 8 * 2048 else 10
    ng = 1 << (lg - 3)
    j0 = ((np.arange(ng, dtype=np.int64) * n_c) >> (lg - 3)) & ~7
    return (j0[:, None] + np.arange(8)[None, :]).ravel()


def test_select_rows_that_defeat_the_sample_bit_exact():
    """Long rows (n > 8192) where the single-read path must give up: all
    values equal (too many gathered), and a row whose large values sit exactly
    where the threshold sample looks, so the sample overestimates the
    threshold (too few gathered).  The exact radix path then decides, and the
    lists must still equal the oracle's."""
    L, Hkv, topk, recent = 16384, 3, 1024, 128
    shape = hs2.Hs2Shape(L=L, Hq=6, Hkv=Hkv, d=128, block=64, topk=topk, recent=recent, kv_dtype=0,
                         q_tok_stride=6 * 128, q_head_stride=128, kv_tok_stride=Hkv * 128, kv_head_stride=128)
    nb = L // 64
    b0, b1 = nb - 2, nb
    rng = np.random.default_rng(9)
    stride = ((orc.n_candidates(64 * b1, recent) + 3) // 4) * 4
    rows = np.full((Hkv, b1 - b0, stride), np.nan, np.float32)
    for bi, b in enumerate(range(b0, b1)):
        n_c = orc.n_candidates(64 * (b + 1), recent)
        sample_pos = _threshold_sample_positions(n_c)
        trap = (rng.random(n_c) * 1e-3).astype(np.float32)
        trap[sample_pos[:500]] = 1.0          # 500 large values, all of them sampled
        rows[0, bi, :n_c] = np.full(n_c, 0.25, np.float32)
        rows[1, bi, :n_c] = trap
        rows[2, bi, :n_c] = rng.random(n_c).astype(np.float32)
    imp = torch.from_numpy(rows).to(DEV)
    idx = torch.full((Hkv, nb, topk + recent), -9, dtype=torch.int32, device=DEV)
    cnt = torch.full((Hkv, nb), -9, dtype=torch.int32, device=DEV)
    hs2.hs2_topk_select(shape, imp, stride, b0, b1, idx, cnt)
    hs2.hs2_sync()
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    for bi, b in enumerate(range(b0, b1)):
        e_b = 64 * (b + 1)
        n_c = orc.n_candidates(e_b, recent)
        for g in range(Hkv):
            want, wc = orc.select(rows[g, bi, :n_c].astype(np.float64), topk, recent, e_b)
            assert cnt_h[g, b] == wc and np.array_equal(idx_h[g, b], want), (b, g)


# ------------------------------------------------------------ kernel (4) --

def test_sparse_matches_oracle_on_gpu_lists():
    L, Hq, Hkv = 4096, 8, 2
    wl = _wl(L, Hq, Hkv, n_sparse=2, seed=17, topk=1000)          # 1128-entry lists: ragged last tile
    x = inputs.make_inputs(wl)
    xd = H.to_dev(x, DEV)
    r = H.run_path(wl, xd, guards=True)
    D = H.decode(x)
    idx, cnt = r["idx"].cpu().numpy(), r["cnt"].cpu().numpy()
    G = wl.G
    for layer, ol in enumerate(r["sparse"], start=1):
        got = ol.float().cpu().numpy()
        ref = np.empty_like(got, dtype=np.float64)
        for b in range(L // 64):
            s_b, e_b = orc.block_rows(b, L, 64)
            for g in range(Hkv):
                ref[s_b:e_b, g * G:(g + 1) * G] = orc.sparse_attn(D["Q"][layer], D["K"], D["V"], idx[g, b],
                                                                  int(cnt[g, b]), b, g, 64)
        H.bf16_close(got, ref, f"sparse layer {layer}")
    assert all(H.guards_intact(bb) for bb in r["bases"])


@pytest.mark.parametrize("L,Hq,Hkv", [(3072, 4, 2), (2048, 16, 2), (2560, 8, 1)])
def test_sparse_group_sizes_match_oracle(L, Hq, Hkv):
    """G = 2 (one M tile per work item) and G = 8 (two items per block and KV
    head); every block against the oracle, on GPU lists of 1128 entries (a
    ragged last key tile)."""
    wl = _wl(L, Hq, Hkv, n_sparse=1, seed=43, topk=1000)
    x = inputs.make_inputs(wl)
    xd = H.to_dev(x, DEV)
    r = H.run_path(wl, xd, guards=True)
    D = H.decode(x)
    idx, cnt = r["idx"].cpu().numpy(), r["cnt"].cpu().numpy()
    G = wl.G
    got = r["sparse"][0].float().cpu().numpy()
    ref = np.empty_like(got, dtype=np.float64)
    for b in range(L // 64):
        s_b, e_b = orc.block_rows(b, L, 64)
        for g in range(Hkv):
            ref[s_b:e_b, g * G:(g + 1) * G] = orc.sparse_attn(D["Q"][1], D["K"], D["V"], idx[g, b], int(cnt[g, b]),
                                                              b, g, 64)
    H.bf16_close(got, ref, f"sparse G={G}")
    assert all(H.guards_intact(bb) for bb in r["bases"])


def test_sparse_bounded_wait_reports_timeout_and_context_survives():
    """The persistent sparse kernel with its load roles switched off (test
    flag): the MMA and softmax waits run out, hs2_sync reports
    HS2_ERR_TIMEOUT, and the next call is correct."""
    wl = _wl(1024, 8, 2, seed=47)
    x = inputs.make_inputs(wl)
    xd = H.to_dev(x, DEV)
    r = H.run_path(wl, xd)
    o = torch.empty_like(xd["q_layers"][1])
    hs2.hs2_debug_set(50_000_000, 1)
    try:
        hs2.hs2_sparse_attn(r["shape"], xd["q_layers"][1], xd["k"], xd["v"], None, None, r["idx"], r["cnt"], o)
        with pytest.raises(hs2.Hs2Error) as e:
            hs2.hs2_sync()
        assert e.value.code == hs2.HS2_ERR_TIMEOUT
    finally:
        hs2.hs2_debug_set(H.WAIT_LIMIT_NS, 0)
    hs2.hs2_sparse_attn(r["shape"], xd["q_layers"][1], xd["k"], xd["v"], None, None, r["idx"], r["cnt"], o)
    hs2.hs2_sync()
    assert torch.equal(o, r["sparse"][0])


@pytest.mark.parametrize("L", [1152, 640])
def test_sparse_equals_dense_when_lists_cover_everything(L):
    wl = _wl(L, 8, 2, n_sparse=1, seed=19)
    x = inputs.make_inputs(wl)
    xd = H.to_dev(x, DEV)
    r = H.run_path(wl, xd)
    cnt = r["cnt"].cpu().numpy()
    assert np.array_equal(cnt, np.broadcast_to(np.arange(1, L // 64 + 1) * 64, cnt.shape))
    D = H.decode(x)
    O1, _ = orc.dense_attn(D["Q"][1], D["K"], D["V"])
    H.bf16_close(r["sparse"][0].float().cpu().numpy(), O1, "sparse == dense")


# ----------------------------------------------------------- whole path --

def test_end_to_end_2k_workload_with_needles():
    wl = inputs.WORKLOADS["c1"]
    x = inputs.make_inputs(wl)
    xd = H.to_dev(x, DEV)
    r = H.run_path(wl, xd, guards=True)
    D = H.decode(x)
    O, LSE = orc.dense_attn(D["Q"][0], D["K"], D["V"])
    H.bf16_close(r["o"].float().cpu().numpy(), O, "full-layer O")
    assert np.abs(r["lse"].cpu().numpy() - LSE).max() <= H.LSE_ATOL
    nb = wl.L // 64
    imp = H.gpu_importance(r["shape"], xd, r["lse"], 0, nb).cpu().numpy().astype(np.float64)
    idx, cnt = r["idx"].cpu().numpy(), r["cnt"].cpu().numpy()
    ref_sp = np.empty((wl.L, wl.Hq, 128))
    for b in range(nb):
        s_b, e_b = orc.block_rows(b, wl.L, 64)
        want, wc = orc.select(imp[0, b, :orc.n_candidates(e_b, 128)], 1024, 128, e_b)
        assert np.array_equal(idx[0, b], want) and cnt[0, b] == wc
        ref_sp[s_b:e_b] = orc.sparse_attn(D["Q"][1], D["K"], D["V"], idx[0, b], wc, b, 0, 64)
    H.bf16_close(r["sparse"][0].float().cpu().numpy(), ref_sp, "sparse layer")
    hit = sum(int(n["p"] in set(idx[n["g"], n["t"] // 64, :cnt[n["g"], n["t"] // 64]].tolist()))
              for n in x["needles"])
    print(f"needle recall {hit}/{len(x['needles'])}")
    assert all(H.guards_intact(bb) for bb in r["bases"])


class _Rows:
    """Rows [s, e) of a [L][H][d] array, addressed by absolute row index, so
    the oracle can evaluate one query block of a long workload."""

    def __init__(self, data, s, L):
        self.data, self.s, self.shape = data, s, (L,) + data.shape[1:]

    def __getitem__(self, key):
        r, rest = key[0], tuple(key[1:])
        if r == slice(None):
            return _Rows(self.data[(slice(None),) + rest], self.s, self.shape[0])
        assert r.start >= self.s
        return self.data[(slice(r.start - self.s, r.stop - self.s),) + rest]


def _sampled_check(wl, blocks, groups):
    xd = inputs.make_inputs(wl, device=DEV)
    r = H.run_path(wl, xd)
    fp8 = xd.get("k_scale") is not None
    G = wl.G
    for b in blocks:
        s_b, e_b = orc.block_rows(b, wl.L, 64)
        imp = H.gpu_importance(r["shape"], xd, r["lse"], b, b + 1).cpu().numpy().astype(np.float64)
        for g in groups:
            hs = slice(g * G, (g + 1) * G)
            Qb = [_Rows(orc.decode_bf16(inputs.as_u16(q[s_b:e_b, hs])), s_b, wl.L) for q in xd["q_layers"]]
            K = H.decode_kv(xd["k"][:e_b, g:g + 1], xd["k_scale"][:e_b, g:g + 1] if fp8 else None)
            V = H.decode_kv(xd["v"][:e_b, g:g + 1], xd["v_scale"][:e_b, g:g + 1] if fp8 else None)
            O, LSE = orc.dense_attn(Qb[0], K, V, s_b, e_b)
            H.bf16_close(r["o"][s_b:e_b, hs].float().cpu().numpy(), O, f"O b{b} g{g}")
            assert np.abs(r["lse"][hs, s_b:e_b].cpu().numpy() - LSE).max() <= H.LSE_ATOL
            lse_full = np.zeros((G, e_b - s_b))
            lse_full[:] = LSE
            ref_imp = orc.importance(Qb[0], K, lse_full, b, 0, 64, wl.recent)
            got_imp = imp[g, 0, :ref_imp.size]
            rel = np.abs(got_imp - ref_imp) / np.maximum(np.abs(ref_imp), 1e-30)
            assert rel.max() <= H.IMP_RTOL, (b, g, rel.max())
            want, wc = orc.select(got_imp, wl.topk, wl.recent, e_b)
            idx_g = r["idx"][g, b].cpu().numpy()
            assert int(r["cnt"][g, b]) == wc and np.array_equal(idx_g, want), (b, g)
            for layer, ol in enumerate(r["sparse"], start=1):
                ref = orc.sparse_attn(Qb[layer], K, V, idx_g, wc, b, 0, 64)
                H.bf16_close(ol[s_b:e_b, hs].float().cpu().numpy(), ref, f"sparse l{layer} b{b} g{g}")
    return r


def test_full_size_32k_workload_sampled():
    wl = inputs.WORKLOADS["c2"]
    rng = np.random.default_rng(1)
    blocks = [18, wl.nb - 1] + [int(b) for b in rng.integers(19, wl.nb - 1, 2)]
    _sampled_check(wl, blocks, groups=[0, 5])


def test_full_size_128k_workload_sampled():
    """The benchmark's workload and launch configuration."""
    wl = inputs.WORKLOADS["c3"]
    rng = np.random.default_rng(2)
    blocks = [18, wl.nb - 1] + [int(b) for b in rng.integers(19, wl.nb - 1, 2)]
    _sampled_check(wl, blocks, groups=[3, 7])
    torch.cuda.empty_cache()


def test_full_size_256k_chain_workload_sampled():
    wl = inputs.WORKLOADS["c4"]
    rng = np.random.default_rng(3)
    blocks = [18, wl.nb - 1, int(rng.integers(19, wl.nb - 1))]
    _sampled_check(wl, blocks, groups=[1])
    torch.cuda.empty_cache()


def test_full_size_1m_fp8_workload_sampled():
    """L = 1M with an e4m3 K/V cache and per-token scales."""
    wl = inputs.WORKLOADS["c5"]
    rng = np.random.default_rng(4)
    blocks = [18, wl.nb - 1, int(rng.integers(19, wl.nb - 1))]
    _sampled_check(wl, blocks, groups=[2])
    torch.cuda.empty_cache()


# ------------------------------------------------------ FP8 (e4m3) cache --

def _fp8_wl(L, Hq, Hkv, n_sparse=1, seed=31, topk=1024):
    return inputs.Workload(f"f{L}_{Hq}x{Hkv}", L, Hq, Hkv, n_sparse, seed, kv_dtype="e4m3", topk=topk)


@pytest.mark.parametrize("L,Hq,Hkv", [(1088, 8, 1), (640, 8, 2), (512, 4, 2)])
def test_fp8_attn_fwd_matches_oracle(L, Hq, Hkv):
    wl = _fp8_wl(L, Hq, Hkv)
    x = inputs.make_inputs(wl)
    xd = H.to_dev(x, DEV)
    shape = H.shape_of(wl, xd)
    o, ob = H.guarded((L, Hq, 128), torch.bfloat16, DEV)
    lse, lb = H.guarded((Hq, L), torch.float32, DEV)
    hs2.hs2_attn_fwd(shape, xd["q_layers"][0], xd["k"], xd["v"], xd["k_scale"], xd["v_scale"], o, lse)
    hs2.hs2_sync()
    D = H.decode(x)
    O, LSE = orc.dense_attn(D["Q"][0], D["K"], D["V"])
    H.bf16_close(o.float().cpu().numpy(), O, "O (fp8 cache)")
    assert np.abs(lse.cpu().numpy() - LSE).max() <= H.LSE_ATOL
    assert H.guards_intact(ob) and H.guards_intact(lb)


def test_fp8_q_at_the_edges_of_f16():
    """With an e4m3 cache Q is rounded bf16 -> f16: exact for magnitudes in
    [2^-14, 65504], subnormal below.  Rows holding 6e4 (sharp softmax) and
    rows scaled by 2^-20 (f16 subnormals: flat softmax) still match the
    oracle on the whole path; a Q value of 1e5 (no f16 value) is reported as
    HS2_ERR_RANGE by hs2_sync for the full-attention and the sparse kernel."""
    L, Hq, Hkv = 1536, 8, 2
    wl = _fp8_wl(L, Hq, Hkv, n_sparse=1, seed=37)
    x = inputs.make_inputs(wl)
    rng = np.random.default_rng(3)
    for q in x["q_layers"]:
        big = rng.choice(L * Hq, 200, replace=False)
        tiny = rng.choice(np.setdiff1d(np.arange(L * Hq), big), 200, replace=False)
        flat = q.view(L * Hq, 128)
        flat[big, 0] = 6.0e4
        flat[big, 1] = -6.0e4
        flat[tiny] = (flat[tiny].float() * 2.0 ** -20).to(torch.bfloat16)
    xd = H.to_dev(x, DEV)
    r = H.run_path(wl, xd)
    D = H.decode(x)
    O, LSE = orc.dense_attn(D["Q"][0], D["K"], D["V"])
    H.bf16_close(r["o"].float().cpu().numpy(), O, "O (Q at the f16 edges)")
    assert (np.abs(r["lse"].cpu().numpy() - LSE) <= H.LSE_ATOL + 1e-6 * np.abs(LSE)).all()
    nb = L // 64
    imp = H.gpu_importance(r["shape"], xd, r["lse"], 0, nb).cpu().numpy().astype(np.float64)
    idx, cnt = r["idx"].cpu().numpy(), r["cnt"].cpu().numpy()
    ref_sp = np.empty((L, Hq, 128))
    for b in range(nb):
        s_b, e_b = orc.block_rows(b, L, 64)
        for g in range(Hkv):
            n_c = orc.n_candidates(e_b, 128)
            want, wc = orc.select(imp[g, b, :n_c], wl.topk, 128, e_b)
            assert cnt[g, b] == wc and np.array_equal(idx[g, b], want), (g, b)
            ref_sp[s_b:e_b, g * 4:(g + 1) * 4] = orc.sparse_attn(D["Q"][1], D["K"], D["V"], idx[g, b], wc, b, g, 64)
    H.bf16_close(r["sparse"][0].float().cpu().numpy(), ref_sp, "sparse (Q at the f16 edges)")

    bad = [q.clone() for q in xd["q_layers"]]
    for q in bad:
        q[100, 3, 17] = 1.0e5
    o = torch.empty_like(bad[0])
    lse = torch.empty((Hq, L), device=DEV)
    hs2.hs2_attn_fwd(r["shape"], bad[0], xd["k"], xd["v"], xd["k_scale"], xd["v_scale"], o, lse)
    with pytest.raises(hs2.Hs2Error) as e:
        hs2.hs2_sync()
    assert e.value.code == hs2.HS2_ERR_RANGE
    hs2.hs2_sparse_attn(r["shape"], bad[1], xd["k"], xd["v"], xd["k_scale"], xd["v_scale"], r["idx"], r["cnt"], o)
    with pytest.raises(hs2.Hs2Error) as e:
        hs2.hs2_sync()
    assert e.value.code == hs2.HS2_ERR_RANGE
    hs2.hs2_sync()   # the status was cleared


@pytest.mark.parametrize("L,Hq,Hkv", [(2304, 8, 1), (1536, 4, 2)])
def test_fp8_importance_select_and_sparse_match_oracle(L, Hq, Hkv):
    wl = _fp8_wl(L, Hq, Hkv, n_sparse=1, topk=1000)
    x = inputs.make_inputs(wl)
    xd = H.to_dev(x, DEV)
    r = H.run_path(wl, xd, guards=True)
    nb = L // 64
    imp = H.gpu_importance(r["shape"], xd, r["lse"], 0, nb).cpu().numpy().astype(np.float64)
    D = H.decode(x)
    _, LSE = orc.dense_attn(D["Q"][0], D["K"], D["V"])
    idx, cnt = r["idx"].cpu().numpy(), r["cnt"].cpu().numpy()
    G = wl.G
    ref_sp = np.empty((L, Hq, 128))
    worst = 0.0
    for b in range(nb):
        s_b, e_b = orc.block_rows(b, L, 64)
        for g in range(Hkv):
            ref = orc.importance(D["Q"][0], D["K"], LSE[:, s_b:e_b], b, g, 64, 128)
            got = imp[g, b, :ref.size]
            if ref.size:
                worst = max(worst, (np.abs(got - ref) / np.maximum(np.abs(ref), 1e-30)).max())
            want, wc = orc.select(got, wl.topk, 128, e_b)
            assert cnt[g, b] == wc and np.array_equal(idx[g, b], want), (g, b)
            ref_sp[s_b:e_b, g * G:(g + 1) * G] = orc.sparse_attn(D["Q"][1], D["K"], D["V"], idx[g, b], wc, b, g, 64)
    assert worst <= H.IMP_RTOL, worst
    H.bf16_close(r["sparse"][0].float().cpu().numpy(), ref_sp, "sparse (fp8 cache)")
    assert all(H.guards_intact(bb) for bb in r["bases"])


@pytest.mark.parametrize("L,Hq,Hkv", [(2368, 8, 1), (1088, 8, 2), (3072, 16, 2)])
def test_fp8_layer_copy_equals_in_kernel_conversion(L, Hq, Hkv):
    """hs2_full_attn_select converts an e4m3 cache to f16 once per layer when
    the workspace also holds that copy, and inside kernels (1) and (2)
    otherwise: both must give the same bits (O, LSE, lists), and the same O /
    LSE as hs2_attn_fwd, which always converts in the kernel."""
    wl = _fp8_wl(L, Hq, Hkv, n_sparse=0, seed=37, topk=1000)
    xd = H.to_dev(inputs.make_inputs(wl), DEV)
    shape = H.shape_of(wl, xd)
    q0, k, v, ks, vs = xd["q_layers"][0], xd["k"], xd["v"], xd["k_scale"], xd["v_scale"]
    nb = L // 64
    ws_min = Hkv * ((L - 128 + 63) // 64 * 64) * 4
    ws_rec = hs2.workspace_bytes(shape)
    assert ws_rec >= ws_min + 2 * L * Hkv * 128 * 2  # room for the f16 copy
    outs = []
    for nbytes in (ws_min, ws_rec):
        o, lse = torch.empty_like(q0), torch.empty((Hq, L), device=DEV, dtype=torch.float32)
        idx = torch.empty((Hkv, nb, wl.topk + wl.recent), device=DEV, dtype=torch.int32)
        cnt = torch.empty((Hkv, nb), device=DEV, dtype=torch.int32)
        ws = torch.empty(nbytes // 4, device=DEV, dtype=torch.float32)
        hs2.hs2_full_attn_select(shape, q0, k, v, ks, vs, o, lse, idx, cnt, ws)
        hs2.hs2_sync()
        outs.append((o, lse, idx, cnt))
    for a, b in zip(*outs):
        assert torch.equal(a, b)
    o1, lse1 = torch.empty_like(q0), torch.empty((Hq, L), device=DEV, dtype=torch.float32)
    hs2.hs2_attn_fwd(shape, q0, k, v, ks, vs, o1, lse1)
    hs2.hs2_sync()
    assert torch.equal(o1, outs[1][0]) and torch.equal(lse1, outs[1][1])
    # kernel (1) alone through the layer copy (hs2_attn_fwd_ws)
    ws1 = torch.empty(hs2.attn_fwd_workspace_bytes(shape) // 4 + 4, device=DEV, dtype=torch.float32)
    o2, lse2 = torch.empty_like(q0), torch.empty((Hq, L), device=DEV, dtype=torch.float32)
    hs2.hs2_attn_fwd_ws(shape, q0, k, v, ks, vs, o2, lse2, ws1)
    hs2.hs2_sync()
    assert torch.equal(o2, o1) and torch.equal(lse2, lse1)
    # a workspace too small for the copy: the kernel converts the tiles itself
    o3, lse3 = torch.empty_like(q0), torch.empty((Hq, L), device=DEV, dtype=torch.float32)
    hs2.hs2_attn_fwd_ws(shape, q0, k, v, ks, vs, o3, lse3, torch.empty(4, device=DEV, dtype=torch.float32))
    hs2.hs2_sync()
    assert torch.equal(o3, o1) and torch.equal(lse3, lse1)


@pytest.mark.parametrize("L,Hq,Hkv", [(4096, 8, 2), (2560, 16, 2)])
def test_strip_sizes_do_not_change_the_result(L, Hq, Hkv):
    """The full-layer call groups query blocks into strips that fit the
    workspace: the minimum (one block per strip), a few blocks per strip, and
    the recommended size must all give the same bits."""
    wl = _wl(L, Hq, Hkv, n_sparse=0, seed=41)
    xd = H.to_dev(inputs.make_inputs(wl), DEV)
    shape = H.shape_of(wl, xd)
    q0, k, v = xd["q_layers"][0], xd["k"], xd["v"]
    nb = L // 64
    row = (L - 128 + 63) // 64 * 64 * 4
    outs = []
    for nbytes in (Hkv * row, 5 * Hkv * row + 64, hs2.workspace_bytes(shape)):
        o, lse = torch.empty_like(q0), torch.empty((Hq, L), device=DEV, dtype=torch.float32)
        idx = torch.empty((Hkv, nb, wl.topk + wl.recent), device=DEV, dtype=torch.int32)
        cnt = torch.empty((Hkv, nb), device=DEV, dtype=torch.int32)
        ws = torch.empty(nbytes // 4, device=DEV, dtype=torch.float32)
        hs2.hs2_full_attn_select(shape, q0, k, v, None, None, o, lse, idx, cnt, ws)
        hs2.hs2_sync()
        outs.append((o, lse, idx, cnt))
    for other in outs[1:]:
        for a, b in zip(outs[0], other):
            assert torch.equal(a, b)


# -------------------------------------------------- device-side failures --

def test_bounded_wait_reports_timeout_and_context_survives():
    """The load role issues nothing (test flag), so the other roles' bounded
    waits run out: hs2_sync reports HS2_ERR_TIMEOUT, and the next call works."""
    wl = _wl(256, 4, 2, seed=23)
    x = inputs.make_inputs(wl)
    xd = H.to_dev(x, DEV)
    shape = hs2.make_shape(xd["q_layers"][0], xd["k"])
    o = torch.empty_like(xd["q_layers"][0])
    lse = torch.empty((4, 256), device=DEV)
    hs2.hs2_debug_set(50_000_000, 1)
    try:
        hs2.hs2_attn_fwd(shape, xd["q_layers"][0], xd["k"], xd["v"], None, None, o, lse)
        with pytest.raises(hs2.Hs2Error) as e:
            hs2.hs2_sync()
        assert e.value.code == hs2.HS2_ERR_TIMEOUT
    finally:
        hs2.hs2_debug_set(H.WAIT_LIMIT_NS, 0)
    hs2.hs2_attn_fwd(shape, xd["q_layers"][0], xd["k"], xd["v"], None, None, o, lse)
    hs2.hs2_sync()
    D = H.decode(x)
    O, _ = orc.dense_attn(D["Q"][0], D["K"], D["V"])
    H.bf16_close(o.float().cpu().numpy(), O, "O after timeout")


def test_host_tensor_map_failure_returns_before_any_launch():
    """Host-side fault injection (hs2_debug_set bit 3): every TMA descriptor
    encoding fails as a driver error would.  Each call returns HS2_ERR_CUDA
    without launching a kernel or touching its outputs, and once the hook is
    cleared the same calls work."""
    wl = _wl(1024, 8, 2, seed=31)
    x = inputs.make_inputs(wl)
    xd = H.to_dev(x, DEV)
    r = H.run_path(wl, xd)  # lists for the sparse call
    q0, k, v = xd["q_layers"][0], xd["k"], xd["v"]
    shape = r["shape"]
    o = torch.full_like(q0, 7.0)
    lse = torch.full((wl.Hq, wl.L), 7.0, device=DEV)
    idx = torch.full_like(r["idx"], 7)
    cnt = torch.full_like(r["cnt"], 7)
    ws = torch.empty(hs2.workspace_bytes(shape) // 4 + 4, device=DEV, dtype=torch.float32)
    torch.cuda.synchronize()
    n0 = hs2.hs2_launch_count()
    hs2.hs2_debug_set(H.WAIT_LIMIT_NS, hs2.DEBUG_FAIL_TMAP)
    try:
        calls = [
            lambda: hs2.hs2_attn_fwd(shape, q0, k, v, None, None, o, lse),
            lambda: hs2.hs2_full_attn_select(shape, q0, k, v, None, None, o, lse, idx, cnt, ws),
            lambda: hs2.hs2_sparse_attn(shape, xd["q_layers"][1], k, v, None, None, r["idx"], r["cnt"], o),
            lambda: hs2.hs2_swa_attn(shape, q0, k, v, 128, o, lse),
        ]
        for call in calls:
            with pytest.raises(hs2.Hs2Error) as e:
                call()
            assert e.value.code == hs2.HS2_ERR_CUDA
    finally:
        hs2.hs2_debug_set(H.WAIT_LIMIT_NS, 0)
    torch.cuda.synchronize()
    assert hs2.hs2_launch_count() == n0
    assert bool((o == 7.0).all()) and bool((lse == 7.0).all())
    assert bool((idx == 7).all()) and bool((cnt == 7).all())
    hs2.hs2_full_attn_select(shape, q0, k, v, None, None, o, lse, idx, cnt, ws)
    hs2.hs2_sync()
    assert torch.equal(o, r["o"]) and torch.equal(lse, r["lse"])
    assert torch.equal(idx, r["idx"]) and torch.equal(cnt, r["cnt"])


def test_out_of_range_list_entries_are_reported_not_read():
    """Listed positions outside [0, e_b) are never dereferenced: the gather
    zero-fills them, the softmax masks them, and hs2_sync reports
    HS2_ERR_INDEX; the remaining entries give the right answer."""
    L, Hq, Hkv = 512, 4, 2
    wl = _wl(L, Hq, Hkv, seed=29)
    x = inputs.make_inputs(wl)
    xd = H.to_dev(x, DEV)
    r = H.run_path(wl, xd)
    idx = r["idx"].clone()
    b = 5
    idx[1, b, 3] = 64 * (b + 1) + 7       # beyond the block end
    idx[1, b, 10] = -5                    # negative
    o = torch.empty_like(xd["q_layers"][1])
    hs2.hs2_sparse_attn(r["shape"], xd["q_layers"][1], xd["k"], xd["v"], None, None, idx, r["cnt"], o)
    with pytest.raises(hs2.Hs2Error) as e:
        hs2.hs2_sync()
    assert e.value.code == hs2.HS2_ERR_INDEX
    D = H.decode(x)
    lst = idx[1, b].cpu().numpy()
    c = int(r["cnt"][1, b])
    keep = lst[:c][(lst[:c] >= 0) & (lst[:c] < 64 * (b + 1))]
    ref = orc.sparse_attn(D["Q"][1], D["K"], D["V"], keep, keep.size, b, 1, 64)
    H.bf16_close(o[64 * b:64 * (b + 1), 2:4].float().cpu().numpy(), ref, "masked bad entries")
    hs2.hs2_sync()   # status was cleared
