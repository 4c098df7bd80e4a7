"""Pins for the fp64 oracle against things other than itself: library routines
(torch SDPA in float64, torch dtype conversions), closed forms, hand-derived
golden values, invariants and brute force on tiny inputs.  Each check is a
function of the oracle routine it pins, so the planted-mistake tests at the end
can show that a plausible bug in the oracle fails the pin."""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import hs2_oracle as orc


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _sdpa(Q, K, V, mask=None, causal=False):
    """torch SDPA in float64 on [L][H][d] arrays (GQA with contiguous groups)."""
    q = torch.from_numpy(Q).permute(1, 0, 2)[None]
    k = torch.from_numpy(K).permute(1, 0, 2)[None]
    v = torch.from_numpy(V).permute(1, 0, 2)[None]
    m = None if mask is None else torch.from_numpy(mask)
    o = F.scaled_dot_product_attention(q, k, v, attn_mask=m, is_causal=causal, enable_gqa=True)
    return o[0].permute(1, 0, 2).numpy()


# ------------------------------------------------------------------ decode --

def test_decode_bf16_all_patterns():
    u = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(u.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = orc.decode_bf16(u)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_decode_e4m3_all_codes():
    u = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(u).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = orc.decode_e4m3(u)
    nan = np.isnan(ref)
    assert nan.sum() == 2                       # S.1111.111 only
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9


# ------------------------------------------------------------ dense attn --

def check_dense_vs_sdpa(dense_fn, L=97, Hq=6, Hkv=2, d=32, seed=1):
    Q, K, V = _rand((L, Hq, d), seed), _rand((L, Hkv, d), seed + 1), _rand((L, Hkv, d), seed + 2)
    O, _ = dense_fn(Q, K, V)
    return np.abs(O - _sdpa(Q, K, V, causal=True)).max()


def check_lse_vs_sdpa_onehot(dense_fn, L=40, Hq=4, Hkv=2, d=48, seed=3):
    """exp(s_ij - lse_i) must equal the attention probability P_ij, which SDPA
    returns when the values are one-hot position vectors (d >= L)."""
    Q, K = _rand((L, Hq, d), seed), _rand((L, Hkv, d), seed + 1)
    E = np.zeros((L, Hkv, d))
    E[np.arange(L), :, np.arange(L)] = 1.0
    P = _sdpa(Q, K, E, causal=True)[:, :, :L]          # [i][h][j]
    _, lse = dense_fn(Q, K, E)
    G = Hq // Hkv
    err = 0.0
    for h in range(Hq):
        s = Q[:, h] @ K[:, h // G].T / math.sqrt(d)
        p = np.tril(np.exp(s - lse[h][:, None]))
        err = max(err, np.abs(p - P[:, h, :]).max())
    return err


def test_dense_matches_sdpa():
    assert check_dense_vs_sdpa(orc.dense_attn) < 1e-12
    assert check_dense_vs_sdpa(orc.dense_attn, L=64, Hq=8, Hkv=1, d=128, seed=9) < 1e-12


def test_dense_row_range_matches_full():
    Q, K, V = _rand((130, 4, 16), 4), _rand((130, 2, 16), 5), _rand((130, 2, 16), 6)
    O, lse = orc.dense_attn(Q, K, V)
    O2, lse2 = orc.dense_attn(Q, K, V, 64, 128)
    assert np.abs(O[64:128] - O2).max() < 1e-13 and np.abs(lse[:, 64:128] - lse2).max() < 1e-13


def test_lse_matches_sdpa_probabilities():
    assert check_lse_vs_sdpa_onehot(orc.dense_attn) < 1e-12


def test_dense_naive_loop():
    """Triple loop in pure Python with math.exp at L <= 16."""
    L, Hq, Hkv, d = 12, 4, 2, 8
    Q, K, V = _rand((L, Hq, d), 7), _rand((L, Hkv, d), 8), _rand((L, Hkv, d), 9)
    O, lse = orc.dense_attn(Q, K, V)
    G = Hq // Hkv
    for h in range(Hq):
        for i in range(L):
            sc = [sum(Q[i, h, c] * K[j, h // G, c] for c in range(d)) / math.sqrt(d) for j in range(i + 1)]
            z = sum(math.exp(x) for x in sc)
            assert abs(lse[h, i] - math.log(z)) < 1e-12
            for c in range(d):
                o = sum(math.exp(sc[j]) / z * V[j, h // G, c] for j in range(i + 1))
                assert abs(O[i, h, c] - o) < 1e-12


def test_dense_invariants():
    Q, K, V = _rand((70, 2, 16), 11), _rand((70, 1, 16), 12), _rand((70, 1, 16), 13)
    _, lse = orc.dense_attn(Q, K, V)
    for h in range(2):
        s = np.tril(Q[:, h] @ K[:, 0].T / 4.0) + np.triu(np.full((70, 70), -np.inf), 1)
        mx = s.max(axis=1)
        assert np.all(lse[h] >= mx - 1e-12)
        assert np.all(lse[h] <= mx + np.log(np.arange(1, 71)) + 1e-12)


def test_handworked_golden(golden_dir):
    with open(os.path.join(golden_dir, "handworked_attention.json")) as f:
        gd = json.load(f)
    num = lambda x: math.log(3) if x == "ln3" else (math.log(4) if x == "ln4" else float(x))
    Q = np.array([[[num(x) for x in r]] for r in gd["q"]])
    K = np.array([[[num(x) for x in r]] for r in gd["k"]])
    V = np.array([[[num(x) for x in r]] for r in gd["v"]])
    O, lse = orc.dense_attn(Q, K, V)
    assert np.abs(O[:, 0, :] - np.array(gd["o"], dtype=float)).max() < 1e-15
    assert np.abs(lse[0] - np.array([num(x) for x in gd["lse"]])).max() < 1e-15
    I = orc.importance(Q, K, lse, 0, 0, B=2, w=0, scope="visible")
    assert np.abs(I - np.array(gd["importance_visible_block0_B2"])).max() < 1e-15


# ------------------------------------------------------------- importance --

def check_importance_vs_sdpa(imp_fn, L=128, Hq=4, Hkv=2, d=128, B=16, w=32, seed=21):
    """Sum of SDPA one-hot probabilities over the block's rows and the group's
    heads equals the importance row."""
    Q, K = _rand((L, Hq, d), seed), _rand((L, Hkv, d), seed + 1)
    E = np.zeros((L, Hkv, d))
    E[np.arange(L), :, np.arange(L)] = 1.0
    P = _sdpa(Q, K, E, causal=True)[:, :, :L]
    _, lse = orc.dense_attn(Q, K, E)
    G = Hq // Hkv
    err = 0.0
    for b in range((L + B - 1) // B):
        s_b, e_b = orc.block_rows(b, L, B)
        for g in range(Hkv):
            ref = P[s_b:e_b, g * G:(g + 1) * G, :].sum(axis=(0, 1))
            got_v = imp_fn(Q, K, lse[:, s_b:e_b], b, g, B, w, scope="visible")
            got_c = imp_fn(Q, K, lse[:, s_b:e_b], b, g, B, w)
            nc = orc.n_candidates(e_b, w)
            err = max(err, np.abs(got_v - ref[:e_b]).max(),
                      np.abs(got_c - ref[:nc]).max() if nc else 0.0)
    return err


def test_importance_matches_sdpa_probabilities():
    assert check_importance_vs_sdpa(orc.importance) < 1e-12
    assert check_importance_vs_sdpa(orc.importance, L=100, Hq=6, Hkv=3, B=32, w=8, seed=5) < 1e-12


@pytest.mark.parametrize("L,Hq,Hkv,B,w", [(256, 4, 1, 64, 128), (200, 8, 2, 64, 128), (90, 4, 2, 16, 16)])
def test_importance_mass_conservation(L, Hq, Hkv, B, w):
    """Summed over every visible key, the block's importance is rows * G."""
    d = 32
    Q, K, V = _rand((L, Hq, d), L), _rand((L, Hkv, d), L + 1), _rand((L, Hkv, d), L + 2)
    _, lse = orc.dense_attn(Q, K, V)
    G = Hq // Hkv
    for b in range((L + B - 1) // B):
        s_b, e_b = orc.block_rows(b, L, B)
        for g in range(Hkv):
            I = orc.importance(Q, K, lse[:, s_b:e_b], b, g, B, w, scope="visible")
            assert abs(I.sum() - (e_b - s_b) * G) < 1e-12 * (e_b - s_b) * G


def test_importance_identical_keys_closed_form():
    """All keys equal: p_ij = 1 / (i + 1), so every candidate gets
    G * sum_{i in block} 1 / (i + 1)."""
    L, Hq, Hkv, d, B, w = 384, 4, 2, 16, 64, 128
    Q = _rand((L, Hq, d), 31)
    K = np.broadcast_to(_rand((1, Hkv, d), 32), (L, Hkv, d)).copy()
    _, lse = orc.dense_attn(Q, K, K)
    G = Hq // Hkv
    for b in range(L // B):
        s_b, e_b = orc.block_rows(b, L, B)
        want = G * sum(1.0 / (i + 1) for i in range(s_b, e_b))
        for g in range(Hkv):
            I = orc.importance(Q, K, lse[:, s_b:e_b], b, g, B, w)
            assert I.size == orc.n_candidates(e_b, w)
            if I.size:
                assert np.abs(I - want).max() < 1e-12


# --------------------------------------------------------------- select --

def check_select_brute(select_fn, seed=0):
    """Return the number of mismatches between select and the brute-force
    rank definition on tiny rows with many ties (k = 64, w = 16, B = 16)."""
    rng = np.random.default_rng(seed)
    k, w, B = 64, 16, 16
    bad = 0
    for L in (16, 17, 40, 96, 100, 200, 512):
        for b in range((L + B - 1) // B):
            _, e_b = orc.block_rows(b, L, B)
            n_c = orc.n_candidates(e_b, w)
            I = rng.integers(0, 7, size=n_c).astype(np.float64) / 4.0   # many ties
            idx, cnt = select_fn(I, k, w, e_b)
            rank = orc.brute_rank(I)
            want = sorted([j for j in range(n_c) if rank[j] < k] + list(range(max(0, e_b - w), e_b)))
            got = list(idx[:cnt])
            bad += int(got != want) + int(np.any(idx[cnt:] != -1))
    return bad


def test_select_brute_force_rank():
    for seed in range(4):
        assert check_select_brute(orc.select, seed) == 0


def test_select_all_equal_takes_first_positions():
    k, w = 1024, 128
    e_b = 4096
    idx, cnt = orc.select(np.ones(e_b - w), k, w, e_b)
    assert cnt == k + w
    assert np.array_equal(idx[:k], np.arange(k))
    assert np.array_equal(idx[k:cnt], np.arange(e_b - w, e_b))


def test_select_invariants_and_golden_sizes(golden_dir):
    with open(os.path.join(golden_dir, "list_sizes_L2048.json")) as f:
        gd = json.load(f)
    L, B, k, w = gd["L"], gd["block"], gd["topk"], gd["recent"]
    rng = np.random.default_rng(3)
    for b in range(L // B):
        _, e_b = orc.block_rows(b, L, B)
        I = rng.random(orc.n_candidates(e_b, w))
        idx, cnt = orc.select(I, k, w, e_b)
        v = idx[:cnt]
        assert cnt == orc.list_size(e_b, k, w) <= gd["max_size"] == k + w
        if str(b) in gd["sizes_by_block"]:
            assert cnt == gd["sizes_by_block"][str(b)]
        assert np.all(np.diff(v) > 0) and v[0] >= 0 and v[-1] == e_b - 1
        assert set(range(max(0, e_b - w), e_b)) <= set(v.tolist())
        assert np.all(idx[cnt:] == -1)


def test_select_scaled_with_w_below_block():
    """w < B exercises the general causal path of importance and sparse attn."""
    L, Hq, Hkv, d, B, k, w = 160, 4, 2, 16, 64, 24, 16
    Q, K, V = _rand((L, Hq, d), 41), _rand((L, Hkv, d), 42), _rand((L, Hkv, d), 43)
    for b in range(L // B):
        for g in range(Hkv):
            r = orc.full_attn_select_block(Q, K, V, b, g, B, k, w)
            rank = orc.brute_rank(r["I"])
            _, e_b = orc.block_rows(b, L, B)
            want = sorted([j for j in range(r["I"].size) if rank[j] < k] + list(range(max(0, e_b - w), e_b)))
            assert list(r["idx"][:r["cnt"]]) == want


# ---------------------------------------------------------- sparse attn --

def check_sparse_vs_masked_sdpa(sparse_fn, L=150, Hq=4, Hkv=2, d=16, B=32, seed=51):
    """Random sorted index lists: sparse attention equals SDPA with an explicit
    boolean mask (listed and causal)."""
    rng = np.random.default_rng(seed)
    Q, K, V = _rand((L, Hq, d), seed), _rand((L, Hkv, d), seed + 1), _rand((L, Hkv, d), seed + 2)
    G = Hq // Hkv
    err = 0.0
    for b in range((L + B - 1) // B):
        s_b, e_b = orc.block_rows(b, L, B)
        for g in range(Hkv):
            extra = rng.choice(max(1, s_b), size=min(s_b, 7), replace=False) if s_b else np.array([], int)
            pos = np.unique(np.concatenate([extra, np.arange(s_b, e_b)])).astype(np.int64)
            idx = np.concatenate([pos, -np.ones(5, np.int64)])
            got = sparse_fn(Q, K, V, idx, pos.size, b, g, B)
            mask = np.zeros((e_b - s_b, L), bool)
            mask[:, pos] = True
            mask &= np.arange(L)[None, :] <= np.arange(s_b, e_b)[:, None]
            mask = np.broadcast_to(mask[None], (G, e_b - s_b, L)).copy()
            qg = Q[s_b:e_b, g * G:(g + 1) * G]
            ref = _sdpa(qg, K[:, g:g + 1], V[:, g:g + 1], mask=mask)
            err = max(err, np.abs(got - ref).max())
    return err


def test_sparse_matches_masked_sdpa():
    assert check_sparse_vs_masked_sdpa(orc.sparse_attn) < 1e-12


@pytest.mark.parametrize("L", [1152, 700])
def test_sparse_equals_dense_when_list_is_everything(L):
    """L <= k + w = 1152: every earlier position is selected, so each sparse
    layer reduces to dense causal attention."""
    Hq, Hkv, d, B, k, w = 4, 2, 16, 64, 1024, 128
    Q, K, V = _rand((L, Hq, d), L), _rand((L, Hkv, d), L + 1), _rand((L, Hkv, d), L + 2)
    Q2 = _rand((L, Hq, d), L + 3)
    O2, _ = orc.dense_attn(Q2, K, V)
    G = Hq // Hkv
    for b in range((L + B - 1) // B):
        s_b, e_b = orc.block_rows(b, L, B)
        for g in range(Hkv):
            r = orc.full_attn_select_block(Q, K, V, b, g, B, k, w)
            assert r["cnt"] == e_b and np.array_equal(r["idx"][:e_b], np.arange(e_b))
            o = orc.sparse_attn(Q2, K, V, r["idx"], r["cnt"], b, g, B)
            assert np.abs(o - O2[s_b:e_b, g * G:(g + 1) * G]).max() < 1e-12


def test_sparse_equals_dense_when_k_covers_L():
    L, Hq, Hkv, d, B, k, w = 90, 2, 1, 8, 16, 128, 16
    Q, K, V = _rand((L, Hq, d), 61), _rand((L, Hkv, d), 62), _rand((L, Hkv, d), 63)
    O, _ = orc.dense_attn(Q, K, V)
    for b in range((L + B - 1) // B):
        s_b, e_b = orc.block_rows(b, L, B)
        r = orc.full_attn_select_block(Q, K, V, b, 0, B, k, w)
        o = orc.sparse_attn(Q, K, V, r["idx"], r["cnt"], b, 0, B)
        assert np.abs(o - O[s_b:e_b]).max() < 1e-12


# ------------------------------------------------------ planted mistakes --
# Each mutant is a plausible oracle bug; the pin it targets must reject it.

def _dense_no_scale(Q, K, V, r0=0, r1=None):
    return orc.dense_attn(Q * math.sqrt(Q.shape[2]), K, V, r0, r1)


def _dense_wrong_gqa(Q, K, V, r0=0, r1=None):
    Hq, Hkv = Q.shape[1], K.shape[1]
    perm = [h % Hkv for h in range(Hq)]          # interleaved instead of contiguous groups
    Kx = K[:, perm, :]
    Vx = V[:, perm, :]
    return orc.dense_attn(Q, Kx, Vx, r0, r1)


def _dense_lse_log2(Q, K, V, r0=0, r1=None):
    O, lse = orc.dense_attn(Q, K, V, r0, r1)
    return O, lse / math.log(2.0)


def _importance_unnormalised(Q, K, lse_block, b, g, B, w, scope="candidates"):
    return orc.importance(Q, K, lse_block * 0.0, b, g, B, w, scope)


def _imp_first_head(Q, K, lse_block, b, g, B, w, scope="candidates"):
    G = Q.shape[1] // K.shape[1]
    Qx = Q.copy()
    for hl in range(1, G):                       # forget every head but the first of the group
        Qx[:, g * G + hl] = Q[:, g * G]
    lx = lse_block.copy()
    for hl in range(1, G):
        lx[g * G + hl] = lse_block[g * G]
    return orc.importance(Qx, K, lx, b, g, B, w, scope)


def _sel_rev(I, k, w, e_b):
    n_c = orc.n_candidates(e_b, w)
    pos = np.arange(n_c)
    order = np.lexsort((-pos, -I))               # ties to the higher position
    top = np.sort(order[:min(n_c, k)])
    chosen = np.concatenate([top, np.arange(max(0, e_b - w), e_b)])
    idx = np.full(k + w, -1, np.int64)
    idx[:chosen.size] = chosen
    return idx, chosen.size


def _select_no_recent(I, k, w, e_b):
    idx, cnt = orc.select(I, k, w, e_b)
    keep = idx[:cnt][idx[:cnt] < e_b - w] if e_b > w else idx[:0]
    out = np.full(k + w, -1, np.int64)
    out[:keep.size] = keep
    return out, keep.size


def _sparse_unmasked(Q, K, V, idx, cnt, b, g, B):
    L, Hq, d = Q.shape
    G = Hq // K.shape[1]
    s_b, e_b = orc.block_rows(b, L, B)
    pos = idx[:cnt]
    O = np.zeros((e_b - s_b, G, d))
    for hl in range(G):
        s = Q[s_b:e_b, g * G + hl] @ K[pos, g].T / math.sqrt(d)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        O[:, hl] = p @ V[pos, g] / p.sum(axis=1, keepdims=True)
    return O


def test_planted_mistakes_are_caught():
    assert check_dense_vs_sdpa(_dense_no_scale) > 1e-3
    assert check_dense_vs_sdpa(_dense_wrong_gqa, Hq=4, Hkv=2) > 1e-3
    assert check_lse_vs_sdpa_onehot(_dense_lse_log2) > 1e-3
    assert check_importance_vs_sdpa(_importance_unnormalised) > 1e-3
    assert check_importance_vs_sdpa(_imp_first_head) > 1e-3
    assert check_select_brute(_sel_rev) > 0
    assert check_select_brute(_select_no_recent) > 0
    assert check_sparse_vs_masked_sdpa(_sparse_unmasked) > 1e-3


# ------------------------------------------------------------ FP8 KV write --

def test_encode_e4m3_matches_torch_round_to_nearest_even():
    rng = np.random.default_rng(7)
    y = np.concatenate([rng.standard_normal(200_000) * 100, rng.uniform(-448, 448, 200_000),
                        rng.uniform(-2.0 ** -6, 2.0 ** -6, 50_000)]).astype(np.float32)
    grid = orc.decode_e4m3(np.arange(0x7F, dtype=np.uint8))
    mids = ((grid[1:] + grid[:-1]) / 2).astype(np.float32)        # exact ties (representable in fp32)
    y = np.concatenate([y, mids, -mids, [0.0, -0.0, 2.0 ** -11, -(2.0 ** -11)]]).astype(np.float32)
    y = np.clip(y, -448, 448)
    ref = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = orc.encode_e4m3(y)
    assert np.array_equal(got, ref)


def test_encode_decode_roundtrip_and_saturation():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = orc.decode_e4m3(codes)
    back = orc.encode_e4m3(vals)
    assert np.array_equal(orc.decode_e4m3(back), vals)
    assert orc.decode_e4m3(orc.encode_e4m3(np.array([1e6, -1e6, 449.0])))[0] == 448.0
    assert orc.decode_e4m3(orc.encode_e4m3(np.array([-1e6])))[0] == -448.0


def test_quantize_kv_row_definition():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((64, 3, 128)).astype(np.float32)
    x[5, 1] = 0.0
    codes, scale = orc.quantize_kv(x)
    assert scale.dtype == np.float32 and scale[5, 1] == 1.0
    amax = np.abs(x).max(axis=-1)
    nz = amax > 0
    assert np.array_equal(scale[nz], (amax / np.float32(448)).astype(np.float32)[nz])
    deq = orc.dequantize(codes, scale)
    # every element within half an e4m3 step of its value; the row max lands on 448 * scale
    assert np.all(np.abs(deq - x) <= np.abs(x) * 2.0 ** -4 + scale[..., None] * 2.0 ** -9 + 1e-12)
    top = np.abs(x).argmax(axis=-1)
    assert np.all(np.abs(np.take_along_axis(orc.decode_e4m3(codes), top[..., None], -1)[..., 0][nz]) == 448.0)


# ------------------------------------------------ block-level selection (v1) --

def _fsum_blocks(I, B=64):
    """Correctly rounded per-block sums by math.fsum over plain Python floats:
    a routine that shares nothing with the oracle's vectorised float64 sum."""
    vals = [float(x) for x in np.asarray(I, np.float32)]
    return [math.fsum(vals[m * B:(m + 1) * B]) for m in range(len(vals) // B)]


def test_pool_blocks_is_the_block_sum():
    rng = np.random.default_rng(9)
    for I in (rng.random(64 * 37).astype(np.float32),
              np.exp(-rng.random(64 * 23) * 80).astype(np.float32),     # 35 binades in one block
              (rng.integers(0, 5, 64 * 11) / 8).astype(np.float32)):
        J = orc.pool_blocks(I)
        ref = np.array(_fsum_blocks(I))
        assert J.dtype == np.float64 and np.all(np.abs(J - ref) <= 1e-14 * ref)
    Iz = np.zeros(64 * 3, np.float32)
    Iz[64 + 7] = 3.0
    assert list(orc.pool_blocks(Iz)) == [0.0, 3.0, 0.0]


def check_select_blocks_brute(sel_fn, seed=0):
    """Brute force at block granularity: block m is kept iff fewer than k/64
    blocks beat it (higher pooled value, or equal and lower index), with the
    pooled values from math.fsum."""
    rng = np.random.default_rng(seed)
    k, w, B = 256, 128, 64
    bad = 0
    for L in (128, 192, 512, 1024, 2048):
        for b in range(L // B):
            e_b = B * (b + 1)
            n_c = orc.n_candidates(e_b, w)
            if seed % 2:
                I = (rng.integers(0, 3, n_c) / 2.0).astype(np.float32)       # many exact block ties
            else:
                I = rng.random(n_c).astype(np.float32)
            idx, cnt = sel_fn(I, k, w, e_b)
            J = _fsum_blocks(I)
            nbk = len(J)
            rank = [sum(1 for m2 in range(nbk) if J[m2] > J[m] or (J[m2] == J[m] and m2 < m)) for m in range(nbk)]
            want = [p for m in range(nbk) if rank[m] < k // B for p in range(m * B, (m + 1) * B)]
            want += list(range(max(0, e_b - w), e_b))
            bad += int(list(idx[:cnt]) != want) + int(np.any(idx[cnt:] != -1))
    return bad


def test_select_blocks_brute_force_and_sizes():
    for seed in range(3):
        assert check_select_blocks_brute(orc.select_blocks, seed) == 0
    e_b = 4096
    idx, cnt = orc.select_blocks(np.ones(e_b - 128, np.float32), 1024, 128, e_b)
    assert cnt == 1152 and np.array_equal(idx[:1024], np.arange(1024))          # ties -> lowest blocks
    assert cnt == orc.list_size(e_b, 1024, 128)


def test_select_blocks_planted_mistake_is_caught():
    def ties_high(I, k, w, e_b, B=64):
        n_c = orc.n_candidates(e_b, w)
        J = orc.pool_blocks(I) if n_c else np.zeros(0)
        m = np.arange(J.size)
        keep = np.sort(np.lexsort((-m, -J))[:min(J.size, k // B)])
        top = (keep[:, None] * B + np.arange(B)[None, :]).reshape(-1)
        ch = np.concatenate([top, np.arange(max(0, e_b - w), e_b)])
        idx = np.full(k + w, -1, np.int64)
        idx[:ch.size] = ch
        return idx, ch.size
    assert check_select_blocks_brute(ties_high, seed=1) > 0

    def first_value_only(I, k, w, e_b, B=64):        # pools by the block's first key instead of its sum
        n_c = orc.n_candidates(e_b, w)
        J = np.asarray(I, np.float64)[::B] if n_c else np.zeros(0)
        keep = np.sort(np.lexsort((np.arange(J.size), -J))[:min(J.size, k // B)])
        ch = np.concatenate([(keep[:, None] * B + np.arange(B)[None, :]).reshape(-1),
                             np.arange(max(0, e_b - w), e_b)])
        idx = np.full(k + w, -1, np.int64)
        idx[:ch.size] = ch
        return idx, ch.size
    assert check_select_blocks_brute(first_value_only, seed=0) > 0


# ------------------------------------------------- sliding-window attention --

def test_swa_matches_sdpa_with_band_mask():
    L, Hq, Hkv, d = 150, 4, 2, 16
    Q, K, V = _rand((L, Hq, d), 71), _rand((L, Hkv, d), 72), _rand((L, Hkv, d), 73)
    for W in (1, 7, 64, 128):
        O, lse = orc.swa_attn(Q, K, V, W)
        i, j = np.arange(L)[:, None], np.arange(L)[None, :]
        band = np.broadcast_to((j <= i) & (j > i - W), (Hq, L, L)).copy()
        assert np.abs(O - _sdpa(Q, K, V, mask=band)).max() < 1e-12
    O1, _ = orc.swa_attn(Q, K, V, 1)                 # each query sees only itself
    G = Hq // Hkv
    assert np.abs(O1 - V[:, np.arange(Hq) // G, :]).max() < 1e-15
    Ofull, lfull = orc.swa_attn(Q, K, V, L)         # window >= L is plain causal attention
    Od, ld = orc.dense_attn(Q, K, V)
    assert np.abs(Ofull - Od).max() < 1e-13 and np.abs(lfull - ld).max() < 1e-13


# ------------------------------------------------ decode-step sparse attention --

def _full_lists(L, Hkv, B):
    """Lists holding every position of [0, e_b): the case k >= L."""
    nb = L // B
    idx = np.full((Hkv, nb, L), -1, dtype=np.int64)
    cnt = np.zeros((Hkv, nb), dtype=np.int64)
    for b in range(nb):
        e = B * (b + 1)
        idx[:, b, :e] = np.arange(e)
        cnt[:, b] = e
    return idx, cnt


def test_decode_with_full_lists_is_causal_attention_rows():
    L, Hq, Hkv, d, B = 192, 4, 2, 16, 64
    Q, K, V = _rand((L, Hq, d), 81), _rand((L, Hkv, d), 82), _rand((L, Hkv, d), 83)
    idx, cnt = _full_lists(L, Hkv, B)
    pos = np.array([0, 1, 63, 64, 100, 191])
    O = orc.sparse_decode(Q[pos], pos, K, V, idx, cnt, B)
    ref = _sdpa(Q, K, V, causal=True)[pos]
    assert np.abs(O - ref).max() < 1e-12


def test_decode_rows_equal_the_block_sparse_layer():
    """Any query of block b, decoded on its own, gets the row the prefill
    sparse layer computes for it from the same list."""
    L, Hq, Hkv, d, B = 256, 8, 2, 16, 64
    Q, K, V = _rand((L, Hq, d), 84), _rand((L, Hkv, d), 85), _rand((L, Hkv, d), 86)
    rng = np.random.default_rng(87)
    nb, width = L // B, 160
    idx = np.full((Hkv, nb, width), -1, dtype=np.int64)
    cnt = np.zeros((Hkv, nb), dtype=np.int64)
    for g in range(Hkv):
        for b in range(nb):
            e = B * (b + 1)
            lst = np.sort(rng.choice(e, size=min(e, width - 40), replace=False))
            idx[g, b, :lst.size], cnt[g, b] = lst, lst.size
    G = Hq // Hkv
    for b in (0, 2, 3):
        pos = np.arange(B * b, B * (b + 1))
        O = orc.sparse_decode(Q[pos], pos, K, V, idx, cnt, B)
        for g in range(Hkv):
            ref = orc.sparse_attn(Q, K, V, idx[g, b], int(cnt[g, b]), b, g, B)
            assert np.abs(O[:, g * G:(g + 1) * G] - ref).max() < 1e-12


def test_decode_hand_case_and_empty_visibility():
    """One head, d = 2, a list of three keys: the softmax written out by hand;
    and a query whose listed keys all lie after it gets a zero row."""
    K = np.zeros((64, 1, 2))
    V = np.zeros((64, 1, 2))
    K[3, 0], K[10, 0], K[40, 0] = [1.0, 0.0], [0.0, 2.0], [3.0, 3.0]
    V[3, 0], V[10, 0], V[40, 0] = [1.0, 2.0], [-1.0, 0.5], [7.0, 7.0]
    idx = np.array([[[3, 10, 40, -1]]])
    cnt = np.array([[3]])
    q = np.array([[[2.0, 1.0]]])
    O = orc.sparse_decode(q, np.array([20]), K, V, idx, cnt, 64)   # key 40 is after t = 20
    s3, s10 = 2.0 / math.sqrt(2), 2.0 / math.sqrt(2)
    w3, w10 = math.exp(s3), math.exp(s10)
    want = [(w3 * 1.0 + w10 * -1.0) / (w3 + w10), (w3 * 2.0 + w10 * 0.5) / (w3 + w10)]
    assert np.abs(O[0, 0] - want).max() < 1e-15
    O2 = orc.sparse_decode(q, np.array([2]), K, V, idx, cnt, 64)
    assert np.all(O2 == 0.0)


def test_swa_and_decode_planted_mistakes_are_caught():
    """Plausible bugs in the window and decode oracles, each rejected by the
    pin above that targets it: a window one key wider (i - W <= j), a decode
    query that reads the next block's list, and one with no causal mask."""
    L, Hq, Hkv, d = 150, 4, 2, 16
    Q, K, V = _rand((L, Hq, d), 71), _rand((L, Hkv, d), 72), _rand((L, Hkv, d), 73)
    i, j = np.arange(L)[:, None], np.arange(L)[None, :]
    W = 7
    band = np.broadcast_to((j <= i) & (j > i - W), (Hq, L, L)).copy()
    O_wide, _ = orc.swa_attn(Q, K, V, W + 1)           # mutant: one key wider
    assert np.abs(O_wide - _sdpa(Q, K, V, mask=band)).max() > 1e-3

    L, Hq, Hkv, d, B = 192, 4, 2, 16, 64
    Q, K, V = _rand((L, Hq, d), 81), _rand((L, Hkv, d), 82), _rand((L, Hkv, d), 83)
    idx, cnt = _full_lists(L, Hkv, B)
    pos = np.array([1, 63, 64, 100])
    ref = _sdpa(Q, K, V, causal=True)[pos]
    O_next = orc.sparse_decode(Q[pos], pos + B, K, V, idx, cnt, B)   # mutant: next block's list
    assert np.abs(O_next - ref).max() > 1e-3
    O_nomask = orc.sparse_decode(Q[pos], np.full_like(pos, L - 1), K, V, idx, cnt, B)  # mutant: no j <= t
    assert np.abs(O_nomask - ref).max() > 1e-3
