"""fp64 CPU oracle for HySparse2-style token-level sparse causal attention.

TEST INFRASTRUCTURE.  This module defines what the prefill path computes, in
plain NumPy float64, so that the CUDA library can be checked against it.  Only
the test suite, the smoke check and the benchmark's CPU-baseline / reference
leg may import it.  It shares no code with the CUDA path and never calls it.

Sources (pages, cited by title and paragraph or section):
  [HS2]   "罗福莉剧透小米MiMo-V3架构：HySparse2让预填充提前退出" -- the HySparse2 /
          MiMo-V3 architecture summary.  Paragraphs used:
            KV-sharing paragraph: sparse layers reuse the full-attention
              layer's KV cache and its token selection (KV Reuse);
            branch-removal paragraph: no separate sliding-window branch, the
              most recent tokens are forced into the sparse selection;
            token-selection paragraph: selection is per token, 1024 global
              tokens plus the 128 most recent, reused by later sparse layers;
            ablation paragraph: the full-attention layer's complete scores
              pick the tokens (no separate retrieval module);
            cost paragraph: FP8 KV cache.
  [SHARP] "企业官网建设流程全解析" (a walk-through of SHARP sparse attention),
          section 1.1: Attention(Q,K,V) = softmax(Q K^T / sqrt(d_k)) V.

Readings where the pages are silent:
  R1  scores are s = q.k / sqrt(d), natural-log LSE;
  R2  grouped-query attention maps query head h to KV head floor(h / G);
  R3  one selection per (query block of 64 tokens, KV head), shared by the
      block's queries and the group's heads;
  R4  importance of key j for block b and KV head g is the sum of the
      normalised probabilities exp(s - lse) over the block's queries and the
      group's heads;
  R5  the recent window is block-aligned: R_b = [e_b - w, e_b), with the
      per-query causal mask j <= i applied inside it;
  R6  global tokens come only from C_b = [0, max(0, e_b - w)); the list holds
      min(|C_b|, k) of them plus min(w, e_b) recent ones;
  R7  ties in importance go to the lower position;
  R8  the list is ascending (global part, then the recent window) and padded
      with -1 to k + w entries; a count gives the valid length;
  R9  a query row with no visible key (possible only when w < block) gives a
      zero output row;
  R10 FP8 is OCP e4m3fn with one fp32 scale per (token, KV head); a stored
      value is code * scale;
  R13 the sliding window of width W lets query i see keys i - W < j <= i;
  R14 a decode-step query at position t reuses the list of the block that
      holds t, with the causal mask j <= t.

Shapes: Q [L][Hq][d], K/V [L][Hkv][d] (token-major), all float64 here.
"""
from __future__ import annotations

import numpy as np

# ---------------------------------------------------------------- decoding --


def decode_bf16(u16: np.ndarray) -> np.ndarray:
    """Exact value of bfloat16 bit patterns: a bf16 is the top half of an IEEE
    binary32, so widening the pattern by 16 zero bits gives the same number."""
    u = np.asarray(u16, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):
        return u.view(np.float32).astype(np.float64)


def decode_e4m3(u8: np.ndarray) -> np.ndarray:
    """Exact value of OCP e4m3fn codes (reading R10): 1 sign bit, 4 exponent
    bits with bias 7, 3 mantissa bits, no infinities, S.1111.111 is NaN.
    Normal: 2^(e-7) * (1 + m/8); subnormal (e = 0): 2^-6 * m/8."""
    c = np.asarray(u8, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, np.ldexp(m / 8.0, -6), np.ldexp(1.0 + m / 8.0, e - 7))
    mag = np.where((e == 0xF) & (m == 0x7), np.nan, mag)
    return sign * mag


def dequantize(codes_u8: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """Stored FP8 value times its per-(token, head) scale (reading R10)."""
    return decode_e4m3(codes_u8) * np.asarray(scale, dtype=np.float64)[..., None]


E4M3_MAX = 448.0


def _e4m3_grid() -> np.ndarray:
    """All non-negative finite e4m3fn values, ascending (code order)."""
    return decode_e4m3(np.arange(0x7F, dtype=np.uint8))   # 0x00..0x7E; 0x7F is NaN


def encode_e4m3(y) -> np.ndarray:
    """Round values to OCP e4m3fn codes: nearest representable value, ties to
    the even code (mantissa LSB 0), magnitudes beyond 448 saturate to 448
    (reading R10); the sign bit follows the input's sign, zero included.
    Works on float32 inputs exactly, by search over the grid."""
    y = np.asarray(y, dtype=np.float64)
    grid = _e4m3_grid()
    mag = np.minimum(np.abs(y), E4M3_MAX)
    hi = np.clip(np.searchsorted(grid, mag, side="left"), 1, grid.size - 1)
    lo = hi - 1
    d_lo, d_hi = mag - grid[lo], grid[hi] - mag
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(mag <= 0.0, 0, np.where(mag >= grid[-1], grid.size - 1, np.where(take_hi, hi, lo)))
    sign = np.where(np.signbit(y), 0x80, 0)   # a negative value keeps its sign, even at zero
    return (code | sign).astype(np.uint8)


def quantize_kv(x_rows):
    """FP8 KV write (HS2 cost paragraph: FP8 KV cache; reading R10): for each
    row of 128 values (one token, one KV head), scale = amax / 448 computed in
    float32 (1 when the row is all zero), codes = e4m3(x / scale) with the
    division in float32.  x_rows [..., d] holds values exactly representable in
    float32.  Returns (codes uint8 [..., d], scale float32 [...])."""
    x = np.asarray(x_rows, dtype=np.float32)
    amax = np.abs(x).max(axis=-1)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    y = (x / scale[..., None]).astype(np.float32)
    return encode_e4m3(y), scale


# ------------------------------------------------------- index arithmetic --


def kv_head(h: int, G: int) -> int:
    """Reading R2: contiguous head groups."""
    return h // G


def block_rows(b: int, L: int, B: int) -> tuple[int, int]:
    """Query rows [s_b, e_b) of query block b."""
    return B * b, min(L, B * (b + 1))


def n_candidates(e_b: int, w: int) -> int:
    """|C_b| = max(0, e_b - w) (reading R6)."""
    return max(0, e_b - w)


def list_size(e_b: int, k: int, w: int) -> int:
    """Number of valid entries in a block's index list (reading R6)."""
    return min(n_candidates(e_b, w), k) + min(w, e_b)


# ------------------------------------------------------ dense attention --


def dense_attn(Q, K, V, r0: int = 0, r1: int | None = None):
    """Causal grouped-query softmax attention ([SHARP] 1.1 with the causal mask
    j <= i; [HS2] full-attention layer) for query rows [r0, r1).

    Returns O [r1-r0][Hq][d] and lse [Hq][r1-r0] with
    lse_{h,i} = log sum_{j<=i} exp(s_{h,i,j}).  Softmax is max-subtracted."""
    L, Hq, d = Q.shape
    G = Hq // K.shape[1]
    r1 = L if r1 is None else r1
    i = np.arange(r0, r1)[:, None]
    j = np.arange(r1)[None, :]
    visible = j <= i
    O = np.empty((r1 - r0, Hq, d))
    lse = np.empty((Hq, r1 - r0))
    for h in range(Hq):
        g = kv_head(h, G)
        s = (Q[r0:r1, h, :] @ K[:r1, g, :].T) / np.sqrt(d)
        s = np.where(visible, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        l = p.sum(axis=1, keepdims=True)
        O[:, h, :] = (p @ V[:r1, g, :]) / l
        lse[h] = (m + np.log(l))[:, 0]
    return O, lse


def swa_attn(Q, K, V, W: int):
    """Causal sliding-window attention: query i attends to keys
    max(0, i - W + 1) <= j <= i ([HS2] two-part paragraph: the self-decoder
    combines full and sliding-window attention; the window width is this
    library's parameter, 128 in the measurements).  Returns O and lse like
    dense_attn."""
    L, Hq, d = Q.shape
    G = Hq // K.shape[1]
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    visible = (j <= i) & (j > i - W)
    O = np.empty((L, Hq, d))
    lse = np.empty((Hq, L))
    for h in range(Hq):
        g = kv_head(h, G)
        s = (Q[:, h, :] @ K[:, g, :].T) / np.sqrt(d)
        s = np.where(visible, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        l = p.sum(axis=1, keepdims=True)
        O[:, h, :] = (p @ V[:, g, :]) / l
        lse[h] = (m + np.log(l))[:, 0]
    return O, lse


# ------------------------------------------------------------ importance --


def importance(Q, K, lse_block, b: int, g: int, B: int, w: int, scope: str = "candidates"):
    """Importance of each key for query block b and KV head g (reading R4):

        I_j = sum_{h in group g} sum_{i in block b, j <= i} exp(s_{h,i,j} - lse_{h,i})

    lse_block is [Hq][e_b - s_b], the natural-log LSE of the block's rows.
    scope "candidates" returns I over C_b = [0, e_b - w) (the keys the top-k
    draws from); scope "visible" returns I over every key j < e_b, which by
    construction sums to (#rows in block) * G.  The causal mask is kept in the
    general form so that scaled tests with w < B stay exact."""
    L, Hq, d = Q.shape
    G = Hq // K.shape[1]
    s_b, e_b = block_rows(b, L, B)
    hi = n_candidates(e_b, w) if scope == "candidates" else e_b
    I = np.zeros(hi)
    if hi == 0:
        return I
    i = np.arange(s_b, e_b)[:, None]
    j = np.arange(hi)[None, :]
    visible = j <= i
    for hl in range(G):
        h = g * G + hl
        s = (Q[s_b:e_b, h, :] @ K[:hi, g, :].T) / np.sqrt(d)
        p = np.exp(s - lse_block[h][:, None])
        I += np.where(visible, p, 0.0).sum(axis=0)
    return I


# -------------------------------------------------------------- selection --


def select(I_row, k: int, w: int, e_b: int):
    """Top-k over the candidates plus the forced recent window ([HS2]
    token-selection and branch-removal paragraphs; readings R5-R8).

    I_row holds the importance of C_b = [0, e_b - w).  A stable sort on
    (-I, j) orders candidates by importance with ties to the lower position;
    the first min(|C_b|, k) are kept, put in ascending order, and the recent
    window [e_b - w, e_b) is appended.  Returns (idx[k + w] padded with -1, cnt).
    """
    n_c = n_candidates(e_b, w)
    I_row = np.asarray(I_row, dtype=np.float64)
    assert I_row.shape == (n_c,), (I_row.shape, n_c)
    pos = np.arange(n_c)
    order = np.lexsort((pos, -I_row))          # primary -I, secondary position
    top = np.sort(order[: min(n_c, k)])
    recent = np.arange(max(0, e_b - w), e_b)
    chosen = np.concatenate([top, recent]).astype(np.int64)
    idx = np.full(k + w, -1, dtype=np.int64)
    idx[: chosen.size] = chosen
    return idx, int(chosen.size)


def pool_blocks(I_row, B: int = 64):
    """Importance of each whole 64-key block: the exact sum of its 64 values,
    taken in float64 (the block-level selection of [HS2]'s block-selection
    paragraph ranks blocks by how much of the row's importance they hold; the
    page fixes no summation order, so the oracle sums in float64, where the
    rounding of 64 float32 terms is far below any float32 difference)."""
    assert B == 64
    x = np.asarray(I_row, dtype=np.float64)
    return x.reshape(-1, B).sum(axis=1)


def select_blocks(I_row, k: int, w: int, e_b: int, B: int = 64):
    """Block-level selection of HySparse v1 ([HS2] block-selection paragraph:
    whole 64-token blocks are chosen) on the same importance, as the variant
    the token-level design is compared with: the candidates C_b are pooled
    into 64-key blocks (pool_blocks), the top min(#blocks, k / 64) blocks by
    pooled importance are kept (ties to the lower block), their positions
    listed in ascending order, and the recent window appended; -1 padded to
    k + w.  Requires k % 64 == 0 and |C_b| % 64 == 0."""
    n_c = n_candidates(e_b, w)
    assert k % B == 0 and n_c % B == 0
    I_row = np.asarray(I_row, dtype=np.float64)
    assert I_row.shape == (n_c,)
    J = pool_blocks(I_row, B) if n_c else np.zeros(0)
    m = np.arange(J.size)
    order = np.lexsort((m, -J))
    keep = np.sort(order[: min(J.size, k // B)])
    top = (keep[:, None] * B + np.arange(B)[None, :]).reshape(-1)
    recent = np.arange(max(0, e_b - w), e_b)
    chosen = np.concatenate([top, recent]).astype(np.int64)
    idx = np.full(k + w, -1, dtype=np.int64)
    idx[: chosen.size] = chosen
    return idx, int(chosen.size)


def brute_rank(I_row):
    """rank_j = #{j' : I_j' > I_j or (I_j' == I_j and j' < j)}; j is among the
    top k exactly when rank_j < k.  Quadratic, independent of any sort."""
    I_row = np.asarray(I_row, dtype=np.float64)
    n = I_row.size
    a = I_row[None, :]
    b = I_row[:, None]
    jj = np.arange(n)
    earlier = jj[None, :] < jj[:, None]
    return ((a > b) | ((a == b) & earlier)).sum(axis=1)


# ------------------------------------------------------ sparse attention --


def sparse_attn(Q, K, V, idx_row, cnt: int, b: int, g: int, B: int):
    """Sparse-layer attention of block b, KV head g over the shared index list
    ([HS2] KV-sharing paragraph: the sparse layer reuses the full layer's KV
    cache and token selection).  For query i the softmax runs over the listed
    positions j with j <= i (causal mask, reading R5); padding (-1) beyond cnt
    is never read.  Returns O [rows][G][d] for the group's heads."""
    L, Hq, d = Q.shape
    G = Hq // K.shape[1]
    s_b, e_b = block_rows(b, L, B)
    pos = np.asarray(idx_row[:cnt], dtype=np.int64)
    assert pos.size == 0 or (pos.min() >= 0 and pos.max() < e_b)
    i = np.arange(s_b, e_b)[:, None]
    visible = pos[None, :] <= i
    O = np.zeros((e_b - s_b, G, d))
    if pos.size == 0:
        return O
    Kp = K[pos, g, :]
    Vp = V[pos, g, :]
    any_vis = visible.any(axis=1)
    for hl in range(G):
        h = g * G + hl
        s = (Q[s_b:e_b, h, :] @ Kp.T) / np.sqrt(d)
        s = np.where(visible, s, -np.inf)
        m = np.where(any_vis, s.max(axis=1), 0.0)[:, None]
        p = np.where(visible, np.exp(s - m), 0.0)
        l = p.sum(axis=1, keepdims=True)
        O[:, hl, :] = np.where(any_vis[:, None], (p @ Vp) / np.where(l > 0, l, 1.0), 0.0)
    return O


def sparse_decode(q_rows, positions, K, V, idx, cnt, B: int):
    """Decode-step sparse attention ([HS2] KV-sharing paragraph: the sparse
    layers reuse the full layer's KV cache and token selection; with early
    exit they mostly run at decode).  Reading R14: a query at position t uses
    the list of the block holding t, floor(t / B), for its KV head, and sees
    the listed positions j <= t.

    q_rows [n][Hq][d], positions [n], K / V [L][Hkv][d], idx [Hkv][nb][*],
    cnt [Hkv][nb].  Returns O [n][Hq][d]; a query with no visible listed key
    gets a zero row (reading R9)."""
    n, Hq, d = q_rows.shape
    G = Hq // K.shape[1]
    O = np.zeros((n, Hq, d))
    for r in range(n):
        t = int(positions[r])
        b = t // B
        for h in range(Hq):
            g = kv_head(h, G)
            listed = np.asarray(idx[g, b, :int(cnt[g, b])], dtype=np.int64)
            vis = listed[listed <= t]
            if vis.size == 0:
                continue
            s = (K[vis, g, :] @ q_rows[r, h, :]) / np.sqrt(d)
            p = np.exp(s - s.max())
            O[r, h, :] = (p @ V[vis, g, :]) / p.sum()
    return O


# ------------------------------------------------- whole-path composition --


def full_attn_select_block(Q, K, V, b: int, g: int, B: int, k: int, w: int):
    """Everything the full-attention layer produces for one (block, KV head):
    the group's dense output rows and LSE, the candidate importance row, and
    the selected index list.  Returns a dict."""
    L, Hq, d = Q.shape
    G = Hq // K.shape[1]
    s_b, e_b = block_rows(b, L, B)
    O, lse = dense_attn(Q[:, g * G:(g + 1) * G], K[:, g:g + 1], V[:, g:g + 1], s_b, e_b)
    lse_block = np.zeros((Hq, e_b - s_b))
    lse_block[g * G:(g + 1) * G] = lse
    I = importance(Q, K, lse_block, b, g, B, w)
    idx, cnt = select(I, k, w, e_b)
    return {"O": O, "lse": lse, "I": I, "idx": idx, "cnt": cnt}


def prefill_units(Q_layers, K, V, units, B: int, k: int, w: int):
    """Run the whole path (full layer + every sparse layer) on a list of
    (block, KV head) units.  Used for the CPU baseline and sampled parity."""
    out = []
    for b, g in units:
        r = full_attn_select_block(Q_layers[0], K, V, b, g, B, k, w)
        r["sparse"] = [sparse_attn(Ql, K, V, r["idx"], r["cnt"], b, g, B) for Ql in Q_layers[1:]]
        out.append(r)
    return out
