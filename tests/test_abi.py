"""The C ABI without a GPU: libhs2.so loads, exports every function that
include/hs2.h declares, answers the workspace query, and rejects bad
arguments with the documented codes before touching the device.

Every call below that passes pointers is built to fail a host-side check
(the fake addresses are never dereferenced or launched on)."""
import ctypes
import os
import re
import subprocess

import pytest

from token_level_sparse_causal_b200 import build, hs2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return hs2.lib()


def _declared():
    with open(os.path.join(ROOT, "include", "hs2.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hs2_[a-z_0-9]+)\s*\(", text)))


def _shape(**kw):
    base = dict(L=2048, Hq=8, Hkv=2, d=128, block=64, topk=1024, recent=128, kv_dtype=0,
                q_tok_stride=8 * 128, q_head_stride=128, kv_tok_stride=2 * 128, kv_head_stride=128)
    base.update(kw)
    return hs2.Hs2Shape(**base)


P = ctypes.c_void_p(0x10000)        # aligned fake address, never dereferenced
MIS = ctypes.c_void_p(0x10008)      # misaligned fake address


def test_exports_match_header(lib):
    names = _declared()
    assert set(names) == set(hs2.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", hs2.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (hs2_[a-z_0-9]+)", out))
    assert set(names) <= exported
    assert not [s for s in exported if not s.startswith("hs2_")], "only hs2_* symbols are exported"


def test_no_link_time_driver_dependency():
    out = subprocess.run(["ldd", hs2.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out and "libtorch" not in out


def test_strerror_and_version(lib):
    assert hs2.strerror(0) == "ok"
    assert "timed out" in hs2.strerror(hs2.HS2_ERR_TIMEOUT)
    assert hs2.strerror(999).startswith("unknown")
    assert lib.hs2_version() >= 100


def test_workspace_query_is_host_only(lib):
    s = _shape(L=131072, Hq=64, Hkv=8, q_tok_stride=64 * 128, kv_tok_stride=8 * 128)
    n = hs2.workspace_bytes(s)
    min_ws = 8 * (131072 - 128) * 4
    row = (131072 - 128) * 4  # the longest importance row
    # strips fit L2 (64 MiB) or, for long rows, hold at least 296 rows (two per SM)
    assert min_ws <= n <= max(min_ws, 64 << 20, 296 * row + 4096)
    assert n >= min(296 * row, 64 << 20)
    small = _shape(L=1024)
    assert hs2.workspace_bytes(small) >= 2 * (1024 - 128) * 4


def test_fp8_workspaces_hold_the_layer_copy(lib):
    """With an e4m3 cache the recommended full-layer workspace, and the one
    hs2_attn_fwd_ws asks for, hold the f16 copy of K and V plus the K column
    scales; a bf16 cache needs none for kernel (1)."""
    L, Hkv = 131072, 8
    copy = 2 * L * Hkv * 128 * 2 + Hkv * L * 4
    s8 = _shape(L=L, Hq=64, Hkv=Hkv, q_tok_stride=64 * 128, kv_tok_stride=Hkv * 128, kv_dtype=hs2.HS2_KV_E4M3)
    assert hs2.workspace_bytes(s8) >= Hkv * (L - 128) * 4 + copy
    assert copy <= hs2.attn_fwd_workspace_bytes(s8) <= copy + 1024
    s16 = _shape(L=L, Hq=64, Hkv=Hkv, q_tok_stride=64 * 128, kv_tok_stride=Hkv * 128)
    assert hs2.attn_fwd_workspace_bytes(s16) == 0
    assert lib.hs2_attn_fwd_ws(ctypes.byref(s8), None, None, None, None, None, None, None, None, None,
                               None) == hs2.HS2_ERR_INVALID_ARG


@pytest.mark.parametrize("kw,code", [
    (dict(d=64), hs2.HS2_ERR_UNSUPPORTED),
    (dict(block=32), hs2.HS2_ERR_UNSUPPORTED),
    (dict(L=2000), hs2.HS2_ERR_UNSUPPORTED),
    (dict(L=0), hs2.HS2_ERR_INVALID_ARG),
    (dict(Hq=6, Hkv=4), hs2.HS2_ERR_INVALID_ARG),
    (dict(Hq=16, Hkv=1, q_tok_stride=16 * 128, kv_tok_stride=128), hs2.HS2_ERR_UNSUPPORTED),
    (dict(Hq=2, Hkv=2, q_tok_stride=2 * 128), hs2.HS2_ERR_UNSUPPORTED),
    (dict(recent=32), hs2.HS2_ERR_UNSUPPORTED),
    (dict(recent=100), hs2.HS2_ERR_UNSUPPORTED),
    (dict(topk=4000), hs2.HS2_ERR_UNSUPPORTED),
    (dict(kv_dtype=7), hs2.HS2_ERR_INVALID_ARG),
    (dict(q_tok_stride=8 * 128 + 4), hs2.HS2_ERR_UNSUPPORTED),
    (dict(q_tok_stride=4 * 128), hs2.HS2_ERR_UNSUPPORTED),
    (dict(kv_head_stride=64), hs2.HS2_ERR_UNSUPPORTED),
])
def test_bad_shapes_rejected(lib, kw, code):
    s = ctypes.byref(_shape(**kw))
    st = ctypes.c_void_p(0)
    assert lib.hs2_attn_fwd(s, P, P, P, None, None, P, P, st) == code
    assert lib.hs2_sparse_attn(s, P, P, P, None, None, P, P, P, st) == code
    n = ctypes.c_size_t(1 << 30)
    assert lib.hs2_full_attn_select(s, P, P, P, None, None, P, P, P, P, P, ctypes.byref(n), None, 0, 0, st) == code
    assert lib.hs2_importance(s, P, P, None, P, 0, 1, P, 4096, st) == code
    assert lib.hs2_topk_select(s, P, 4096, 0, 1, P, P, st) == code


def test_null_and_misaligned_pointers_rejected(lib):
    s = ctypes.byref(_shape())
    st = ctypes.c_void_p(0)
    assert lib.hs2_attn_fwd(s, None, P, P, None, None, P, P, st) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_attn_fwd(s, P, None, P, None, None, P, P, st) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_attn_fwd(s, P, P, P, None, None, P, None, st) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_attn_fwd(s, MIS, P, P, None, None, P, P, st) == hs2.HS2_ERR_UNSUPPORTED
    assert lib.hs2_attn_fwd(s, P, MIS, P, None, None, P, P, st) == hs2.HS2_ERR_UNSUPPORTED
    assert lib.hs2_sparse_attn(s, P, P, P, None, None, None, P, P, st) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_sparse_attn(s, P, P, P, None, None, P, P, MIS, st) == hs2.HS2_ERR_UNSUPPORTED
    assert lib.hs2_topk_select(s, None, 4096, 0, 1, P, P, st) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_topk_select(s, MIS, 4096, 0, 1, P, P, st) == hs2.HS2_ERR_UNSUPPORTED


def test_block_ranges_and_strides_rejected(lib):
    s = ctypes.byref(_shape())
    st = ctypes.c_void_p(0)
    assert lib.hs2_importance(s, P, P, None, P, 3, 3, P, 4096, st) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_importance(s, P, P, None, P, 0, 33, P, 4096, st) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_importance(s, P, P, None, P, 0, 32, P, 1900, st) == hs2.HS2_ERR_INVALID_ARG   # < |C_31|
    assert lib.hs2_importance(s, P, P, None, P, 0, 32, P, 4098, st) == hs2.HS2_ERR_INVALID_ARG   # not % 4
    assert lib.hs2_topk_select(s, P, 4096, -1, 4, P, P, st) == hs2.HS2_ERR_INVALID_ARG


def test_importance_launch_rows_are_capped(lib):
    """One importance launch covers at most 65535 (KV head, block) rows (its
    grid's y extent): a wider range is refused before anything is launched."""
    L, Hkv = 524288, 8
    s = ctypes.byref(_shape(L=L, Hq=16, Hkv=Hkv, q_tok_stride=16 * 128, kv_tok_stride=Hkv * 128))
    st = ctypes.c_void_p(0)
    nb = L // 64
    assert Hkv * nb > 65535
    assert lib.hs2_importance(s, P, P, None, P, 0, nb, P, L, st) == hs2.HS2_ERR_UNSUPPORTED


def test_workspace_too_small_rejected(lib):
    s = _shape()
    n = ctypes.c_size_t(2 * (2048 - 128) * 4 - 16)
    rc = lib.hs2_full_attn_select(ctypes.byref(s), P, P, P, None, None, P, P, P, P, P, ctypes.byref(n), None, 0, 0,
                                  ctypes.c_void_p(0))
    assert rc == hs2.HS2_ERR_WORKSPACE
    assert lib.hs2_full_attn_select(ctypes.byref(s), P, P, P, None, None, P, P, P, P, P, None, None, 0, 0,
                                    ctypes.c_void_p(0)) == hs2.HS2_ERR_INVALID_ARG


def test_importance_export_range_checked(lib):
    """The optional importance export of hs2_full_attn_select takes a block
    range inside [0, L/64) and a 4-byte aligned buffer; both are checked
    before anything is launched."""
    s = _shape()
    n = ctypes.c_size_t(1 << 30)
    st = ctypes.c_void_p(0)
    call = lambda out, b0, b1: lib.hs2_full_attn_select(ctypes.byref(s), P, P, P, None, None, P, P, P, P, P,
                                                        ctypes.byref(n), out, b0, b1, st)
    assert call(P, 3, 3) == hs2.HS2_ERR_INVALID_ARG
    assert call(P, -1, 2) == hs2.HS2_ERR_INVALID_ARG
    assert call(P, 0, 33) == hs2.HS2_ERR_INVALID_ARG        # L = 2048: 32 blocks
    assert call(ctypes.c_void_p(0x1002), 0, 4) == hs2.HS2_ERR_UNSUPPORTED
    assert hs2.importance_row_stride(s, 32) == 1920 and hs2.importance_row_stride(s, 1) == 64


def test_fp8_needs_scales(lib):
    s = ctypes.byref(_shape(kv_dtype=1))
    st = ctypes.c_void_p(0)
    assert lib.hs2_attn_fwd(s, P, P, P, None, None, P, P, st) in (hs2.HS2_ERR_INVALID_ARG, hs2.HS2_ERR_UNSUPPORTED)


def test_debug_set_validates(lib):
    assert lib.hs2_debug_set(0, 0) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_debug_set(2_000_000_000, 0) == hs2.HS2_OK


def test_quantize_kv_argument_checks(lib):
    st = ctypes.c_void_p(0)
    assert lib.hs2_quantize_kv(0, 2, P, 256, 128, P, 256, 128, P, st) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_quantize_kv(16, 2, None, 256, 128, P, 256, 128, P, st) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_quantize_kv(16, 2, P, 256, 64, P, 256, 128, P, st) == hs2.HS2_ERR_UNSUPPORTED
    assert lib.hs2_quantize_kv(16, 2, P, 200, 128, P, 256, 128, P, st) == hs2.HS2_ERR_UNSUPPORTED
    assert lib.hs2_quantize_kv(16, 2, ctypes.c_void_p(0x10008), 256, 128, P, 256, 128, P, st) == \
        hs2.HS2_ERR_UNSUPPORTED
    assert lib.hs2_quantize_kv(16, 2, P, 256, 128, P, 260, 128, P, st) == hs2.HS2_ERR_UNSUPPORTED


def test_block_select_longest_sequence(lib):
    """Block-level selection holds a row's pooled values (L / 64 floats) in
    64 KiB of shared memory: L = 2^20 passes the size check (and fails on the
    null index buffer), L = 2^21 is refused before anything is launched."""
    st = ctypes.c_void_p(0)
    for L, code in ((1 << 20, hs2.HS2_ERR_INVALID_ARG), (1 << 21, hs2.HS2_ERR_UNSUPPORTED)):
        s = ctypes.byref(_shape(L=L, Hq=16, Hkv=2, q_tok_stride=16 * 128))
        assert lib.hs2_block_select(s, P, L, 0, 1, None, P, st) == code
    s = ctypes.byref(_shape(L=1 << 21, Hq=16, Hkv=2, q_tok_stride=16 * 128))
    n = ctypes.c_size_t(1 << 40)
    assert lib.hs2_full_attn_select_blocks(s, P, P, P, None, None, P, P, P, P, P, ctypes.byref(n), st) == \
        hs2.HS2_ERR_UNSUPPORTED


def test_block_select_needs_topk_multiple_of_64(lib):
    s = ctypes.byref(_shape(topk=1000))
    st = ctypes.c_void_p(0)
    assert lib.hs2_block_select(s, P, 4096, 0, 1, P, P, st) == hs2.HS2_ERR_UNSUPPORTED
    n = ctypes.c_size_t(1 << 30)
    assert lib.hs2_full_attn_select_blocks(s, P, P, P, None, None, P, P, P, P, P, ctypes.byref(n), st) == \
        hs2.HS2_ERR_UNSUPPORTED
    s2 = ctypes.byref(_shape())
    assert lib.hs2_block_select(s2, None, 4096, 0, 1, P, P, st) == hs2.HS2_ERR_INVALID_ARG


def test_swa_argument_checks(lib):
    st = ctypes.c_void_p(0)
    s = ctypes.byref(_shape())
    assert lib.hs2_swa_attn(s, P, P, P, 0, P, None, st) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_swa_attn(s, P, P, P, 2049, P, None, st) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_swa_attn(s, None, P, P, 128, P, None, st) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_swa_attn(s, P, P, P, 128, None, None, st) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_swa_attn(s, P, P, P, 128, P, MIS, st) == hs2.HS2_ERR_UNSUPPORTED
    assert lib.hs2_swa_attn(s, MIS, P, P, 128, P, None, st) == hs2.HS2_ERR_UNSUPPORTED
    assert lib.hs2_swa_attn(ctypes.byref(_shape(kv_dtype=1)), P, P, P, 128, P, None, st) == \
        hs2.HS2_ERR_UNSUPPORTED
    assert lib.hs2_swa_attn(ctypes.byref(_shape(d=64)), P, P, P, 128, P, None, st) == hs2.HS2_ERR_UNSUPPORTED


def test_decode_workspace_plan_and_argument_checks(lib):
    st = ctypes.c_void_p(0)
    s = _shape(L=131072, Hq=64, Hkv=8, q_tok_stride=64 * 128, kv_tok_stride=8 * 128)
    one = hs2.sparse_decode_workspace_bytes(s, 1)        # 8 units split over 18 chunks
    assert one >= 8 * 18 * 8 * 128 * 4
    assert hs2.sparse_decode_workspace_bytes(s, 64) == 0  # 512 units: one CTA each, no partials
    n = ctypes.c_size_t(0)
    assert lib.hs2_sparse_decode_workspace(ctypes.byref(s), 0, ctypes.byref(n)) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_sparse_decode_workspace(ctypes.byref(s), 65536, ctypes.byref(n)) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_sparse_decode_workspace(ctypes.byref(s), 1, None) == hs2.HS2_ERR_INVALID_ARG
    sp = ctypes.byref(s)
    args = lambda q=P, pos=P, nq=1, o=P, ws=P, wsb=one: (sp, q, pos, nq, P, P, None, None, P, P, o, ws, wsb, st)
    assert lib.hs2_sparse_decode(*args(ws=P, wsb=one - 4)) == hs2.HS2_ERR_WORKSPACE
    assert lib.hs2_sparse_decode(*args(ws=None)) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_sparse_decode(*args(q=None)) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_sparse_decode(*args(pos=None)) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_sparse_decode(*args(nq=0)) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_sparse_decode(*args(q=MIS)) == hs2.HS2_ERR_UNSUPPORTED
    assert lib.hs2_sparse_decode(*args(ws=MIS)) == hs2.HS2_ERR_UNSUPPORTED
    assert lib.hs2_sparse_decode(ctypes.byref(_shape(d=64)), P, P, 1, P, P, None, None, P, P, P, P, one, st) == \
        hs2.HS2_ERR_UNSUPPORTED
