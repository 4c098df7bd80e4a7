"""Thin ctypes binding over libhs2.so (argument marshalling only).

Every step of the prefill path runs in the library's CUDA kernels; this
module only turns torch tensors into device pointers and sizes, picks the
current CUDA stream, and raises Hs2Error on a non-zero status.  If the shared
library is missing or fails to load, importing the functions raises: there is
no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libhs2.so")

(HS2_OK, HS2_ERR_INVALID_ARG, HS2_ERR_UNSUPPORTED, HS2_ERR_WORKSPACE, HS2_ERR_CUDA, HS2_ERR_TIMEOUT, HS2_ERR_INDEX,
 HS2_ERR_RANGE) = range(8)
HS2_KV_BF16, HS2_KV_E4M3 = 0, 1

EXPORTS = ("hs2_full_attn_select", "hs2_sparse_attn", "hs2_sync", "hs2_attn_fwd", "hs2_importance",
           "hs2_topk_select", "hs2_strerror", "hs2_debug_set", "hs2_version", "hs2_launch_count",
           "hs2_full_attn_select_static", "hs2_exp2_check", "hs2_quantize_kv", "hs2_block_select",
           "hs2_full_attn_select_blocks", "hs2_swa_attn", "hs2_sparse_decode",
           "hs2_sparse_decode_workspace", "hs2_attn_fwd_ws")


class Hs2Shape(ctypes.Structure):
    _fields_ = [("L", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("d", ctypes.c_int32),
                ("block", ctypes.c_int32), ("topk", ctypes.c_int32), ("recent", ctypes.c_int32),
                ("kv_dtype", ctypes.c_int32), ("q_tok_stride", ctypes.c_int64), ("q_head_stride", ctypes.c_int64),
                ("kv_tok_stride", ctypes.c_int64), ("kv_head_stride", ctypes.c_int64)]


class Hs2Error(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: hs2 status {code} ({strerror(code)})")
        self.code = code


_lib: Optional[ctypes.CDLL] = None

_vp, _i32, _i64, _u32, _u64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32, ctypes.c_uint64
_SIGS = {
    "hs2_full_attn_select": [ctypes.POINTER(Hs2Shape), _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                             ctypes.POINTER(ctypes.c_size_t), _vp, _i32, _i32, _vp],
    "hs2_full_attn_select_static": [ctypes.POINTER(Hs2Shape), _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp],
    "hs2_full_attn_select_blocks": [ctypes.POINTER(Hs2Shape), _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                    ctypes.POINTER(ctypes.c_size_t), _vp],
    "hs2_block_select": [ctypes.POINTER(Hs2Shape), _vp, _i64, _i32, _i32, _vp, _vp, _vp],
    "hs2_sparse_attn": [ctypes.POINTER(Hs2Shape), _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp],
    "hs2_sync": [_vp],
    "hs2_attn_fwd": [ctypes.POINTER(Hs2Shape), _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp],
    "hs2_attn_fwd_ws": [ctypes.POINTER(Hs2Shape), _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                        ctypes.POINTER(ctypes.c_size_t), _vp],
    "hs2_swa_attn": [ctypes.POINTER(Hs2Shape), _vp, _vp, _vp, _i32, _vp, _vp, _vp],
    "hs2_sparse_decode": [ctypes.POINTER(Hs2Shape), _vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                          ctypes.c_size_t, _vp],
    "hs2_sparse_decode_workspace": [ctypes.POINTER(Hs2Shape), _i32, ctypes.POINTER(ctypes.c_size_t)],
    "hs2_importance": [ctypes.POINTER(Hs2Shape), _vp, _vp, _vp, _vp, _i32, _i32, _vp, _i64, _vp],
    "hs2_topk_select": [ctypes.POINTER(Hs2Shape), _vp, _i64, _i32, _i32, _vp, _vp, _vp],
    "hs2_debug_set": [_u64, _u32],
    "hs2_exp2_check": [_vp, _vp, _vp, _vp, _i64, _vp],
    "hs2_quantize_kv": [_i32, _i32, _vp, _i64, _i64, _vp, _i64, _i64, _vp, _vp],
    "hs2_version": [],
}


def lib() -> ctypes.CDLL:
    """Load libhs2.so (built in-tree by token_level_sparse_causal_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libhs2.so not built at {LIB_PATH}; run token_level_sparse_causal_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        L.hs2_launch_count.argtypes = []
        L.hs2_launch_count.restype = ctypes.c_uint64
        L.hs2_strerror.argtypes = [ctypes.c_int]
        L.hs2_strerror.restype = ctypes.c_char_p
        _lib = L
    return _lib


def strerror(code: int) -> str:
    return lib().hs2_strerror(int(code)).decode()


def _check(rc: int, what: str) -> None:
    if rc != HS2_OK:
        raise Hs2Error(rc, what)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def make_shape(q: torch.Tensor, k: torch.Tensor, topk: int = 1024, recent: int = 128, block: int = 64,
               kv_dtype: int = HS2_KV_BF16) -> Hs2Shape:
    """hs2_shape for Q [L][Hq][d] and K [L][Hkv][d] tensors (element strides)."""
    L, Hq, d = q.shape
    return Hs2Shape(L=L, Hq=Hq, Hkv=k.shape[1], d=d, block=block, topk=topk, recent=recent, kv_dtype=kv_dtype,
                    q_tok_stride=q.stride(0), q_head_stride=q.stride(1), kv_tok_stride=k.stride(0),
                    kv_head_stride=k.stride(1))


def workspace_bytes(shape: Hs2Shape) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().hs2_full_attn_select(ctypes.byref(shape), None, None, None, None, None, None, None, None, None,
                                      None, ctypes.byref(n), None, 0, 0, None), "hs2_full_attn_select(size query)")
    return int(n.value)


def importance_row_stride(shape, b1: int) -> int:
    """Row stride (floats) of hs2_full_attn_select's importance export for the
    block range ending at b1: max(64, roundup(e_{b1-1} - recent, 64))."""
    n_c = max(0, min(shape.L, shape.block * b1) - shape.recent)
    return max(64, (n_c + 63) // 64 * 64)


def hs2_full_attn_select(shape, q, k, v, k_scale, v_scale, o, lse, idx, cnt, workspace, stream=None,
                         importance_out=None, strip=(0, 0)) -> None:
    """importance_out: optional fp32 tensor of Hkv * (b1 - b0) * importance_row_stride(shape, b1)
    elements receiving the importance rows of blocks strip = (b0, b1) that the selection consumed."""
    n = ctypes.c_size_t(workspace.numel() * workspace.element_size())
    _check(lib().hs2_full_attn_select(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(k_scale), _ptr(v_scale),
                                      _ptr(o), _ptr(lse), _ptr(idx), _ptr(cnt), _ptr(workspace), ctypes.byref(n),
                                      _ptr(importance_out), int(strip[0]), int(strip[1]), _stream(stream)),
           "hs2_full_attn_select")


def hs2_full_attn_select_static(shape, q, k, v, k_scale, v_scale, o, lse, idx, cnt, stream=None) -> None:
    """Same as hs2_full_attn_select, scratch taken from the library's fixed
    16 MiB device array (for callers that cannot allocate)."""
    _check(lib().hs2_full_attn_select_static(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(k_scale),
                                             _ptr(v_scale), _ptr(o), _ptr(lse), _ptr(idx), _ptr(cnt),
                                             _stream(stream)), "hs2_full_attn_select_static")


def hs2_full_attn_select_blocks(shape, q, k, v, k_scale, v_scale, o, lse, idx, cnt, workspace, stream=None) -> None:
    n = ctypes.c_size_t(workspace.numel() * workspace.element_size())
    _check(lib().hs2_full_attn_select_blocks(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(k_scale),
                                             _ptr(v_scale), _ptr(o), _ptr(lse), _ptr(idx), _ptr(cnt), _ptr(workspace),
                                             ctypes.byref(n), _stream(stream)), "hs2_full_attn_select_blocks")


def hs2_block_select(shape, imp, row_stride, b0, b1, idx, cnt, stream=None) -> None:
    _check(lib().hs2_block_select(ctypes.byref(shape), _ptr(imp), int(row_stride), int(b0), int(b1), _ptr(idx),
                                  _ptr(cnt), _stream(stream)), "hs2_block_select")


def hs2_sparse_attn(shape, q, k, v, k_scale, v_scale, idx, cnt, o, stream=None) -> None:
    _check(lib().hs2_sparse_attn(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(k_scale), _ptr(v_scale),
                                 _ptr(idx), _ptr(cnt), _ptr(o), _stream(stream)), "hs2_sparse_attn")


def hs2_attn_fwd(shape, q, k, v, k_scale, v_scale, o, lse, stream=None) -> None:
    _check(lib().hs2_attn_fwd(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(k_scale), _ptr(v_scale),
                              _ptr(o), _ptr(lse), _stream(stream)), "hs2_attn_fwd")


def attn_fwd_workspace_bytes(shape) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().hs2_attn_fwd_ws(ctypes.byref(shape), None, None, None, None, None, None, None, None,
                                 ctypes.byref(n), None), "hs2_attn_fwd_ws(size query)")
    return int(n.value)


def hs2_attn_fwd_ws(shape, q, k, v, k_scale, v_scale, o, lse, workspace, stream=None) -> None:
    """Kernel (1) as the full layer runs it.  A null workspace pointer is the
    C call's size query, so without a workspace this is hs2_attn_fwd."""
    if workspace is None or workspace.numel() == 0:
        hs2_attn_fwd(shape, q, k, v, k_scale, v_scale, o, lse, stream)
        return
    n = ctypes.c_size_t(workspace.numel() * workspace.element_size())
    _check(lib().hs2_attn_fwd_ws(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(k_scale), _ptr(v_scale),
                                 _ptr(o), _ptr(lse), _ptr(workspace), ctypes.byref(n), _stream(stream)),
           "hs2_attn_fwd_ws")


def sparse_decode_workspace_bytes(shape, n: int) -> int:
    nbytes = ctypes.c_size_t(0)
    _check(lib().hs2_sparse_decode_workspace(ctypes.byref(shape), int(n), ctypes.byref(nbytes)),
           "hs2_sparse_decode_workspace")
    return int(nbytes.value)


def hs2_sparse_decode(shape, q, positions, k, v, k_scale, v_scale, idx, cnt, o, workspace=None,
                      stream=None) -> None:
    """q / o [n][Hq][d] with the strides in `shape`; positions int32 [n] on the device."""
    n = int(positions.numel())
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().hs2_sparse_decode(ctypes.byref(shape), _ptr(q), _ptr(positions), n, _ptr(k), _ptr(v),
                                   _ptr(k_scale), _ptr(v_scale), _ptr(idx), _ptr(cnt), _ptr(o), _ptr(workspace),
                                   nbytes, _stream(stream)), "hs2_sparse_decode")


def hs2_swa_attn(shape, q, k, v, window, o, lse=None, stream=None) -> None:
    _check(lib().hs2_swa_attn(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), int(window), _ptr(o), _ptr(lse),
                              _stream(stream)), "hs2_swa_attn")


def hs2_importance(shape, q, k, k_scale, lse, b0, b1, imp, row_stride, stream=None) -> None:
    _check(lib().hs2_importance(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(k_scale), _ptr(lse), int(b0), int(b1),
                                _ptr(imp), int(row_stride), _stream(stream)), "hs2_importance")


def hs2_topk_select(shape, imp, row_stride, b0, b1, idx, cnt, stream=None) -> None:
    _check(lib().hs2_topk_select(ctypes.byref(shape), _ptr(imp), int(row_stride), int(b0), int(b1), _ptr(idx),
                                 _ptr(cnt), _stream(stream)), "hs2_topk_select")


def hs2_quantize_kv(src, dst, scale, stream=None) -> None:
    """bf16 [L][Hkv][128] -> e4m3 codes (uint8, same shape) + fp32 scales [L][Hkv]."""
    L, Hkv, _ = src.shape
    _check(lib().hs2_quantize_kv(int(L), int(Hkv), _ptr(src), src.stride(0), src.stride(1), _ptr(dst), dst.stride(0),
                                 dst.stride(1), _ptr(scale), _stream(stream)), "hs2_quantize_kv")


def hs2_sync(stream=None) -> None:
    _check(lib().hs2_sync(_stream(stream)), "hs2_sync")


def hs2_launch_count() -> int:
    return int(lib().hs2_launch_count())


def hs2_exp2_check(x, y_mufu, y_fma3, y_fma4, stream=None) -> None:
    _check(lib().hs2_exp2_check(_ptr(x), _ptr(y_mufu), _ptr(y_fma3), _ptr(y_fma4), x.numel(), _stream(stream)),
           "hs2_exp2_check")


# hs2_debug_set flag bits (include/hs2.h)
DEBUG_SKIP_LOADS, DEBUG_IMP_VISIBLE, DEBUG_FA_CTA_PAIRS, DEBUG_FAIL_TMAP = 1, 2, 4, 8


def hs2_debug_set(wait_limit_ns: int = 2_000_000_000, flags: int = 0) -> None:
    _check(lib().hs2_debug_set(int(wait_limit_ns), int(flags)), "hs2_debug_set")


# ------------------------------------------------------------ conveniences --

def alloc_outputs(shape: Hs2Shape, q: torch.Tensor, with_workspace: bool = True) -> dict:
    """Device buffers for one full-layer call (torch supplies the memory)."""
    dev = q.device
    nb = shape.L // shape.block
    out = {
        "o": torch.empty_like(q),
        "lse": torch.empty((shape.Hq, shape.L), device=dev, dtype=torch.float32),
        "idx": torch.empty((shape.Hkv, nb, shape.topk + shape.recent), device=dev, dtype=torch.int32),
        "cnt": torch.empty((shape.Hkv, nb), device=dev, dtype=torch.int32),
    }
    if with_workspace:
        out["workspace"] = torch.empty(workspace_bytes(shape) // 4 + 4, device=dev, dtype=torch.float32)
    return out
