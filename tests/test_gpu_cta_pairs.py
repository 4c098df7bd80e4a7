"""Kernel (1) on clusters of two CTAs (tcgen05 cta_group::2, the
hs2_debug_set bit 2 variant): the same products and the same per-row softmax
arithmetic as the default kernel, so every output must be bit for bit the
default kernel's (whose parity with the fp64 oracle the other files check);
one shape is also checked against the oracle directly.  The in-kernel e4m3
conversion (no layer copy) is outside the variant and falls back."""
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
    yield
    hs2.hs2_debug_set(H.WAIT_LIMIT_NS, 0)


def _wl(L, Hq, Hkv, kv="bf16", seed=41):
    return inputs.Workload(f"p{L}_{Hq}x{Hkv}", L, Hq, Hkv, 1, seed, kv_dtype=kv)


def _attn(shape, xd, flags):
    """hs2_attn_fwd_ws with a workspace (the e4m3 layer copy), under `flags`."""
    q0 = xd["q_layers"][0]
    o = torch.full_like(q0, float("nan"))
    lse = torch.full((shape.Hq, shape.L), float("nan"), device=DEV)
    ws = torch.empty(max(16, hs2.attn_fwd_workspace_bytes(shape)), dtype=torch.uint8, device=DEV)
    hs2.hs2_debug_set(H.WAIT_LIMIT_NS, flags)
    try:
        hs2.hs2_attn_fwd_ws(shape, q0, xd["k"], xd["v"], xd["k_scale"], xd["v_scale"], o, lse, ws)
        hs2.hs2_sync()
    finally:
        hs2.hs2_debug_set(H.WAIT_LIMIT_NS, 0)
    return o, lse


@pytest.mark.parametrize("L,Hq,Hkv,kv", [(1088, 8, 2, "bf16"), (2048, 16, 2, "bf16"), (4096, 8, 4, "bf16"),
                                         (640, 16, 8, "bf16"), (1088, 8, 2, "e4m3"), (2944, 16, 2, "e4m3")])
def test_cta_pairs_are_bitwise_the_default_kernel(L, Hq, Hkv, kv):
    wl = _wl(L, Hq, Hkv, kv)
    xd = H.to_dev(inputs.make_inputs(wl), DEV)
    shape = H.shape_of(wl, xd)
    o0, lse0 = _attn(shape, xd, 0)
    o1, lse1 = _attn(shape, xd, hs2.DEBUG_FA_CTA_PAIRS)
    assert torch.equal(o0, o1)
    assert torch.equal(lse0, lse1)


def test_cta_pairs_match_the_oracle():
    wl = _wl(1152, 4, 2, seed=43)
    x = inputs.make_inputs(wl)
    xd = H.to_dev(x, DEV)
    o, lse = _attn(H.shape_of(wl, xd), xd, hs2.DEBUG_FA_CTA_PAIRS)
    D = H.decode(x)
    O, LSE = orc.dense_attn(D["Q"][0], D["K"], D["V"])
    H.bf16_close(o.float().cpu().numpy(), O, "O (CTA pairs)")
    assert abs(lse.cpu().double().numpy() - LSE).max() <= H.LSE_ATOL


def test_in_kernel_e4m3_conversion_falls_back_to_the_default_kernel():
    """An e4m3 cache without the layer's f16 copy (hs2_attn_fwd, no
    workspace) runs the default kernel's in-kernel conversion either way."""
    wl = _wl(1088, 8, 2, kv="e4m3", seed=45)
    xd = H.to_dev(inputs.make_inputs(wl), DEV)
    shape = H.shape_of(wl, xd)
    q0 = xd["q_layers"][0]
    outs = []
    for flags in (0, hs2.DEBUG_FA_CTA_PAIRS):
        o = torch.full_like(q0, float("nan"))
        lse = torch.full((wl.Hq, wl.L), float("nan"), device=DEV)
        hs2.hs2_debug_set(H.WAIT_LIMIT_NS, flags)
        try:
            hs2.hs2_attn_fwd(shape, q0, xd["k"], xd["v"], xd["k_scale"], xd["v_scale"], o, lse)
            hs2.hs2_sync()
        finally:
            hs2.hs2_debug_set(H.WAIT_LIMIT_NS, 0)
        outs.append((o, lse))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


def test_cta_pairs_inside_the_full_layer_call():
    """hs2_full_attn_select with the variant: O, LSE and every list equal."""
    wl = _wl(4096, 8, 2, seed=47)
    xd = H.to_dev(inputs.make_inputs(wl), DEV)
    r0 = H.run_path(wl, xd)
    hs2.hs2_debug_set(H.WAIT_LIMIT_NS, hs2.DEBUG_FA_CTA_PAIRS)
    try:
        r1 = H.run_path(wl, xd)
    finally:
        hs2.hs2_debug_set(H.WAIT_LIMIT_NS, 0)
    for key in ("o", "lse", "idx", "cnt"):
        assert torch.equal(r0[key], r1[key]), key
    for a, b in zip(r0["sparse"], r1["sparse"]):
        assert torch.equal(a, b)


def test_cta_pairs_bounded_waits_report_timeout_and_context_survives():
    """The load role issues nothing (bit 0), so every other role of both CTAs
    runs out its bounded waits: hs2_sync reports HS2_ERR_TIMEOUT, and the next
    call on the pair kernel is right."""
    wl = _wl(512, 4, 2, seed=49)
    xd = H.to_dev(inputs.make_inputs(wl), DEV)
    shape = H.shape_of(wl, xd)
    q0 = xd["q_layers"][0]
    o = torch.empty_like(q0)
    lse = torch.empty((wl.Hq, wl.L), device=DEV)
    hs2.hs2_debug_set(50_000_000, hs2.DEBUG_SKIP_LOADS | hs2.DEBUG_FA_CTA_PAIRS)
    try:
        hs2.hs2_attn_fwd(shape, q0, xd["k"], xd["v"], None, None, o, lse)
        with pytest.raises(hs2.Hs2Error) as e:
            hs2.hs2_sync()
        assert e.value.code == hs2.HS2_ERR_TIMEOUT
    finally:
        hs2.hs2_debug_set(H.WAIT_LIMIT_NS, 0)
    o0, lse0 = _attn(shape, xd, 0)
    o1, lse1 = _attn(shape, xd, hs2.DEBUG_FA_CTA_PAIRS)
    assert torch.equal(o0, o1) and torch.equal(lse0, lse1)
