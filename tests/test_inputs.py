"""The seeded input generator: determinism, shapes, needle placement and the
FP8 encoding of the KV cache (decoded by the oracle's own decoder)."""
import numpy as np
import torch

from oracle import hs2_oracle as orc
from token_level_sparse_causal_b200 import inputs


def _small(**kw):
    return inputs.WORKLOADS["c1"].scaled(L=512, **kw)


def test_deterministic_and_shapes():
    wl = _small()
    a, b = inputs.make_inputs(wl), inputs.make_inputs(wl)
    assert len(a["q_layers"]) == 1 + wl.n_sparse
    for x, y in zip(a["q_layers"] + [a["k"], a["v"]], b["q_layers"] + [b["k"], b["v"]]):
        assert torch.equal(x, y)
    assert a["q_layers"][0].shape == (512, 4, 128) and a["k"].shape == (512, 1, 128)
    assert a["q_layers"][0].dtype == torch.bfloat16
    assert not torch.equal(a["q_layers"][0], a["q_layers"][1])


def test_needles_sit_before_the_recent_window():
    wl = _small()
    x = inputs.make_inputs(wl)
    assert len(x["needles"]) == 16
    for n in x["needles"]:
        e_b = min(wl.L, (n["t"] // wl.block + 1) * wl.block)
        assert 0 <= n["p"] < e_b - wl.recent
        kq = x["q_layers"][0][n["t"], n["h"]].float()
        kk = x["k"][n["p"], n["g"]].float()
        cos = (kq @ kk) / (kq.norm() * kk.norm())
        assert abs(kk.norm().item() - 4.0) < 0.05 or cos > 0.99


def test_chain_needles_are_ordered():
    wl = inputs.WORKLOADS["c4"].scaled(L=4096, Hq=4, Hkv=2, n_sparse=1)
    x = inputs.make_inputs(wl)
    assert len(x["needles"]) == 8 * 4
    for c in range(8):
        ps = [n["p"] for n in x["needles"] if n["chain"] == c]
        assert ps == sorted(ps) and len(set(ps)) == 4


def test_fp8_cache_roundtrip_within_e4m3_precision():
    wl = inputs.WORKLOADS["c5"].scaled(L=1024, Hq=8, Hkv=2)
    x = inputs.make_inputs(wl, with_needles=False)
    assert x["k"].dtype == torch.uint8 and x["k_scale"].shape == (1024, 2)
    ref = inputs.make_inputs(wl.scaled(kv_dtype="bf16"), with_needles=False)
    kd = orc.dequantize(inputs.as_u8(x["k"]), x["k_scale"].numpy())
    kr = orc.decode_bf16(inputs.as_u16(ref["k"]))
    amax = np.abs(kr).max(axis=-1, keepdims=True)
    assert np.all(np.abs(kd - kr) <= amax * 2.0 ** -4 + 1e-12)      # e4m3 keeps 3 mantissa bits
    assert np.all(np.abs(orc.decode_e4m3(inputs.as_u8(x["k"]))) <= 448.0)
