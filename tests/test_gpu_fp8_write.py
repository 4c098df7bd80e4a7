"""FP8 KV write (hs2_quantize_kv) against the oracle's quantiser: codes and
scales bit-exact (the oracle divides in IEEE float32 and rounds to nearest
even; the kernel reaches the same float32 quotients through a per-row
reciprocal and two FMA corrections, or the IEEE division for rows of tiny
amax)."""
import numpy as np
import pytest
import torch

from oracle import hs2_oracle as orc
from token_level_sparse_causal_b200 import build, hs2, inputs

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    hs2.hs2_debug_set(500_000_000, 0)


def _check(src_bf16, dst, scale):
    codes, sc = orc.quantize_kv(orc.decode_bf16(inputs.as_u16(src_bf16)))
    assert np.array_equal(scale.cpu().numpy(), sc)
    assert np.array_equal(dst.cpu().numpy(), codes)


def test_random_rows_with_zeros_and_extremes():
    g = torch.Generator().manual_seed(11)
    x = (torch.randn((777, 3, 128), generator=g) * torch.logspace(-3, 3, 777)[:, None, None]).to(torch.bfloat16)
    x[5] = 0
    x[6, 1, :] = -0.0
    x[7, 2, 3] = 3.0e38
    x[8, 0, ::2] = -1e-30
    xd = x.to(DEV)
    dst = torch.full((777, 3, 128), 0xAA, dtype=torch.uint8, device=DEV)
    scale = torch.empty((777, 3), device=DEV)
    hs2.hs2_quantize_kv(xd, dst, scale)
    hs2.hs2_sync()
    _check(x, dst, scale)


def test_padded_strides_leave_padding_untouched():
    g = torch.Generator().manual_seed(12)
    big = torch.randn((301, 5, 136), generator=g).to(torch.bfloat16).to(DEV)
    src = big[:301, 1:4, :128]
    out = torch.full((301, 4, 136), 0x5A, dtype=torch.uint8, device=DEV)
    dst = out[:, :3, :128]
    scale = torch.empty((301, 3), device=DEV)
    hs2.hs2_quantize_kv(src, dst, scale)
    hs2.hs2_sync()
    _check(src.contiguous(), dst.contiguous(), scale)
    assert bool((out[:, 3] == 0x5A).all()) and bool((out[:, :3, 128:] == 0x5A).all())


def test_matches_the_generators_fp8_cache_on_the_1m_workload_rows():
    wl = inputs.WORKLOADS["c5"].scaled(L=65536)
    x = inputs.make_inputs(wl.scaled(kv_dtype="bf16"), device=DEV, with_needles=False)
    q8 = inputs.make_inputs(wl, device=DEV, with_needles=False)
    dst = torch.empty_like(q8["k"])
    scale = torch.empty_like(q8["k_scale"])
    hs2.hs2_quantize_kv(x["k"], dst, scale)
    hs2.hs2_sync()
    assert torch.equal(dst, q8["k"]) and torch.equal(scale, q8["k_scale"])   # same bytes as the torch path
    rows = np.random.default_rng(0).integers(0, 65536, 64)
    _check(x["k"][rows].cpu(), dst[rows], scale[rows])


def test_every_bf16_value_under_many_scales():
    """All finite bf16 magnitudes from 2^-20 to 2^15 (both signs), each row
    completed by an amax that sets one of 41 scales: the codes stay bit-exact
    wherever x / scale lands, on and next to every e4m3 rounding midpoint."""
    u = np.arange(0x3580, 0x4700, dtype=np.uint32)            # 2^-20 .. 2^15 as bf16 bit patterns
    vals = torch.from_numpy((u << 16).view(np.float32)).to(torch.bfloat16)
    vals = torch.cat([vals, -vals])
    n = vals.numel() // 127 * 127
    rows = vals[:n].view(-1, 127)
    out_rows = []
    for i, amax in enumerate(np.geomspace(2.0 ** -3, 2.0 ** 16, 41)):
        a = torch.tensor([amax], dtype=torch.float32).to(torch.bfloat16)
        r = rows[(torch.arange(rows.shape[0]) % 41) == i]
        r = r.float().clamp(-float(a), float(a)).to(torch.bfloat16)
        out_rows.append(torch.cat([r, a.expand(r.shape[0], 1)], dim=1))
    x = torch.cat(out_rows).view(-1, 1, 128)
    xd = x.to(DEV)
    dst = torch.empty(x.shape, dtype=torch.uint8, device=DEV)
    scale = torch.empty(x.shape[:2], device=DEV)
    hs2.hs2_quantize_kv(xd, dst, scale)
    hs2.hs2_sync()
    _check(x, dst, scale)


def test_every_scale_mantissa_and_tiny_rows():
    """Rows whose amax takes each of the 128 bf16 mantissas at three binades
    (every scale mantissa the kernel can meet), each filled with every bf16
    value from amax * 2^-20 up to amax of both signs, plus rows of amax below
    448 * 2^-90 (the kernel's IEEE-division branch) and bf16 subnormals."""
    rows = []
    for e in (-3, 4, 12):
        for m in range(128):
            a = np.float32((128 + m) / 128 * 2.0 ** e)
            hi = int(np.array([a], dtype=np.float32).view(np.uint32)[0] >> 16)
            pats = np.arange(hi - 20 * 128, hi + 1, dtype=np.uint32)
            vals = (pats << 16).view(np.float32)
            vals = np.concatenate([vals, -vals[:-1]])
            n = vals.size // 127 * 127
            r = vals[:n].reshape(-1, 127)
            rows.append(np.concatenate([r, np.full((r.shape[0], 1), a, dtype=np.float32)], axis=1))
    tiny = np.float32(2.0 ** -100)
    t = (np.arange(1, 128 * 128 + 1, dtype=np.float32) / (128 * 128)).reshape(-1, 128) * tiny
    t[:, 0] = tiny
    t[1::2] *= -1
    rows.append(t.astype(np.float32))
    sub = (np.arange(1, 129, dtype=np.uint32) << 16).view(np.float32).reshape(1, 128)  # bf16 subnormals
    rows.append(np.concatenate([sub, -sub]))
    x = torch.from_numpy(np.concatenate(rows)).to(torch.bfloat16).view(-1, 1, 128)
    xd = x.to(DEV)
    dst = torch.empty(x.shape, dtype=torch.uint8, device=DEV)
    scale = torch.empty(x.shape[:2], device=DEV)
    hs2.hs2_quantize_kv(xd, dst, scale)
    hs2.hs2_sync()
    _check(x, dst, scale)
