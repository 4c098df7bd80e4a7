// FP8 KV write (the step that produces the e4m3 cache the other kernels read;
// HySparse2 architecture summary, cost paragraph: FP8 KV cache).
//
// For every (token, KV head) row of 128 bf16 values: amax over the row,
// scale = amax / 448 in fp32 (1 for an all-zero row), and codes =
// e4m3(x / scale) with the quotient correctly rounded to fp32 (the IEEE
// quotient) and saturating round-to-nearest-even conversion.  Grid-stride
// over rows.  Memory-bound: 256 B read, 128 B + 4 B written per row.
#pragma once

#include "common.cuh"

namespace hs2 {

struct QuantParams {
  int rows;  // L * Hkv (< 2^31, checked on the host)
  int Hkv;
  const __nv_bfloat16* src;
  int64_t src_tok, src_head;  // elements
  uint8_t* dst;
  int64_t dst_tok, dst_head;  // bytes
  float* scale;               // [L][Hkv]
};

__device__ __forceinline__ uint32_t e4m3x2_from_f32(float lo, float hi) {
  uint16_t c;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(c) : "f"(hi), "f"(lo));
  return c;
}

// A half-warp covers one row with 16-byte loads (8 values per lane); each warp
// issues the loads of 8 rows before converting any, to keep bytes in flight.
__global__ void __launch_bounds__(256) quantize_kv_kernel(const QuantParams p) {
  constexpr int ROWS = 8;  // rows per warp and iteration (2 per load step)
  const int lane = threadIdx.x & 31;
  const int sub = lane >> 4, l16 = lane & 15;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * 8;
  for (int64_t base = (static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5)) * ROWS; base < p.rows;
       base += nwarps * ROWS) {
    uint4 raw[ROWS / 2];
    int rowi[ROWS / 2];
#pragma unroll
    for (int k = 0; k < ROWS / 2; ++k) {
      rowi[k] = static_cast<int>(base) + 2 * k + sub;
      raw[k] = make_uint4(0, 0, 0, 0);
      if (rowi[k] < p.rows) {
        const int t = rowi[k] / p.Hkv;
        const int hd = rowi[k] - t * p.Hkv;
        raw[k] = ld_nc_v4(p.src + static_cast<int64_t>(t) * p.src_tok + hd * p.src_head + l16 * 8);
      }
    }
#pragma unroll
    for (int k = 0; k < ROWS / 2; ++k) {
      const uint32_t w[4] = {raw[k].x, raw[k].y, raw[k].z, raw[k].w};
      float v[8];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        v[2 * q] = __uint_as_float(w[q] << 16);
        v[2 * q + 1] = __uint_as_float(w[q] & 0xFFFF0000u);
      }
      float a = 0.f;
#pragma unroll
      for (int q = 0; q < 8; ++q) a = fmaxf(a, fabsf(v[q]));
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));  // within the half-warp
      const float scale = (a > 0.f) ? a / 448.0f : 1.0f;
      uint32_t c[4];
      if (scale >= 0x1p-90f) {
        // x / scale, correctly rounded, without a division per value:
        // Markstein's method (P. Markstein, "Computation of elementary
        // functions on the IBM RISC System/6000 processor", IBM J. Res. Dev.
        // 34(1), 1990) with y = RN(1 / scale) once per row, q = RN(x y), then
        // q = RN(q + RN(x - q scale) y) by two FMAs, on value pairs.  Exact
        // rational arithmetic over every pair of bf16 mantissas of x and of
        // the row's amax gives RN(x / scale) (tests/test_markstein_division.py;
        // exponents shift every quantity alike while all stay normal, and the
        // scale bound keeps the residuals normal for every quotient above
        // 2^-12, below which both round to a zero code).
        const float y = __frcp_rn(scale);
        const uint64_t y2 = f2_pack(y, y), ns2 = f2_pack(-scale, -scale);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint64_t x2 = f2_pack(v[2 * q], v[2 * q + 1]);
          uint64_t q2 = f2_mul(x2, y2);
          q2 = f2_fma(f2_fma(q2, ns2, x2), y2, q2);
          float q0, q1;
          f2_unpack(q2, q0, q1);
          // the quotient has x's sign; the correction's RN(+0 + -0) = +0
          // would lose it for x = -0
          c[q] = e4m3x2_from_f32(copysignf(q0, v[2 * q]), copysignf(q1, v[2 * q + 1]));
        }
      } else {  // rows of amax below 448 * 2^-90: the IEEE division
#pragma unroll
        for (int q = 0; q < 4; ++q) c[q] = e4m3x2_from_f32(v[2 * q] / scale, v[2 * q + 1] / scale);
      }
      if (rowi[k] < p.rows) {
        const int t = rowi[k] / p.Hkv;
        const int hd = rowi[k] - t * p.Hkv;
        *reinterpret_cast<uint2*>(p.dst + static_cast<int64_t>(t) * p.dst_tok + hd * p.dst_head + l16 * 8) =
            make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
        if (l16 == 0) p.scale[rowi[k]] = scale;
      }
    }
  }
}

}  // namespace hs2

namespace hs2 {

// Once-per-layer dequantisation of the e4m3 cache for the dense passes.
//
// The full-attention kernel and the importance pass read every K/V tile of a
// KV head once per query tile and query head; converting the codes inside
// those kernels repeats the same conversion G * (tiles before it) times and
// competes with the softmax for the conversion units.  This pass converts the
// cache once into f16 buffers the dense kernels load by TMA, with exactly the
// arithmetic of the in-kernel converters:
//   kf[t][g][:]  = f16(code)                (exact: every e4m3 value is an f16)
//   vf[t][g][:]  = f16(code) * f16(vscale)  (one f16 multiply, as in the gather)
//   kcol[g][t]   = kscale[t][g] * log2(e)/sqrt(d)   (fp32; 0 for L <= t < Lp)
// Memory-bound: 2 x 128 B + 8 B read, 2 x 256 B + 4 B written per row.
struct DequantParams {
  int L, Hkv, Lp;  // Lp: kcol row stride (L rounded up to the key tile)
  const uint8_t* k8;
  const uint8_t* v8;
  int64_t kv_tok, kv_head;  // bytes
  const float* ksc;         // [L][Hkv]
  const float* vsc;
  uint16_t* kf;  // f16 bits, [L][Hkv][128] contiguous
  uint16_t* vf;
  float* kcol;  // [Hkv][Lp]
  float scale_log2;
};

// Eight threads per (token, head) row, 16 codes of K and 16 of V each; every
// thread issues the loads of ROWS rows before converting any.
__global__ void __launch_bounds__(256) dequant_kv_kernel(const DequantParams p) {
  constexpr int ROWS = 4;  // row steps per thread and iteration
  const int64_t rows = static_cast<int64_t>(p.Lp) * p.Hkv;
  const int c8 = threadIdx.x & 7;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 3);
  for (int64_t r0 = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 3) + (threadIdx.x >> 3); r0 < rows;
       r0 += stride * ROWS) {
    uint4 rk[ROWS], rv[ROWS];
    float sk[ROWS], sv[ROWS];
#pragma unroll
    for (int u = 0; u < ROWS; ++u) {
      const int64_t row = r0 + u * stride;
      const int t = static_cast<int>(row / p.Hkv), g = static_cast<int>(row % p.Hkv);
      rk[u] = rv[u] = make_uint4(0, 0, 0, 0);
      sk[u] = sv[u] = 0.f;
      if (row < rows && t < p.L) {
        const int64_t off = static_cast<int64_t>(t) * p.kv_tok + static_cast<int64_t>(g) * p.kv_head + c8 * 16;
        rk[u] = ld_nc_v4(p.k8 + off);
        rv[u] = ld_nc_v4(p.v8 + off);
        sk[u] = p.ksc[static_cast<int64_t>(t) * p.Hkv + g];
        sv[u] = p.vsc[static_cast<int64_t>(t) * p.Hkv + g];
      }
    }
#pragma unroll
    for (int u = 0; u < ROWS; ++u) {
      const int64_t row = r0 + u * stride;
      if (row >= rows) continue;
      const int t = static_cast<int>(row / p.Hkv), g = static_cast<int>(row % p.Hkv);
      if (c8 == 0) p.kcol[static_cast<int64_t>(g) * p.Lp + t] = (t < p.L) ? sk[u] * p.scale_log2 : 0.f;
      if (t >= p.L) continue;
      const uint32_t wk[4] = {rk[u].x, rk[u].y, rk[u].z, rk[u].w};
      const uint32_t wv[4] = {rv[u].x, rv[u].y, rv[u].z, rv[u].w};
      const uint32_t s2 = pack_f16x2(sv[u], sv[u]);
      uint32_t fk[8], fv[8];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        fk[2 * q] = e4m3x2_to_f16x2(wk[q]);
        fk[2 * q + 1] = e4m3x2_to_f16x2(wk[q] >> 16);
        fv[2 * q] = hmul2_u32(e4m3x2_to_f16x2(wv[q]), s2);
        fv[2 * q + 1] = hmul2_u32(e4m3x2_to_f16x2(wv[q] >> 16), s2);
      }
      const int64_t o = (static_cast<int64_t>(t) * p.Hkv + g) * 128 + c8 * 16;
      uint4* dk = reinterpret_cast<uint4*>(p.kf + o);
      uint4* dv = reinterpret_cast<uint4*>(p.vf + o);
      dk[0] = make_uint4(fk[0], fk[1], fk[2], fk[3]);
      dk[1] = make_uint4(fk[4], fk[5], fk[6], fk[7]);
      dv[0] = make_uint4(fv[0], fv[1], fv[2], fv[3]);
      dv[1] = make_uint4(fv[4], fv[5], fv[6], fv[7]);
    }
  }
}

}  // namespace hs2
