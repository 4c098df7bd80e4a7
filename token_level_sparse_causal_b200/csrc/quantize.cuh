// FP8 KV write (the step that produces the e4m3 cache the other kernels read;
// HySparse2 architecture summary, cost paragraph: FP8 KV cache).
//
// For every (token, KV head) row of 128 bf16 values: amax over the row,
// scale = amax / 448 in fp32 (1 for an all-zero row), and codes =
// e4m3(x / scale) with the division in fp32 and saturating round-to-nearest-
// even conversion.  Grid-stride over rows.  Memory-bound: 256 B read, 128 B +
// 4 B written per row.
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
#pragma unroll
      for (int q = 0; q < 4; ++q) c[q] = e4m3x2_from_f32(v[2 * q] / scale, v[2 * q + 1] / scale);
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
