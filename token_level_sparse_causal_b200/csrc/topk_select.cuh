// Kernel (3): per (KV head, query block) top-k over the candidate importance
// row plus the forced recent window (HySparse2 architecture summary,
// token-selection paragraph: 1024 global tokens + the 128 most recent;
// branch-removal paragraph: the recent tokens replace the sliding-window
// branch).
//
// One CTA of 512 threads per row.  With n = |C_b| candidates:
//   n <= k : every candidate is selected; the row is never read.
//   n >  k : radix select on order-preserving 32-bit keys of the fp32 values
//            (three histogram passes of 11, 11 and 10 bits) finds the k-th
//            largest key T and how many keys equal to T are taken (krem);
//            one ordered compaction pass then emits, in ascending position,
//            every j with key > T and the first krem positions with key == T.
//            Output order is ascending by construction (no sort), and ties
//            go to the lower position exactly as a stable sort on (-I, j).
// The recent window [e_b - recent, e_b) follows, then -1 padding.
#pragma once

#include "common.cuh"

namespace hs2 {

constexpr int SEL_THREADS = 512;

struct SelParams {
  int L, Hkv, nb, recent, topk, b0, nbs, list_len;
  const float* imp;
  int64_t row_stride;
  int32_t* idx;
  int32_t* cnt;
};

// Monotone map from float to uint32 (-0.0 folded onto +0.0 first).
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;  // -0.0 ranks with +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Block-wide exclusive prefix sum of one uint32 per thread; returns the
// exclusive prefix and writes the block total to *total.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* warp_sums, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = (lane < SEL_THREADS / 32) ? warp_sums[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < SEL_THREADS / 32) warp_sums[lane] = w;  // inclusive
  }
  __syncthreads();
  const uint32_t before = (warp > 0) ? warp_sums[warp - 1] : 0u;
  *total = warp_sums[SEL_THREADS / 32 - 1];
  __syncthreads();  // warp_sums is reused by the next call
  return before + x - v;
}

__global__ void __launch_bounds__(SEL_THREADS) topk_select_kernel(const SelParams p) {
  __shared__ uint32_t hist[2048];
  __shared__ uint32_t warp_sums[32];
  __shared__ uint32_t sh_digit, sh_above;

  const int y = blockIdx.x;
  const int g = y / p.nbs;
  const int b = p.b0 + y % p.nbs;
  const int e_b = min(p.L, 64 * (b + 1));
  const int n_c = max(0, e_b - p.recent);
  const int nrec = min(p.recent, e_b);
  const int kk = min(n_c, p.topk);
  const int total = kk + nrec;
  int32_t* list = p.idx + (static_cast<int64_t>(g) * p.nb + b) * p.list_len;
  const int tid = threadIdx.x;

  if (n_c > p.topk) {
    const float* row = p.imp + (static_cast<int64_t>(g) * p.nbs + (b - p.b0)) * p.row_stride;
    const float4* row4 = reinterpret_cast<const float4*>(row);
    const int n4 = n_c >> 2;  // n_c is a multiple of 64
    uint32_t prefix = 0, pmask = 0;
    uint32_t krem = static_cast<uint32_t>(p.topk);
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
      const int shift = (pass == 0) ? 21 : (pass == 1) ? 10 : 0;  // digits of 11, 11 and 10 bits
      const int nbins = (pass == 2) ? 1024 : 2048;
      for (int i = tid; i < nbins; i += SEL_THREADS) hist[i] = 0;
      __syncthreads();
      for (int i = tid; i < n4; i += SEL_THREADS) {
        const float4 v = __ldg(row4 + i);
        const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t key = order_key(vv[e]);
          if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & (nbins - 1)], 1u);
        }
      }
      __syncthreads();
      // Thread t owns the bins [nbins - (t+1)*per, nbins - t*per), scanned
      // from the top bin down.
      const int per = nbins / SEL_THREADS;
      uint32_t loc = 0;
      for (int q = 0; q < per; ++q) loc += hist[nbins - 1 - (tid * per + q)];
      uint32_t tot;
      const uint32_t ex = block_excl_scan(loc, warp_sums, &tot);
      if (ex < krem && ex + loc >= krem) {
        uint32_t run = ex;
        for (int q = 0; q < per; ++q) {
          const int bin = nbins - 1 - (tid * per + q);
          const uint32_t c = hist[bin];
          if (run + c >= krem) {
            sh_digit = static_cast<uint32_t>(bin);
            sh_above = run;
            break;
          }
          run += c;
        }
      }
      __syncthreads();
      prefix |= sh_digit << shift;
      pmask |= static_cast<uint32_t>(nbins - 1) << shift;
      krem -= sh_above;
      __syncthreads();
    }
    const uint32_t T = prefix;
    const uint32_t n_gt = static_cast<uint32_t>(p.topk) - krem;
    // ---- ordered compaction
    uint32_t gt_carry = 0, eq_carry = 0;
#pragma unroll 1
    for (int base4 = 0; base4 < n4; base4 += SEL_THREADS) {
      const int i4 = base4 + tid;
      uint32_t gt_m = 0, eq_m = 0;
      if (i4 < n4) {
        const float4 v = __ldg(row4 + i4);
        const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t key = order_key(vv[e]);
          gt_m |= (key > T ? 1u : 0u) << e;
          eq_m |= (key == T ? 1u : 0u) << e;
        }
      }
      const uint32_t packed = (static_cast<uint32_t>(__popc(gt_m)) << 16) | static_cast<uint32_t>(__popc(eq_m));
      uint32_t tot;
      const uint32_t ex = block_excl_scan(packed, warp_sums, &tot);
      uint32_t gt_before = gt_carry + (ex >> 16);
      uint32_t eq_before = eq_carry + (ex & 0xFFFFu);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = i4 * 4 + e;
        if (gt_m & (1u << e)) {
          list[gt_before + min(eq_before, krem)] = j;
          ++gt_before;
        } else if (eq_m & (1u << e)) {
          if (eq_before < krem) list[gt_before + eq_before] = j;
          ++eq_before;
        }
      }
      gt_carry += tot >> 16;
      eq_carry += tot & 0xFFFFu;
      if (gt_carry >= n_gt && eq_carry >= krem) break;  // block-uniform
    }
  } else {
    for (int i = tid; i < kk; i += SEL_THREADS) list[i] = i;
  }
  for (int i = tid; i < nrec; i += SEL_THREADS) list[kk + i] = e_b - nrec + i;
  for (int i = total + tid; i < p.list_len; i += SEL_THREADS) list[i] = -1;
  if (tid == 0) p.cnt[static_cast<int64_t>(g) * p.nb + b] = total;
}

// Block-level selection (HySparse v1, the design the token-level selection
// replaces; HySparse2 architecture summary, block-selection paragraph): each
// candidate row is pooled into 64-key blocks, the top topk/64 blocks by pooled
// importance are kept (ties to the lower block) and expanded to positions.
// The pooled sum of a block is defined in a fixed fp32 order: 16 lanes each
// add 4 consecutive values left to right, then a butterfly over the 16 lanes
// (l ^ 8, ^ 4, ^ 2, ^ 1); every step is commutative, so all lanes hold the
// same bits.  One 512-thread CTA per row; pooled values live in shared memory.
__global__ void __launch_bounds__(SEL_THREADS) block_select_kernel(const SelParams p) {
  extern __shared__ float pooled[];  // [n_blk]
  __shared__ uint32_t hist[2048];
  __shared__ uint32_t warp_sums[32];
  __shared__ uint32_t sh_digit, sh_above;
  __shared__ int sel[64];

  const int y = blockIdx.x;
  const int g = y / p.nbs;
  const int b = p.b0 + y % p.nbs;
  const int e_b = min(p.L, 64 * (b + 1));
  const int n_c = max(0, e_b - p.recent);
  const int nrec = min(p.recent, e_b);
  const int n_blk = n_c / 64, kb = p.topk / 64;
  const int nsel = min(n_blk, kb);
  int32_t* list = p.idx + (static_cast<int64_t>(g) * p.nb + b) * p.list_len;
  const int tid = threadIdx.x;

  if (n_blk > kb) {
    const float4* row4 = reinterpret_cast<const float4*>(p.imp + (static_cast<int64_t>(g) * p.nbs + (b - p.b0)) *
                                                                    p.row_stride);
    const int l16 = tid & 15;
    // a half-warp per block; the loop bound is warp-uniform (full-mask shuffles)
    for (int m0 = (tid >> 5) * 2; m0 < n_blk; m0 += SEL_THREADS / 16) {
      const int m = m0 + ((tid >> 4) & 1);
      const float4 v = (m < n_blk) ? __ldg(row4 + m * 16 + l16) : make_float4(0.f, 0.f, 0.f, 0.f);
      float a = ((v.x + v.y) + v.z) + v.w;
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) a = a + __shfl_xor_sync(0xffffffffu, a, o);
      if (m < n_blk && l16 == 0) pooled[m] = a;
    }
    __syncthreads();
    uint32_t prefix = 0, pmask = 0, krem = static_cast<uint32_t>(kb);
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
      const int shift = (pass == 0) ? 21 : (pass == 1) ? 10 : 0;
      const int nbins = (pass == 2) ? 1024 : 2048;
      for (int i = tid; i < nbins; i += SEL_THREADS) hist[i] = 0;
      __syncthreads();
      for (int m = tid; m < n_blk; m += SEL_THREADS) {
        const uint32_t key = order_key(pooled[m]);
        if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & (nbins - 1)], 1u);
      }
      __syncthreads();
      const int per = nbins / SEL_THREADS;
      uint32_t loc = 0;
      for (int q = 0; q < per; ++q) loc += hist[nbins - 1 - (tid * per + q)];
      uint32_t tot;
      const uint32_t ex = block_excl_scan(loc, warp_sums, &tot);
      if (ex < krem && ex + loc >= krem) {
        uint32_t run = ex;
        for (int q = 0; q < per; ++q) {
          const int bin = nbins - 1 - (tid * per + q);
          const uint32_t c = hist[bin];
          if (run + c >= krem) {
            sh_digit = static_cast<uint32_t>(bin);
            sh_above = run;
            break;
          }
          run += c;
        }
      }
      __syncthreads();
      prefix |= sh_digit << shift;
      pmask |= static_cast<uint32_t>(nbins - 1) << shift;
      krem -= sh_above;
      __syncthreads();
    }
    const uint32_t T = prefix;
    uint32_t gt_carry = 0, eq_carry = 0;
#pragma unroll 1
    for (int base = 0; base < n_blk; base += SEL_THREADS) {
      const int m = base + tid;
      bool gt = false, eq = false;
      if (m < n_blk) {
        const uint32_t key = order_key(pooled[m]);
        gt = key > T;
        eq = key == T;
      }
      uint32_t tot;
      const uint32_t ex = block_excl_scan((gt ? 1u << 16 : 0u) | (eq ? 1u : 0u), warp_sums, &tot);
      const uint32_t gt_before = gt_carry + (ex >> 16), eq_before = eq_carry + (ex & 0xFFFFu);
      if (gt) sel[gt_before + min(eq_before, krem)] = m;
      else if (eq && eq_before < krem) sel[gt_before + eq_before] = m;
      gt_carry += tot >> 16;
      eq_carry += tot & 0xFFFFu;
    }
  } else {
    for (int i = tid; i < nsel; i += SEL_THREADS) sel[i] = i;
  }
  __syncthreads();
  for (int i = tid; i < nsel * 64; i += SEL_THREADS) list[i] = sel[i >> 6] * 64 + (i & 63);
  for (int i = tid; i < nrec; i += SEL_THREADS) list[nsel * 64 + i] = e_b - nrec + i;
  for (int i = nsel * 64 + nrec + tid; i < p.list_len; i += SEL_THREADS) list[i] = -1;
  if (tid == 0) p.cnt[static_cast<int64_t>(g) * p.nb + b] = nsel * 64 + nrec;
}

}  // namespace hs2
