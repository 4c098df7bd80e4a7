// Kernel (3): per (KV head, query block) top-k over the candidate importance
// row plus the forced recent window (HySparse2 architecture summary,
// token-selection paragraph: 1024 global tokens + the 128 most recent;
// branch-removal paragraph: the recent tokens replace the sliding-window
// branch).
//
// One CTA of 512 threads per row.  With n = |C_b| candidates:
//   n <= k : every candidate is selected; the row is never read.
//   n >  k : the set is {j : key_j > T} plus the krem lowest positions with
//            key_j == T, where T is the k-th largest order-preserving 32-bit
//            key of the fp32 values and krem = k - #{key > T}, emitted in
//            ascending position -- exactly a stable sort on (-I, j) followed
//            by a sort of the first k positions.  The fast path (sample,
//            one filtering pass, exact resolution in shared memory) finds it
//            with one read of the row; a three-pass radix path over the row
//            is the fallback when the sample's threshold gathers too few or
//            too many values.
// The recent window [e_b - recent, e_b) follows, then -1 padding.
#pragma once

#include "common.cuh"

namespace hs2 {

constexpr int SEL_THREADS = 512;
constexpr int SEL_CAP = 4096;      // candidates the fast path gathers in shared memory
constexpr int SEL_SAMPLES = 4096;  // most sampled values that set its threshold
constexpr int SEL_BITMAP_BITS = 32 * SEL_SAMPLES;  // rows up to this long emit through a bitmap

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

// The exact three-pass radix path over a row in global memory: radix select
// of the k-th largest key T on order-preserving keys (digits of 11, 11 and 10
// bits), then one ordered compaction pass that emits, in ascending position,
// every j with key > T and the first krem positions with key == T.
__device__ void select_radix_global(const float4* row4, int n4, uint32_t k, uint32_t* hist, uint32_t* warp_sums,
                                    uint32_t* sh, int32_t* list) {
  const int tid = threadIdx.x;
  uint32_t prefix = 0, pmask = 0;
  uint32_t krem = k;
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
          sh[0] = static_cast<uint32_t>(bin);
          sh[1] = run;
          break;
        }
        run += c;
      }
    }
    __syncthreads();
    prefix |= sh[0] << shift;
    pmask |= static_cast<uint32_t>(nbins - 1) << shift;
    krem -= sh[1];
    __syncthreads();
  }
  const uint32_t T = prefix;
  const uint32_t n_gt = k - krem;
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
}

// k-th largest of n keys in shared memory, by radix select (digits of 11, 11
// and 10 bits, histogram in `hist`): returns T and sets *krem to the number
// of keys equal to T among the k largest.  Requires 1 <= k <= n.  Every
// thread gets the same result.  passes = 2 stops after the top 22 bits and
// returns the lower edge of the bin holding the k-th largest (a lower bound
// within 2^10 key steps; *krem is then meaningless).
__device__ uint32_t smem_kth_largest(const uint32_t* keys, int n, uint32_t k, uint32_t* hist, uint32_t* warp_sums,
                                     uint32_t* sh, uint32_t* krem_out, int passes = 3) {
  const int tid = threadIdx.x;
  uint32_t prefix = 0, pmask = 0, krem = k;
#pragma unroll 1
  for (int pass = 0; pass < passes; ++pass) {
    const int shift = (pass == 0) ? 21 : (pass == 1) ? 10 : 0;
    const int nbins = (pass == 2) ? 1024 : 2048;
    for (int i = tid; i < nbins; i += SEL_THREADS) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += SEL_THREADS) {
      const uint32_t key = keys[i];
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
          sh[0] = static_cast<uint32_t>(bin);
          sh[1] = run;
          break;
        }
        run += c;
      }
    }
    __syncthreads();
    prefix |= sh[0] << shift;
    pmask |= static_cast<uint32_t>(nbins - 1) << shift;
    krem -= sh[1];
    __syncthreads();
  }
  *krem_out = krem;
  return prefix;
}

// Ascending bitonic sort of a[0, np) in shared memory; np a power of two,
// at most 2 * SEL_THREADS * 4.  Called by the whole CTA.
__device__ void bitonic_sort_smem(uint32_t* a, int np) {
#pragma unroll 1
  for (int size = 2; size <= np; size <<= 1) {
#pragma unroll 1
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = threadIdx.x; t < (np >> 1); t += SEL_THREADS) {
        const int lo = 2 * t - (t & (stride - 1));
        const int hi = lo + stride;
        const uint32_t x = a[lo], y = a[hi];
        if ((x > y) == ((lo & size) == 0)) {
          a[lo] = y;
          a[hi] = x;
        }
      }
      __syncthreads();
    }
  }
}

// One streaming pass over a row: appends the raw bits and the position of
// every value whose order key is >= tau to (ckey, cpos) (at most SEL_CAP are
// stored; *count receives the total).  FAST: tau is the key of a positive
// float, and for any fp32 v, order_key(v) >= tau exactly when the bits of v
// as a signed integer are >= those of that float (negative values, -0.0 and
// negative NaNs are negative integers; positive NaNs lie above +inf in both
// orders), so one integer compare decides.  Each thread first counts its
// values (16 in flight); a thread with hits reserves that many slots with one
// shared atomic and stores them.  The slot order is not deterministic, and
// nothing downstream depends on it (the set is order-free; emission is by
// position).
template <bool FAST>
__device__ __forceinline__ void gather_pass(const float4* row4, int n4, uint32_t tau, uint32_t* ckey,
                                            uint32_t* cpos, uint32_t* count) {
  constexpr int U = 4;  // float4 loads in flight per thread
  const int tid = threadIdx.x;
  const int tau_i = static_cast<int>(tau & 0x7FFFFFFFu);
  auto hit = [&](float f, bool live) -> bool {
    return FAST ? (__float_as_int(f) >= tau_i) : (live && order_key(f) >= tau);
  };
#pragma unroll 1
  for (int base4 = 0; base4 < n4; base4 += SEL_THREADS * U) {
    float4 v[U];
    bool live[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i4 = base4 + u * SEL_THREADS + tid;
      live[u] = i4 < n4;
      // -inf pads the tail: a negative integer, never >= a positive float
      v[u] = live[u] ? __ldg(row4 + i4) : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    }
    uint32_t c = 0;
#pragma unroll
    for (int u = 0; u < U; ++u)
      c += (hit(v[u].x, live[u]) ? 1u : 0u) + (hit(v[u].y, live[u]) ? 1u : 0u) + (hit(v[u].z, live[u]) ? 1u : 0u) +
           (hit(v[u].w, live[u]) ? 1u : 0u);
    if (c) {
      // hits are sparse (about 2k of a row's values pass tau), so the few
      // lanes with any reserve their slots with one shared atomic each
      uint32_t at = atomicAdd(count, c);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint32_t p0 = static_cast<uint32_t>(base4 + u * SEL_THREADS + tid) * 4u;
        const float vv[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (hit(vv[e], live[u])) {
            if (at < SEL_CAP) {
              ckey[at] = __float_as_uint(vv[e]);
              cpos[at] = p0 + e;
            }
            ++at;
          }
        }
      }
    }
  }
}

// Shared memory of topk_select_kernel (dynamic).
struct SelSmem {
  uint32_t ckey[SEL_CAP];    // gathered candidates: order keys ...
  uint32_t cpos[SEL_CAP];    // ... and positions
  uint32_t samp[SEL_SAMPLES];
  uint32_t hist[2048];
  uint32_t warp_sums[32];
  uint32_t sh[8];  // [0, 1] radix select; [2] winners; [3] keys == T; [4] ties gathered
  uint32_t count;
};

// Kernel (3).  For rows with n > k candidates, the fast path reads the row
// once: a sample of up to SEL_SAMPLES values (groups of 8 consecutive values
// spread evenly over the row) gives a threshold tau (a lower bound, within
// 2^10 key steps, of the sample's q-th largest, q chosen so that about 2k
// values are expected at or above it; tau = 0 when the whole row fits in
// shared memory), every value >= tau is gathered into shared memory, and
// there the k-th largest T and the tie count are found exactly; the winners
// are emitted through a position bitmap, or sorted bitonically for very long
// rows and for ties at T that do not all fit.  The k-th largest of the row is
// >= tau whenever at least k values were gathered, so the set is exactly the
// one of the three-pass radix path below; that path runs instead when fewer
// than k or more than SEL_CAP values were gathered.
__global__ void __launch_bounds__(SEL_THREADS, 3) topk_select_kernel(const SelParams p) {
  extern __shared__ __align__(16) uint8_t sel_raw[];
  SelSmem& S = *reinterpret_cast<SelSmem*>(sel_raw);

  const int y = blockIdx.x;
  const int g = y / p.nbs;
  const int b = p.b0 + y % p.nbs;
  const int e_b = min(p.L, 64 * (b + 1));
  const int n_c = max(0, e_b - p.recent);
  const int nrec = min(p.recent, e_b);
  const int kk = min(n_c, p.topk);
  const int total = kk + nrec;
  int32_t* list = p.idx + (static_cast<int64_t>(g) * p.nb + b) * p.list_len;
  const int tid = threadIdx.x, lane = tid & 31;

  if (n_c > p.topk) {
    const float* row = p.imp + (static_cast<int64_t>(g) * p.nbs + (b - p.b0)) * p.row_stride;
    const float4* row4 = reinterpret_cast<const float4*>(row);
    const int n4 = n_c >> 2;  // n_c is a multiple of 64
    const uint32_t k = static_cast<uint32_t>(p.topk);

    // ---- threshold from a sample of whole 32-byte sectors: groups of 8
    // consecutive values spread evenly over the row (a scattered sample
    // would touch a separate DRAM burst per value)
    uint32_t tau = 0;
    if (n_c > SEL_CAP) {
      // 1024, 2048 or 4096 sampled values (128, 256 or 512 groups)
      const int lg = n_c >= 8 * SEL_SAMPLES ? 12 : n_c >= 8 * 2048 ? 11 : 10;
      const int ns = 1 << lg;
      if (tid < (ns >> 3)) {  // group tid starts at a multiple of 8, ends before n_c
        const int j0 = static_cast<int>((static_cast<int64_t>(tid) * n_c) >> (lg - 3)) & ~7;
        const float4 a = __ldg(row4 + (j0 >> 2)), c = __ldg(row4 + (j0 >> 2) + 1);
        uint4 o0 = make_uint4(order_key(a.x), order_key(a.y), order_key(a.z), order_key(a.w));
        uint4 o1 = make_uint4(order_key(c.x), order_key(c.y), order_key(c.z), order_key(c.w));
        *reinterpret_cast<uint4*>(S.samp + 8 * tid) = o0;
        *reinterpret_cast<uint4*>(S.samp + 8 * tid + 4) = o1;
      }
      __syncthreads();
      const int64_t qq = (2 * static_cast<int64_t>(k) * ns + n_c - 1) / n_c;
      const uint32_t q = static_cast<uint32_t>(qq < 1 ? 1 : (qq > ns ? ns : qq));
      uint32_t unused;  // a lower bound of the sample's q-th largest is enough for tau
      tau = smem_kth_largest(S.samp, ns, q, S.hist, S.warp_sums, S.sh, &unused, 2);
    }
    // ---- gather every value >= tau: the raw fp32 bits and positions go to
    // shared memory (warp-aggregated appends; order is restored below), then
    // the bits are mapped to order keys
    if (tid == 0) S.count = 0;
    __syncthreads();
    if (tau > 0x80000000u)
      gather_pass<true>(row4, n4, tau, S.ckey, S.cpos, &S.count);
    else
      gather_pass<false>(row4, n4, tau, S.ckey, S.cpos, &S.count);
    __syncthreads();
    {
      const int ng = static_cast<int>(min(S.count, static_cast<uint32_t>(SEL_CAP)));
      for (int i = tid; i < ng; i += SEL_THREADS) S.ckey[i] = order_key(__uint_as_float(S.ckey[i]));
    }
    __syncthreads();
    const uint32_t cnt_g = S.count;
    if (cnt_g >= k && cnt_g <= SEL_CAP) {
      const int nc = static_cast<int>(cnt_g);
      uint32_t krem;
      const uint32_t T = smem_kth_largest(S.ckey, nc, k, S.hist, S.warp_sums, S.sh, &krem);
      const int ncr = (nc + 31) & ~31;  // warp-uniform trip count
      // ---- how many gathered keys equal T
      if (tid == 0) S.sh[2] = S.sh[3] = S.sh[4] = 0;
      __syncthreads();
      for (int i = tid; i < ncr; i += SEL_THREADS) {
        const uint32_t m = __ballot_sync(0xffffffffu, i < nc && S.ckey[i < nc ? i : 0] == T);
        if (lane == 0 && m) atomicAdd(&S.sh[3], static_cast<uint32_t>(__popc(m)));
      }
      __syncthreads();
      if (S.sh[3] == krem && n_c <= SEL_BITMAP_BITS) {
        // ---- every key >= T wins: mark positions in a bitmap (over the
        // sample buffer), then emit set bits in ascending order
        uint32_t* bm = S.samp;
        const int nw = (n_c + 31) >> 5;
        for (int i = tid; i < nw; i += SEL_THREADS) bm[i] = 0u;
        __syncthreads();
        for (int i = tid; i < nc; i += SEL_THREADS)
          if (S.ckey[i] >= T) atomicOr(&bm[S.cpos[i] >> 5], 1u << (S.cpos[i] & 31));
        __syncthreads();
        const int per = (nw + SEL_THREADS - 1) / SEL_THREADS;  // <= 8 words per thread
        const int w0 = min(nw, tid * per), w1 = min(nw, w0 + per);
        uint32_t cntw = 0;
        for (int w = w0; w < w1; ++w) cntw += static_cast<uint32_t>(__popc(bm[w]));
        uint32_t tot;
        uint32_t out = block_excl_scan(cntw, S.warp_sums, &tot);
        for (int w = w0; w < w1; ++w) {
          uint32_t bits = bm[w];
          while (bits) {
            const int bit = __ffs(bits) - 1;
            bits &= bits - 1;
            list[out++] = w * 32 + bit;
          }
        }
      } else {
      // ---- the winners: every key > T, then the krem lowest positions with
      // key == T (all of them when there are krem); sorted by position
      if (tid == 0) S.sh[2] = S.sh[3] = S.sh[4] = 0;
      __syncthreads();
      const uint32_t lt_mask = (1u << lane) - 1u;
      auto append = [&](bool f, uint32_t val, uint32_t* dst, uint32_t* counter) {
        const uint32_t m = __ballot_sync(0xffffffffu, f);
        if (m) {
          uint32_t at = 0;
          if (lane == 0) at = atomicAdd(counter, static_cast<uint32_t>(__popc(m)));
          at = __shfl_sync(0xffffffffu, at, 0) + static_cast<uint32_t>(__popc(m & lt_mask));
          if (f) dst[at] = val;
        }
      };
      for (int i = tid; i < ncr; i += SEL_THREADS) {
        const uint32_t key = (i < nc) ? S.ckey[i] : 0u;
        const bool live = i < nc;
        append(live && key > T, S.cpos[i < nc ? i : 0], S.samp, &S.sh[2]);
        if (live && key == T) S.cpos[i] |= 0x80000000u;  // positions are < 2^24
        const uint32_t m = __ballot_sync(0xffffffffu, live && key == T);
        if (lane == 0 && m) atomicAdd(&S.sh[3], static_cast<uint32_t>(__popc(m)));
      }
      __syncthreads();
      const uint32_t n_tie = S.sh[3];
      if (n_tie == krem) {
        for (int i = tid; i < ncr; i += SEL_THREADS) {
          const uint32_t cp = (i < nc) ? S.cpos[i] : 0u;
          append((i < nc) && (cp & 0x80000000u), cp & 0x7FFFFFFFu, S.samp, &S.sh[2]);
        }
      } else {  // more ties than places: the lowest positions win
        for (int i = tid; i < ncr; i += SEL_THREADS) {
          const uint32_t cp = (i < nc) ? S.cpos[i] : 0u;
          append((i < nc) && (cp & 0x80000000u), cp & 0x7FFFFFFFu, S.ckey, &S.sh[4]);
        }
        __syncthreads();
        const int nt = static_cast<int>(n_tie);
        int np = 1;
        while (np < nt) np <<= 1;
        for (int i = nt + tid; i < np; i += SEL_THREADS) S.ckey[i] = 0xFFFFFFFFu;
        __syncthreads();
        bitonic_sort_smem(S.ckey, np);
        const uint32_t n_gt = k - krem;
        for (int i = tid; i < static_cast<int>(krem); i += SEL_THREADS) S.samp[n_gt + i] = S.ckey[i];
      }
      __syncthreads();
      int np = 1;
      while (np < static_cast<int>(k)) np <<= 1;
      for (int i = static_cast<int>(k) + tid; i < np; i += SEL_THREADS) S.samp[i] = 0xFFFFFFFFu;
      __syncthreads();
      bitonic_sort_smem(S.samp, np);
      for (int i = tid; i < static_cast<int>(k); i += SEL_THREADS) list[i] = static_cast<int32_t>(S.samp[i]);
      }
    } else {
      select_radix_global(row4, n4, k, S.hist, S.warp_sums, S.sh, list);
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
// A block's pooled sum is taken in fp32: 16 lanes each add 4 consecutive
// values left to right, then a butterfly over the 16 lanes (l ^ 8, ^ 4, ^ 2,
// ^ 1); every step is commutative, so all lanes hold the same bits.  Blocks
// whose exact sums differ by less than the rounding of a 64-term fp32 sum
// may rank either way.  One 512-thread CTA per row; pooled values live in
// shared memory.
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
