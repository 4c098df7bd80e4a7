// Flash-attention forward on tcgen05 tensor cores (the sparse layers' and
// the sliding window's persistent kernel in sparse_attn.cuh is built on the
// same pipeline):
//
// Kernel (1): causal grouped-query attention of the full layer, one CTA per
// (pair of 128-query tiles, query head), K/V tiles of 128 keys streamed
// through shared memory; writes O and the per-query natural-log LSE.
// (HySparse2 architecture summary, ablation paragraph: the full layer's
// complete scores; SHARP walk-through, section 1.1: softmax(Q K^T / sqrt(d)) V.)
//
// CTA = 12 warps:
//   warp 0      TMA: Q tiles, K/V tiles (bf16 cache, or the f16 copy of an
//               FP8 cache with its K column scales)
//   warp 1      TMEM allocation; one thread issues every tcgen05.mma
//   warps 2-3   with an FP8 cache: convert Q to f16 in place; when reading
//               the e4m3 codes directly, also load, convert and scale every
//               K/V tile
//   warps 4-7   softmax / rescale / epilogue of query tile A (thread r <-> row r)
//   warps 8-11  the same for query tile B
//
// FP8 e4m3 cache: every e4m3 value is an f16 value, so codes convert exactly
// to f16, Q is converted bf16 -> f16 in shared memory after its TMA load, and
// all MMAs run kind::f16 on f16 operands.  The per-token K scale (times
// log2(e)/sqrt(d)) multiplies the S columns in fp32; the V scale is folded
// into the f16 V rows.  Two ways to get the f16 tiles, same values:
//   KVM_E4M3  warps 2-3 load the codes and convert every tile in the kernel
//             (no scratch memory);
//   KVM_F16   the cache was converted once for the layer (dequant_kv_kernel)
//             and warp 0 loads f16 tiles by TMA plus each tile's 128 column
//             scales by a bulk copy -- the conversion is not repeated for
//             every query head and query tile that reads the tile.
// (HySparse2 architecture summary, cost paragraph: FP8 KV cache.)
//
// Tensor memory (512 columns): S_A [0,128), S_B [128,256), O_A [256,384),
// O_B [384,512).  P (bf16) is written over the first 64 columns of its S and
// fed to the PV product straight from tensor memory.
//
// Per key tile j the MMA thread issues PV_A(j), S_A(j+1), PV_B(j), S_B(j+1),
// so while softmax A works on S_A(j+1) the tensor core runs PV_B(j) and
// S_B(j+1), and vice versa: the two softmax warpgroups take turns and the
// tensor core always has the other tile's work.  Only P stands between a
// softmax phase and the products that follow it: the MMA thread checks that
// V(j) and K(j + 1) landed before it waits for P; a stage's K is released
// after both S products of its tile, its V after both P V products; the
// softmax needs no wait on the previous P V (s_full's commit covers it, as a
// commit covers every earlier MMA of the thread), and O is signalled only
// after a tile's last product.
//
// Softmax runs in the log2 domain with a lazily updated reference max: O is
// rescaled only when a row max grows by more than 8 (P stays below 256; the
// final O / l is exact up to rounding).  Arguments and row sums use packed
// f32x2 FMA/ADD and the row max 3-input max, in independent partial chains:
// the softmax is bound by instruction issue, not by the MUFU exponential
// unit (moving exponentials to FMA-pipe polynomials measured slower).
#pragma once

#include "common.cuh"

namespace hs2 {

constexpr int HD = 128;
constexpr int FL_STAGES = 2;
constexpr int FL_THREADS = 384;
constexpr uint32_t TILE_BYTES = 128u * 128u * 2u;  // one 128 x 128 bf16 tile
constexpr uint32_t HALF_BYTES = 128u * 64u * 2u;   // its d-half (128 rows x 128 B)
constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, 0, 0);
constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 128, 0, 1);
constexpr uint32_t IDESC_S_F16 = idesc_f16_f32(128, 128, 0, 0);
constexpr uint32_t IDESC_PV_F16 = idesc_f16_f32(128, 128, 0, 1);
// K/V cache modes of the dense kernels
constexpr int KVM_BF16 = 0;  // bf16 cache, TMA
constexpr int KVM_E4M3 = 1;  // e4m3 codes, converted in the kernel
constexpr int KVM_F16 = 2;   // f16 copy of an e4m3 cache (+ K column scales), TMA
constexpr uint32_t FLAG_SKIP_LOADS = 1u;
constexpr uint32_t FLAG_IMP_VISIBLE = 2u;  // hs2_importance over every visible key (checking mode)
constexpr int MAX_LIST = 4096;

struct FlashParams {
  int L, Hq, Hkv, G, nqt, npairs;      // dense: 128-row query tiles, tile pairs
  int nb, list_len, mtiles, rows_tok;  // sparse: blocks, list stride, M tiles per (b,g), tokens per M tile
  int mpairs;                          // sparse: pairs of M tiles per (b,g)
  float scale_log2;                    // log2(e) / sqrt(d)
  int window;                          // window mode of the persistent kernel: keys i - window < j <= i
  const __nv_bfloat16* k;              // gather sources (sparse)
  const __nv_bfloat16* v;
  const uint8_t* k8;                   // e4m3 codes and fp32 scales [L][Hkv] (KV8)
  const uint8_t* v8;
  const float* ksc;
  const float* vsc;
  const float* kcol;  // KVM_F16: K scale x log2(e)/sqrt(d), [Hkv][kcol_stride]
  int kcol_stride;    // L rounded up to 128
  int64_t kv_tok, kv_head;
  const int32_t* idx;
  const int32_t* cnt;
  __nv_bfloat16* o;
  int64_t o_tok, o_head;
  float* lse;  // [Hq][L] (dense)
  uint64_t limit_ns;
  uint32_t flags;
};

struct FlashBars {
  uint64_t q_raw;  // KV8: Q landed (bf16), before its conversion
  uint64_t q_full;
  uint64_t full_k[FL_STAGES];
  uint64_t full_v[FL_STAGES];
  uint64_t empty_k[FL_STAGES];  // the stage's K tile (with an FP8 cache also its column scales) may be replaced
  uint64_t empty_v[FL_STAGES];  // the stage's V tile may be replaced
  uint64_t s_full[2];  // per query tile
  uint64_t p_ready[2];
  uint64_t o_done[2];
  uint64_t fin;
  uint32_t tmem_slot;
  int abort;
};

constexpr uint32_t FL_Q_OFF = 0;                // Q_A, then Q_B
constexpr uint32_t FL_KV_OFF = 2 * TILE_BYTES;  // stage s: K at +0, V at +TILE_BYTES
constexpr uint32_t FL_BAR_OFF = FL_KV_OFF + FL_STAGES * 2 * TILE_BYTES;
constexpr uint32_t FL_POS_OFF = FL_BAR_OFF + 256;
constexpr uint32_t FL_SMEM_DENSE = FL_POS_OFF + 1024;  // + alignment slack
constexpr uint32_t FL_KSC_OFF = FL_POS_OFF + MAX_LIST * 4;  // KV8: [stage][128] column scales
constexpr uint32_t FL_SMEM_KV8 = FL_KSC_OFF + FL_STAGES * 128 * 4 + 1024;

// mbar_wait taken by every lane of a warp, with a warp-uniform result, for
// roles that go on to issue warp-collective tcgen05.ld / tcgen05.st.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                          volatile int* abort, int where) {
  const bool ok = mbar_wait(bar, parity, limit_ns, abort, where);
  return __all_sync(0xffffffffu, ok);
}

// Waits for work already in flight (TMA or MMA completion), ignoring the
// abort flag: such work always finishes, and the CTA must not release its
// shared or tensor memory while it is outstanding.
__device__ __forceinline__ bool wait_done(uint64_t* bar, uint32_t parity, uint64_t limit_ns, int where) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(a, parity)) return true;
    if ((it & 31u) == 31u && globaltimer_ns() - t0 > limit_ns) {
      report(HS2_ERR_TIMEOUT, where);
      return false;
    }
  }
}

template <int KVM>
__global__ void __launch_bounds__(FL_THREADS, 1)
    flash_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const FlashParams p) {
  constexpr bool KV8 = KVM != KVM_BF16;   // f16 operands, K column scales
  constexpr bool CONV = KVM == KVM_E4M3;  // K/V tiles converted by warps 2-3
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  FlashBars* bars = reinterpret_cast<FlashBars*>(smem + FL_BAR_OFF);
  float* ksc_s = reinterpret_cast<float*>(smem + FL_KSC_OFF);
  const uint32_t q_base = smem_u32(smem + FL_Q_OFF);
  const uint32_t kv_base = smem_u32(smem + FL_KV_OFF);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &bars->abort;

  // ---- work item: query tiles A and B (B may be absent); query tile x uses
  // key tiles 0 .. (x ? nB : nA) - 1
  // KV-group-major order, longest tile pairs first within a group: the CTAs
  // resident at any time share one group's K/V, which then stays in L2.
  const int per_g = p.npairs * p.G;
  const int g = static_cast<int>(blockIdx.x) / per_g;
  const int rem = static_cast<int>(blockIdx.x) % per_g;
  const int pair = p.npairs - 1 - rem / p.G;
  const int h = g * p.G + rem % p.G;
  const int nA = 2 * pair + 1;
  const int nB = (2 * pair + 1 < p.nqt) ? 2 * pair + 2 : 0;
  const int n = max(nA, nB);

  const bool has_b = nB > 0;

  if (threadIdx.x == 0) {
    const uint32_t kv_arrivals = CONV ? 64u : 1u;
    mbar_init(&bars->q_raw, 1);
    mbar_init(&bars->q_full, KV8 ? 64u : 1u);
    for (int s = 0; s < FL_STAGES; ++s) {
      mbar_init(&bars->full_k[s], kv_arrivals);
      mbar_init(&bars->full_v[s], kv_arrivals);
      mbar_init(&bars->empty_k[s], 1);
      mbar_init(&bars->empty_v[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->s_full[x], 1);
      mbar_init(&bars->p_ready[x], 4);  // one arrival per softmax warp
      mbar_init(&bars->o_done[x], 1);
    }
    mbar_init(&bars->fin, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_slot;

  if (warp == 0) {
    // =========================================================== TMA loads
    if (lane == 0 && !(p.flags & FLAG_SKIP_LOADS) && n > 0) {
      tma_prefetch_desc(&tmQ);
      const int nq = has_b ? 2 : 1;
      uint64_t* qbar = KV8 ? &bars->q_raw : &bars->q_full;
      mbar_arrive_expect_tx(qbar, static_cast<uint32_t>(nq) * TILE_BYTES);
      for (int x = 0; x < nq; ++x) {
        uint8_t* qd = smem + FL_Q_OFF + x * TILE_BYTES;
        tma_load_3d(qd, &tmQ, qbar, 0, h, (2 * pair + x) * 128);
        tma_load_3d(qd + HALF_BYTES, &tmQ, qbar, 64, h, (2 * pair + x) * 128);
      }
      if (!CONV) {
        int last = -1;
        // A stage's K is replaced once both S products of its tile executed,
        // its V once both P V products did (with an FP8 cache the K column
        // scales are read by the softmax of the tile, so K goes with V).
        for (int j = 0; j < n; ++j) {
          const int s = j % FL_STAGES;
          const uint32_t par = ((j / FL_STAGES) - 1) & 1;
          if (j >= FL_STAGES && !mbar_wait(&bars->empty_k[s], par, p.limit_ns, abort_flag, 101)) break;
          uint8_t* kd = smem + FL_KV_OFF + s * 2 * TILE_BYTES;
          mbar_arrive_expect_tx(&bars->full_k[s], TILE_BYTES + (KV8 ? 512u : 0u));
          if (KV8) bulk_load(ksc_s + s * 128, p.kcol + static_cast<int64_t>(g) * p.kcol_stride + j * 128, 512u,
                             &bars->full_k[s]);
          tma_load_3d(kd, &tmK, &bars->full_k[s], 0, g, j * 128);
          tma_load_3d(kd + HALF_BYTES, &tmK, &bars->full_k[s], 64, g, j * 128);
          if (j >= FL_STAGES && !mbar_wait(&bars->empty_v[s], par, p.limit_ns, abort_flag, 105)) {
            wait_done(&bars->full_k[s], (j / FL_STAGES) & 1, p.limit_ns, 106);  // K(j) in flight
            break;
          }
          mbar_arrive_expect_tx(&bars->full_v[s], TILE_BYTES);
          tma_load_3d(kd + TILE_BYTES, &tmV, &bars->full_v[s], 0, g, j * 128);
          tma_load_3d(kd + TILE_BYTES + HALF_BYTES, &tmV, &bars->full_v[s], 64, g, j * 128);
          last = j;
        }
        // Never leave a TMA write in flight into memory the CTA gives back.
        for (int u = max(0, last - FL_STAGES + 1); u <= last; ++u) {
          const int s = u % FL_STAGES;
          wait_done(&bars->full_k[s], (u / FL_STAGES) & 1, p.limit_ns, 102);
          wait_done(&bars->full_v[s], (u / FL_STAGES) & 1, p.limit_ns, 103);
        }
      }
      wait_done(qbar, 0, p.limit_ns, 104);
    }
  } else if (warp == 1) {
    // ========================================================== MMA issue
    if (lane == 0 && n > 0) {
      const int nx[2] = {nA, nB};
      auto issue_s = [&](int x, int j) {
        const uint32_t kb = kv_base + (j % FL_STAGES) * 2 * TILE_BYTES;
        const uint32_t qb = q_base + x * TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
          umma_ss(tmem + x * 128, sdesc_sw128(qb + koff, 16, 1024), sdesc_sw128(kb + koff, 16, 1024),
                  KV8 ? IDESC_S_F16 : IDESC_S, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars->s_full[x]);
      };
      auto issue_pv = [&](int x, int j) {
        const uint32_t vb = kv_base + (j % FL_STAGES) * 2 * TILE_BYTES + TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bdesc = sdesc_sw128(vb + kk * 2048, HALF_BYTES, 1024);
          umma_ts(tmem + 256 + x * 128, tmem + x * 128 + kk * 8, bdesc, KV8 ? IDESC_PV_F16 : IDESC_PV,
                  (j > 0 || kk > 0) ? 1u : 0u);
        }
        // O is final after the tile's last product (earlier products are
        // known complete through s_full: a commit covers every MMA issued
        // before it)
        if (j == nx[x] - 1) umma_commit(&bars->o_done[x]);
      };
      bool ok = mbar_wait(&bars->q_full, 0, p.limit_ns, abort_flag, 111);
      if (ok) ok = mbar_wait(&bars->full_k[0], 0, p.limit_ns, abort_flag, 112);
      if (ok) {
        tc_fence_after();
        for (int x = 0; x < 2; ++x)
          if (nx[x] > 0) issue_s(x, 0);
        if (!KV8) umma_commit(&bars->empty_k[0]);  // K(0) multiplied by both query tiles
      }
      for (int j = 0; j < n && ok; ++j) {
        const int u = j;
        const int s = u % FL_STAGES;
        // V(j) and K(j + 1) normally landed long ago: check them before
        // blocking on the softmax, so nothing but P stands between its
        // arrival and the products
        if (!mbar_wait(&bars->full_v[s], (u / FL_STAGES) & 1, p.limit_ns, abort_flag, 114)) break;
        if (j + 1 < n &&
            !mbar_wait(&bars->full_k[(u + 1) % FL_STAGES], ((u + 1) / FL_STAGES) & 1, p.limit_ns, abort_flag, 115))
          break;
        for (int x = 0; x < 2 && ok; ++x) {
          if (j >= nx[x]) continue;
          if (!mbar_wait(&bars->p_ready[x], j & 1, p.limit_ns, abort_flag, 113)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_pv(x, j);
          if (j + 1 < nx[x]) issue_s(x, j + 1);
        }
        if (ok) {
          // V(j) is read by no later product; K(j + 1) neither, once both S
          // products of tile j + 1 are queued
          umma_commit(&bars->empty_v[s]);
          if (KV8)
            umma_commit(&bars->empty_k[s]);
          else if (j + 1 < n)
            umma_commit(&bars->empty_k[(u + 1) % FL_STAGES]);
        }
      }
      umma_commit(&bars->fin);
      wait_done(&bars->fin, 0, p.limit_ns, 116);
    }
  } else if (warp < 4) {
    // ============================================ KV8: convert Q, load K/V
    if (KV8 && n > 0 && !(p.flags & FLAG_SKIP_LOADS)) {
      const int pt = threadIdx.x - 64;  // 0..63
      if (mbar_wait(&bars->q_raw, 0, p.limit_ns, abort_flag, 141)) {
        const int nchunks = (has_b ? 2 : 1) * static_cast<int>(TILE_BYTES / 16);
        bool q_over = false;
        for (int c = pt; c < nchunks; c += 64) {
          const uint32_t a = q_base + c * 16;
          st_shared_v4(a, bf16x8_to_f16x8_checked(ld_shared_v4(a), q_over));
        }
        if (q_over) report(HS2_ERR_RANGE, 149);
        fence_proxy_async_smem();
        mbar_arrive(&bars->q_full);
        // K/V tiles: 8 threads per 128-byte code row, 16 codes -> two f16 chunks each
        const int rsub = pt >> 3, c8 = pt & 7;
        const uint8_t* kb8 = p.k8 + static_cast<int64_t>(g) * p.kv_head + c8 * 16;
        const uint8_t* vb8 = p.v8 + static_cast<int64_t>(g) * p.kv_head + c8 * 16;
        for (int j = 0; j < (CONV ? n : 0); ++j) {  // KVM_F16: K/V tiles come by TMA
          const int s = j % FL_STAGES;
          if (j >= FL_STAGES &&
              (!mbar_wait(&bars->empty_k[s], ((j / FL_STAGES) - 1) & 1, p.limit_ns, abort_flag, 142) ||
               !mbar_wait(&bars->empty_v[s], ((j / FL_STAGES) - 1) & 1, p.limit_ns, abort_flag, 143)))
            break;
          const uint32_t kd = kv_base + s * 2 * TILE_BYTES;
#pragma unroll 1
          for (int half = 0; half < 2; ++half) {  // 0: K, 1: V
            const uint8_t* base8 = half ? vb8 : kb8;
            const float* scale = half ? p.vsc : p.ksc;
            // every row's codes and scale in flight before any is converted
            uint4 raw[16];
            float sgv[16];
#pragma unroll
            for (int it = 0; it < 16; ++it) {
              const int pj = j * 128 + rsub + 8 * it;
              raw[it] = make_uint4(0, 0, 0, 0);
              sgv[it] = 0.f;
              if (pj < p.L) {
                raw[it] = ld_nc_v4(base8 + static_cast<int64_t>(pj) * p.kv_tok);
                sgv[it] = scale[static_cast<int64_t>(pj) * p.Hkv + g];
              }
            }
#pragma unroll
            for (int it = 0; it < 16; ++it) {
              const int r = rsub + 8 * it;
              const float sg = sgv[it];
              const uint32_t w[4] = {raw[it].x, raw[it].y, raw[it].z, raw[it].w};
              uint32_t f[8];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                f[2 * q] = e4m3x2_to_f16x2(w[q]);
                f[2 * q + 1] = e4m3x2_to_f16x2(w[q] >> 16);
              }
              if (half) {
                const uint32_t s2 = pack_f16x2(sg, sg);
#pragma unroll
                for (int q = 0; q < 8; ++q) f[q] = hmul2_u32(f[q], s2);
              } else if (c8 == 0) {
                ksc_s[s * 128 + r] = sg * p.scale_log2;
              }
              const uint32_t dst = kd + half * TILE_BYTES;
              st_shared_v4(dst + sw128_chunk_offset(r, 2 * c8, 128), make_uint4(f[0], f[1], f[2], f[3]));
              st_shared_v4(dst + sw128_chunk_offset(r, 2 * c8 + 1, 128), make_uint4(f[4], f[5], f[6], f[7]));
            }
            fence_proxy_async_smem();
            mbar_arrive(half ? &bars->full_v[s] : &bars->full_k[s]);
          }
        }
      }
    }
  } else {
    // ============================================ softmax / rescale / epilogue
    const int x = (warp >= 8) ? 1 : 0;  // query tile of this warpgroup
    const int nX = x ? nB : nA;
    const int r = threadIdx.x - 128 - 128 * x;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t s_tm = tmem + lane_off + x * 128;
    const uint32_t o_tm = tmem + lane_off + 256 + x * 128;
    const int qt = 2 * pair + x;
    const int i_row = qt * 128 + r, hh = h, diag = qt;
    const float sc = KV8 ? 1.f : p.scale_log2;  // KV8 folds the scale into the columns
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nX; ++j) {
      const int t = j;  // tiles this query tile has seen before j
      if (!warp_wait(&bars->s_full[x], t & 1, p.limit_ns, abort_flag, 131)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[4][32];
      tmem_ld32(s_tm, sr[0]);
      tmem_ld32(s_tm + 32, sr[1]);
      tmem_ld32(s_tm + 64, sr[2]);
      tmem_ld32(s_tm + 96, sr[3]);
      tmem_ld_wait();
      reg_fence(sr[0]);
      reg_fence(sr[1]);
      reg_fence(sr[2]);
      reg_fence(sr[3]);
      if (KV8) {  // per-key scale (already times log2(e)/sqrt(d)) on every column
        const uint64_t* ks2 = reinterpret_cast<const uint64_t*>(ksc_s + (j % FL_STAGES) * 128);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float a0, a1;
            f2_unpack(f2_mul(f2_pack(__uint_as_float(sr[c][2 * e]), __uint_as_float(sr[c][2 * e + 1])),
                             ks2[c * 16 + e]),
                      a0, a1);
            sr[c][2 * e] = __float_as_uint(a0);
            sr[c][2 * e + 1] = __float_as_uint(a1);
          }
        }
      }
      // ---- mask (after any scaling, so a masked column is exactly -inf)
      if (j == diag) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c > r) sr[c >> 5][c & 31] = __float_as_uint(-INFINITY);
      }
      // ---- row max: 8 independent chains of 3-input max over 16 values each
      float mx8[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint32_t* v = &sr[q >> 1][(q & 1) * 16];
        float m = fmax3(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]));
#pragma unroll
        for (int e = 0; e < 6; ++e) m = fmax3(m, __uint_as_float(v[3 + 2 * e]), __uint_as_float(v[4 + 2 * e]));
        mx8[q] = fmaxf(m, __uint_as_float(v[15]));
      }
      const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
      const float m_new = fmaxf(m_used, mx * sc);
      float alpha = 1.f;
      const bool resc = m_new > m_used + 8.f;
      if (resc) {
        alpha = ex2_approx(m_used - m_new);
        m_used = m_new;
      }
      const float mu = (m_used == -INFINITY) ? 0.f : m_used;
      l *= alpha;
      // ---- P = exp2(s * scale - m) into TMEM over S (arguments and row sums
      // as packed f32x2)
      const uint64_t sc2 = f2_pack(sc, sc), nmu2 = f2_pack(-mu, -mu);
      uint64_t sum2[2] = {0ull, 0ull};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const uint64_t a2 =
              f2_fma(f2_pack(__uint_as_float(sr[c][2 * e]), __uint_as_float(sr[c][2 * e + 1])), sc2, nmu2);
          const uint64_t p2 = ex2_x2(a2);
          sum2[e & 1] = f2_add(sum2[e & 1], p2);
          float e0, e1;
          f2_unpack(p2, e0, e1);
          pk[e] = KV8 ? pack_f16x2(e0, e1) : pack_bf16x2(e0, e1);
        }
        tmem_st16(s_tm + c * 16, pk);
      }
      {
        float a0, a1, b0, b1;
        f2_unpack(sum2[0], a0, a1);
        f2_unpack(sum2[1], b0, b1);
        l += (a0 + a1) + (b0 + b1);
      }
      // ---- O rescale: P V(j - 1) completed before S(j) (it was issued
      // first by the same thread, and s_full's commit covers it)
      if (t > 0) {
        if (__any_sync(0xffffffffu, resc)) {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t orr[32];
            tmem_ld32(o_tm + c * 32, orr);
            tmem_ld_wait();
            reg_fence(orr);
#pragma unroll
            for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
            tmem_st32(o_tm + c * 32, orr);
          }
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();  // one arrival per warp, once all its lanes' stores completed
      if (lane == 0) mbar_arrive(&bars->p_ready[x]);
    }
    // ---- epilogue
    const bool row_live = i_row < p.L && (x == 0 || has_b);  // a last dense tile may hang past L
    __nv_bfloat16* orow = p.o + static_cast<int64_t>(i_row) * p.o_tok + static_cast<int64_t>(hh) * p.o_head;
    const int nT = nX;  // key tiles of this query tile
    if (ok && nT > 0 && warp_wait(&bars->o_done[x], 0, p.limit_ns, abort_flag, 133)) {
      tc_fence_after();
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t orr[32];
        tmem_ld32(o_tm + c * 32, orr);
        tmem_ld_wait();
        reg_fence(orr);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(orr[2 * e]) * inv, __uint_as_float(orr[2 * e + 1]) * inv);
        uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
        if (row_live) {
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
        }
      }
      if (row_live)
        p.lse[static_cast<int64_t>(hh) * p.L + i_row] = (m_used + log2f(l)) * 0.69314718055994530942f;
    }
  }

  // ---- teardown: every role has drained its asynchronous work
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace hs2
