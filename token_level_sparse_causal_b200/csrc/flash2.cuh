// Kernel (1) on CTA pairs: the causal grouped-query attention and LSE of
// flash_fwd_kernel (HySparse2 architecture summary, ablation paragraph: the
// full layer's complete scores; SHARP walk-through, section 1.1:
// softmax(Q K^T / sqrt(d)) V), with each product issued once for two CTAs
// (tcgen05.mma.cta_group::2, M = 256) so that each CTA holds only half of
// every K and V tile.
//
// A cluster of two CTAs takes one pair of 128-query tiles (A, B) of two query
// heads of one KV group (CTA rank r: head 2m + r).  Per key tile j:
//   S_x(j) = Q_x K_j^T      M = 256 (128 query rows from each CTA's Q_x),
//                           N = 128 keys: CTA r holds keys [64r, 64r + 64)
//   O_x += P_x(j) V_j       M = 256 (P from each CTA's tensor memory),
//                           N = 128 dims: CTA r holds V's dims [64r, 64r + 64)
// Every CTA's tensor memory holds its own rows of S_A, S_B, O_A, O_B (128
// columns each), so each CTA's softmax warpgroups and epilogue are those of
// flash_fwd_kernel.  Per SM, the K/V bytes brought into shared memory and the
// shared-memory operand reads of both products are half of the one-CTA
// kernel's, and the ring has room for four stages.
//
// Roles (both CTAs): warp 0 issues the TMA loads of its Q tiles and its K/V
// halves; the halves of both CTAs complete on the leader CTA's full
// barriers (cta_group::2 TMA).  Warps 2-3 forward "Q ready" to the leader
// (converting Q to f16 first with an FP8 cache).  In the leader (rank 0) one
// thread of warp 1 issues every MMA; each of its commits arrives on the
// barriers of both CTAs.  The softmax warps of both CTAs arrive on the
// leader's p_ready barriers.  Every wait is bounded.
//
// K/V modes: the bf16 cache, or the layer's f16 copy of an e4m3 cache (K
// column scales loaded by each CTA for all 128 keys of a tile); the in-kernel
// e4m3 conversion uses flash_fwd_kernel.  The two heads of a cluster belong to
// one KV group because every supported group size (2, 4, 8) is even.
//
// Results are bit for bit those of flash_fwd_kernel (same products, same
// softmax arithmetic per row).  Measured against it at 128k (64/8 heads) the
// pair kernel is within 1%, and 7% slower at 32k, so flash_fwd_kernel stays
// the default and this one runs when the FLAG_FA_CTA_PAIRS test hook is set.
#pragma once

#include "flash.cuh"

namespace hs2 {

constexpr uint32_t FLAG_FA_CTA_PAIRS = 4u;  // run kernel (1) on CTA pairs (bf16 cache or its f16 layer copy)
constexpr int F2_STAGES = 4;
constexpr uint32_t F2_KHALF = 64u * 128u * 2u;  // 64 keys x 128 dims: this CTA's half of a K tile
constexpr uint32_t F2_KQUART = F2_KHALF / 2;    // its dims [0, 64) or [64, 128) (64 rows x 128 B)
constexpr uint32_t F2_VHALF = 128u * 64u * 2u;  // 128 keys x 64 dims: this CTA's half of a V tile
constexpr uint32_t F2_STAGE_BYTES = F2_KHALF + F2_VHALF;
constexpr uint32_t F2_Q_OFF = 0;  // Q_A, then Q_B
constexpr uint32_t F2_KV_OFF = 2 * TILE_BYTES;
constexpr uint32_t F2_BAR_OFF = F2_KV_OFF + F2_STAGES * F2_STAGE_BYTES;
constexpr uint32_t F2_KSC_OFF = F2_BAR_OFF + 256;  // KV8: [stage][128] column scales
constexpr uint32_t F2_SMEM = F2_KSC_OFF + F2_STAGES * 128 * 4 + 1024;  // + alignment slack
constexpr uint32_t F2_Q_ARRIVALS = 128;  // warps 2-3 of both CTAs
constexpr uint32_t IDESC2_S = idesc_bf16_f32(256, 128, 0, 0);
constexpr uint32_t IDESC2_PV = idesc_bf16_f32(256, 128, 0, 1);
constexpr uint32_t IDESC2_S_F16 = idesc_f16_f32(256, 128, 0, 0);
constexpr uint32_t IDESC2_PV_F16 = idesc_f16_f32(256, 128, 0, 1);

struct F2Bars {
  uint64_t q_raw;                // this CTA's Q tiles landed
  uint64_t q_full;               // leader: Q of both CTAs ready for the tensor core
  uint64_t full_k[F2_STAGES];    // leader: both halves of the stage's K tile landed
  uint64_t full_v[F2_STAGES];    // leader: both halves of the stage's V tile landed
  uint64_t empty_k[F2_STAGES];   // the stage's K half may be replaced
  uint64_t empty_v[F2_STAGES];   // the stage's V half may be replaced
  uint64_t ksc_full[F2_STAGES];  // KV8: this CTA's copy of the tile's column scales landed
  uint64_t s_full[2];            // per query tile
  uint64_t p_ready[2];           // leader: per query tile, one arrival per softmax warp of both CTAs
  uint64_t o_done[2];
  uint64_t fin;
  uint32_t tmem_slot;
  int abort;
};
static_assert(sizeof(F2Bars) <= 256, "barriers fit their slot");
static_assert(F2_SMEM <= 232448, "shared memory of one CTA");

// ------------------------------------------------------ cluster helpers --

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
// Address of the same shared-memory variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
  uint32_t d;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(smem_u32(p)), "r"(rank));
  return d;
}
// Every thread of both CTAs (like __syncthreads for the pair).
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
// Arrive on a barrier of either CTA of the pair.  The data it publishes is
// tensor memory (completed by tcgen05.wait::st and ordered by
// tcgen05.fence::before_thread_sync) or shared memory handed to the tensor
// core (fence.proxy.async): the default CTA-scope release suffices, and a
// cluster-scope release costs a fence on every arrival.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}
// TMA load into this CTA's shared memory (this CTA only) completing on a
// barrier of either CTA of the pair.
__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* map, uint32_t cluster_bar, int c0,
                                                 int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(cluster_bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D[tmem of both CTAs] (+)= A[smem of both] * B[smem of both]
__device__ __forceinline__ void umma_ss_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem of both] (+)= A[tmem of both] * B[smem of both]
__device__ __forceinline__ void umma_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on `bar` in both CTAs when every MMA issued so far completed.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(static_cast<uint16_t>(3))
      : "memory");
}

template <int KVM>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(FL_THREADS, 1)
    flash2_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK64,
                      const __grid_constant__ CUtensorMap tmV, const FlashParams p) {
  static_assert(KVM == KVM_BF16 || KVM == KVM_F16, "tiles by TMA");
  constexpr bool KV8 = KVM == KVM_F16;  // f16 operands, K column scales
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  F2Bars* bars = reinterpret_cast<F2Bars*>(smem + F2_BAR_OFF);
  float* ksc_s = reinterpret_cast<float*>(smem + F2_KSC_OFF);
  const uint32_t q_base = smem_u32(smem + F2_Q_OFF);
  const uint32_t kv_base = smem_u32(smem + F2_KV_OFF);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &bars->abort;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  // ---- work item: query tiles A and B (B may be absent) of head h; both
  // CTAs of the cluster take the same tiles of two heads of one KV group.
  // KV-group-major order, longest tile pairs first within a group.
  const int hpg = p.G >> 1;  // head pairs per group
  const int c = static_cast<int>(cluster_id_x());
  const int per_g = p.npairs * hpg;
  const int g = c / per_g;
  const int rem = c % per_g;
  const int pair = p.npairs - 1 - rem / hpg;
  const int h = g * p.G + 2 * (rem % hpg) + static_cast<int>(rank);
  const int nA = 2 * pair + 1;
  const int nB = (2 * pair + 1 < p.nqt) ? 2 * pair + 2 : 0;
  const int n = max(nA, nB);
  const bool has_b = nB > 0;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_raw, 1);
    mbar_init(&bars->q_full, F2_Q_ARRIVALS);
    for (int s = 0; s < F2_STAGES; ++s) {
      mbar_init(&bars->full_k[s], 1);
      mbar_init(&bars->full_v[s], 1);
      mbar_init(&bars->empty_k[s], 1);
      mbar_init(&bars->empty_v[s], 1);
      mbar_init(&bars->ksc_full[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->s_full[x], 1);
      mbar_init(&bars->p_ready[x], 8);  // 4 softmax warps in each CTA
      mbar_init(&bars->o_done[x], 1);
    }
    mbar_init(&bars->fin, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(&bars->tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers exist before either signals the other
  tc_fence_after();
  const uint32_t tmem = bars->tmem_slot;

  if (warp == 0) {
    // =========================================================== TMA loads
    if (lane == 0 && !(p.flags & FLAG_SKIP_LOADS)) {
      tma_prefetch_desc(&tmQ);
      const int nq = has_b ? 2 : 1;
      mbar_arrive_expect_tx(&bars->q_raw, static_cast<uint32_t>(nq) * TILE_BYTES);
      for (int x = 0; x < nq; ++x) {
        uint8_t* qd = smem + F2_Q_OFF + x * TILE_BYTES;
        tma_load_3d(qd, &tmQ, &bars->q_raw, 0, h, (2 * pair + x) * 128);
        tma_load_3d(qd + HALF_BYTES, &tmQ, &bars->q_raw, 64, h, (2 * pair + x) * 128);
      }
      int last = -1;
      // A stage's K half is replaced once both S products of its tile
      // executed, its V half once both P V products did (with an FP8 cache
      // K goes with V: the softmax reads the tile's column scales).
      for (int j = 0; j < n; ++j) {
        const int s = j % F2_STAGES;
        const uint32_t par = ((j / F2_STAGES) - 1) & 1;
        if (j >= F2_STAGES && !mbar_wait(&bars->empty_k[s], par, p.limit_ns, abort_flag, 301)) break;
        uint8_t* kd = smem + F2_KV_OFF + s * F2_STAGE_BYTES;
        if (leader) mbar_arrive_expect_tx(&bars->full_k[s], 2 * F2_KHALF);
        if (KV8) {
          mbar_arrive_expect_tx(&bars->ksc_full[s], 512u);
          bulk_load(ksc_s + s * 128, p.kcol + static_cast<int64_t>(g) * p.kcol_stride + j * 128, 512u,
                    &bars->ksc_full[s]);
        }
        const uint32_t fk = cluster_addr(&bars->full_k[s], 0);
        tma_load_3d_pair(kd, &tmK64, fk, 0, g, j * 128 + 64 * static_cast<int>(rank));
        tma_load_3d_pair(kd + F2_KQUART, &tmK64, fk, 64, g, j * 128 + 64 * static_cast<int>(rank));
        if (j >= F2_STAGES && !mbar_wait(&bars->empty_v[s], par, p.limit_ns, abort_flag, 302)) {
          if (leader) wait_done(&bars->full_k[s], (j / F2_STAGES) & 1, p.limit_ns, 303);  // K(j) in flight
          break;
        }
        if (leader) mbar_arrive_expect_tx(&bars->full_v[s], 2 * F2_VHALF);
        tma_load_3d_pair(kd + F2_KHALF, &tmV, cluster_addr(&bars->full_v[s], 0), 64 * static_cast<int>(rank), g,
                         j * 128);
        last = j;
      }
      // Never leave a TMA write in flight into memory a CTA gives back: the
      // leader's barriers count both CTAs' bytes, and neither CTA passes the
      // closing cluster barrier before the leader has seen them land.
      for (int u = max(0, last - F2_STAGES + 1); u <= last; ++u) {
        const int s = u % F2_STAGES;
        if (leader) {
          wait_done(&bars->full_k[s], (u / F2_STAGES) & 1, p.limit_ns, 304);
          wait_done(&bars->full_v[s], (u / F2_STAGES) & 1, p.limit_ns, 305);
        }
        if (KV8) wait_done(&bars->ksc_full[s], (u / F2_STAGES) & 1, p.limit_ns, 306);
      }
      wait_done(&bars->q_raw, 0, p.limit_ns, 307);
    }
  } else if (warp == 1) {
    // ========================================================== MMA issue
    if (leader && lane == 0) {
      const int nx[2] = {nA, nB};
      auto issue_s = [&](int x, int j) {
        const uint32_t kb = kv_base + (j % F2_STAGES) * F2_STAGE_BYTES;
        const uint32_t qb = q_base + x * TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t qoff = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
          const uint32_t koff = (kk >> 2) * F2_KQUART + (kk & 3) * 32;
          umma_ss_pair(tmem + x * 128, sdesc_sw128(qb + qoff, 16, 1024), sdesc_sw128(kb + koff, 16, 1024),
                       KV8 ? IDESC2_S_F16 : IDESC2_S, kk > 0 ? 1u : 0u);
        }
        umma_commit_pair(&bars->s_full[x]);
      };
      auto issue_pv = [&](int x, int j) {
        const uint32_t vb = kv_base + (j % F2_STAGES) * F2_STAGE_BYTES + F2_KHALF;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bdesc = sdesc_sw128(vb + kk * 2048, F2_VHALF, 1024);
          umma_ts_pair(tmem + 256 + x * 128, tmem + x * 128 + kk * 8, bdesc, KV8 ? IDESC2_PV_F16 : IDESC2_PV,
                       (j > 0 || kk > 0) ? 1u : 0u);
        }
        // O is final after the tile's last product (earlier products are
        // known complete through s_full: a commit covers every MMA issued
        // before it)
        if (j == nx[x] - 1) umma_commit_pair(&bars->o_done[x]);
      };
      bool ok = mbar_wait(&bars->q_full, 0, p.limit_ns, abort_flag, 311);
      if (ok) ok = mbar_wait(&bars->full_k[0], 0, p.limit_ns, abort_flag, 312);
      if (ok) {
        tc_fence_after();
        for (int x = 0; x < 2; ++x)
          if (nx[x] > 0) issue_s(x, 0);
        if (!KV8) umma_commit_pair(&bars->empty_k[0]);  // K(0) multiplied by both query tiles
      }
      for (int j = 0; j < n && ok; ++j) {
        const int s = j % F2_STAGES;
        // V(j) and K(j + 1) normally landed long ago: check them before
        // blocking on the softmax
        if (!mbar_wait(&bars->full_v[s], (j / F2_STAGES) & 1, p.limit_ns, abort_flag, 314)) break;
        if (j + 1 < n && !mbar_wait(&bars->full_k[(j + 1) % F2_STAGES], ((j + 1) / F2_STAGES) & 1, p.limit_ns,
                                    abort_flag, 315))
          break;
        for (int x = 0; x < 2 && ok; ++x) {
          if (j >= nx[x]) continue;
          if (!mbar_wait(&bars->p_ready[x], j & 1, p.limit_ns, abort_flag, 313)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_pv(x, j);
          if (j + 1 < nx[x]) issue_s(x, j + 1);
        }
        if (ok) {
          umma_commit_pair(&bars->empty_v[s]);
          if (KV8)
            umma_commit_pair(&bars->empty_k[s]);
          else if (j + 1 < n)
            umma_commit_pair(&bars->empty_k[(j + 1) % F2_STAGES]);
        }
      }
      umma_commit_pair(&bars->fin);
      wait_done(&bars->fin, 0, p.limit_ns, 316);
    }
  } else if (warp < 4) {
    // ====================== Q ready (converted to f16 with an FP8 cache)
    const int pt = threadIdx.x - 64;  // 0..63
    if (mbar_wait(&bars->q_raw, 0, p.limit_ns, abort_flag, 321)) {
      if (KV8) {
        const int nchunks = (has_b ? 2 : 1) * static_cast<int>(TILE_BYTES / 16);
        bool q_over = false;
        for (int cc = pt; cc < nchunks; cc += 64) {
          const uint32_t a = q_base + cc * 16;
          st_shared_v4(a, bf16x8_to_f16x8_checked(ld_shared_v4(a), q_over));
        }
        if (q_over) report(HS2_ERR_RANGE, 329);
      }
      fence_proxy_async_smem();
      mbar_arrive_remote(cluster_addr(&bars->q_full, 0));
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
    const int i_row = qt * 128 + r;
    const float sc = KV8 ? 1.f : p.scale_log2;  // KV8 folds the scale into the columns
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nX; ++j) {
      if (!warp_wait(&bars->s_full[x], j & 1, p.limit_ns, abort_flag, 331)) {
        ok = false;
        break;
      }
      if (KV8 && !warp_wait(&bars->ksc_full[j % F2_STAGES], (j / F2_STAGES) & 1, p.limit_ns, abort_flag, 332)) {
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
        const uint64_t* ks2 = reinterpret_cast<const uint64_t*>(ksc_s + (j % F2_STAGES) * 128);
#pragma unroll
        for (int cq = 0; cq < 4; ++cq) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float a0, a1;
            f2_unpack(f2_mul(f2_pack(__uint_as_float(sr[cq][2 * e]), __uint_as_float(sr[cq][2 * e + 1])),
                             ks2[cq * 16 + e]),
                      a0, a1);
            sr[cq][2 * e] = __float_as_uint(a0);
            sr[cq][2 * e + 1] = __float_as_uint(a1);
          }
        }
      }
      // ---- mask (after any scaling, so a masked column is exactly -inf)
      if (j == qt) {
#pragma unroll
        for (int cc = 0; cc < 128; ++cc)
          if (cc > r) sr[cc >> 5][cc & 31] = __float_as_uint(-INFINITY);
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
      // ---- P = exp2(s * scale - m) into TMEM over S
      const uint64_t sc2 = f2_pack(sc, sc), nmu2 = f2_pack(-mu, -mu);
      uint64_t sum2[2] = {0ull, 0ull};
#pragma unroll
      for (int cq = 0; cq < 4; ++cq) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const uint64_t a2 =
              f2_fma(f2_pack(__uint_as_float(sr[cq][2 * e]), __uint_as_float(sr[cq][2 * e + 1])), sc2, nmu2);
          const uint64_t p2 = ex2_x2(a2);
          sum2[e & 1] = f2_add(sum2[e & 1], p2);
          float e0, e1;
          f2_unpack(p2, e0, e1);
          pk[e] = KV8 ? pack_f16x2(e0, e1) : pack_bf16x2(e0, e1);
        }
        tmem_st16(s_tm + cq * 16, pk);
      }
      {
        float a0, a1, b0, b1;
        f2_unpack(sum2[0], a0, a1);
        f2_unpack(sum2[1], b0, b1);
        l += (a0 + a1) + (b0 + b1);
      }
      // ---- O rescale: P V(j - 1) completed before S(j) (it was issued
      // first by the same thread, and s_full's commit covers it)
      if (j > 0 && __any_sync(0xffffffffu, resc)) {
#pragma unroll 1
        for (int cq = 0; cq < 4; ++cq) {
          uint32_t orr[32];
          tmem_ld32(o_tm + cq * 32, orr);
          tmem_ld_wait();
          reg_fence(orr);
#pragma unroll
          for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
          tmem_st32(o_tm + cq * 32, orr);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();  // one arrival per warp, once all its lanes' stores completed
      if (lane == 0) mbar_arrive_remote(cluster_addr(&bars->p_ready[x], 0));
    }
    // ---- epilogue
    const bool row_live = i_row < p.L && (x == 0 || has_b);  // a last dense tile may hang past L
    __nv_bfloat16* orow = p.o + static_cast<int64_t>(i_row) * p.o_tok + static_cast<int64_t>(h) * p.o_head;
    if (ok && nX > 0 && warp_wait(&bars->o_done[x], 0, p.limit_ns, abort_flag, 333)) {
      tc_fence_after();
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll 1
      for (int cq = 0; cq < 4; ++cq) {
        uint32_t orr[32];
        tmem_ld32(o_tm + cq * 32, orr);
        tmem_ld_wait();
        reg_fence(orr);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(orr[2 * e]) * inv, __uint_as_float(orr[2 * e + 1]) * inv);
        uint4* dst = reinterpret_cast<uint4*>(orow + cq * 32);
        if (row_live) {
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
        }
      }
      if (row_live) p.lse[static_cast<int64_t>(h) * p.L + i_row] = (m_used + log2f(l)) * 0.69314718055994530942f;
    }
  }

  // ---- teardown: every role of both CTAs has drained its asynchronous work
  // (the leader's MMA thread saw every product complete, its producer saw
  // every load of both CTAs land) before either CTA frees tensor memory or
  // exits
  tc_fence_before();
  __syncwarp();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace hs2
