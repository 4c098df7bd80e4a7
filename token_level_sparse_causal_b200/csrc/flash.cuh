// Flash-attention forward on tcgen05 tensor cores, in two modes sharing one
// pipeline:
//
//   FLASH_DENSE  -- kernel (1): causal grouped-query attention of the full
//                   layer, one CTA per (128-query tile, query head), K/V tiles
//                   of 128 keys streamed by TMA; writes O and the per-query
//                   natural-log LSE.  (HySparse2 architecture summary, ablation
//                   paragraph: the full layer's complete scores; SHARP
//                   walk-through, section 1.1: softmax(Q K^T / sqrt(d)) V.)
//   FLASH_SPARSE -- kernel (4): a sparse layer (KV Reuse, KV-sharing
//                   paragraph), one CTA per (query block b, KV head g, 128-row
//                   M tile); the 128 rows are (128/G tokens) x (G heads) of the
//                   block, all sharing the block's index list, whose K/V rows
//                   are gathered with 16-byte cp.async into swizzled shared
//                   memory; the causal mask j <= i applies to listed positions.
//
// CTA = 8 warps:
//   warp 0      TMA: Q tile (both modes), K/V tiles (dense)
//   warp 1      TMEM allocation; one thread issues every tcgen05.mma
//   warps 2-3   K/V gather (sparse)
//   warps 4-7   softmax, O rescale and epilogue; thread r owns row r (TMEM
//               lane r) of S, P and O
//
// Tensor memory (512 columns): S0 = [0,128), S1 = [128,256), O = [256,384).
// P (bf16) is written over the first 64 columns of the S buffer it came from
// and fed to the PV product straight from tensor memory.
//
// Per key tile j:  S_j = Q K_j^T (SS MMA, M=N=128, K=d=128 in 8 steps);
// softmax rows in the log2 domain with a lazily updated reference max: O is
// rescaled only when the running max grows by more than 2^8, so P stays
// below 256 and the final O / l is exact up to rounding; O += P_j V_j (TS
// MMA, V as an MN-major operand).  Issue order of the MMA thread is
// S_0, S_1, PV_0, S_2, PV_1, ... so the tensor core works on S_{j+1} while
// the softmax warps process S_j.
#pragma once

#include "common.cuh"

namespace hs2 {

constexpr int HD = 128;
constexpr int FL_STAGES = 2;
constexpr uint32_t TILE_BYTES = 128u * 128u * 2u;  // one 128 x 128 bf16 tile
constexpr uint32_t HALF_BYTES = 128u * 64u * 2u;   // its d-half (128 rows x 128 B)
constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, 0, 0);
constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 128, 0, 1);
constexpr int FLASH_DENSE = 0;
constexpr int FLASH_SPARSE = 1;
constexpr uint32_t FLAG_SKIP_LOADS = 1u;
constexpr int MAX_LIST = 4096;

struct FlashParams {
  int L, Hq, Hkv, G, nqt;  // nqt: 128-row query tiles (dense)
  int nb, list_len, mtiles, rows_tok;  // sparse: blocks, list stride, M tiles per (b,g), tokens per M tile
  float scale_log2;                    // log2(e) / sqrt(d)
  const __nv_bfloat16* k;              // gather sources (sparse)
  const __nv_bfloat16* v;
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
  uint64_t q_full;
  uint64_t full_k[FL_STAGES];
  uint64_t full_v[FL_STAGES];
  uint64_t empty[FL_STAGES];
  uint64_t s_full[2];
  uint64_t p_ready;
  uint64_t o_done;
  uint64_t fin;
  uint32_t tmem_slot;
  int abort;
};

constexpr uint32_t FL_Q_OFF = 0;
constexpr uint32_t FL_KV_OFF = TILE_BYTES;
constexpr uint32_t FL_BAR_OFF = TILE_BYTES + FL_STAGES * 2 * TILE_BYTES;
constexpr uint32_t FL_POS_OFF = FL_BAR_OFF + 256;
constexpr uint32_t FL_SMEM_DENSE = FL_POS_OFF + 1024;  // + alignment slack
constexpr uint32_t FL_SMEM_SPARSE = FL_POS_OFF + MAX_LIST * 4 + 1024;

// mbar_wait taken by every lane of a warp, with a warp-uniform result, for
// roles that go on to issue warp-collective tcgen05.ld / tcgen05.st.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                          volatile int* abort, int where) {
  const bool ok = mbar_wait(bar, parity, limit_ns, abort, where);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ bool wait_done(uint64_t* bar, uint32_t parity, uint64_t limit_ns, int where) {
  // Waits for work already in flight (TMA or MMA completion), ignoring the
  // abort flag: such work always finishes, and the CTA must not release its
  // shared or tensor memory while it is outstanding.
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

template <int MODE>
__global__ void __launch_bounds__(256, 1)
    flash_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const FlashParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  FlashBars* bars = reinterpret_cast<FlashBars*>(smem + FL_BAR_OFF);
  int32_t* pos_s = reinterpret_cast<int32_t*>(smem + FL_POS_OFF);
  const uint32_t q_base = smem_u32(smem + FL_Q_OFF);
  const uint32_t kv_base = smem_u32(smem + FL_KV_OFF);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &bars->abort;

  // ---- work item
  int qt = 0, h = 0, g = 0, b = 0, mt = 0, ntiles = 0, cnt = 0, e_b = 0;
  if (MODE == FLASH_DENSE) {
    qt = p.nqt - 1 - static_cast<int>(blockIdx.x) / p.Hq;  // longest rows first
    h = static_cast<int>(blockIdx.x) % p.Hq;
    g = h / p.G;
    ntiles = qt + 1;
  } else {
    mt = static_cast<int>(blockIdx.x) % p.mtiles;
    const int bg = static_cast<int>(blockIdx.x) / p.mtiles;
    g = bg % p.Hkv;
    b = bg / p.Hkv;
    e_b = min(p.L, 64 * (b + 1));
    cnt = p.cnt[static_cast<int64_t>(g) * p.nb + b];
    cnt = max(0, min(cnt, p.list_len));
    ntiles = (cnt + 127) / 128;
    const int32_t* list = p.idx + (static_cast<int64_t>(g) * p.nb + b) * p.list_len;
    for (int i = threadIdx.x; i < ntiles * 128; i += blockDim.x) pos_s[i] = (i < cnt) ? list[i] : -1;
  }

  if (threadIdx.x == 0) {
    const uint32_t kv_arrivals = (MODE == FLASH_DENSE) ? 1u : 64u;
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < FL_STAGES; ++s) {
      mbar_init(&bars->full_k[s], kv_arrivals);
      mbar_init(&bars->full_v[s], kv_arrivals);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->s_full[0], 1);
    mbar_init(&bars->s_full[1], 1);
    mbar_init(&bars->p_ready, 128);
    mbar_init(&bars->o_done, 1);
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
    if (lane == 0 && !(p.flags & FLAG_SKIP_LOADS) && ntiles > 0) {
      tma_prefetch_desc(&tmQ);
      mbar_arrive_expect_tx(&bars->q_full, TILE_BYTES);
      if (MODE == FLASH_DENSE) {
        tma_load_3d(smem + FL_Q_OFF, &tmQ, &bars->q_full, 0, h, qt * 128);
        tma_load_3d(smem + FL_Q_OFF + HALF_BYTES, &tmQ, &bars->q_full, 64, h, qt * 128);
      } else {
        const int t0 = 64 * b + mt * p.rows_tok;
        tma_load_3d(smem + FL_Q_OFF, &tmQ, &bars->q_full, 0, g * p.G, t0);
        tma_load_3d(smem + FL_Q_OFF + HALF_BYTES, &tmQ, &bars->q_full, 64, g * p.G, t0);
      }
      if (MODE == FLASH_DENSE) {
        int last = -1;
        for (int j = 0; j < ntiles; ++j) {
          const int s = j % FL_STAGES;
          if (j >= FL_STAGES &&
              !mbar_wait(&bars->empty[s], ((j / FL_STAGES) - 1) & 1, p.limit_ns, abort_flag, 101))
            break;
          uint8_t* kd = smem + FL_KV_OFF + s * 2 * TILE_BYTES;
          mbar_arrive_expect_tx(&bars->full_k[s], TILE_BYTES);
          tma_load_3d(kd, &tmK, &bars->full_k[s], 0, g, j * 128);
          tma_load_3d(kd + HALF_BYTES, &tmK, &bars->full_k[s], 64, g, j * 128);
          mbar_arrive_expect_tx(&bars->full_v[s], TILE_BYTES);
          tma_load_3d(kd + TILE_BYTES, &tmV, &bars->full_v[s], 0, g, j * 128);
          tma_load_3d(kd + TILE_BYTES + HALF_BYTES, &tmV, &bars->full_v[s], 64, g, j * 128);
          last = j;
        }
        // Never leave a TMA write in flight into memory the CTA gives back.
        for (int j = max(0, last - FL_STAGES + 1); j <= last; ++j) {
          const int s = j % FL_STAGES;
          wait_done(&bars->full_k[s], (j / FL_STAGES) & 1, p.limit_ns, 102);
          wait_done(&bars->full_v[s], (j / FL_STAGES) & 1, p.limit_ns, 103);
        }
      }
      wait_done(&bars->q_full, 0, p.limit_ns, 104);
    }
  } else if (warp == 1) {
    // ========================================================== MMA issue
    if (lane == 0 && ntiles > 0) {
      bool ok = mbar_wait(&bars->q_full, 0, p.limit_ns, abort_flag, 111);
      auto do_pv = [&](int t) -> bool {
        const int s = t % FL_STAGES;
        if (!mbar_wait(&bars->p_ready, t & 1, p.limit_ns, abort_flag, 112)) return false;
        if (!mbar_wait(&bars->full_v[s], (t / FL_STAGES) & 1, p.limit_ns, abort_flag, 113)) return false;
        tc_fence_after();
        const uint32_t vb = kv_base + s * 2 * TILE_BYTES + TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bdesc = sdesc_sw128(vb + kk * 2048, HALF_BYTES, 1024);
          umma_ts(tmem + 256, tmem + (t & 1) * 128 + kk * 8, bdesc, IDESC_PV, (t > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&bars->o_done);
        umma_commit(&bars->empty[s]);
        return true;
      };
      if (ok) {
        tc_fence_after();
        for (int j = 0; j < ntiles && ok; ++j) {
          const int s = j % FL_STAGES;
          if (!mbar_wait(&bars->full_k[s], (j / FL_STAGES) & 1, p.limit_ns, abort_flag, 114)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t kb = kv_base + s * 2 * TILE_BYTES;
          const uint32_t d = tmem + (j & 1) * 128;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t koff = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
            umma_ss(d, sdesc_sw128(q_base + koff, 16, 1024), sdesc_sw128(kb + koff, 16, 1024), IDESC_S,
                    kk > 0 ? 1u : 0u);
          }
          umma_commit(&bars->s_full[j & 1]);
          if (j > 0) ok = do_pv(j - 1);
        }
        if (ok) do_pv(ntiles - 1);
      }
      umma_commit(&bars->fin);
      wait_done(&bars->fin, 0, p.limit_ns, 115);
    }
  } else if (warp < 4) {
    // ========================================================= K/V gather
    if (MODE == FLASH_SPARSE && !(p.flags & FLAG_SKIP_LOADS)) {
      const int pt = threadIdx.x - 64;  // 0..63
      const int row_sub = (pt >> 4) & 1, chunk = pt & 15, pw = pt >> 5;
      const __nv_bfloat16* kg = p.k + static_cast<int64_t>(g) * p.kv_head + chunk * 8;
      const __nv_bfloat16* vg = p.v + static_cast<int64_t>(g) * p.kv_head + chunk * 8;
      for (int j = 0; j < ntiles; ++j) {
        const int s = j % FL_STAGES;
        if (j >= FL_STAGES &&
            !mbar_wait(&bars->empty[s], ((j / FL_STAGES) - 1) & 1, p.limit_ns, abort_flag, 121))
          break;
        const uint32_t kd = kv_base + s * 2 * TILE_BYTES;
        int64_t src[32];
        uint32_t nbytes[32];
#pragma unroll
        for (int it = 0; it < 32; ++it) {
          const int r = pw * 2 + row_sub + 4 * it;
          const int gi = j * 128 + r;
          const int pj = pos_s[gi];
          const bool listed = gi < cnt;
          const bool valid = listed && pj >= 0 && pj < e_b;
          if (listed && !valid) report(HS2_ERR_INDEX, 122);
          src[it] = static_cast<int64_t>(valid ? pj : 0) * p.kv_tok;
          nbytes[it] = valid ? 16u : 0u;
          cp_async_16(kd + sw128_chunk_offset(r, chunk, 128), kg + src[it], nbytes[it]);
        }
        cp_async_commit();
#pragma unroll
        for (int it = 0; it < 32; ++it) {
          const int r = pw * 2 + row_sub + 4 * it;
          cp_async_16(kd + TILE_BYTES + sw128_chunk_offset(r, chunk, 128), vg + src[it], nbytes[it]);
        }
        cp_async_commit();
        cp_async_wait<1>();
        fence_proxy_async_smem();
        mbar_arrive(&bars->full_k[s]);
        cp_async_wait<0>();
        fence_proxy_async_smem();
        mbar_arrive(&bars->full_v[s]);
      }
      cp_async_wait<0>();
    }
  } else {
    // ============================================ softmax / rescale / epilogue
    const int r = threadIdx.x - 128;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    int i_row, hh;
    if (MODE == FLASH_DENSE) {
      i_row = qt * 128 + r;
      hh = h;
    } else {
      i_row = 64 * b + mt * p.rows_tok + r / p.G;
      hh = g * p.G + r % p.G;
    }
    const int i_min = (MODE == FLASH_DENSE) ? qt * 128 : 64 * b + mt * p.rows_tok;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      const int buf = j & 1;
      if (!warp_wait(&bars->s_full[buf], (j >> 1) & 1, p.limit_ns, abort_flag, 131)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t s_addr = tmem + lane_off + buf * 128;
      uint32_t sr[4][32];
      tmem_ld32(s_addr, sr[0]);
      tmem_ld32(s_addr + 32, sr[1]);
      tmem_ld32(s_addr + 64, sr[2]);
      tmem_ld32(s_addr + 96, sr[3]);
      tmem_ld_wait();
      reg_fence(sr[0]);
      reg_fence(sr[1]);
      reg_fence(sr[2]);
      reg_fence(sr[3]);
      // ---- mask
      bool need_mask;
      if (MODE == FLASH_DENSE) {
        need_mask = (j == qt);
      } else {
        const int last = j * 128 + 127;
        need_mask = (last >= cnt) || (pos_s[last] > i_min);
      }
      if (need_mask) {
        if (MODE == FLASH_DENSE) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c > r) sr[c >> 5][c & 31] = __float_as_uint(-INFINITY);
        } else {
          const int4* pv4 = reinterpret_cast<const int4*>(pos_s + j * 128);
#pragma unroll
          for (int c4 = 0; c4 < 32; ++c4) {
            const int4 q4 = pv4[c4];  // same address in every lane: a broadcast
            const int pj[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = c4 * 4 + e;
              const bool keep = (j * 128 + c < cnt) && (pj[e] >= 0) && (pj[e] <= i_row);
              if (!keep) sr[c >> 5][c & 31] = __float_as_uint(-INFINITY);
            }
          }
        }
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) mx = fmaxf(mx, __uint_as_float(sr[c >> 5][c & 31]));
      const float m_new = fmaxf(m_used, mx * p.scale_log2);
      float alpha = 1.f;
      const bool resc = m_new > m_used + 8.f;
      if (resc) {
        alpha = ex2_approx(m_used - m_new);
        m_used = m_new;
      }
      const float mu = (m_used == -INFINITY) ? 0.f : m_used;
      l *= alpha;
      // ---- P = exp2(s * scale - m), into TMEM over S
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float a = ex2_approx(fmaf(__uint_as_float(sr[c][2 * e]), p.scale_log2, -mu));
          const float bb = ex2_approx(fmaf(__uint_as_float(sr[c][2 * e + 1]), p.scale_log2, -mu));
          rs += a + bb;
          pk[e] = pack_bf16x2(a, bb);
        }
        tmem_st16(s_addr + c * 16, pk);
      }
      l += rs;
      // ---- O rescale (needs PV_{j-1} complete)
      if (j > 0) {
        if (!warp_wait(&bars->o_done, (j - 1) & 1, p.limit_ns, abort_flag, 132)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, resc)) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t orr[32];
            tmem_ld32(tmem + lane_off + 256 + c * 32, orr);
            tmem_ld_wait();
            reg_fence(orr);
#pragma unroll
            for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
            tmem_st32(tmem + lane_off + 256 + c * 32, orr);
          }
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->p_ready);
    }
    // ---- epilogue
    const bool row_live = i_row < p.L;  // a last dense tile may hang past L
    if (ok && ntiles > 0 && warp_wait(&bars->o_done, (ntiles - 1) & 1, p.limit_ns, abort_flag, 133)) {
      tc_fence_after();
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
      __nv_bfloat16* orow = p.o + static_cast<int64_t>(i_row) * p.o_tok + static_cast<int64_t>(hh) * p.o_head;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t orr[32];
        tmem_ld32(tmem + lane_off + 256 + c * 32, orr);
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
      if (MODE == FLASH_DENSE && row_live) {
        p.lse[static_cast<int64_t>(hh) * p.L + i_row] = (m_used + log2f(l)) * 0.69314718055994530942f;
      }
    } else if (ntiles == 0 && MODE == FLASH_SPARSE) {
      __nv_bfloat16* orow = p.o + static_cast<int64_t>(i_row) * p.o_tok + static_cast<int64_t>(hh) * p.o_head;
      uint4* dst = reinterpret_cast<uint4*>(orow);
      for (int v4 = 0; v4 < 16; ++v4) dst[v4] = make_uint4(0, 0, 0, 0);
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
