// Kernel (4), persistent: the sparse layers' attention over the shared index
// lists (HySparse2 architecture summary, KV-sharing paragraph: the sparse
// layers reuse the full layer's KV cache and token selection), with the
// causal mask j <= i on listed positions.  Window mode (WIN): the same
// pipeline computes causal sliding-window attention (the self-decoder's window
// layers; HySparse2 architecture summary, paragraph on the self-decoder /
// cross-decoder split): an item's keys are the contiguous range its block's
// windows cover, loaded as whole tiles by TMA, with the band mask
// i - W < j <= i.
//
// The per-tile arithmetic is that of kernel (1) (flash_fwd_kernel): an
// item is (query block b, KV head g, pair of 128-row M tiles), each M tile
// 128/G tokens x G heads of the block sharing the block's list, whose K/V rows
// are gathered with 16-byte cp.async into 128-byte-swizzled shared memory
// and multiplied on tcgen05 tensor cores (S in TMEM, P written back over S,
// O += P V from TMEM).  An item touches only 1152 keys (9 key tiles), so a
// CTA per item spends as long on its start and end -- TMEM allocation,
// barrier set-up, the Q and list loads, the first gathers, the last softmax
// and the O write -- as on the tiles themselves.  Here one CTA per SM loops
// over items instead, and every pipeline keeps running across item
// boundaries:
//
//   * the K/V ring, the per-tile barriers and TMEM carry over: phases are
//     counted over the CTA's whole tile stream, not per item;
//   * Q of the next item is loaded as soon as the last S of the current one
//     has executed (q_empty), while its last P V products and softmax run;
//   * the index list is double-buffered (list_full / list_empty), so the
//     gather of the next item starts while the current one is finishing;
//   * the first P V of an item waits only for the previous epilogue of the
//     same M tile to have read O (o_free); its S products do not wait.
//
// Roles, as in flash_fwd_kernel: warp 1 issues every MMA, warps 4-7 / 8-11
// run the softmax and epilogue of M tile A / B; with a bf16 cache warps 0, 2,
// 3 and 12-15 load the lists, gather K/V and (one thread) load Q; with an FP8
// cache warp 0 loads Q by TMA and warps 2, 3, 12 and 13 convert it and gather
// and convert the K/V codes to f16; in window mode (12 warps) warp 0 loads Q
// and whole K/V tiles by TMA.  The list modes run 16 warps with registers
// moved to the softmax warpgroups (the gather's issue rate was the critical
// path with 3 gather warps).  Every wait is bounded; a wait that runs out
// records HS2_ERR_TIMEOUT and the CTA winds down.
#pragma once

#include "flash.cuh"

namespace hs2 {

struct SparseBars {
  uint64_t q_raw;    // KV8: Q landed (bf16), before its conversion
  uint64_t q_full;   // Q of the current item ready for the MMAs
  uint64_t q_empty;  // the item's last S products have executed
  uint64_t full_k[FL_STAGES];
  uint64_t full_v[FL_STAGES];
  uint64_t empty[FL_STAGES];  // a stage's K/V rows: both P V products of its tile have executed
  uint64_t s_full[2];
  uint64_t p_ready[2];
  uint64_t o_done[2];
  uint64_t o_free[2];  // epilogue of M tile x has read O
  uint64_t list_full[2];
  uint64_t list_empty[2];
  uint64_t fin;
  uint32_t tmem_slot;
  int abort;
};
static_assert(sizeof(SparseBars) <= 256, "barriers fit their slot");

// The list modes run 16 warps: the bf16 gather uses 7 of them (0, 2, 3,
// 12-15), the FP8 converter 4 (2, 3, 12, 13), with registers moved from the
// copy/MMA warpgroups (0 and 3) to the two softmax warpgroups:
// 2 x 128 x SP_REG_COPY + 256 x SP_REG_SOFTMAX = 65536 = 512 x 128, the
// registers the CTA is launched with.  The window mode keeps 12 warps.
constexpr int SP_THREADS_LIST = 512;
constexpr uint32_t SP_REG_COPY = 80, SP_REG_SOFTMAX = 176;  // 56 / 200 and 88, 96 measured slower
static_assert(2 * 128 * SP_REG_COPY + 256 * SP_REG_SOFTMAX <= SP_THREADS_LIST * (65536 / SP_THREADS_LIST),
              "register split within the launch's registers");
__host__ __device__ constexpr int sp_threads(bool kv8, bool win) { return !win ? SP_THREADS_LIST : FL_THREADS; }

constexpr uint32_t SP_POS_OFF = FL_POS_OFF;                      // int [2][MAX_LIST]
constexpr uint32_t SP_KSC_OFF = SP_POS_OFF + 2 * MAX_LIST * 4;   // KV8: [stage][128]
constexpr uint32_t SP_SMEM = SP_KSC_OFF + 1024;                  // + alignment slack
constexpr uint32_t SP_SMEM_KV8 = SP_KSC_OFF + FL_STAGES * 128 * 4 + 1024;

struct SpItem {
  int b, g, pair, cnt, nt, nB, e_b;
  int lo;  // window mode: the first key of the item's contiguous key range
  bool has_b;
};

// The list length of item `it` (0 past the last item).
// Window mode's item order: CTA c takes it = c, c + grid, ...; this maps
// each full run of grid * mpairs such indices so that one CTA takes the M-tile
// pairs of one (block, KV head) back to back, the second finding the window's
// K/V tiles in L2 right after the first (2.46 -> 2.37 ms at 128k, 64/8 heads,
// W = 128; the list modes measured 3% slower with it and keep the plain
// order).  The last, partial run keeps the plain order; the map is a
// bijection on [0, n_items).
__device__ __forceinline__ int item_id(const FlashParams& p, int it, int n_items) {
  if (p.mpairs == 1) return it;
  const int step = static_cast<int>(gridDim.x);
  const int run = step * p.mpairs;
  const int r0 = (it / run) * run;
  if (r0 + run > n_items) return it;
  const int l = it - r0;
  return r0 + (l % step) * p.mpairs + l / step;
}

__device__ __forceinline__ int item_cnt(const FlashParams& p, int it, int n_items) {
  if (it >= n_items) return 0;
  const int bg = it / p.mpairs;
  return __ldg(p.cnt + static_cast<int64_t>(bg % p.Hkv) * p.nb + bg / p.Hkv);
}

// Item `it` given its list length c (read one item ahead, off the critical
// path).  In window mode the keys are the contiguous range the block's
// windows cover, [max(0, 64 b - W + 1), 64 b + 63], and c is not used.
template <bool WIN>
__device__ __forceinline__ SpItem sparse_item(const FlashParams& p, int it, int c, int n_items) {
  SpItem w;
  const int id = WIN ? item_id(p, it, n_items) : it;
  w.pair = id % p.mpairs;
  const int bg = id / p.mpairs;
  w.g = bg % p.Hkv;
  w.b = bg / p.Hkv;
  w.e_b = min(p.L, 64 * (w.b + 1));
  w.lo = 0;
  if (WIN) {
    w.lo = max(0, 64 * w.b - p.window + 1);
    c = w.e_b - w.lo;
  }
  w.cnt = max(0, min(c, WIN ? c : p.list_len));
  w.nt = (w.cnt + 127) / 128;
  w.has_b = 2 * w.pair + 1 < p.mtiles;
  w.nB = w.has_b ? w.nt : 0;
  return w;
}

template <bool KV8, bool WIN>
__global__ void __launch_bounds__(sp_threads(KV8, WIN), 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const FlashParams p, int n_items) {
  static_assert(!(KV8 && WIN), "the window mode reads a bf16 cache");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  SparseBars* bars = reinterpret_cast<SparseBars*>(smem + FL_BAR_OFF);
  int32_t* pos_base = reinterpret_cast<int32_t*>(smem + SP_POS_OFF);
  float* ksc_s = reinterpret_cast<float*>(smem + SP_KSC_OFF);
  const uint32_t q_base = smem_u32(smem + FL_Q_OFF);
  const uint32_t kv_base = smem_u32(smem + FL_KV_OFF);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &bars->abort;
  const int first = blockIdx.x, step = gridDim.x;
  // loader threads: warps 2-3 with an FP8 cache (warp 0 then only loads Q);
  // warps 0, 2, 3 and 12-15 with bf16 lists, warp 0's lane 0 also loading Q
  constexpr bool SPLIT = !WIN;  // 16 warps, registers moved to the softmax
  constexpr int NLD = KV8 ? 128 : (WIN ? 96 : 224);

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_raw, 1);
    mbar_init(&bars->q_full, KV8 ? static_cast<uint32_t>(NLD) : 1u);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < FL_STAGES; ++s) {
      mbar_init(&bars->full_k[s], WIN ? 1 : NLD);
      mbar_init(&bars->full_v[s], WIN ? 1 : NLD);
      mbar_init(&bars->empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->s_full[x], 1);
      mbar_init(&bars->p_ready[x], 4);  // one arrival per softmax warp
      mbar_init(&bars->o_done[x], 1);
      mbar_init(&bars->o_free[x], 128);
      mbar_init(&bars->list_full[x], NLD);
      mbar_init(&bars->list_empty[x], 256);
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
  // warpgroup index, visibly uniform for the compiler
  const int wgi = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x) / 128, 0);
  if (wgi == 0 || wgi == 3) {
  if (SPLIT) reg_release<SP_REG_COPY>();
  if ((KV8 || WIN) && warp == 0) {
    // ============================ Q by TMA (and, in window mode, K/V tiles)
    if (lane == 0 && !(p.flags & FLAG_SKIP_LOADS)) {
      tma_prefetch_desc(&tmQ);
      if (WIN) {
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
      }
      int u0 = 0, last_u = -1;
      uint64_t* qbar = KV8 ? &bars->q_raw : &bars->q_full;
      int ii = 0, loaded = 0;
      int c_cur = WIN ? 0 : item_cnt(p, first, n_items), c_nxt = 0;
      for (int it = first; it < n_items; it += step, ++ii, c_cur = c_nxt) {
        c_nxt = WIN ? 0 : item_cnt(p, it + step, n_items);
        const SpItem w = sparse_item<WIN>(p, it, c_cur, n_items);
        if (w.nt == 0) continue;
        bool ok = true;
        // window mode: key tile j of the item into its ring stage
        auto load_tile = [&](int j) -> bool {
          const int u = u0 + j;
          const int s = u % FL_STAGES;
          if (u >= FL_STAGES &&
              !mbar_wait(&bars->empty[s], ((u / FL_STAGES) - 1) & 1, p.limit_ns, abort_flag, 305))
            return false;
          uint8_t* kd = smem + FL_KV_OFF + s * 2 * TILE_BYTES;
          const int t0 = w.lo + j * 128;
          mbar_arrive_expect_tx(&bars->full_k[s], TILE_BYTES);
          tma_load_3d(kd, &tmK, &bars->full_k[s], 0, w.g, t0);
          tma_load_3d(kd + HALF_BYTES, &tmK, &bars->full_k[s], 64, w.g, t0);
          mbar_arrive_expect_tx(&bars->full_v[s], TILE_BYTES);
          tma_load_3d(kd + TILE_BYTES, &tmV, &bars->full_v[s], 0, w.g, t0);
          tma_load_3d(kd + TILE_BYTES + HALF_BYTES, &tmV, &bars->full_v[s], 64, w.g, t0);
          last_u = u;
          return true;
        };
        if (loaded > 0 && !mbar_wait(&bars->q_empty, (loaded - 1) & 1, p.limit_ns, abort_flag, 301)) break;
        const int nq = w.has_b ? 2 : 1;
        mbar_arrive_expect_tx(qbar, static_cast<uint32_t>(nq) * TILE_BYTES);
        for (int x = 0; x < nq; ++x) {
          uint8_t* qd = smem + FL_Q_OFF + x * TILE_BYTES;
          const int t0 = 64 * w.b + (2 * w.pair + x) * p.rows_tok;
          tma_load_3d(qd, &tmQ, qbar, 0, w.g * p.G, t0);
          tma_load_3d(qd + HALF_BYTES, &tmQ, qbar, 64, w.g * p.G, t0);
        }
        ++loaded;
        for (int j = 0; WIN && j < w.nt && ok; ++j) ok = load_tile(j);
        if (!ok) break;
        u0 += w.nt;
      }
      // never leave a TMA write in flight into memory the CTA gives back
      if (loaded > 0) wait_done(qbar, (loaded - 1) & 1, p.limit_ns, 302);
      for (int u = max(0, last_u - FL_STAGES + 1); u <= last_u; ++u) {
        wait_done(&bars->full_k[u % FL_STAGES], (u / FL_STAGES) & 1, p.limit_ns, 306);
        wait_done(&bars->full_v[u % FL_STAGES], (u / FL_STAGES) & 1, p.limit_ns, 307);
      }
    }
  } else if (warp == 1) {
    // ========================================================== MMA issue
    if (lane == 0) {
      int u0 = 0, qi = 0;            // tiles of the CTA's stream so far; items with Q
      int tx[2] = {0, 0}, jx[2] = {0, 0};  // tiles / items per M tile so far
      bool ok = true;
      int c_cur = WIN ? 0 : item_cnt(p, first, n_items), c_nxt = 0;
      for (int it = first; it < n_items && ok; it += step, c_cur = c_nxt) {
        c_nxt = WIN ? 0 : item_cnt(p, it + step, n_items);
        const SpItem w = sparse_item<WIN>(p, it, c_cur, n_items);
        const int nt = w.nt;
        if (nt == 0) continue;
        const int nx[2] = {nt, w.nB};
        auto issue_s = [&](int x, int j) {
          const uint32_t kb = kv_base + ((u0 + j) % FL_STAGES) * 2 * TILE_BYTES;
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
          const uint32_t vb = kv_base + ((u0 + j) % FL_STAGES) * 2 * TILE_BYTES + TILE_BYTES;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t bdesc = sdesc_sw128(vb + kk * 2048, HALF_BYTES, 1024);
            umma_ts(tmem + 256 + x * 128, tmem + x * 128 + kk * 8, bdesc, KV8 ? IDESC_PV_F16 : IDESC_PV,
                    (j > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&bars->o_done[x]);
        };
        ok = mbar_wait(&bars->q_full, qi & 1, p.limit_ns, abort_flag, 311);
        if (ok) ok = mbar_wait(&bars->full_k[u0 % FL_STAGES], (u0 / FL_STAGES) & 1, p.limit_ns, abort_flag, 312);
        if (!ok) break;
        tc_fence_after();
        for (int x = 0; x < 2; ++x)
          if (nx[x] > 0) issue_s(x, 0);
        if (nt == 1) umma_commit(&bars->q_empty);
        for (int j = 0; j < nt && ok; ++j) {
          const int u = u0 + j;
          const int s = u % FL_STAGES;
          bool v_ready = false, k_next = false;
          for (int x = 0; x < 2 && ok; ++x) {
            if (j >= nx[x]) continue;
            if (!mbar_wait(&bars->p_ready[x], (tx[x] + j) & 1, p.limit_ns, abort_flag, 313)) {
              ok = false;
              break;
            }
            if (!v_ready) {
              if (!mbar_wait(&bars->full_v[s], (u / FL_STAGES) & 1, p.limit_ns, abort_flag, 314)) {
                ok = false;
                break;
              }
              v_ready = true;
            }
            // the first P V of an item overwrites O: the previous epilogue must have read it
            if (j == 0 && jx[x] > 0 &&
                !mbar_wait(&bars->o_free[x], (jx[x] - 1) & 1, p.limit_ns, abort_flag, 315)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_pv(x, j);
            // the tile's last P V is issued: its stage is released as soon as
            // that executes, before the next tile's S products are queued
            if (x == 1 || j >= nx[1]) umma_commit(&bars->empty[s]);
            if (j + 1 < nx[x]) {
              if (!k_next) {
                const int s1 = (u + 1) % FL_STAGES;
                if (!mbar_wait(&bars->full_k[s1], ((u + 1) / FL_STAGES) & 1, p.limit_ns, abort_flag, 316)) {
                  ok = false;
                  break;
                }
                k_next = true;
                tc_fence_after();
              }
              issue_s(x, j + 1);
            }
          }
          if (ok && j + 2 == nt) umma_commit(&bars->q_empty);  // the item's last S products are issued
        }
        u0 += nt;
        ++qi;
        for (int x = 0; x < 2; ++x) {
          tx[x] += nx[x];
          jx[x] += nx[x] > 0 ? 1 : 0;
        }
      }
      umma_commit(&bars->fin);
      wait_done(&bars->fin, 0, p.limit_ns, 317);
    }
  } else if (!WIN && (KV8 ? (warp == 2 || warp == 3 || warp == 12 || warp == 13)
                          : (warp == 0 || warp == 2 || warp == 3 || warp >= 12))) {
    // ===================================== lists and K/V (gather / convert)
    if (!(p.flags & FLAG_SKIP_LOADS)) {
      const int pt = KV8 ? (warp < 4 ? threadIdx.x - 64 : threadIdx.x - 320)
                         : (warp == 0 ? lane : (warp < 4 ? threadIdx.x - 32 : threadIdx.x - 288));  // 0 .. NLD-1
      const bool q_thread = !KV8 && warp == 0 && lane == 0;
      if (q_thread) tma_prefetch_desc(&tmQ);
      int ii = 0, u0 = 0, qi = 0, loaded = 0;
      bool ok = true;
      int c_cur = WIN ? 0 : item_cnt(p, first, n_items), c_nxt = 0;
      for (int it = first; it < n_items && ok; it += step, ++ii, c_cur = c_nxt) {
        c_nxt = WIN ? 0 : item_cnt(p, it + step, n_items);
        const SpItem w = sparse_item<WIN>(p, it, c_cur, n_items);
        const int buf = ii & 1;
        int32_t* pos_s = pos_base + buf * MAX_LIST;
        // ---- the item's list (the buffer's previous item is done with it)
        if (ii >= 2 && !mbar_wait(&bars->list_empty[buf], ((ii >> 1) - 1) & 1, p.limit_ns, abort_flag, 321)) {
          ok = false;
          break;
        }
        // entries past the count, and entries outside [0, e_b) (reported),
        // become -1: never read, always masked
        const int32_t* list = p.idx + (static_cast<int64_t>(w.g) * p.nb + w.b) * p.list_len;
        constexpr int LB = 6;  // list loads in flight per thread (a 1152-entry list: 2 or 3 rounds)
        for (int i0 = pt; i0 < w.nt * 128; i0 += LB * NLD) {
          int e[LB];
#pragma unroll
          for (int v = 0; v < LB; ++v) {
            const int i = i0 + v * NLD;
            e[v] = (i < w.cnt) ? __ldg(list + i) : -1;
          }
#pragma unroll
          for (int v = 0; v < LB; ++v) {
            const int i = i0 + v * NLD;
            if (i < w.nt * 128) {
              if (i < w.cnt && (e[v] < 0 || e[v] >= w.e_b)) {
                report(HS2_ERR_INDEX, 328);
                e[v] = -1;
              }
              pos_s[i] = e[v];
            }
          }
        }
        mbar_arrive(&bars->list_full[buf]);
        // bf16: Q of the item, once the previous item's S products ran (after
        // this thread's share of the list, so the list is not held up)
        if (q_thread && w.nt > 0) {
          if (loaded > 0 && !mbar_wait(&bars->q_empty, (loaded - 1) & 1, p.limit_ns, abort_flag, 301)) {
            ok = false;
            break;
          }
          const int nq = w.has_b ? 2 : 1;
          mbar_arrive_expect_tx(&bars->q_full, static_cast<uint32_t>(nq) * TILE_BYTES);
          for (int x = 0; x < nq; ++x) {
            uint8_t* qd = smem + FL_Q_OFF + x * TILE_BYTES;
            const int t0 = 64 * w.b + (2 * w.pair + x) * p.rows_tok;
            tma_load_3d(qd, &tmQ, &bars->q_full, 0, w.g * p.G, t0);
            tma_load_3d(qd + HALF_BYTES, &tmQ, &bars->q_full, 64, w.g * p.G, t0);
          }
          ++loaded;
        }
        // the loaders read each other's entries too: wait for all of them (bounded)
        if (!mbar_wait(&bars->list_full[buf], (ii >> 1) & 1, p.limit_ns, abort_flag, 327)) {
          ok = false;
          break;
        }
        if (w.nt == 0) continue;
        if (KV8) {
          // ---- Q: bf16 -> f16 in place, once its TMA has landed
          if (!mbar_wait(&bars->q_raw, qi & 1, p.limit_ns, abort_flag, 322)) {
            ok = false;
            break;
          }
          const int nchunks = (w.has_b ? 2 : 1) * static_cast<int>(TILE_BYTES / 16);
          bool q_over = false;
          for (int c = pt; c < nchunks; c += NLD) {
            const uint32_t a = q_base + c * 16;
            st_shared_v4(a, bf16x8_to_f16x8_checked(ld_shared_v4(a), q_over));
          }
          if (q_over) report(HS2_ERR_RANGE, 349);
          fence_proxy_async_smem();
          mbar_arrive(&bars->q_full);
          // ---- K/V tiles: 8 threads per 128-byte code row, RPT rows each
          constexpr int RSTEP = NLD / 8, RPT = 128 / RSTEP;
          static_assert(!KV8 || RSTEP * RPT == 128, "converter rows cover the tile");
          const int rsub = pt >> 3, c8 = pt & 7;
          const uint8_t* kb8 = p.k8 + static_cast<int64_t>(w.g) * p.kv_head + c8 * 16;
          const uint8_t* vb8 = p.v8 + static_cast<int64_t>(w.g) * p.kv_head + c8 * 16;
          for (int j = 0; j < w.nt && ok; ++j) {
            const int u = u0 + j;
            const int s = u % FL_STAGES;
            if (u >= FL_STAGES &&
                !mbar_wait(&bars->empty[s], ((u / FL_STAGES) - 1) & 1, p.limit_ns, abort_flag, 323)) {
              ok = false;
              break;
            }
            const uint32_t kd = kv_base + s * 2 * TILE_BYTES;
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {  // 0: K, 1: V
              const uint8_t* base8 = half ? vb8 : kb8;
              const float* scale = half ? p.vsc : p.ksc;
              // every row's codes and scale in flight before any is converted
              uint4 raw[RPT];
              float sgv[RPT];
#pragma unroll
              for (int i = 0; i < RPT; ++i) {
                const int pj = pos_s[j * 128 + rsub + RSTEP * i];
                raw[i] = make_uint4(0, 0, 0, 0);
                sgv[i] = 0.f;
                if (pj >= 0) {
                  raw[i] = ld_nc_v4(base8 + static_cast<int64_t>(pj) * p.kv_tok);
                  sgv[i] = scale[static_cast<int64_t>(pj) * p.Hkv + w.g];
                }
              }
#pragma unroll
              for (int i = 0; i < RPT; ++i) {
                const int r = rsub + RSTEP * i;
                const float sg = sgv[i];
                const uint32_t wd[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
                uint32_t f[8];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  f[2 * q] = e4m3x2_to_f16x2(wd[q]);
                  f[2 * q + 1] = e4m3x2_to_f16x2(wd[q] >> 16);
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
        } else {
          // ---- bf16 gather: per key tile, 16 threads per row (one 16-byte
          // chunk each) and 6 rows at a time, K and V of a row together
          const int rg = pt >> 4, chunk = pt & 15;
          const uint32_t half_off = static_cast<uint32_t>((chunk >> 3) * 128 * 128);
          const __nv_bfloat16* kg = p.k + static_cast<int64_t>(w.g) * p.kv_head + chunk * 8;
          const __nv_bfloat16* vg = p.v + static_cast<int64_t>(w.g) * p.kv_head + chunk * 8;
          for (int j = 0; j < w.nt && ok; ++j) {
            const int u = u0 + j;
            const int s = u % FL_STAGES;
            // the next tile's rows start moving into L2 now: its gather can
            // only begin once a stage frees, and rows missing L2 would
            // otherwise set that gather's length
            if (j + 1 < w.nt) {  // 4 lines of 128 B per listed position (K and V rows)
              for (int q = pt; q < 4 * 128; q += NLD) {
                const int pj = pos_s[(j + 1) * 128 + (q >> 2)];
                if (pj >= 0) {
                  const int64_t off = static_cast<int64_t>(pj) * p.kv_tok - chunk * 8 + (q & 1) * 64;
                  prefetch_l2(((q & 2) ? vg : kg) + off);
                }
              }
            }
            if (u >= FL_STAGES &&
                !mbar_wait(&bars->empty[s], ((u / FL_STAGES) - 1) & 1, p.limit_ns, abort_flag, 325)) {
              ok = false;
              break;
            }
            const uint32_t kd = kv_base + s * 2 * TILE_BYTES + half_off;
            const int32_t* pj_row = pos_s + j * 128;
#pragma unroll 6
            for (int r = rg; r < 128; r += NLD / 16) {
              const int pj = pj_row[r];
              const bool valid = pj >= 0;
              const int64_t off = static_cast<int64_t>(valid ? pj : 0) * p.kv_tok;
              const uint32_t d = kd + static_cast<uint32_t>(r * 128 + (((chunk & 7) ^ (r & 7)) << 4));
              cp_async_16(d, kg + off, valid ? 16u : 0u);
              cp_async_16(d + TILE_BYTES, vg + off, valid ? 16u : 0u);
            }
            cp_async_commit();
            cp_async_wait<0>();
            fence_proxy_async_smem();
            mbar_arrive(&bars->full_k[s]);
            mbar_arrive(&bars->full_v[s]);
          }
        }
        u0 += w.nt;
        ++qi;
      }
      cp_async_wait<0>();
      if (q_thread && loaded > 0) wait_done(&bars->q_full, (loaded - 1) & 1, p.limit_ns, 302);
    }
  }
  } else {
    if (SPLIT) reg_acquire<SP_REG_SOFTMAX>();
    // ============================================ softmax / rescale / epilogue
    const int x = (warp >= 8) ? 1 : 0;  // M tile of this warpgroup
    const int r = threadIdx.x - 128 - 128 * x;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t s_tm = tmem + lane_off + x * 128;
    const uint32_t o_tm = tmem + lane_off + 256 + x * 128;
    const float sc = KV8 ? 1.f : p.scale_log2;  // KV8 folds the scale into the columns
    int ii = 0, u0 = 0, tx = 0;
    bool ok = true;
    int c_cur = WIN ? 0 : item_cnt(p, first, n_items), c_nxt = 0;
    for (int it = first; it < n_items && ok; it += step, ++ii, c_cur = c_nxt) {
      c_nxt = WIN ? 0 : item_cnt(p, it + step, n_items);
      const SpItem w = sparse_item<WIN>(p, it, c_cur, n_items);
      const int buf = ii & 1;
      const int32_t* pos_s = pos_base + buf * MAX_LIST;
      const int nX = x ? w.nB : w.nt;
      const int mt = 2 * w.pair + x;
      const int i_row = 64 * w.b + mt * p.rows_tok + r / p.G;
      const int hh = w.g * p.G + r % p.G;
      const int i_min = 64 * w.b + mt * p.rows_tok;
      if (!WIN && !warp_wait(&bars->list_full[buf], (ii >> 1) & 1, p.limit_ns, abort_flag, 330)) {
        ok = false;
        break;
      }
      float m_used = -INFINITY, l = 0.f;
      for (int j = 0; j < nX; ++j) {
        const int t = tx + j;  // tiles this M tile has seen before j
        if (!warp_wait(&bars->s_full[x], t & 1, p.limit_ns, abort_flag, 331)) {
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
          const uint64_t* ks2 = reinterpret_cast<const uint64_t*>(ksc_s + ((u0 + j) % FL_STAGES) * 128);
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
        // ---- mask (after any scaling): the window band, or causal on listed positions
        const int last = j * 128 + 127;
        if (WIN) {  // keep i - W < key <= i, key = lo + 128 j + c
          const int c_hi = i_row - (w.lo + j * 128), c_lo = c_hi - p.window;
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c > c_hi || c <= c_lo) sr[c >> 5][c & 31] = __float_as_uint(-INFINITY);
        } else if ((last >= w.cnt) || (pos_s[last] > i_min)) {
          const int4* pv4 = reinterpret_cast<const int4*>(pos_s + j * 128);
#pragma unroll
          for (int c4 = 0; c4 < 32; ++c4) {
            const int4 q4 = pv4[c4];  // same address in every lane: a broadcast
            const int pj[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = c4 * 4 + e;
              const bool keep = (j * 128 + c < w.cnt) && (pj[e] >= 0) && (pj[e] <= i_row);
              if (!keep) sr[c >> 5][c & 31] = __float_as_uint(-INFINITY);
            }
          }
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
        const float mx =
            fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
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
        // ---- O rescale: P V of the previous tile completed before S of this
        // one (the MMA thread issues P V(j - 1) first, and s_full's commit
        // covers every MMA issued before it)
        if (j > 0 && __any_sync(0xffffffffu, resc)) {
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
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();  // one arrival per warp, once all its lanes' stores completed
        if (lane == 0) mbar_arrive(&bars->p_ready[x]);
      }
      if (!WIN) mbar_arrive(&bars->list_empty[buf]);  // masking is done with this list
      if (!ok) break;
      // ---- epilogue
      const bool row_live = x == 0 || w.has_b;
      __nv_bfloat16* orow = p.o + static_cast<int64_t>(i_row) * p.o_tok + static_cast<int64_t>(hh) * p.o_head;
      if (nX > 0) {
        if (!warp_wait(&bars->o_done[x], (tx + nX - 1) & 1, p.limit_ns, abort_flag, 333)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float inv = (l > 0.f) ? 1.f / l : 0.f;
        // O in two halves of 64 columns, one TMEM wait each; once the second
        // half is in registers the next item's P V may overwrite O, so o_free
        // is signalled before the last stores
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          uint32_t orr[2][32];
          tmem_ld32(o_tm + (2 * half) * 32, orr[0]);
          tmem_ld32(o_tm + (2 * half + 1) * 32, orr[1]);
          tmem_ld_wait();
          reg_fence(orr[0]);
          reg_fence(orr[1]);
          if (half == 1) {
            tc_fence_before();
            mbar_arrive(&bars->o_free[x]);
          }
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
              pk[e] = pack_bf16x2(__uint_as_float(orr[cc][2 * e]) * inv, __uint_as_float(orr[cc][2 * e + 1]) * inv);
            uint4* dst = reinterpret_cast<uint4*>(orow + (2 * half + cc) * 32);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
          }
        }
        if (WIN && p.lse != nullptr)  // natural-log LSE of the row
          p.lse[static_cast<int64_t>(hh) * p.L + i_row] = (m_used + log2f(l)) * 0.69314718055994530942f;
      } else if (w.nt == 0 && row_live) {
        // an empty list: the rows attend to nothing
        uint4* dst = reinterpret_cast<uint4*>(orow);
        for (int v4 = 0; v4 < 16; ++v4) dst[v4] = make_uint4(0, 0, 0, 0);
      }
      u0 += w.nt;
      tx += nX;
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
