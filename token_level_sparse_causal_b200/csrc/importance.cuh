// Kernel (2): block importance from the full layer's scores.
//
// For query block b (64 tokens), KV head g and every candidate key
// j in C_b = [0, e_b - recent):
//     I_j = sum_{h in group g} sum_{i in block b} exp(s_hij - lse_hi)
// (HySparse2 architecture summary, ablation paragraph: the full layer's
// complete attention scores choose the tokens; the aggregation is this
// library's reading.)  Because every candidate lies before the block's
// recent window and recent >= 64, j < i holds for all of the block's
// queries and no causal mask is needed.
//
// Mapping: keys sit on the MMA M dimension.  D = K_tile (128 keys x d) *
// Q_block^T (d x 64G query-head rows), so TMEM lane r holds key r's scores
// against every (query, head) of the block, and the thread that owns lane r
// sums exp2(s * log2e/sqrt(d) - lse_n * log2e) along its row.  The 64G
// columns are split in sub-tiles of N = min(256, 64G); two TMEM buffers let
// the tensor core fill one sub-tile while the epilogue drains the other.
//
// CTA = 20 warps: warp 0 TMA (Q block once, then K tiles), warp 1 MMA issue
// and TMEM owner, warps 4-19 four epilogue warpgroups that split the columns
// of each sub-tile in quarters (thread r of every group <-> key r of the
// tile).  Each thread issues all of its TMEM loads for a sub-tile before one
// wait, and groups 2-4 hand their partial sums to group 1 through shared
// memory, which adds them in a fixed order (the result is deterministic, so
// hs2_importance reproduces exactly what the selection saw).  Arguments and
// sums use packed f32x2 FMA/ADD; a quarter of the exponentials run on the FMA
// pipes (exp2_fma3), the rest on the MUFU unit -- the share measured fastest.
// FP8 e4m3 cache: warps 2-3 convert the Q block to f16 in place, and the K
// tiles are f16 (MMAs run kind::f16): either converted exactly from the codes
// by warps 2-3 (KVM_E4M3) or loaded by TMA from the layer's f16 copy
// (KVM_F16, see dequant_kv_kernel); each key's fp32 scale multiplies its row
// of scores in the epilogue.
// Work item = (KV head, block, chunk of IMP_CK keys); the grid is
// (chunks of the longest row of the strip) x (Hkv * blocks).
#pragma once

#include <type_traits>

#include "common.cuh"
#include "flash.cuh"

namespace hs2 {

constexpr int IMP_CK = 4096;   // keys per CTA (2048 and 8192 measured slower overall)
constexpr int IMP_STAGES = 2;  // K tile ring (deeper rings measured no faster)

struct ImpParams {
  int L, Hq, Hkv, G, recent, b0, nbs;
  const uint8_t* k8;  // e4m3 K codes and fp32 scales [L][Hkv] (KV8)
  const float* ksc;
  int64_t kv_tok, kv_head;
  int skip_le;       // rows with |C_b| <= skip_le are not computed (-1: compute all)
  int visible;       // checking mode: rows over every key j < e_b, causal mask applied
  float scale_log2;  // log2(e) / sqrt(d)
  const float* lse;  // [Hq][L]
  float* imp;
  int64_t row_stride;
  uint64_t limit_ns;
  uint32_t flags;
};

struct ImpBars {
  uint64_t q_raw;  // KV8: Q block landed (bf16), before its conversion to f16
  uint64_t q_full;
  uint64_t k_full[IMP_STAGES];
  uint64_t k_empty[IMP_STAGES];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t part_full[2];   // group 2's partial sums of a tile are in `part`
  uint64_t part_empty[2];  // group 1 has read them
  uint64_t fin;
  uint32_t tmem_slot;
  int abort;
};

__host__ __device__ constexpr uint32_t imp_q_bytes(int G) { return static_cast<uint32_t>(64 * G) * 256u; }
__host__ __device__ constexpr uint32_t imp_kv_off(int G) { return imp_q_bytes(G); }
__host__ __device__ constexpr uint32_t imp_bar_off(int G) { return imp_q_bytes(G) + IMP_STAGES * TILE_BYTES; }
__host__ __device__ constexpr uint32_t imp_lse_off(int G) { return imp_bar_off(G) + 256; }
__host__ __device__ constexpr uint32_t imp_part_off(int G) { return imp_lse_off(G) + static_cast<uint32_t>(64 * G) * 4u; }
constexpr int IMP_GROUPS = 4;  // epilogue warpgroups
constexpr int IMP_THREADS = 128 + 128 * IMP_GROUPS;
__host__ __device__ constexpr uint32_t imp_smem_bytes(int G) {
  return imp_part_off(G) + (IMP_GROUPS - 1) * 2u * 128u * 4u + 1024u;
}

template <int G, int KVM>
__global__ void __launch_bounds__(IMP_THREADS, 1)
    importance_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const ImpParams p) {
  constexpr bool KV8 = KVM != KVM_BF16;   // f16 operands, per-key scales
  constexpr bool CONV = KVM == KVM_E4M3;  // K tiles converted by warps 2-3
  constexpr int NQ = 64 * G;                    // query-head rows of a block
  constexpr int NSUB = (NQ < 256) ? NQ : 256;   // MMA N per sub-tile
  constexpr int SUBS = NQ / NSUB;
  constexpr uint32_t QHALF = static_cast<uint32_t>(NQ) * 128u;
  constexpr uint32_t IDESC = KV8 ? idesc_f16_f32(128, NSUB, 0, 0) : idesc_bf16_f32(128, NSUB, 0, 0);
  constexpr uint32_t TMEM_COLS = (2 * NSUB <= 256) ? 256u : 512u;

  const int y = blockIdx.y;
  const int g = y / p.nbs;
  const int b = p.b0 + y % p.nbs;
  const int e_b = min(p.L, 64 * (b + 1));
  const int n_c = p.visible ? e_b : max(0, e_b - p.recent);
  const int j0 = static_cast<int>(blockIdx.x) * IMP_CK;
  if (j0 >= n_c || n_c <= p.skip_le) return;  // uniform exit before any allocation
  const int ntiles = (min(IMP_CK, n_c - j0) + 127) / 128;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  ImpBars* bars = reinterpret_cast<ImpBars*>(smem + imp_bar_off(G));
  float* nlse = reinterpret_cast<float*>(smem + imp_lse_off(G));
  float* part = reinterpret_cast<float*>(smem + imp_part_off(G));  // [groups-1][2][128] partial sums
  const uint32_t q_base = smem_u32(smem);
  const uint32_t k_base = smem_u32(smem + imp_kv_off(G));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &bars->abort;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_raw, 1);
    mbar_init(&bars->q_full, KV8 ? 64u : 1u);
    for (int s = 0; s < IMP_STAGES; ++s) {
      mbar_init(&bars->k_full[s], CONV ? 64u : 1u);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->acc_full[s], 1);
      mbar_init(&bars->acc_empty[s], 128 * IMP_GROUPS);
      mbar_init(&bars->part_full[s], 128 * (IMP_GROUPS - 1));
      mbar_init(&bars->part_empty[s], 128);
    }
    mbar_init(&bars->fin, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  // -lse * log2(e) for every (query, head) column n = t * G + hl of the block
  for (int n = threadIdx.x; n < NQ; n += blockDim.x) {
    const int t = n / G, hl = n % G;
    nlse[n] = -p.lse[static_cast<int64_t>(g * G + hl) * p.L + 64 * b + t] * 1.44269504088896340736f;
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_slot;

  if (warp == 0) {
    if (lane == 0 && !(p.flags & FLAG_SKIP_LOADS)) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      uint64_t* qbar = KV8 ? &bars->q_raw : &bars->q_full;
      mbar_arrive_expect_tx(qbar, 2 * QHALF);
      tma_load_3d(smem, &tmQ, qbar, 0, g * G, 64 * b);
      tma_load_3d(smem + QHALF, &tmQ, qbar, 64, g * G, 64 * b);
      int last = -1;
      for (int t = 0; t < (CONV ? 0 : ntiles); ++t) {
        const int s = t % IMP_STAGES;
        if (t >= IMP_STAGES &&
            !mbar_wait(&bars->k_empty[s], ((t / IMP_STAGES) - 1) & 1, p.limit_ns, abort_flag, 201))
          break;
        uint8_t* kd = smem + imp_kv_off(G) + s * TILE_BYTES;
        mbar_arrive_expect_tx(&bars->k_full[s], TILE_BYTES);
        tma_load_3d(kd, &tmK, &bars->k_full[s], 0, g, j0 + t * 128);
        tma_load_3d(kd + HALF_BYTES, &tmK, &bars->k_full[s], 64, g, j0 + t * 128);
        last = t;
      }
      for (int t = max(0, last - IMP_STAGES + 1); t <= last; ++t)
        wait_done(&bars->k_full[t % IMP_STAGES], (t / IMP_STAGES) & 1, p.limit_ns, 202);
      wait_done(qbar, 0, p.limit_ns, 203);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = mbar_wait(&bars->q_full, 0, p.limit_ns, abort_flag, 211);
      if (ok) tc_fence_after();
      int u = 0;
      for (int t = 0; t < ntiles && ok; ++t) {
        const int s = t % IMP_STAGES;
        if (!mbar_wait(&bars->k_full[s], (t / IMP_STAGES) & 1, p.limit_ns, abort_flag, 212)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t kb = k_base + s * TILE_BYTES;
        for (int sub = 0; sub < SUBS; ++sub, ++u) {
          const int buf = u & 1;
          if (u >= 2 && !mbar_wait(&bars->acc_empty[buf], ((u >> 1) - 1) & 1, p.limit_ns, abort_flag, 213)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem + buf * NSUB;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t koff = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
            const uint32_t qoff = (kk >> 2) * QHALF + sub * NSUB * 128 + (kk & 3) * 32;
            umma_ss(d, sdesc_sw128(kb + koff, 16, 1024), sdesc_sw128(q_base + qoff, 16, 1024), IDESC,
                    kk > 0 ? 1u : 0u);
          }
          umma_commit(&bars->acc_full[buf]);
        }
        if (ok) umma_commit(&bars->k_empty[s]);
      }
      umma_commit(&bars->fin);
      wait_done(&bars->fin, 0, p.limit_ns, 214);
    }
  } else if (warp < 4) {
    // FP8 cache: convert the Q block to f16 in place; KVM_E4M3 then loads,
    // converts (exactly, e4m3 -> f16) and stores every K tile, 8 threads per
    // 128-byte code row.
    if (KV8 && !(p.flags & FLAG_SKIP_LOADS)) {
      const int pt = threadIdx.x - 64;
      if (mbar_wait(&bars->q_raw, 0, p.limit_ns, abort_flag, 241)) {
        bool q_over = false;
        for (int c = pt; c < static_cast<int>(2 * QHALF / 16); c += 64) {
          const uint32_t a = q_base + c * 16;
          st_shared_v4(a, bf16x8_to_f16x8_checked(ld_shared_v4(a), q_over));
        }
        if (q_over) report(HS2_ERR_RANGE, 249);
        fence_proxy_async_smem();
        mbar_arrive(&bars->q_full);
        const int rsub = pt >> 3, c8 = pt & 7;
        const uint8_t* kb8 = p.k8 + static_cast<int64_t>(g) * p.kv_head + c8 * 16;
        for (int t = 0; t < (CONV ? ntiles : 0); ++t) {  // KVM_F16: K tiles come by TMA
          const int s = t % IMP_STAGES;
          if (t >= IMP_STAGES &&
              !mbar_wait(&bars->k_empty[s], ((t / IMP_STAGES) - 1) & 1, p.limit_ns, abort_flag, 242))
            break;
          const uint32_t kd = k_base + s * TILE_BYTES;
#pragma unroll 4
          for (int it = 0; it < 16; ++it) {
            const int r = rsub + 8 * it;
            const uint4 raw = ld_nc_v4(kb8 + static_cast<int64_t>(j0 + t * 128 + r) * p.kv_tok);  // < L
            const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
            uint32_t f[8];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              f[2 * q] = e4m3x2_to_f16x2(w[q]);
              f[2 * q + 1] = e4m3x2_to_f16x2(w[q] >> 16);
            }
            st_shared_v4(kd + sw128_chunk_offset(r, 2 * c8, 128), make_uint4(f[0], f[1], f[2], f[3]));
            st_shared_v4(kd + sw128_chunk_offset(r, 2 * c8 + 1, 128), make_uint4(f[4], f[5], f[6], f[7]));
          }
          fence_proxy_async_smem();
          mbar_arrive(&bars->k_full[s]);
        }
      }
    }
  } else if (warp >= 4) {
    const int grp = (warp - 4) >> 2;              // epilogue group 0..IMP_GROUPS-1
    const int r = threadIdx.x - 128 - 128 * grp;  // key row of the tile
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    constexpr int QCOLS = NSUB / IMP_GROUPS;      // columns per group and sub-tile (32 or 64)
    constexpr int NLD = QCOLS / 32;
    float* out = p.imp + (static_cast<int64_t>(g) * p.nbs + (b - p.b0)) * p.row_stride;
    const uint64_t c2p = f2_pack(p.scale_log2, p.scale_log2);
    int u = 0;
    bool ok = true;
    for (int t = 0; t < ntiles && ok; ++t) {
      uint64_t acc2[2] = {0ull, 0ull};
      uint64_t c2t = c2p;
      if (KV8) {  // this key's scale multiplies its whole row of scores
        const int jk = min(j0 + t * 128 + r, p.L - 1);
        const float cs = p.scale_log2 * p.ksc[static_cast<int64_t>(jk) * p.Hkv + g];
        c2t = f2_pack(cs, cs);
      }
      for (int sub = 0; sub < SUBS; ++sub, ++u) {
        const int buf = u & 1;
        if (!warp_wait(&bars->acc_full[buf], (u >> 1) & 1, p.limit_ns, abort_flag, 221)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int col0 = grp * QCOLS;
        uint32_t sr[NLD][32];
#pragma unroll
        for (int c = 0; c < NLD; ++c) tmem_ld32(tmem + lane_off + buf * NSUB + col0 + c * 32, sr[c]);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < NLD; ++c) reg_fence(sr[c]);
        tc_fence_before();
        mbar_arrive(&bars->acc_empty[buf]);  // the buffer's data is in registers now
        const float4* nl4 = reinterpret_cast<const float4*>(nlse + sub * NSUB + col0);
        // MASK (checking mode only, on the tiles that reach the block's own
        // positions): key j is visible to column n (query 64b + n / G) iff
        // n >= (j - 64b) * G.
        auto accumulate = [&](auto mask_tag) {
          constexpr bool MASK = decltype(mask_tag)::value;
          const int nmin = MASK ? (j0 + t * 128 + r - 64 * b) * G - (sub * NSUB + col0) : 0;
#pragma unroll
          for (int c = 0; c < NLD; ++c) {
#pragma unroll
            for (int e4 = 0; e4 < 8; ++e4) {
              const float4 nl = nl4[c * 8 + e4];  // broadcast read
              const uint64_t a01 = f2_fma(
                  f2_pack(__uint_as_float(sr[c][4 * e4]), __uint_as_float(sr[c][4 * e4 + 1])), c2t,
                  f2_pack(nl.x, nl.y));
              const uint64_t a23 = f2_fma(
                  f2_pack(__uint_as_float(sr[c][4 * e4 + 2]), __uint_as_float(sr[c][4 * e4 + 3])), c2t,
                  f2_pack(nl.z, nl.w));
              // 2 of every 8 columns take the FMA-pipe exponential (exp2_fma3,
              // relative error 7.5e-5): measured fastest at this share
              float x0, x1, x2, x3;
              f2_unpack(a01, x0, x1);
              f2_unpack(a23, x2, x3);
              float y0 = ((e4 & 1) == 0) ? exp2_fma3(x0) : ex2_approx(x0);
              float y1 = ex2_approx(x1);
              float y2 = ((e4 & 1) == 1) ? exp2_fma3(x2) : ex2_approx(x2);
              float y3 = ex2_approx(x3);
              if (MASK) {
                const int n0 = c * 32 + 4 * e4;
                y0 = (n0 >= nmin) ? y0 : 0.f;
                y1 = (n0 + 1 >= nmin) ? y1 : 0.f;
                y2 = (n0 + 2 >= nmin) ? y2 : 0.f;
                y3 = (n0 + 3 >= nmin) ? y3 : 0.f;
              }
              acc2[0] = f2_add(acc2[0], f2_pack(y0, y1));
              acc2[1] = f2_add(acc2[1], f2_pack(y2, y3));
            }
          }
        };
        if (p.visible && j0 + t * 128 + 127 >= 64 * b)
          accumulate(std::true_type{});
        else
          accumulate(std::false_type{});
      }
      if (!ok) break;
      // Groups 2..IMP_GROUPS hand their partial sums to group 1 through a
      // double-buffered shared array guarded by mbarriers (bounded waits: no
      // CTA barrier inside the loop, so an aborted role never strands others).
      float m0, m1, m2, m3;
      f2_unpack(acc2[0], m0, m1);
      f2_unpack(acc2[1], m2, m3);
      const float mine = (m0 + m1) + (m2 + m3);
      const int pb = t & 1;
      if (grp > 0) {
        if (t >= 2 && !mbar_wait(&bars->part_empty[pb], ((t >> 1) - 1) & 1, p.limit_ns, abort_flag, 222)) {
          ok = false;
          break;
        }
        part[((grp - 1) * 2 + pb) * 128 + r] = mine;
        mbar_arrive(&bars->part_full[pb]);
      } else {
        if (!mbar_wait(&bars->part_full[pb], (t >> 1) & 1, p.limit_ns, abort_flag, 223)) {
          ok = false;
          break;
        }
        float total = mine;
#pragma unroll
        for (int q = 0; q < IMP_GROUPS - 1; ++q) total += part[(q * 2 + pb) * 128 + r];
        mbar_arrive(&bars->part_empty[pb]);
        const int j = j0 + t * 128 + r;
        if (j < n_c) out[j] = total;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace hs2
