// Decode-step sparse attention: a few query tokens at arbitrary positions t,
// each attending to the index list of the block that holds t over the shared
// K/V cache, with the causal mask j <= t.  (HySparse2 architecture summary,
// KV-sharing paragraph: the sparse layers reuse the full layer's KV cache and
// token selection; with early exit they mostly run at decode.)
//
// The work is a gather: per (query, KV head) at most k + w listed rows of K
// and V (256 B each in bf16, 128 B as e4m3) shared by the G <= 8 query heads
// of the group.  Its two products are 16 x 64 x 128 per 64 listed keys (the
// G heads padded to 16 rows), below tcgen05's 64-row minimum, and at
// 4 MAC per gathered byte too much work for the FMA pipes to keep up with
// HBM; so each warp runs them as warp-level m16n8k16 MMAs from registers:
//
//   grid   = (splits, Hkv, n); a CTA takes a contiguous range of the list in
//            chunks of 64 entries, two chunks in flight (16-byte cp.async
//            into rows padded to avoid bank conflicts; rows a query cannot
//            see are zero-filled, never read); list entries are read one
//            chunk ahead, off the critical path;
//   warp w = keys 16w .. 16w+15 of every chunk: S = Q K^T (2 n-tiles x 8
//            k-steps), its own online softmax in registers (log2 domain),
//            O += P V (16 n-tiles, P straight from the S accumulators);
//   merge  = the 4 warps' (m, l, O) in shared memory, then either the
//            normalised bf16 output (one split) or a partial per split; the
//            last CTA of a (query, KV head) to finish -- one atomic ticket,
//            no waiting -- merges the partials in split order, so the result
//            does not depend on which CTA finishes last.
//
// With an e4m3 cache the MMAs run on f16: codes convert exactly to f16, Q is
// rounded bf16 -> f16, the K scale (times log2(e)/sqrt(d)) multiplies the
// score columns in fp32 and the V scale multiplies P before it is rounded to
// f16 (the softmax sum uses the unscaled P).
#pragma once

#include "common.cuh"

namespace hs2 {

constexpr int DEC_THREADS = 128;
constexpr int DEC_CHUNK = 64;
constexpr int DEC_MAX_G = 8;
constexpr int DEC_MAX_SPLITS = 64;

struct DecodeParams {
  const __nv_bfloat16* q;  // [n][Hq][128], element strides q_tok / q_head
  int64_t q_tok, q_head;
  const int32_t* pos;      // [n] query positions
  const uint8_t* k;        // bf16 rows or e4m3 codes, element strides kv_tok / kv_head
  const uint8_t* v;
  const float* ksc;        // [L][Hkv] (e4m3 only)
  const float* vsc;
  int64_t kv_tok, kv_head;
  const int32_t* idx;      // [Hkv][nb][list_len]
  const int32_t* cnt;      // [Hkv][nb]
  __nv_bfloat16* o;        // [n][Hq][128], strides o_tok / o_head
  int64_t o_tok, o_head;
  float* part_o;           // [n][Hkv][splits][G][128]   (splits > 1)
  float* part_ml;          // [n][Hkv][splits][G][2]
  unsigned* ticket;        // [n][Hkv], zero at launch
  int L, Hkv, G, nb, list_len, block;
  int splits, chunks_per_split;
  float scale_log2;
};

template <bool KV8>
struct DecSmem {
  static constexpr int ROW = KV8 ? 128 : 256;  // bytes of one cached row
  static constexpr int PITCH = ROW + 16;       // padded: 8 consecutive rows hit 8 distinct bank groups
  static constexpr int TILE = DEC_CHUNK * PITCH;
  static constexpr int K_OFF = 0;                       // [2 stages][64][PITCH]
  static constexpr int V_OFF = 2 * TILE;                // [2 stages][64][PITCH]
  static constexpr int POS_OFF = 4 * TILE;              // int [2][64]: position, or -1 if not visible
  static constexpr int KS_OFF = POS_OFF + 2 * DEC_CHUNK * 4;  // float [2][64] (e4m3)
  static constexpr int VS_OFF = KS_OFF + 2 * DEC_CHUNK * 4;   // float [2][64] (e4m3)
  static constexpr int FLAG_OFF = VS_OFF + 2 * DEC_CHUNK * 4;
  static constexpr int BYTES = FLAG_OFF + 16;
  // after the main loop the stage buffers are reused for the merges
  static constexpr int MRG_O = 0;                                    // float [4][G][128]
  static constexpr int MRG_ML = MRG_O + 4 * DEC_MAX_G * 128 * 4;     // float [4][G][2]
  static constexpr int SPL_ML = MRG_ML + 4 * DEC_MAX_G * 2 * 4;      // float [splits][G][2]
  static constexpr int SPL_W = SPL_ML + DEC_MAX_SPLITS * DEC_MAX_G * 2 * 4;  // float [splits][G]
  static constexpr int SPL_L = SPL_W + DEC_MAX_SPLITS * DEC_MAX_G * 4;       // float [G]
  static constexpr int MERGE_END = SPL_L + DEC_MAX_G * 4;
  static_assert(MERGE_END <= 4 * TILE, "merge scratch fits in the stage buffers");
};

__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// D[16x8] += A[16x16] B[16x8].  A's rows 8..15 are zero here, so only its
// first and third registers (row gq; columns 2tq.. and 8+2tq..) are passed.
template <bool F16>
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  if (F16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
  }
}

__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t lds_u8(uint32_t addr) {
  unsigned short v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}

template <bool KV8>
__global__ void __launch_bounds__(DEC_THREADS, 3) sparse_decode_kernel(const DecodeParams p) {
  using SM = DecSmem<KV8>;
  extern __shared__ __align__(128) uint8_t dsm[];
  int* pos_s = reinterpret_cast<int*>(dsm + SM::POS_OFF);
  float* ks_s = reinterpret_cast<float*>(dsm + SM::KS_OFF);
  float* vs_s = reinterpret_cast<float*>(dsm + SM::VS_OFF);
  int* flag_s = reinterpret_cast<int*>(dsm + SM::FLAG_OFF);
  const uint32_t base = smem_u32(dsm);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, tq = lane & 3;  // fragment row / column pair
  const int split = blockIdx.x, g = blockIdx.y, r = blockIdx.z;
  const int G = p.G;

  // ---- the query's block and the list range of this split
  int t = p.pos[r];
  const bool t_ok = t >= 0 && t < p.L;
  if (!t_ok) {
    if (tid == 0 && split == 0 && g == 0) report(HS2_ERR_INDEX, 201);
    t = 0;
  }
  const int b = t / p.block;
  const int e_b = min(p.L, p.block * (b + 1));
  int c_all = p.cnt[static_cast<int64_t>(g) * p.nb + b];
  if (c_all < 0 || c_all > p.list_len) {
    if (tid == 0) report(HS2_ERR_INDEX, 202);
    c_all = max(0, min(c_all, p.list_len));
  }
  if (!t_ok) c_all = 0;
  const int32_t* list = p.idx + (static_cast<int64_t>(g) * p.nb + b) * p.list_len;
  const int e_lo = split * p.chunks_per_split * DEC_CHUNK;
  const int e_hi = min(c_all, e_lo + p.chunks_per_split * DEC_CHUNK);
  const int nchunks = e_hi > e_lo ? (e_hi - e_lo + DEC_CHUNK - 1) / DEC_CHUNK : 0;

  // ---- Q as A fragments (rows = the group's heads; rows >= G are zero)
  uint32_t qa[8][2];
  {
    const bool live = gq < G;
    const __nv_bfloat16* qr =
        p.q + static_cast<int64_t>(r) * p.q_tok + static_cast<int64_t>(g * G + (live ? gq : 0)) * p.q_head;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
      for (int hlf = 0; hlf < 2; ++hlf) {
        uint32_t w = live ? *reinterpret_cast<const uint32_t*>(qr + 16 * ks + 8 * hlf + 2 * tq) : 0u;
        if (KV8) {
          const uint32_t h = pack_f16x2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
          if (f16_overflowed(w, h)) report(HS2_ERR_RANGE, 399);
          w = h;
        }
        qa[ks][hlf] = w;
      }
    }
  }

  // ---- gather role: 16-byte chunks, CPR per row, RPI rows per instruction
  constexpr int CPR = SM::ROW / 16;
  constexpr int RPI = DEC_THREADS / CPR;
  constexpr int NR = DEC_CHUNK / RPI;  // rows each thread copies per chunk
  const int my_chunk = tid % CPR, my_row0 = tid / CPR;
  const int64_t rb_tok = p.kv_tok * (KV8 ? 1 : 2), rb_head = p.kv_head * (KV8 ? 1 : 2);
  const uint8_t* kg = p.k + static_cast<int64_t>(g) * rb_head + my_chunk * 16;
  const uint8_t* vg = p.v + static_cast<int64_t>(g) * rb_head + my_chunk * 16;
  int ent[NR];  // list entries of the next chunk to issue
  auto fetch = [&](int c) {
#pragma unroll
    for (int i = 0; i < NR; ++i) {
      const int e = e_lo + c * DEC_CHUNK + my_row0 + RPI * i;
      ent[i] = (c < nchunks && e < e_hi) ? __ldg(list + e) : -1;
    }
  };
  auto issue = [&](int c) {
    const int st = c & 1;
#pragma unroll
    for (int i = 0; i < NR; ++i) {
      const int row = my_row0 + RPI * i;
      const int e = e_lo + c * DEC_CHUNK + row;
      const int pj = ent[i];
      const bool listed = e < e_hi;
      const bool in_range = pj >= 0 && pj < e_b;
      if (listed && !in_range) report(HS2_ERR_INDEX, 203);
      const bool vis = listed && in_range && pj <= t;
      const int64_t off = static_cast<int64_t>(vis ? pj : 0) * rb_tok;
      const uint32_t dst = st * SM::TILE + row * SM::PITCH + my_chunk * 16;
      cp_async_16(base + SM::K_OFF + dst, kg + off, vis ? 16u : 0u);
      cp_async_16(base + SM::V_OFF + dst, vg + off, vis ? 16u : 0u);
      if (my_chunk == 0) {
        pos_s[st * DEC_CHUNK + row] = vis ? pj : -1;
        if (KV8) {
          const int64_t si = static_cast<int64_t>(vis ? pj : 0) * p.Hkv + g;
          cp_async_4(smem_u32(ks_s + st * DEC_CHUNK + row), p.ksc + si, vis ? 4u : 0u);
          cp_async_4(smem_u32(vs_s + st * DEC_CHUNK + row), p.vsc + si, vis ? 4u : 0u);
        }
      }
    }
    cp_async_commit();
  };

  // ---- per-warp softmax state (row gq) and O fragments
  float m_run = -INFINITY, l_run = 0.f;
  float o[16][4];
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
  const float sc = p.scale_log2;
  const int kw0 = warp * 16;  // this warp's keys within a chunk

  if (nchunks > 0) {
    fetch(0);
    issue(0);
    fetch(1);
  }
  for (int c = 0; c < nchunks; ++c) {
    const int st = c & 1;
    if (c + 1 < nchunks) {
      issue(c + 1);
      fetch(c + 2);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint32_t kt = base + SM::K_OFF + st * SM::TILE, vt = base + SM::V_OFF + st * SM::TILE;

    // ---- S = Q K^T for keys kw0 .. kw0+15 (n-tiles 0, 1)
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    if (KV8) {
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const uint32_t ra = kt + (kw0 + nt * 8 + gq) * SM::PITCH + 16 * ks + 2 * tq;
          const uint32_t b0 = e4m3x2_to_f16x2(lds_u16(ra)), b1 = e4m3x2_to_f16x2(lds_u16(ra + 8));
          mma16816<true>(s[nt], qa[ks][0], qa[ks][1], b0, b1);
        }
      }
    } else {
      const int mat = lane >> 3, mrow = lane & 7;
      const uint32_t ra = kt + (kw0 + mrow + (mat >> 1) * 8) * SM::PITCH + (mat & 1) * 16;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t bb[4];
        ldsm_x4(ra + ks * 32, bb);
        mma16816<false>(s[0], qa[ks][0], qa[ks][1], bb[0], bb[1]);
        mma16816<false>(s[1], qa[ks][0], qa[ks][1], bb[2], bb[3]);
      }
    }
    // ---- mask, scale, online softmax of row gq over the warp's 16 keys
    float mx = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int key = kw0 + nt * 8 + 2 * tq + e;
        const bool vis = pos_s[st * DEC_CHUNK + key] >= 0;
        const float f = KV8 ? ks_s[st * DEC_CHUNK + key] * sc : sc;
        s[nt][e] = vis ? s[nt][e] * f : -INFINITY;
        mx = fmaxf(mx, s[nt][e]);
      }
    }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m_run, mx);
    const float mu = (m_new == -INFINITY) ? 0.f : m_new;
    const float alpha = (m_new == -INFINITY) ? 1.f : ex2_approx(m_run - m_new);
    m_run = m_new;
    float pr[2][2];
    float psum = 0.f;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        pr[nt][e] = ex2_approx(s[nt][e] - mu);
        psum += pr[nt][e];
      }
    }
    l_run = l_run * alpha + psum;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      o[nt][0] *= alpha;
      o[nt][1] *= alpha;
    }
    // ---- P as the A fragment (keys 2tq.., 8+2tq..), then O += P V
    uint32_t pa0, pa2;
    if (KV8) {
      const float* vs = vs_s + st * DEC_CHUNK + kw0 + 2 * tq;
      pa0 = pack_f16x2(pr[0][0] * vs[0], pr[0][1] * vs[1]);
      pa2 = pack_f16x2(pr[1][0] * vs[8], pr[1][1] * vs[9]);
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        const uint32_t ca = vt + (kw0 + 2 * tq) * SM::PITCH + nt * 8 + gq;
        const uint32_t lo0 = lds_u8(ca), hi0 = lds_u8(ca + SM::PITCH);
        const uint32_t lo1 = lds_u8(ca + 8 * SM::PITCH), hi1 = lds_u8(ca + 9 * SM::PITCH);
        const uint32_t b0 = e4m3x2_to_f16x2(lo0 | (hi0 << 8)), b1 = e4m3x2_to_f16x2(lo1 | (hi1 << 8));
        mma16816<true>(o[nt], pa0, pa2, b0, b1);
      }
    } else {
      pa0 = pack_bf16x2(pr[0][0], pr[0][1]);
      pa2 = pack_bf16x2(pr[1][0], pr[1][1]);
      const int mat = lane >> 3, mrow = lane & 7;
      const uint32_t ra = vt + (kw0 + mrow + (mat & 1) * 8) * SM::PITCH + (mat >> 1) * 16;
#pragma unroll
      for (int pp = 0; pp < 8; ++pp) {
        uint32_t bb[4];
        ldsm_x4_t(ra + pp * 32, bb);
        mma16816<false>(o[2 * pp], pa0, pa2, bb[0], bb[1]);
        mma16816<false>(o[2 * pp + 1], pa0, pa2, bb[2], bb[3]);
      }
    }
    __syncthreads();  // stage st is refilled by the next iteration's issue
  }

  // ---- merge the 4 warps (stage buffers are free now)
  float* mrg_o = reinterpret_cast<float*>(dsm + SM::MRG_O);
  float* mrg_ml = reinterpret_cast<float*>(dsm + SM::MRG_ML);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  if (gq < G) {
#pragma unroll
    for (int nt = 0; nt < 16; ++nt)
      *reinterpret_cast<float2*>(mrg_o + (warp * DEC_MAX_G + gq) * 128 + nt * 8 + 2 * tq) =
          make_float2(o[nt][0], o[nt][1]);
    if (tq == 0) {
      mrg_ml[(warp * DEC_MAX_G + gq) * 2] = m_run;
      mrg_ml[(warp * DEC_MAX_G + gq) * 2 + 1] = l_run;
    }
  }
  __syncthreads();
  float acc[DEC_MAX_G], mh[DEC_MAX_G], lh[DEC_MAX_G];
#pragma unroll
  for (int h = 0; h < DEC_MAX_G; ++h) {
    acc[h] = 0.f;
    mh[h] = -INFINITY;
    lh[h] = 0.f;
    if (h < G) {
#pragma unroll
      for (int w = 0; w < 4; ++w) mh[h] = fmaxf(mh[h], mrg_ml[(w * DEC_MAX_G + h) * 2]);
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float mw = mrg_ml[(w * DEC_MAX_G + h) * 2];
        const float wt = (mw == -INFINITY) ? 0.f : ex2_approx(mw - mh[h]);
        lh[h] = fmaf(mrg_ml[(w * DEC_MAX_G + h) * 2 + 1], wt, lh[h]);
        acc[h] = fmaf(mrg_o[(w * DEC_MAX_G + h) * 128 + tid], wt, acc[h]);
      }
    }
  }

  const int64_t og = static_cast<int64_t>(r) * p.o_tok;
  if (p.splits == 1) {
#pragma unroll
    for (int h = 0; h < DEC_MAX_G; ++h)
      if (h < G)
        p.o[og + static_cast<int64_t>(g * G + h) * p.o_head + tid] =
            __float2bfloat16(lh[h] > 0.f ? acc[h] / lh[h] : 0.f);
    return;
  }

  // ---- several splits: publish this split's partial; the last CTA merges
  const int64_t unit = static_cast<int64_t>(r) * p.Hkv + g;
  const int64_t slot = unit * p.splits + split;
#pragma unroll
  for (int h = 0; h < DEC_MAX_G; ++h)
    if (h < G) p.part_o[(slot * G + h) * 128 + tid] = acc[h];
  if (tid == 0) {  // (m, l) are the same in every thread
#pragma unroll
    for (int h = 0; h < DEC_MAX_G; ++h) {
      if (h < G) {
        p.part_ml[(slot * G + h) * 2] = mh[h];
        p.part_ml[(slot * G + h) * 2 + 1] = lh[h];
      }
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) flag_s[0] = (atomicAdd(p.ticket + unit, 1u) == static_cast<unsigned>(p.splits - 1)) ? 1 : 0;
  __syncthreads();
  if (!flag_s[0]) return;
  __threadfence();
  float* spl_ml = reinterpret_cast<float*>(dsm + SM::SPL_ML);
  float* spl_w = reinterpret_cast<float*>(dsm + SM::SPL_W);
  float* spl_l = reinterpret_cast<float*>(dsm + SM::SPL_L);
  const int nml = p.splits * G * 2;
  for (int i = tid; i < nml; i += DEC_THREADS) spl_ml[i] = __ldcg(p.part_ml + unit * p.splits * G * 2 + i);
  __syncthreads();
  if (tid < G) {  // per head: the largest split max, the weighted sum in split order
    float M = -INFINITY;
    for (int s2 = 0; s2 < p.splits; ++s2) M = fmaxf(M, spl_ml[(s2 * G + tid) * 2]);
    float Ls = 0.f;
    for (int s2 = 0; s2 < p.splits; ++s2) {
      const float ms = spl_ml[(s2 * G + tid) * 2];
      const float w = (ms == -INFINITY) ? 0.f : ex2_approx(ms - M);
      spl_w[s2 * G + tid] = w;
      Ls = fmaf(spl_ml[(s2 * G + tid) * 2 + 1], w, Ls);
    }
    spl_l[tid] = Ls;
  }
  __syncthreads();
  float out[DEC_MAX_G];
#pragma unroll
  for (int h = 0; h < DEC_MAX_G; ++h) out[h] = 0.f;
  const float* po = p.part_o + unit * p.splits * G * 128 + tid;
#pragma unroll 2
  for (int s2 = 0; s2 < p.splits; ++s2) {
#pragma unroll
    for (int h = 0; h < DEC_MAX_G; ++h)
      if (h < G) out[h] = fmaf(__ldcg(po + (s2 * G + h) * 128), spl_w[s2 * G + h], out[h]);
  }
#pragma unroll
  for (int h = 0; h < DEC_MAX_G; ++h)
    if (h < G)
      p.o[og + static_cast<int64_t>(g * G + h) * p.o_head + tid] =
          __float2bfloat16(spl_l[h] > 0.f ? out[h] / spl_l[h] : 0.f);
}

}  // namespace hs2
