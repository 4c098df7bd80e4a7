// libhs2: host side of the C ABI declared in include/hs2.h, plus the single
// translation unit that instantiates every sm_100a kernel.
//
// Host responsibilities: argument validation (nothing is launched when a
// check fails), TMA tensor-map encoding, the strip schedule of the importance
// and select passes, launches on the caller's stream, and the device status
// word read back by hs2_sync.  No device memory is ever allocated here.
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/hs2.h"
#include "common.cuh"
#include "flash.cuh"
#include "flash2.cuh"
#include "sparse_attn.cuh"
#include "importance.cuh"
#include "topk_select.cuh"
#include "quantize.cuh"
#include "decode.cuh"

namespace hs2 {
namespace {

uint64_t g_wait_limit_ns = 2000000000ull;
uint32_t g_flags = 0;
std::atomic<uint64_t> g_launches{0};

inline int cuda_ok(cudaError_t e) { return e == cudaSuccess ? HS2_OK : HS2_ERR_CUDA; }

// NVTX range around each kernel's launch (and each composite call), so that a
// profiler can attribute and filter launches by name; free when no tool is
// attached.
struct Range {
  explicit Range(const char* name) { nvtxRangePushA(name); }
  ~Range() { nvtxRangePop(); }
  Range(const Range&) = delete;
  Range& operator=(const Range&) = delete;
};

// Test hook (hs2_debug_set bit 3): every TMA descriptor encoding reports a
// failure, as a driver error would, so that tests can check that a call
// fails with HS2_ERR_CUDA before launching anything.
constexpr uint32_t FLAG_FAIL_TMAP = 8u;

inline int launched() {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return HS2_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return HS2_OK;
}

// ------------------------------------------------------------ validation --

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

int check_shape(const hs2_shape* s) {
  if (!s) return HS2_ERR_INVALID_ARG;
  if (s->L <= 0 || s->Hq <= 0 || s->Hkv <= 0 || s->d <= 0 || s->block <= 0 || s->topk <= 0 || s->recent <= 0)
    return HS2_ERR_INVALID_ARG;
  if (s->Hq % s->Hkv != 0) return HS2_ERR_INVALID_ARG;
  if (s->kv_dtype != HS2_KV_BF16 && s->kv_dtype != HS2_KV_E4M3) return HS2_ERR_INVALID_ARG;
  if (s->q_tok_stride <= 0 || s->q_head_stride <= 0 || s->kv_tok_stride <= 0 || s->kv_head_stride <= 0)
    return HS2_ERR_INVALID_ARG;
  const int G = s->Hq / s->Hkv;
  if (s->d != HD || s->block != 64) return HS2_ERR_UNSUPPORTED;
  if (s->L % 64 != 0 || s->L > (1 << 24)) return HS2_ERR_UNSUPPORTED;
  if (s->recent % 64 != 0 || s->recent < s->block) return HS2_ERR_UNSUPPORTED;
  if (s->topk + s->recent > MAX_LIST) return HS2_ERR_UNSUPPORTED;
  if (G != 2 && G != 4 && G != 8) return HS2_ERR_UNSUPPORTED;
  if (s->q_tok_stride % 8 || s->q_head_stride % 8) return HS2_ERR_UNSUPPORTED;
  const int64_t kv_align = (s->kv_dtype == HS2_KV_E4M3) ? 16 : 8;
  if (s->kv_tok_stride % kv_align || s->kv_head_stride % kv_align) return HS2_ERR_UNSUPPORTED;
  // rows must not overlap: d contiguous elements per head, heads within a token
  if (s->q_head_stride < HD || s->kv_head_stride < HD) return HS2_ERR_UNSUPPORTED;
  if (s->q_tok_stride < static_cast<int64_t>(s->Hq) * s->q_head_stride) return HS2_ERR_UNSUPPORTED;
  if (s->kv_tok_stride < static_cast<int64_t>(s->Hkv) * s->kv_head_stride) return HS2_ERR_UNSUPPORTED;
  return HS2_OK;
}

int check_kv(const hs2_shape* s, const void* k, const void* v, const float* ks, const float* vs) {
  if (!k || !v) return HS2_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v)) return HS2_ERR_UNSUPPORTED;
  if (s->kv_dtype == HS2_KV_E4M3 && (!ks || !vs)) return HS2_ERR_INVALID_ARG;
  return HS2_OK;
}

// --------------------------------------------------------- tensor maps --

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 3-D bf16 map over [tokens][heads][128] with the d dimension contiguous and
// a box of (64 d, box_h heads, box_t tokens), 128-byte swizzle.
int make_map(CUtensorMap* m, const void* base, int L, int H, int64_t tok_stride, int64_t head_stride, int box_h,
             int box_t) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || (g_flags & FLAG_FAIL_TMAP)) return HS2_ERR_CUDA;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(HD), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(L)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_stride) * 2, static_cast<cuuint64_t>(tok_stride) * 2};
  const cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(box_h), static_cast<cuuint32_t>(box_t)};
  const cuuint32_t es[3] = {1u, 1u, 1u};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? HS2_OK : HS2_ERR_CUDA;
}

// Streaming multiprocessors of the current device (queried once per process).
int sm_count() {
  static int n = [] {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return 148;
    return v > 0 ? v : 148;
  }();
  return n;
}

float scale_log2(int d) { return static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(d))); }

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current
// device, once per (kernel, device): the attribute is per device, so a
// process that drives several GPUs sets it on each.
template <typename K>
int set_smem(K kernel, uint32_t bytes) {
  struct Done {
    const void* fn;
    int dev;
    uint32_t bytes;
  };
  static std::mutex mu;
  static Done done[256];
  static int n_done = 0;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return HS2_ERR_CUDA;
  const void* fn = reinterpret_cast<const void*>(kernel);
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < n_done; ++i)
    if (done[i].fn == fn && done[i].dev == dev && done[i].bytes >= bytes) return HS2_OK;
  if (int rc = cuda_ok(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            static_cast<int>(bytes))))
    return rc;
  if (n_done < 256) done[n_done++] = Done{fn, dev, bytes};
  return HS2_OK;
}

// ------------------------------------------------------------- launches --

// The f16 copy of an e4m3 cache made once per layer by dequant_kv_kernel
// (inside a caller workspace): K and V [L][Hkv][128] f16, K column scales
// [Hkv][Lp].
struct DequantBuf {
  uint16_t* kf;
  uint16_t* vf;
  float* kcol;
  int Lp;
};

int kcol_stride(const hs2_shape* s) { return (s->L + 127) / 128 * 128; }

size_t dequant_bytes(const hs2_shape* s) {
  const size_t kv = static_cast<size_t>(s->L) * s->Hkv * HD * 2u;
  return 2 * kv + static_cast<size_t>(s->Hkv) * kcol_stride(s) * 4u + 3 * 256;
}

// Carves a DequantBuf from [base, base + dequant_bytes(s)).
DequantBuf dequant_carve(const hs2_shape* s, uint8_t* base) {
  auto up = [](uint8_t* x) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(x) + 255) & ~static_cast<uintptr_t>(255));
  };
  const size_t kv = static_cast<size_t>(s->L) * s->Hkv * HD * 2u;
  DequantBuf d{};
  uint8_t* x = up(base);
  d.kf = reinterpret_cast<uint16_t*>(x);
  x = up(x + kv);
  d.vf = reinterpret_cast<uint16_t*>(x);
  x = up(x + kv);
  d.kcol = reinterpret_cast<float*>(x);
  d.Lp = kcol_stride(s);
  return d;
}

int launch_dequant(const hs2_shape* s, const void* k, const void* v, const float* ks, const float* vs,
                   const DequantBuf& d, cudaStream_t st) {
  const Range range("hs2 dequant_kv");
  DequantParams p{};
  p.L = s->L;
  p.Hkv = s->Hkv;
  p.Lp = d.Lp;
  p.k8 = static_cast<const uint8_t*>(k);
  p.v8 = static_cast<const uint8_t*>(v);
  p.kv_tok = s->kv_tok_stride;
  p.kv_head = s->kv_head_stride;
  p.ksc = ks;
  p.vsc = vs;
  p.kf = d.kf;
  p.vf = d.vf;
  p.kcol = d.kcol;
  p.scale_log2 = scale_log2(s->d);
  const int64_t rows = static_cast<int64_t>(d.Lp) * s->Hkv;
  const int64_t blocks = std::min<int64_t>((rows + 31) / 32, static_cast<int64_t>(sm_count()) * 8);
  dequant_kv_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(p);
  return launched();
}

// Kernel (1).  dq: the layer's f16 copy of an e4m3 cache (KVM_F16), or null
// to read the cache itself (bf16 by TMA, or e4m3 converted in the kernel).
int launch_attn_fwd(const hs2_shape* s, const void* q, const void* k, const void* v, const float* ks,
                    const float* vs, void* o, float* lse, cudaStream_t st, const DequantBuf* dq = nullptr) {
  const Range range("hs2 attn_fwd (kernel 1)");
  const bool kv8 = s->kv_dtype == HS2_KV_E4M3;
  CUtensorMap mq, mk, mv;
  int rc;
  if ((rc = make_map(&mq, q, s->L, s->Hq, s->q_tok_stride, s->q_head_stride, 1, 128))) return rc;
  if (!kv8) {
    if ((rc = make_map(&mk, k, s->L, s->Hkv, s->kv_tok_stride, s->kv_head_stride, 1, 128))) return rc;
    if ((rc = make_map(&mv, v, s->L, s->Hkv, s->kv_tok_stride, s->kv_head_stride, 1, 128))) return rc;
  } else if (dq) {
    if ((rc = make_map(&mk, dq->kf, s->L, s->Hkv, int64_t(s->Hkv) * HD, HD, 1, 128))) return rc;
    if ((rc = make_map(&mv, dq->vf, s->L, s->Hkv, int64_t(s->Hkv) * HD, HD, 1, 128))) return rc;
  } else {
    mk = mq;
    mv = mq;
  }
  FlashParams p{};
  p.k8 = static_cast<const uint8_t*>(k);
  p.v8 = static_cast<const uint8_t*>(v);
  p.ksc = ks;
  p.vsc = vs;
  if (dq) {
    p.kcol = dq->kcol;
    p.kcol_stride = dq->Lp;
  }
  p.kv_tok = s->kv_tok_stride;
  p.kv_head = s->kv_head_stride;
  p.L = s->L;
  p.Hq = s->Hq;
  p.Hkv = s->Hkv;
  p.G = s->Hq / s->Hkv;
  p.nqt = s->L / 128 + (s->L % 128 ? 1 : 0);
  p.npairs = (p.nqt + 1) / 2;
  p.scale_log2 = scale_log2(s->d);
  p.o = static_cast<__nv_bfloat16*>(o);
  p.o_tok = s->q_tok_stride;
  p.o_head = s->q_head_stride;
  p.lse = lse;
  p.limit_ns = g_wait_limit_ns;
  p.flags = g_flags;
  if ((g_flags & FLAG_FA_CTA_PAIRS) && p.G % 2 == 0 && (!kv8 || dq)) {
    // CTA pairs: two heads of a group per cluster (check_shape admits G = 2,
    // 4, 8), K tiles loaded as 64-key halves
    CUtensorMap mk64;
    if (!kv8) {
      if ((rc = make_map(&mk64, k, s->L, s->Hkv, s->kv_tok_stride, s->kv_head_stride, 1, 64))) return rc;
    } else {
      if ((rc = make_map(&mk64, dq->kf, s->L, s->Hkv, int64_t(s->Hkv) * HD, HD, 1, 64))) return rc;
    }
    const unsigned grid2 = static_cast<unsigned>(p.npairs * s->Hq);
    if (kv8) {
      if (int rc_smem = set_smem(flash2_fwd_kernel<KVM_F16>, F2_SMEM)) return rc_smem;
      flash2_fwd_kernel<KVM_F16><<<grid2, FL_THREADS, F2_SMEM, st>>>(mq, mk64, mv, p);
    } else {
      if (int rc_smem = set_smem(flash2_fwd_kernel<KVM_BF16>, F2_SMEM)) return rc_smem;
      flash2_fwd_kernel<KVM_BF16><<<grid2, FL_THREADS, F2_SMEM, st>>>(mq, mk64, mv, p);
    }
    return launched();
  }
  const unsigned grid = static_cast<unsigned>(p.npairs * s->Hq);
  if (kv8 && dq) {
    if (int rc_smem = set_smem(flash_fwd_kernel<KVM_F16>, FL_SMEM_KV8)) return rc_smem;
    flash_fwd_kernel<KVM_F16><<<grid, FL_THREADS, FL_SMEM_KV8, st>>>(mq, mk, mv, p);
  } else if (kv8) {
    if (int rc_smem = set_smem(flash_fwd_kernel<KVM_E4M3>, FL_SMEM_KV8)) return rc_smem;
    flash_fwd_kernel<KVM_E4M3><<<grid, FL_THREADS, FL_SMEM_KV8, st>>>(mq, mk, mv, p);
  } else {
    if (int rc_smem = set_smem(flash_fwd_kernel<KVM_BF16>, FL_SMEM_DENSE)) return rc_smem;
    flash_fwd_kernel<KVM_BF16><<<grid, FL_THREADS, FL_SMEM_DENSE, st>>>(mq, mk, mv, p);
  }
  return launched();
}

// The persistent kernel (4): over index lists, or (window > 0) over each
// block's sliding windows, bf16 cache, optionally writing the LSE.
int launch_sparse(const hs2_shape* s, const void* q, const void* k, const void* v, const float* ks,
                  const float* vs, const int32_t* idx, const int32_t* cnt, void* o, cudaStream_t st, int window = 0,
                  float* lse = nullptr) {
  const Range range(window > 0 ? "hs2 swa_attn (kernel 4, window)" : "hs2 sparse_attn (kernel 4)");
  const int G = s->Hq / s->Hkv;
  const int rows_tok = 128 / G;
  CUtensorMap mq, mk, mv;
  int rc;
  if ((rc = make_map(&mq, q, s->L, s->Hq, s->q_tok_stride, s->q_head_stride, G, rows_tok))) return rc;
  mk = mq;
  mv = mq;
  if (window > 0) {
    if ((rc = make_map(&mk, k, s->L, s->Hkv, s->kv_tok_stride, s->kv_head_stride, 1, 128))) return rc;
    if ((rc = make_map(&mv, v, s->L, s->Hkv, s->kv_tok_stride, s->kv_head_stride, 1, 128))) return rc;
  }
  FlashParams p{};
  p.L = s->L;
  p.Hq = s->Hq;
  p.Hkv = s->Hkv;
  p.G = G;
  p.nb = s->L / 64;
  p.list_len = s->topk + s->recent;
  p.mtiles = (64 * G) / 128;
  p.mpairs = (p.mtiles + 1) / 2;
  p.rows_tok = rows_tok;
  p.scale_log2 = scale_log2(s->d);
  p.window = window;
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.k8 = static_cast<const uint8_t*>(k);
  p.v8 = static_cast<const uint8_t*>(v);
  p.ksc = ks;
  p.vsc = vs;
  p.kv_tok = s->kv_tok_stride;
  p.kv_head = s->kv_head_stride;
  p.idx = idx;
  p.cnt = cnt;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.o_tok = s->q_tok_stride;
  p.o_head = s->q_head_stride;
  p.lse = lse;
  p.limit_ns = g_wait_limit_ns;
  p.flags = g_flags;
  // persistent: one CTA per SM walks the (block, KV head, M-tile pair) items
  const int n_items = p.nb * s->Hkv * p.mpairs;
  const unsigned grid = static_cast<unsigned>(std::min(n_items, sm_count()));
  if (window > 0) {
    if (int rc_smem = set_smem(sparse_attn_kernel<false, true>, SP_SMEM)) return rc_smem;
    sparse_attn_kernel<false, true><<<grid, FL_THREADS, SP_SMEM, st>>>(mq, mk, mv, p, n_items);
  } else if (s->kv_dtype == HS2_KV_E4M3) {
    if (int rc_smem = set_smem(sparse_attn_kernel<true, false>, SP_SMEM_KV8)) return rc_smem;
    sparse_attn_kernel<true, false><<<grid, sp_threads(true, false), SP_SMEM_KV8, st>>>(mq, mk, mv, p, n_items);
  } else {
    if (int rc_smem = set_smem(sparse_attn_kernel<false, false>, SP_SMEM)) return rc_smem;
    sparse_attn_kernel<false, false><<<grid, sp_threads(false, false), SP_SMEM, st>>>(mq, mk, mv, p, n_items);
  }
  return launched();
}

// Decode: split each (query, KV head) list so that about three CTAs per SM
// are in flight even for a single query; a split covers whole 64-entry
// chunks, and no split is empty for a full list.
struct DecodePlan {
  int splits, chunks_per_split;
  size_t ticket_off, ml_off, part_off, ws_bytes;
};

DecodePlan decode_plan(const hs2_shape* s, int n) {
  const int list_len = s->topk + s->recent;
  const int chunks = (list_len + DEC_CHUNK - 1) / DEC_CHUNK;
  const int64_t units = static_cast<int64_t>(n) * s->Hkv;
  const int64_t target = 148 * 3;
  int splits = static_cast<int>(std::min<int64_t>(chunks, std::max<int64_t>(1, (target + units - 1) / units)));
  const int cps = (chunks + splits - 1) / splits;
  splits = (chunks + cps - 1) / cps;
  DecodePlan pl{splits, cps, 0, 0, 0, 0};
  if (splits > 1) {
    const int G = s->Hq / s->Hkv;
    auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    pl.ticket_off = 0;
    pl.ml_off = up(static_cast<size_t>(units) * 4);
    pl.part_off = pl.ml_off + up(static_cast<size_t>(units) * splits * G * 2 * 4);
    pl.ws_bytes = pl.part_off + static_cast<size_t>(units) * splits * G * 128 * 4;
  }
  return pl;
}

int launch_decode(const hs2_shape* s, const void* q, const int32_t* positions, int n, const void* k, const void* v,
                  const float* ks, const float* vs, const int32_t* idx, const int32_t* cnt, void* o, void* ws,
                  const DecodePlan& pl, cudaStream_t st) {
  const Range range("hs2 sparse_decode");
  DecodeParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.q_tok = s->q_tok_stride;
  p.q_head = s->q_head_stride;
  p.pos = positions;
  p.k = static_cast<const uint8_t*>(k);
  p.v = static_cast<const uint8_t*>(v);
  p.ksc = ks;
  p.vsc = vs;
  p.kv_tok = s->kv_tok_stride;
  p.kv_head = s->kv_head_stride;
  p.idx = idx;
  p.cnt = cnt;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.o_tok = s->q_tok_stride;
  p.o_head = s->q_head_stride;
  p.L = s->L;
  p.Hkv = s->Hkv;
  p.G = s->Hq / s->Hkv;
  p.nb = s->L / 64;
  p.list_len = s->topk + s->recent;
  p.block = s->block;
  p.splits = pl.splits;
  p.chunks_per_split = pl.chunks_per_split;
  p.scale_log2 = scale_log2(s->d);
  if (pl.splits > 1) {
    uint8_t* w = static_cast<uint8_t*>(ws);
    p.ticket = reinterpret_cast<unsigned*>(w + pl.ticket_off);
    p.part_ml = reinterpret_cast<float*>(w + pl.ml_off);
    p.part_o = reinterpret_cast<float*>(w + pl.part_off);
    if (int rc = cuda_ok(cudaMemsetAsync(p.ticket, 0, static_cast<size_t>(n) * s->Hkv * 4, st))) return rc;
  }
  const dim3 grid(static_cast<unsigned>(pl.splits), static_cast<unsigned>(s->Hkv), static_cast<unsigned>(n));
  if (s->kv_dtype == HS2_KV_E4M3) {
    if (int rc_smem = set_smem(sparse_decode_kernel<true>, DecSmem<true>::BYTES)) return rc_smem;
    sparse_decode_kernel<true><<<grid, DEC_THREADS, DecSmem<true>::BYTES, st>>>(p);
  } else {
    if (int rc_smem = set_smem(sparse_decode_kernel<false>, DecSmem<false>::BYTES)) return rc_smem;
    sparse_decode_kernel<false><<<grid, DEC_THREADS, DecSmem<false>::BYTES, st>>>(p);
  }
  return launched();
}

int n_cand(const hs2_shape* s, int b) { return std::max(0, std::min(s->L, 64 * (b + 1)) - s->recent); }

template <int G, int KVM>
int launch_importance_g(const CUtensorMap& mq, const CUtensorMap& mk, const ImpParams& p, dim3 grid,
                        cudaStream_t st) {
  if (int rc_smem = set_smem(importance_kernel<G, KVM>, imp_smem_bytes(G))) return rc_smem;
  importance_kernel<G, KVM><<<grid, IMP_THREADS, imp_smem_bytes(G), st>>>(mq, mk, p);
  return launched();
}

// Kernel (2) for blocks [b0, b1).  dq as in launch_attn_fwd.
int launch_importance(const hs2_shape* s, const void* q, const void* k, const float* ks, const float* lse, int b0,
                      int b1, float* imp, int64_t row_stride, int skip_le, cudaStream_t st,
                      const DequantBuf* dq = nullptr, bool visible = false) {
  const Range range("hs2 importance (kernel 2)");
  const bool kv8 = s->kv_dtype == HS2_KV_E4M3;
  const int G = s->Hq / s->Hkv;
  const int longest = visible ? std::min(s->L, 64 * b1) : n_cand(s, b1 - 1);
  if (longest <= 0 || longest <= skip_le) return HS2_OK;
  CUtensorMap mq, mk;
  int rc;
  if ((rc = make_map(&mq, q, s->L, s->Hq, s->q_tok_stride, s->q_head_stride, G, 64))) return rc;
  if (!kv8) {
    if ((rc = make_map(&mk, k, s->L, s->Hkv, s->kv_tok_stride, s->kv_head_stride, 1, 128))) return rc;
  } else if (dq) {
    if ((rc = make_map(&mk, dq->kf, s->L, s->Hkv, int64_t(s->Hkv) * HD, HD, 1, 128))) return rc;
  } else {
    mk = mq;
  }
  ImpParams p{};
  p.k8 = static_cast<const uint8_t*>(k);
  p.ksc = ks;
  p.kv_tok = s->kv_tok_stride;
  p.kv_head = s->kv_head_stride;
  p.L = s->L;
  p.Hq = s->Hq;
  p.Hkv = s->Hkv;
  p.G = G;
  p.recent = s->recent;
  p.b0 = b0;
  p.nbs = b1 - b0;
  p.skip_le = skip_le;
  p.visible = visible ? 1 : 0;
  p.scale_log2 = scale_log2(s->d);
  p.lse = lse;
  p.imp = imp;
  p.row_stride = row_stride;
  p.limit_ns = g_wait_limit_ns;
  p.flags = g_flags;
  const dim3 grid(static_cast<unsigned>((longest + IMP_CK - 1) / IMP_CK), static_cast<unsigned>(s->Hkv * (b1 - b0)));
  const int kvm = !kv8 ? KVM_BF16 : (dq ? KVM_F16 : KVM_E4M3);
  switch (G * 4 + kvm) {
    case 8: return launch_importance_g<2, KVM_BF16>(mq, mk, p, grid, st);
    case 9: return launch_importance_g<2, KVM_E4M3>(mq, mk, p, grid, st);
    case 10: return launch_importance_g<2, KVM_F16>(mq, mk, p, grid, st);
    case 16: return launch_importance_g<4, KVM_BF16>(mq, mk, p, grid, st);
    case 17: return launch_importance_g<4, KVM_E4M3>(mq, mk, p, grid, st);
    case 18: return launch_importance_g<4, KVM_F16>(mq, mk, p, grid, st);
    case 32: return launch_importance_g<8, KVM_BF16>(mq, mk, p, grid, st);
    case 33: return launch_importance_g<8, KVM_E4M3>(mq, mk, p, grid, st);
    case 34: return launch_importance_g<8, KVM_F16>(mq, mk, p, grid, st);
    default: return HS2_ERR_UNSUPPORTED;
  }
}

// Pooled block values of one row live in shared memory: L / 64 * 4 bytes,
// at most 64 KiB, so block-level selection covers L <= 2^20.
constexpr uint32_t kBlockSelectSmem = 64u * 1024u;

int launch_select(const hs2_shape* s, const float* imp, int64_t row_stride, int b0, int b1, int32_t* idx,
                  int32_t* cnt, cudaStream_t st, bool blocks = false) {
  const Range range(blocks ? "hs2 block_select" : "hs2 topk_select (kernel 3)");
  SelParams p{};
  p.L = s->L;
  p.Hkv = s->Hkv;
  p.nb = s->L / 64;
  p.recent = s->recent;
  p.topk = s->topk;
  p.b0 = b0;
  p.nbs = b1 - b0;
  p.list_len = s->topk + s->recent;
  p.imp = imp;
  p.row_stride = row_stride;
  p.idx = idx;
  p.cnt = cnt;
  const unsigned grid = static_cast<unsigned>(s->Hkv * (b1 - b0));
  if (blocks) {
    const uint32_t dyn = static_cast<uint32_t>(s->L / 64) * 4u;  // pooled values of the longest row
    if (dyn > kBlockSelectSmem) return HS2_ERR_UNSUPPORTED;
    if (int rc_smem = set_smem(block_select_kernel, kBlockSelectSmem)) return rc_smem;
    block_select_kernel<<<grid, SEL_THREADS, dyn, st>>>(p);
  } else {
    if (int rc_smem = set_smem(topk_select_kernel, sizeof(SelSmem))) return rc_smem;
    topk_select_kernel<<<grid, SEL_THREADS, sizeof(SelSmem), st>>>(p);
  }
  return launched();
}

__global__ void exp2_check_kernel(const float* x, float* y0, float* y3, float* y4, int64_t n) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float v = x[i];
    y0[i] = ex2_approx(v);
    y3[i] = exp2_fma3(v);
    y4[i] = exp2_fma4(v);
  }
}

int64_t strip_stride(const hs2_shape* s, int b_last) {
  const int64_t n = n_cand(s, b_last);
  return std::max<int64_t>(64, (n + 63) / 64 * 64);
}

size_t min_workspace(const hs2_shape* s) {
  return static_cast<size_t>(s->Hkv) * static_cast<size_t>(strip_stride(s, s->L / 64 - 1)) * 4u;
}

constexpr size_t kStripCap = size_t(64) << 20;  // keep one strip L2-resident
// Rows (KV heads x blocks) of one importance launch: its grid's y extent.
constexpr int64_t kMaxStripRows = 65535;

// Rows a select launch should have at least: two per SM of a B200 (148 SMs),
// so that the per-row latency of long rows is overlapped across the GPU.
constexpr size_t kSelectRows = 296;

// Strips in as few launches as the L2 cap allows, but never fewer rows per
// strip than kSelectRows (long rows then stream from HBM instead of L2:
// cheaper than launches of a few latency-bound rows); with an e4m3 cache,
// plus room for the layer's f16 copy (dequant_bytes).
size_t recommended_workspace(const hs2_shape* s) {
  size_t whole = 0;
  const int nb = s->L / 64;
  for (int b = 0; b < nb; ++b) whole += static_cast<size_t>(s->Hkv) * strip_stride(s, b) * 4u;
  const size_t row_bytes = static_cast<size_t>(strip_stride(s, nb - 1)) * 4u;
  const size_t cap = std::max(kStripCap, kSelectRows * row_bytes);
  const size_t strips = std::max(min_workspace(s), std::min(whole, cap));
  return strips + (s->kv_dtype == HS2_KV_E4M3 ? dequant_bytes(s) : 0u);
}

// Scratch for hs2_full_attn_select_static: the importance strips of callers
// that cannot allocate.  Host code must not use the symbol as an address; the
// device address is looked up per device with cudaGetSymbolAddress.
constexpr size_t kStaticScratchBytes = size_t(16) << 20;
__device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[128] = {};

// Device address of g_static_scratch on the current device (looked up once per
// device, with that device current).
int static_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return HS2_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return HS2_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return HS2_OK;
}

}  // namespace
}  // namespace hs2

using namespace hs2;

extern "C" {

const char* hs2_strerror(int code) {
  switch (code) {
    case HS2_OK: return "ok";
    case HS2_ERR_INVALID_ARG: return "invalid argument";
    case HS2_ERR_UNSUPPORTED: return "unsupported shape, dtype or alignment";
    case HS2_ERR_WORKSPACE: return "workspace too small";
    case HS2_ERR_CUDA: return "CUDA error";
    case HS2_ERR_TIMEOUT: return "device wait timed out";
    case HS2_ERR_INDEX: return "index list entry out of range";
    case HS2_ERR_RANGE: return "input value outside the supported range (Q too large for f16 with an e4m3 cache)";
    default: return "unknown hs2 status";
  }
}

int hs2_version(void) { return 100; }

int hs2_exp2_check(const float* x, float* y_mufu, float* y_fma3, float* y_fma4, int64_t n, void* stream) {
  if (n < 0 || (n > 0 && (!x || !y_mufu || !y_fma3 || !y_fma4))) return HS2_ERR_INVALID_ARG;
  if (n == 0) return HS2_OK;
  const int blocks = static_cast<int>(std::min<int64_t>((n + 255) / 256, 4096));
  exp2_check_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y_mufu, y_fma3, y_fma4, n);
  return launched();
}

uint64_t hs2_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int hs2_debug_set(uint64_t wait_limit_ns, uint32_t flags) {
  if (wait_limit_ns == 0) return HS2_ERR_INVALID_ARG;
  g_wait_limit_ns = wait_limit_ns;
  g_flags = flags;
  return HS2_OK;
}

int hs2_attn_fwd(const hs2_shape* shape, const void* q, const void* k, const void* v, const float* k_scale,
                 const float* v_scale, void* o, float* lse, void* stream) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if ((rc = check_kv(shape, k, v, k_scale, v_scale))) return rc;
  if (!q || !o || !lse) return HS2_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o) || !aligned16(lse)) return HS2_ERR_UNSUPPORTED;
  return launch_attn_fwd(shape, q, k, v, k_scale, v_scale, o, lse, static_cast<cudaStream_t>(stream));
}

int hs2_attn_fwd_ws(const hs2_shape* shape, const void* q, const void* k, const void* v, const float* k_scale,
                    const float* v_scale, void* o, float* lse, void* workspace, size_t* workspace_bytes,
                    void* stream) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!workspace_bytes) return HS2_ERR_INVALID_ARG;
  const bool kv8 = shape->kv_dtype == HS2_KV_E4M3;
  if (!workspace) {
    *workspace_bytes = kv8 ? dequant_bytes(shape) : 0u;
    return HS2_OK;
  }
  if ((rc = check_kv(shape, k, v, k_scale, v_scale))) return rc;
  if (!q || !o || !lse) return HS2_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o) || !aligned16(lse) || !aligned16(workspace)) return HS2_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (kv8 && *workspace_bytes >= dequant_bytes(shape)) {
    const DequantBuf dqb = dequant_carve(shape, static_cast<uint8_t*>(workspace));
    if ((rc = launch_dequant(shape, k, v, k_scale, v_scale, dqb, st))) return rc;
    return launch_attn_fwd(shape, q, k, v, k_scale, v_scale, o, lse, st, &dqb);
  }
  return launch_attn_fwd(shape, q, k, v, k_scale, v_scale, o, lse, st);
}

int hs2_swa_attn(const hs2_shape* shape, const void* q, const void* k, const void* v, int32_t window, void* o,
                 float* lse, void* stream) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (shape->kv_dtype != HS2_KV_BF16) return HS2_ERR_UNSUPPORTED;
  if ((rc = check_kv(shape, k, v, nullptr, nullptr))) return rc;
  if (!q || !o) return HS2_ERR_INVALID_ARG;
  if (window < 1 || window > shape->L) return HS2_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o) || (lse && !aligned16(lse))) return HS2_ERR_UNSUPPORTED;
  return launch_sparse(shape, q, k, v, nullptr, nullptr, nullptr, nullptr, o, static_cast<cudaStream_t>(stream),
                       window, lse);
}

int hs2_importance(const hs2_shape* shape, const void* q, const void* k, const float* k_scale, const float* lse,
                   int32_t b0, int32_t b1, float* imp, int64_t row_stride, void* stream) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if ((rc = check_kv(shape, k, k, k_scale, k_scale))) return rc;
  if (!q || !lse || !imp) return HS2_ERR_INVALID_ARG;
  const int nb = shape->L / 64;
  if (b0 < 0 || b1 > nb || b0 >= b1) return HS2_ERR_INVALID_ARG;
  const bool visible = (g_flags & FLAG_IMP_VISIBLE) != 0;
  const int64_t longest = visible ? std::min(shape->L, 64 * b1) : n_cand(shape, b1 - 1);
  if (row_stride % 4 || row_stride < longest) return HS2_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(imp)) return HS2_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(shape->Hkv) * (b1 - b0) > kMaxStripRows) return HS2_ERR_UNSUPPORTED;
  return launch_importance(shape, q, k, k_scale, lse, b0, b1, imp, row_stride, -1,
                           static_cast<cudaStream_t>(stream), nullptr, visible);
}

int hs2_topk_select(const hs2_shape* shape, const float* imp, int64_t row_stride, int32_t b0, int32_t b1,
                    int32_t* idx, int32_t* cnt, void* stream) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!imp || !idx || !cnt) return HS2_ERR_INVALID_ARG;
  const int nb = shape->L / 64;
  if (b0 < 0 || b1 > nb || b0 >= b1) return HS2_ERR_INVALID_ARG;
  if (row_stride % 4 || row_stride < n_cand(shape, b1 - 1)) return HS2_ERR_INVALID_ARG;
  if (!aligned16(imp)) return HS2_ERR_UNSUPPORTED;
  return launch_select(shape, imp, row_stride, b0, b1, idx, cnt, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace hs2 {
namespace {
// Optional export of the importance rows a full-layer call computed for
// blocks [b0, b1) (see hs2_full_attn_select in hs2.h).
struct ImpExport {
  float* out = nullptr;
  int b0 = 0, b1 = 0;
};
int full_attn_select_impl(const hs2_shape* shape, const void* q, const void* k, const void* v, const float* k_scale,
                          const float* v_scale, void* o, float* lse, int32_t* idx, int32_t* cnt, void* workspace,
                          size_t* workspace_bytes, void* stream, bool blocks, const ImpExport& ex);
}  // namespace
}  // namespace hs2

extern "C" {

int hs2_full_attn_select(const hs2_shape* shape, const void* q, const void* k, const void* v, const float* k_scale,
                         const float* v_scale, void* o, float* lse, int32_t* idx, int32_t* cnt, void* workspace,
                         size_t* workspace_bytes, float* importance_out, int32_t strip_b0, int32_t strip_b1,
                         void* stream) {
  ImpExport ex;
  if (importance_out) {
    if (!shape) return HS2_ERR_INVALID_ARG;
    if (strip_b0 < 0 || strip_b0 >= strip_b1 || shape->block <= 0 || strip_b1 > shape->L / shape->block)
      return HS2_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(importance_out) & 3u) return HS2_ERR_UNSUPPORTED;
    ex.out = importance_out;
    ex.b0 = strip_b0;
    ex.b1 = strip_b1;
  }
  return full_attn_select_impl(shape, q, k, v, k_scale, v_scale, o, lse, idx, cnt, workspace, workspace_bytes, stream,
                               false, ex);
}

int hs2_full_attn_select_blocks(const hs2_shape* shape, const void* q, const void* k, const void* v,
                                const float* k_scale, const float* v_scale, void* o, float* lse, int32_t* idx,
                                int32_t* cnt, void* workspace, size_t* workspace_bytes, void* stream) {
  if (shape && shape->topk % 64) return HS2_ERR_UNSUPPORTED;
  if (shape && shape->L > 0 && static_cast<uint32_t>(shape->L / 64) * 4u > kBlockSelectSmem) return HS2_ERR_UNSUPPORTED;
  return full_attn_select_impl(shape, q, k, v, k_scale, v_scale, o, lse, idx, cnt, workspace, workspace_bytes, stream,
                               true, ImpExport{});
}

int hs2_block_select(const hs2_shape* shape, const float* imp, int64_t row_stride, int32_t b0, int32_t b1,
                     int32_t* idx, int32_t* cnt, void* stream) {
  using namespace hs2;
  int rc = check_shape(shape);
  if (rc) return rc;
  if (shape->topk % 64) return HS2_ERR_UNSUPPORTED;
  if (static_cast<uint32_t>(shape->L / 64) * 4u > kBlockSelectSmem) return HS2_ERR_UNSUPPORTED;
  if (!imp || !idx || !cnt) return HS2_ERR_INVALID_ARG;
  const int nb = shape->L / 64;
  if (b0 < 0 || b1 > nb || b0 >= b1) return HS2_ERR_INVALID_ARG;
  if (row_stride % 4 || row_stride < n_cand(shape, b1 - 1)) return HS2_ERR_INVALID_ARG;
  if (!aligned16(imp)) return HS2_ERR_UNSUPPORTED;
  return launch_select(shape, imp, row_stride, b0, b1, idx, cnt, static_cast<cudaStream_t>(stream), true);
}

}  // extern "C"

namespace hs2 {
namespace {
// Copies the rows of strip [sb0, sb1) (row stride `stride` in the workspace)
// that fall in the export range to the caller's buffer.
int export_rows(const hs2_shape* s, const float* imp, int sb0, int sb1, int64_t stride, const ImpExport& ex,
                cudaStream_t st) {
  const int lo = std::max(sb0, ex.b0), hi = std::min(sb1, ex.b1);
  if (!ex.out || lo >= hi) return HS2_OK;
  const int64_t ostride = strip_stride(s, ex.b1 - 1);
  const size_t width = static_cast<size_t>(std::min(stride, ostride)) * 4u;
  for (int g = 0; g < s->Hkv; ++g) {
    float* dst = ex.out + (static_cast<int64_t>(g) * (ex.b1 - ex.b0) + (lo - ex.b0)) * ostride;
    const float* src = imp + (static_cast<int64_t>(g) * (sb1 - sb0) + (lo - sb0)) * stride;
    if (cudaMemcpy2DAsync(dst, static_cast<size_t>(ostride) * 4u, src, static_cast<size_t>(stride) * 4u, width,
                          static_cast<size_t>(hi - lo), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return HS2_ERR_CUDA;
  }
  return HS2_OK;
}

int full_attn_select_impl(const hs2_shape* shape, const void* q, const void* k, const void* v, const float* k_scale,
                          const float* v_scale, void* o, float* lse, int32_t* idx, int32_t* cnt, void* workspace,
                          size_t* workspace_bytes, void* stream, bool blocks, const ImpExport& ex) {
  const Range range(blocks ? "hs2_full_attn_select_blocks" : "hs2_full_attn_select");
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!workspace_bytes) return HS2_ERR_INVALID_ARG;
  if (!workspace) {
    *workspace_bytes = recommended_workspace(shape);
    return HS2_OK;
  }
  if ((rc = check_kv(shape, k, v, k_scale, v_scale))) return rc;
  if (!q || !o || !lse || !idx || !cnt) return HS2_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o) || !aligned16(lse) || !aligned16(workspace)) return HS2_ERR_UNSUPPORTED;
  size_t ws = *workspace_bytes;
  if (ws < min_workspace(shape)) return HS2_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // An e4m3 cache is converted to f16 once for the layer when the workspace
  // also holds that copy (at its end); otherwise kernels (1) and (2) convert
  // the tiles they load.  The results are the same.
  DequantBuf dqb{};
  const DequantBuf* dq = nullptr;
  if (shape->kv_dtype == HS2_KV_E4M3 && ws >= min_workspace(shape) + dequant_bytes(shape)) {
    ws -= dequant_bytes(shape);
    dqb = dequant_carve(shape, static_cast<uint8_t*>(workspace) + ws);
    dq = &dqb;
    if ((rc = launch_dequant(shape, k, v, k_scale, v_scale, dqb, st))) return rc;
  }
  if ((rc = launch_attn_fwd(shape, q, k, v, k_scale, v_scale, o, lse, st, dq))) return rc;

  // Strips of query blocks.  Blocks whose candidates all fit in the top-k
  // need no importance; the rest are grouped so that a strip's rows
  // (Hkv x blocks x stride floats) fit the workspace.
  float* imp = static_cast<float*>(workspace);
  const int nb = shape->L / 64;
  int b = 0;
  while (b < nb) {
    int b1 = b + 1;
    if (n_cand(shape, b) <= shape->topk) {
      while (b1 < nb && n_cand(shape, b1) <= shape->topk) ++b1;
      if ((rc = launch_select(shape, imp, 64, b, b1, idx, cnt, st))) return rc;
    } else {
      while (b1 < nb && static_cast<int64_t>(shape->Hkv) * (b1 + 1 - b) <= kMaxStripRows &&
             static_cast<size_t>(shape->Hkv) * (b1 + 1 - b) * strip_stride(shape, b1) * 4u <= ws)
        ++b1;
      const int64_t stride = strip_stride(shape, b1 - 1);
      if ((rc = launch_importance(shape, q, k, k_scale, lse, b, b1, imp, stride, shape->topk, st, dq))) return rc;
      if ((rc = launch_select(shape, imp, stride, b, b1, idx, cnt, st, blocks))) return rc;
      if ((rc = export_rows(shape, imp, b, b1, stride, ex, st))) return rc;
    }
    b = b1;
  }
  return HS2_OK;
}
}  // namespace
}  // namespace hs2

extern "C" {

int hs2_full_attn_select_static(const hs2_shape* shape, const void* q, const void* k, const void* v,
                                const float* k_scale, const float* v_scale, void* o, float* lse, int32_t* idx,
                                int32_t* cnt, void* stream) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (min_workspace(shape) > kStaticScratchBytes) return HS2_ERR_WORKSPACE;  // before any CUDA call
  if (!q || !k || !v || !o || !lse || !idx || !cnt) return HS2_ERR_INVALID_ARG;
  void* scratch = nullptr;
  if ((rc = static_scratch(&scratch))) return rc;
  size_t n = kStaticScratchBytes;
  return hs2_full_attn_select(shape, q, k, v, k_scale, v_scale, o, lse, idx, cnt, scratch, &n, nullptr, 0, 0, stream);
}

int hs2_quantize_kv(int32_t L, int32_t Hkv, const void* src, int64_t src_tok_stride, int64_t src_head_stride,
                    void* dst, int64_t dst_tok_stride, int64_t dst_head_stride, float* scale, void* stream) {
  if (L <= 0 || Hkv <= 0 || !src || !dst || !scale) return HS2_ERR_INVALID_ARG;
  if (static_cast<int64_t>(L) * Hkv >= (int64_t(1) << 31)) return HS2_ERR_UNSUPPORTED;
  if (src_tok_stride <= 0 || src_head_stride <= 0 || dst_tok_stride <= 0 || dst_head_stride <= 0)
    return HS2_ERR_INVALID_ARG;
  if (src_head_stride < HD || dst_head_stride < HD || src_tok_stride < static_cast<int64_t>(Hkv) * src_head_stride ||
      dst_tok_stride < static_cast<int64_t>(Hkv) * dst_head_stride)
    return HS2_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(src) & 15u) || (reinterpret_cast<uintptr_t>(dst) & 7u) ||
      (reinterpret_cast<uintptr_t>(scale) & 3u) || src_tok_stride % 8 || src_head_stride % 8 ||
      dst_tok_stride % 8 || dst_head_stride % 8)
    return HS2_ERR_UNSUPPORTED;
  QuantParams p{};
  p.rows = L * Hkv;
  p.Hkv = Hkv;
  p.src = static_cast<const __nv_bfloat16*>(src);
  p.src_tok = src_tok_stride;
  p.src_head = src_head_stride;
  p.dst = static_cast<uint8_t*>(dst);
  p.dst_tok = dst_tok_stride;
  p.dst_head = dst_head_stride;
  p.scale = scale;
  const int64_t blocks = std::min<int64_t>((static_cast<int64_t>(p.rows) + 63) / 64, 148 * 16);
  const Range range("hs2 quantize_kv");
  quantize_kv_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
  return launched();
}

int hs2_sparse_attn(const hs2_shape* shape, const void* q, const void* k, const void* v, const float* k_scale,
                    const float* v_scale, const int32_t* idx, const int32_t* cnt, void* o, void* stream) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if ((rc = check_kv(shape, k, v, k_scale, v_scale))) return rc;
  if (!q || !o || !idx || !cnt) return HS2_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o) || !aligned16(idx)) return HS2_ERR_UNSUPPORTED;
  return launch_sparse(shape, q, k, v, k_scale, v_scale, idx, cnt, o, static_cast<cudaStream_t>(stream));
}

int hs2_sparse_decode_workspace(const hs2_shape* shape, int32_t n, size_t* workspace_bytes) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!workspace_bytes || n < 1 || n > 65535) return HS2_ERR_INVALID_ARG;
  *workspace_bytes = decode_plan(shape, n).ws_bytes;
  return HS2_OK;
}

int hs2_sparse_decode(const hs2_shape* shape, const void* q, const int32_t* positions, int32_t n, const void* k,
                      const void* v, const float* k_scale, const float* v_scale, const int32_t* idx,
                      const int32_t* cnt, void* o, void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (n < 1 || n > 65535) return HS2_ERR_INVALID_ARG;
  const DecodePlan plan = decode_plan(shape, n);
  if ((rc = check_kv(shape, k, v, k_scale, v_scale))) return rc;
  if (!q || !positions || !idx || !cnt || !o) return HS2_ERR_INVALID_ARG;
  if (plan.ws_bytes > 0 && !workspace) return HS2_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o) || (workspace && !aligned16(workspace))) return HS2_ERR_UNSUPPORTED;
  if (workspace_bytes < plan.ws_bytes) return HS2_ERR_WORKSPACE;
  return launch_decode(shape, q, positions, n, k, v, k_scale, v_scale, idx, cnt, o, workspace, plan,
                       static_cast<cudaStream_t>(stream));
}

int hs2_sync(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const cudaError_t e = cudaStreamSynchronize(st);
  DevStatus ds{};
  DevStatus zero{};
  if (cudaMemcpyFromSymbol(&ds, g_status, sizeof(ds)) != cudaSuccess) return HS2_ERR_CUDA;
  if (ds.code != 0 && cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return HS2_ERR_CUDA;
  if (ds.code != 0) return ds.code;
  return e == cudaSuccess ? HS2_OK : HS2_ERR_CUDA;
}

}  // extern "C"
