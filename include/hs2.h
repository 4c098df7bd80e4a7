/*
 * hs2.h -- C ABI of libhs2: token-level sparse causal attention for
 * long-context prefill on one NVIDIA B200 (sm_100a).
 *
 * The method (HySparse2 architecture summary, "罗福莉剧透小米MiMo-V3架构：
 * HySparse2让预填充提前退出"):
 *   - a full-attention layer computes causal grouped-query attention and, from
 *     its own complete scores, picks the tokens worth attending to
 *     (ablation paragraph);
 *   - selection is per token: the 1024 most important earlier tokens plus the
 *     128 most recent ones (token-selection paragraph), the recent tokens
 *     replacing the removed sliding-window branch (branch-removal paragraph);
 *   - the following sparse layers reuse the full layer's KV cache and the
 *     selected positions (KV-sharing paragraph, "KV Reuse").
 * The attention itself is softmax(Q K^T / sqrt(d)) V (SHARP walk-through page,
 * section 1.1) with the causal mask j <= i.
 *
 * Readings fixed by this library where the pages are silent:
 *   - query head h uses KV head floor(h / G), G = Hq / Hkv;
 *   - one index list per (query block of 64 tokens, KV head);
 *   - importance of key j for block b, KV head g:
 *       I_j = sum over the group's heads h and the block's queries i of
 *             exp(s_hij - lse_hi),  s = q.k / sqrt(d), lse = natural-log LSE;
 *   - candidates C_b = [0, e_b - recent), e_b = end of block b; the recent
 *     window R_b = [e_b - recent, e_b) is always listed; ties in importance go
 *     to the lower position; the list is ascending, -1 padded.
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The
 *     library allocates no device memory; calls are asynchronous on `stream`
 *     (a cudaStream_t; NULL = the legacy default stream).  Only hs2_sync
 *     blocks the host.
 *   - Layouts are token-major, batch 1:
 *       Q, O      : bf16 [L][Hq][d]     strides q_tok_stride / q_head_stride
 *                                         (elements; O uses the same strides)
 *       K, V      : bf16 or e4m3 [L][Hkv][d]   strides kv_tok_stride /
 *                                         kv_head_stride (elements); the last
 *                                         dimension is contiguous
 *       k/v_scale : fp32 [L][Hkv] contiguous (only for kv_dtype = E4M3:
 *                   stored value = e4m3(code) * scale)
 *   - With an e4m3 cache (kv_dtype = HS2_KV_E4M3) the tensor-core products run
 *     on f16 operands: e4m3 codes convert to f16 exactly, and Q is rounded
 *     from bf16 to f16, which is exact for magnitudes in [2^-14, 65504].
 *     Smaller magnitudes become f16 subnormals (multiples of 2^-24, so they
 *     keep fewer bits); a magnitude of 65520 or more has no f16 value, and
 *     a Q holding one is reported by the next hs2_sync as HS2_ERR_RANGE (the
 *     outputs of that call are then meaningless).  A bf16 cache has no such
 *     limit.
 *       lse       : fp32 [Hq][L]  (natural log)
 *       idx       : int32 [Hkv][nb][topk + recent], nb = L / block,
 *                   ascending positions, -1 padded
 *       cnt       : int32 [Hkv][nb], valid entries per list
 *   - Errors are returned as HS2_* codes; nothing is launched when an argument
 *     check fails.  Faults found on the device (a bounded wait that ran out,
 *     an index out of range) are recorded in a device status word and
 *     returned by the next hs2_sync.
 *   - Supported shapes: d = 128, block = 64, L a multiple of 64, recent a
 *     multiple of 64 with recent >= block, 1 <= topk <= 4096 - recent,
 *     G = Hq / Hkv in {2, 4, 8}, base pointers 16-byte aligned, strides
 *     multiples of 8 elements (16 bytes for the byte-wide e4m3 cache: 16
 *     elements).  Anything else returns HS2_ERR_UNSUPPORTED.
 */
#ifndef HS2_H_
#define HS2_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum hs2_status {
  HS2_OK = 0,
  HS2_ERR_INVALID_ARG = 1,  /* null pointer, negative size, inconsistent shape */
  HS2_ERR_UNSUPPORTED = 2,  /* shape/alignment outside the supported set above */
  HS2_ERR_WORKSPACE = 3,    /* workspace smaller than the minimum */
  HS2_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed */
  HS2_ERR_TIMEOUT = 5,      /* a device-side bounded wait ran out */
  HS2_ERR_INDEX = 6,        /* an index list held a position outside [0, e_b) */
  HS2_ERR_RANGE = 7         /* an input value outside the supported range (see
                               kv_dtype = HS2_KV_E4M3 below) */
};

enum hs2_kv_dtype { HS2_KV_BF16 = 0, HS2_KV_E4M3 = 1 };

typedef struct hs2_shape {
  int32_t L, Hq, Hkv, d, block, topk, recent, kv_dtype;
  int64_t q_tok_stride, q_head_stride;   /* elements of Q and O */
  int64_t kv_tok_stride, kv_head_stride; /* elements of K and V */
} hs2_shape;

/*
 * Full-attention layer + selection (the whole first half of the prefill path).
 * Computes O and lse (causal GQA flash attention on tcgen05 tensor cores),
 * then, in strips of query blocks that fit the workspace, the importance rows
 * and their top-k selection, writing idx and cnt for every (KV head, block).
 *
 * workspace / workspace_bytes: scratch device memory for importance strips.
 *   workspace == NULL: *workspace_bytes receives the recommended size (whole
 *   path in as few strips as possible, capped at 64 MiB so a strip stays
 *   L2-resident, but never below 296 of the longest rows, two per SM, so that
 *   a select launch over long rows keeps the GPU busy) and nothing else
 *   happens.  Otherwise *workspace_bytes is the size of
 *   `workspace` (16-byte aligned); it must be at least
 *   Hkv * roundup(L - recent, 64) * 4 bytes (one block per strip), else
 *   HS2_ERR_WORKSPACE.  The workspace holds no state between calls.
 *   With an e4m3 cache the recommended size also holds an f16 copy of the
 *   layer's K and V (2 * L * Hkv * 128 * 2 bytes, plus Hkv * roundup(L, 128)
 *   * 4 bytes of K scales and 768 bytes of alignment), taken from the end of
 *   the workspace whenever it fits beside the minimum: the cache is then
 *   converted once instead of inside every tile load of the attention and
 *   importance kernels.  Results are identical either way.
 *
 * importance_out / strip_b0 / strip_b1: optional export, for checking, of the
 *   very importance rows the selection consumed.  NULL: no export (strip_b0
 *   and strip_b1 are ignored).  Otherwise, for the query blocks
 *   b in [strip_b0, strip_b1) (0 <= strip_b0 < strip_b1 <= L / 64) and every
 *   KV head g, row (g, b) is copied out of the workspace, after kernel (2)
 *   wrote it and before the next strip overwrites it, to
 *     importance_out[((g * (strip_b1 - strip_b0)) + (b - strip_b0)) * S + j],
 *   j in C_b = [0, e_b - recent), with the row stride
 *     S = max(64, roundup(e_{strip_b1 - 1} - recent, 64)) floats
 *   (the Python binding's importance_row_stride computes it).  Entries past
 *   |C_b| are unspecified; the rows of blocks with |C_b| <= topk (every
 *   candidate is selected there, so no importance is computed) are left
 *   untouched.
 *   importance_out: device memory of Hkv * (strip_b1 - strip_b0) * S floats,
 *   4-byte aligned; a bad range returns HS2_ERR_INVALID_ARG.
 */
int hs2_full_attn_select(const hs2_shape* shape, const void* q, const void* k, const void* v,
                         const float* k_scale, const float* v_scale, void* o, float* lse, int32_t* idx,
                         int32_t* cnt, void* workspace, size_t* workspace_bytes, float* importance_out,
                         int32_t strip_b0, int32_t strip_b1, void* stream);

/*
 * hs2_full_attn_select without a caller workspace.  (The paper has no
 * counterpart: this is a deployment convenience.)
 *
 * For callers that cannot allocate device memory where they call this: a
 * plugin inside a host framework that owns the whole device pool and hands
 * plugins only the pointers of their tensors, or a latency-critical path where
 * a cudaMalloc could synchronise the device.  The importance strips live in a
 * fixed 16 MiB array inside the library (a file-scope __device__ array, held on
 * every GPU that loads the library until the process exits); nothing is
 * allocated or freed.
 *
 *   - Shapes whose one-block strip needs more than 16 MiB
 *     (Hkv * roundup(L - recent, 64) * 4 bytes > 16 MiB, e.g. L = 1M with
 *     Hkv = 8) return HS2_ERR_WORKSPACE before anything is launched.
 *   - The first call on a device looks up the array's device address with that
 *     device current; make that first call before any stream capture, and pass
 *     a stream of the current device.
 *   - Every call shares the one array, which keeps the previous call's
 *     contents; nothing in it has to start at zero (each importance entry the
 *     select reads is written earlier in the same call).  Calls that overlap on
 *     the GPU (e.g. on two streams of one device) race on it: serialise them.
 * Results equal those of hs2_full_attn_select on the same inputs.
 */
int hs2_full_attn_select_static(const hs2_shape* shape, const void* q, const void* k, const void* v,
                                const float* k_scale, const float* v_scale, void* o, float* lse, int32_t* idx,
                                int32_t* cnt, void* stream);

/*
 * One sparse layer (KV Reuse): for every query i of block b and head h,
 * softmax over the listed positions j <= i of q_hi . k_j / sqrt(d), times V,
 * using the shared K/V and the index lists written by hs2_full_attn_select.
 * q is this layer's own Q; o (same layout and strides as q) is written.
 * Padding entries (-1) are never dereferenced.
 */
int hs2_sparse_attn(const hs2_shape* shape, const void* q, const void* k, const void* v,
                    const float* k_scale, const float* v_scale, const int32_t* idx, const int32_t* cnt,
                    void* o, void* stream);

/*
 * FP8 KV write: quantise a bf16 K or V cache to OCP e4m3fn codes with one fp32
 * scale per (token, KV head), the format hs2_shape.kv_dtype = HS2_KV_E4M3 reads
 * (HySparse2 architecture summary, cost paragraph: FP8 KV cache).  For each row
 * of d = 128 values: scale = amax / 448 in fp32 (1 for an all-zero row),
 * code = e4m3(x / scale) with fp32 division and saturating round-to-nearest-
 * even.  src: bf16 [L][Hkv][128], element strides (multiples of 8, base
 * 16-byte aligned); dst: uint8 [L][Hkv][128], byte strides (multiples of 8,
 * base 8-byte aligned); scale: fp32 [L][Hkv] contiguous.  Device pointers;
 * asynchronous on `stream`.
 */
int hs2_quantize_kv(int32_t L, int32_t Hkv, const void* src, int64_t src_tok_stride, int64_t src_head_stride,
                    void* dst, int64_t dst_tok_stride, int64_t dst_head_stride, float* scale, void* stream);

/*
 * Blocks until `stream` is idle, then returns the first error recorded on the
 * device since the previous hs2_sync (and clears it), or HS2_ERR_CUDA if the
 * stream reported an error, else HS2_OK.
 */
int hs2_sync(void* stream);

/* ---- stage-level entry points (same kernels as above, one stage each) ---- */

/*
 * Full causal attention forward with LSE only (kernel 1 of the path).  With an
 * e4m3 cache the kernel converts every K/V tile it loads (no scratch memory);
 * hs2_attn_fwd_ws below converts the cache once instead, as the full layer
 * does.  Both give the same bits.
 */
int hs2_attn_fwd(const hs2_shape* shape, const void* q, const void* k, const void* v, const float* k_scale,
                 const float* v_scale, void* o, float* lse, void* stream);

/*
 * hs2_attn_fwd as hs2_full_attn_select runs it: with an e4m3 cache and a
 * workspace of at least the size this call reports (workspace == NULL: the
 * size goes to *workspace_bytes, nothing else happens; 0 for a bf16 cache),
 * the cache is first converted once into the workspace (an f16 copy of K and
 * V plus the K column scales) and kernel (1) loads f16 tiles from it;
 * otherwise this is hs2_attn_fwd.  Results are identical to hs2_attn_fwd.
 * workspace: 16-byte aligned; no state is kept between calls.
 */
int hs2_attn_fwd_ws(const hs2_shape* shape, const void* q, const void* k, const void* v, const float* k_scale,
                    const float* v_scale, void* o, float* lse, void* workspace, size_t* workspace_bytes,
                    void* stream);

/*
 * Importance rows (kernel 2) for query blocks [b0, b1), given the full
 * layer's lse.  Row (g, b) holds I_j for j in C_b = [0, e_b - recent) at
 * imp[((g * (b1 - b0)) + (b - b0)) * row_stride + j]; entries past |C_b| are
 * not written.  row_stride (floats) must be a multiple of 4 and at least
 * |C_{b1-1}|.  One call covers at most 65535 rows (Hkv * (b1 - b0)), else
 * HS2_ERR_UNSUPPORTED; hs2_full_attn_select splits its strips accordingly.
 */
int hs2_importance(const hs2_shape* shape, const void* q, const void* k, const float* k_scale,
                   const float* lse, int32_t b0, int32_t b1, float* imp, int64_t row_stride, void* stream);

/*
 * Top-k + recent-window selection (kernel 3) over caller-supplied importance
 * rows laid out as in hs2_importance, for blocks [b0, b1); writes the lists
 * of those blocks into idx / cnt (full [Hkv][nb] layout).  Rows must hold
 * finite values; -0.0 and +0.0 compare equal.
 */
int hs2_topk_select(const hs2_shape* shape, const float* imp, int64_t row_stride, int32_t b0, int32_t b1,
                    int32_t* idx, int32_t* cnt, void* stream);

/* ---- block-level selection (HySparse v1), the design token-level replaces ---- */

/*
 * Like hs2_topk_select, at the granularity of the earlier HySparse (HySparse2
 * architecture summary, block-selection paragraph: a whole 64-token block
 * spends budget): each candidate row is pooled into 64-key blocks -- the sum
 * of a block in a fixed fp32 order: 16 partial sums of 4 consecutive values
 * added left to right, then combined pairwise at distances 8, 4, 2, 1 -- the
 * top topk/64 blocks are kept (ties to the lower block) and listed as
 * ascending positions, followed by the recent window.  Same layouts and list
 * sizes as the token-level lists.  Blocks whose sums agree to within the fp32
 * rounding of a 64-term sum may rank either way.  Requires topk % 64 == 0 and
 * L <= 2^20 (a row's pooled values are held in 64 KiB of shared memory), else
 * HS2_ERR_UNSUPPORTED.
 */
int hs2_block_select(const hs2_shape* shape, const float* imp, int64_t row_stride, int32_t b0, int32_t b1,
                     int32_t* idx, int32_t* cnt, void* stream);

/* hs2_full_attn_select with block-level instead of token-level selection
 * (same limits as hs2_block_select; no importance export). */
int hs2_full_attn_select_blocks(const hs2_shape* shape, const void* q, const void* k, const void* v,
                                const float* k_scale, const float* v_scale, void* o, float* lse, int32_t* idx,
                                int32_t* cnt, void* workspace, size_t* workspace_bytes, void* stream);

/* ---- decode-step sparse attention ---- */

/*
 * Sparse-layer attention for n single query tokens at arbitrary positions
 * (HySparse2 architecture summary, KV-sharing paragraph: the sparse layers
 * reuse the full layer's KV cache and token selection; with early exit they
 * mostly run at decode).  Query r at position t = positions[r] attends, for
 * each KV head g, to the listed positions j <= t of the list of block
 * floor(t / 64), idx[g][floor(t / 64)][0 .. cnt), with softmax(q.k / sqrt(d)).
 * A query with no visible listed key gets a zero row.
 *
 * shape: the prefill's shape (L, heads, d, topk, recent, kv_dtype, K/V
 *   strides); its q strides are the strides of `q` and `o` here.
 * q: bf16 [n][Hq][d]; o: bf16 [n][Hq][d] (written); positions: int32 [n],
 *   device memory, each in [0, L) (an entry outside it, a count outside
 *   [0, topk + recent] or a listed position outside [0, e_b) is reported by
 *   hs2_sync as HS2_ERR_INDEX and never dereferenced; its row is zero).
 * k, v, k_scale, v_scale, idx, cnt: as hs2_sparse_attn.
 * workspace: device scratch of hs2_sparse_decode_workspace(shape, n) bytes
 *   (may be NULL when that is 0), 16-byte aligned; a smaller size returns
 *   HS2_ERR_WORKSPACE.  It holds no state between calls, but two calls in
 *   flight at once must not share it.
 * 1 <= n <= 65535, else HS2_ERR_INVALID_ARG.  Asynchronous on `stream`.
 */
int hs2_sparse_decode(const hs2_shape* shape, const void* q, const int32_t* positions, int32_t n, const void* k,
                      const void* v, const float* k_scale, const float* v_scale, const int32_t* idx,
                      const int32_t* cnt, void* o, void* workspace, size_t workspace_bytes, void* stream);

/* Workspace size in bytes hs2_sparse_decode needs for (shape, n); host only. */
int hs2_sparse_decode_workspace(const hs2_shape* shape, int32_t n, size_t* workspace_bytes);

/* ---- sliding-window attention (self-decoder window layers) ---- */

/*
 * Causal sliding-window attention: o_i = softmax over j in (i - window, i] of
 * q_i . k_j / sqrt(d), applied to v (HySparse2 architecture summary, paragraph
 * on the self-decoder / cross-decoder split: the front half mixes full and
 * sliding-window attention).  Same q / k / v / o layouts and strides as
 * hs2_attn_fwd; the cache must be bf16 (kv_dtype = HS2_KV_BF16, else
 * HS2_ERR_UNSUPPORTED); topk / recent are checked as in every call but not
 * used.  1 <= window <= L, else HS2_ERR_INVALID_ARG.  lse (fp32 [Hq][L],
 * natural log) is optional: NULL skips it, otherwise it must be 16-byte
 * aligned.  Device pointers owned by the caller; asynchronous on `stream`;
 * device-side failures surface through hs2_sync.
 */
int hs2_swa_attn(const hs2_shape* shape, const void* q, const void* k, const void* v, int32_t window, void* o,
                 float* lse, void* stream);

/* ---- diagnostics ---- */

/* Short text for an hs2_status code (static storage). */
const char* hs2_strerror(int code);

/*
 * Limit for every device-side wait, in nanoseconds (default 2e9).  Test hook
 * flags: bit 0 makes the attention kernels' load role issue nothing, so the
 * bounded waits of the other roles must run out and hs2_sync must report
 * HS2_ERR_TIMEOUT.  Bit 1 (checking mode) makes hs2_importance compute each
 * row over every visible key j < e_b with the causal mask j <= i, not only
 * over the candidates C_b (row_stride must then be at least e_{b1-1}): such
 * a row sums to 64 * G (every query's probabilities sum to one), which a test
 * checks; its first |C_b| entries equal the normal row's.  hs2_full_attn_select
 * ignores bit 1.  Bit 2 runs the full layer's attention (hs2_attn_fwd and
 * inside hs2_full_attn_select) on clusters of two CTAs that share every
 * product (tcgen05 cta_group::2) when the cache is bf16 or its f16 layer copy
 * is in the workspace: the results are bit for bit those of the default
 * kernel.  Bit 3 makes every TMA descriptor encoding fail as a driver error
 * would: calls that encode one return HS2_ERR_CUDA before launching anything
 * (host-side fault injection for tests).  Flags are 0 in normal use.
 *
 * Each kernel launch (and each hs2_full_attn_select call) is wrapped in an
 * NVTX range named after it ("hs2 attn_fwd (kernel 1)", ...), which
 * profilers can use to attribute and filter launches.
 */
int hs2_debug_set(uint64_t wait_limit_ns, uint32_t flags);

/*
 * Evaluates, on the device, the exponentials the kernels use for x[0..n):
 * y_mufu = hardware ex2.approx, y_fma3 / y_fma4 = the software 2^x on the FMA
 * pipes (degree-3 and degree-4 polynomials; valid for x >= -125).  Device
 * pointers, n >= 0; for checking their error against an fp64 reference.
 */
int hs2_exp2_check(const float* x, float* y_mufu, float* y_fma3, float* y_fma4, int64_t n, void* stream);

/* Library version as major * 10000 + minor * 100 + patch. */
int hs2_version(void);

/* Number of kernels this library has launched since it was loaded (host-side
 * counter, incremented once per successful launch; for accounting). */
uint64_t hs2_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* HS2_H_ */
