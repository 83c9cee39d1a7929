/*
 * cslc.h -- C ABI of the hybrid compressed attention library (libcslc.so).
 *
 * The library implements the attention path of the CSA / HCA hybrid layer
 * described on the DeepSeek-V4 explainer pages:
 *   CSA  ("从论文出发，逐层剖析 CSA / HCA 混注意力…", §1.1 and its 工程细节 paragraph;
 *         "读完这篇你就搞懂 DeepSeek v4 了", §三 CSA steps 1-3): every m=4 tokens become
 *         one KV entry compressed from an overlapped 2m-token window, a lightning
 *         indexer scores every entry per query, the top-k (1024) entries are
 *         selected, and all query heads attend to that selection with one KV head.
 *   HCA  (same pages, §1.2 / HCA 步骤简化): every m'=128 tokens become one entry,
 *         followed by dense causal attention over the short sequence.
 *   Decode KV layout (first page, §1.4 存储格式混): RoPE dims in BF16, the other
 *         dims in FP8 (e4m3) with one fp32 scale per entry.
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     never allocates or frees device memory. Scratch memory comes from a
 *     caller-provided workspace whose size the matching *_workspace_bytes()
 *     function reports (returns 0 when none is needed). One exception: the
 *     library's module holds a static 16 MiB device array on every device
 *     where it is loaded, until the process exits; only
 *     cslc_decode_topk_noalloc (at the end of this header) uses it.
 *   - Tensors are dense, row-major (last index fastest) with the shapes given
 *     below. bf16 tensors are passed as cslc_bf16 (raw bfloat16 bits).
 *     Every pointer must be 16-byte aligned (CSLC_ERR_ALIGN otherwise).
 *   - Calls are asynchronous on `stream` (NULL = the legacy default stream) and
 *     return after the launches are enqueued. Arguments are validated before
 *     anything is launched: on any error status nothing has been written.
 *     Errors from the CUDA launch itself return CSLC_ERR_CUDA.
 *   - No exception or abort crosses the ABI. cslc_last_error() returns a
 *     thread-local text for the last non-OK status.
 *   - Supported shapes: D = 128 (compressed entry / head dim), d_I = 64, H a
 *     multiple of 16 up to 128, H_I <= 16, 1 <= topk <= 2048, m a power of two
 *     in [1, 128] for compression (any m >= 1 for visibility). Anything else
 *     returns CSLC_ERR_UNSUPPORTED.
 *
 * Geometry shared by every call (the pages leave it open; this is the reading
 * the library follows): entry i of a compression with ratio m covers the
 * tokens up to position (i+1)m-1; a query at absolute position p sees entry i
 * iff (i+1)m-1 <= p, so n_vis(p) = min(N_c, floor((p+1)/m)). Only complete
 * windows are compressed: N_c = floor(L/m).
 */
#ifndef CSLC_H_
#define CSLC_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define CSLC_ABI_VERSION 1
#define CSLC_WAIT_LIMIT_NS_DEFAULT 2000000000ull   /* a pipeline wait gives up after 2 s */
#define CSLC_WAIT_SLEEP_NS_DEFAULT 200000u         /* a waiting thread re-checks every <= 0.2 ms */

typedef uint16_t cslc_bf16;              /* raw bfloat16 bits */
typedef struct CUstream_st* cslc_stream_t; /* the same handle as cudaStream_t */

typedef enum {
  CSLC_OK = 0,
  CSLC_ERR_NULL = 1,          /* a required pointer is NULL */
  CSLC_ERR_SHAPE = 2,         /* a size is negative / inconsistent */
  CSLC_ERR_ALIGN = 3,         /* a pointer is not 16-byte aligned */
  CSLC_ERR_UNSUPPORTED = 4,   /* shape outside the supported set */
  CSLC_ERR_WORKSPACE = 5,     /* workspace missing or too small */
  CSLC_ERR_CUDA = 6,          /* a CUDA call or launch failed */
  CSLC_ERR_DEVICE_CHECK = 7   /* a kernel's own check failed (see cslc_sync_status) */
} cslc_status;

/* Version of this ABI (CSLC_ABI_VERSION). Never fails. */
int cslc_abi_version(void);

/* Text of the last non-OK status returned on the calling thread. */
const char* cslc_last_error(void);

/* Waits for `stream`, then reports (and clears) any error a kernel recorded in
 * its device-side status word; returns CSLC_OK when none. */
cslc_status cslc_sync_status(cslc_stream_t stream);

/* Testing hook (no counterpart on the pages): the time after which a
 * pipelined kernel's wait gives up, and how long a waiting thread sleeps
 * between checks, for the kernels launched after the call on the current
 * device (defaults CSLC_WAIT_LIMIT_NS_DEFAULT, CSLC_WAIT_SLEEP_NS_DEFAULT).
 * A wait that gives up raises its CTA's abort: every role of the CTA leaves
 * its loop, products and copies already issued complete, TMEM is released,
 * and cslc_sync_status reports CSLC_ERR_DEVICE_CHECK; later calls run
 * normally. Synchronises with the legacy default stream. Tests use it to make
 * waits run out on small grids; production code leaves the defaults. */
cslc_status cslc_testing_set_wait_limits(uint64_t limit_ns, uint32_t sleep_ns);

/* ------------------------------------------------------------------------ */
/* Compression ("读完这篇你就搞懂 DeepSeek v4 了", §三 压缩机制; first page §1.1 工程细节)
 *
 * For entry i and channel j:
 *   e_i[j] = sum_{t in W_i} softmax_t( z_t[j] + pos_bias[slot(t)][j] ) * c_t[j]
 * computed in fp32, stored bf16 (round to nearest even).
 * CSA window W_i: C^b = tokens (i-1)m .. im-1 in slots 0..m-1 (absent for
 * i = 0) and C^a = tokens im .. im+m-1 in slots m..2m-1.
 *
 *   c, z      [B, L, D] bf16  candidate vectors and compression logits
 *   c_b, z_b  [B, L, D] bf16  optional separate streams read for the C^b half;
 *                             pass both NULL to read c, z there too
 *   pos_bias  [2m, D] bf16    positional bias per window slot
 *   out       [B, floor(L/m), D] bf16
 * Requires D == 128 (KV entries) or D == 64 (indexer keys compressed from
 * per-token key candidates, see cslc_decode_append), m a power of two in
 * [1, 128]. L < m gives 0 entries (nothing launched).
 */
cslc_status csa_compress(const cslc_bf16* c, const cslc_bf16* z,
                         const cslc_bf16* c_b, const cslc_bf16* z_b,
                         const cslc_bf16* pos_bias, int B, int L, int D, int m,
                         cslc_bf16* out, cslc_stream_t stream);

/* HCA compression (first page §1.2; "读完这篇…" §三 HCA 步骤简化): one window of
 * m' tokens per entry, no overlap: W_i = tokens im' .. im'+m'-1, slot = t - im'.
 *   pos_bias [m', D] bf16; out [B, floor(L/m'), D] bf16; D == 128 or 64. */
cslc_status hca_compress(const cslc_bf16* c, const cslc_bf16* z,
                         const cslc_bf16* pos_bias, int B, int L, int D,
                         int m_prime, cslc_bf16* out, cslc_stream_t stream);

/* Compressor front end ("读完这篇…" §三 压缩机制: 4 learnable W matrices and 2
 * learnable B matrices): the compressed entries straight from the hidden
 * states, the projections and the window compression in one pass.
 *
 * CSA: W [4, 128, d_model] bf16 holds W^{a,KV}, W^{b,KV}, W^{a,Z}, W^{b,Z},
 * each in [output, input] layout: per token t, c^a_t = W^{a,KV} h_t,
 * c^b_t = W^{b,KV} h_t, z^a_t = W^{a,Z} h_t, z^b_t = W^{b,Z} h_t (fp32
 * accumulation of bf16 products, not rounded); entry i is csa_compress's
 * window softmax with the C^a half reading (c^a, z^a) and the C^b half
 * (c^b, z^b): pos_bias [2m, 128] bf16 holds B^b (slots 0..m-1) then B^a.
 *   h [B, L, d_model] bf16; out [B, floor(L/m), 128] bf16.
 * Requires d_model a multiple of 64 (<= 65536), m a power of two <= 64,
 * B * L < 2^31. One launch; no workspace.
 *
 * HCA: W [2, 128, d_model] (W^{KV}, W^{Z}), pos_bias [m', 128], m' = 128;
 * entry i compresses tokens im' .. im'+m'-1 with c = W^{KV} h, z = W^{Z} h.
 */
cslc_status csa_compress_front_end(const cslc_bf16* h, const cslc_bf16* W, const cslc_bf16* pos_bias,
                                   int B, int L, int d_model, int m, cslc_bf16* out,
                                   cslc_stream_t stream);
cslc_status hca_compress_front_end(const cslc_bf16* h, const cslc_bf16* W, const cslc_bf16* pos_bias,
                                   int B, int L, int d_model, int m_prime, cslc_bf16* out,
                                   cslc_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Lightning indexer + top-k ("读完这篇…" §三 闪电索引; first page §1.1 top-k=1024)
 *
 *   S[b,t,i] = sum_h w[b,t,h] * max(0, q_idx[b,t,h,:] . k_idx[b,i,:])
 * for the entries visible to query row t (absolute position q_pos0 + t),
 * computed with fp32 accumulation of bf16 products and stored fp32.
 * idx[b,t,:] = the min(topk, n_vis) visible entries with the largest S (ties
 * to the smaller entry index; -0 and +0 tie), in ascending index order, then
 * -1 padding. Scores may be +-inf; a row holding a NaN score gets some valid
 * selection of distinct visible entries, not a defined one.
 *
 *   q_idx  [B, L, H_I, d_I] bf16     w [B, L, H_I] bf16     k_idx [B, Nc, d_I] bf16
 *   scores [B, L, Nc] fp32 or NULL.  When given, row t holds S for entries
 *          0..n_vis(t)-1; entries from n_vis(t) on are left unspecified.
 *          When NULL the scores live only in the workspace, in blocks of
 *          rows, two blocks in flight: the top-k of one block runs on an
 *          internal stream (one per host thread and device) beside the
 *          indexer of the next. All of it is ordered on `stream`: work queued
 *          there before the call happens before, and work queued after the
 *          call happens after (also under stream capture).
 *   idx    [B, L, topk] int32
 *   ws     workspace of csa_indexer_topk_workspace_bytes() bytes (may be NULL
 *          when that is 0).
 * Requires d_I == 64, 1 <= H_I <= 16, 1 <= topk <= 2048, q_pos0 >= 0,
 * Nc <= 786432 (a row's selection masks, Nc / 4 bytes, stay in shared memory;
 * the 1M-token CSA context has 262,144 entries).
 */
size_t csa_indexer_topk_workspace_bytes(int B, int L, int Nc, int HI, int topk, int scores_given);
cslc_status csa_indexer_topk(const cslc_bf16* q_idx, const cslc_bf16* w,
                             const cslc_bf16* k_idx, int B, int L, int Nc, int HI,
                             int dI, int m, int q_pos0, int topk, float* scores,
                             int32_t* idx, void* ws, size_t ws_bytes,
                             cslc_stream_t stream);

/* The top-k stage alone, on given scores [B, L, Nc] fp32 (same selection rule
 * and output layout as csa_indexer_topk; only the first n_vis(q_pos0+t)
 * entries of row t are read). */
cslc_status csa_topk(const float* scores, int B, int L, int Nc, int m, int q_pos0,
                     int topk, int32_t* idx, cslc_stream_t stream);

/* The indexer and top-k with BF16-stored scores (first page §1.4: the
 * indexer's scores are quantised from FP32 to BF16 to halve the top-k's
 * traffic). Each score is computed as in csa_indexer_topk (fp32 accumulation)
 * and rounded to the nearest bf16 (ties to even) before it is stored; idx is
 * the exact top-k of those bf16 scores under the same rule (ties, which bf16
 * makes frequent, go to the smaller index). scores [B, L, Nc] bf16 or NULL;
 * the workspace holds bf16 score blocks (csa_indexer_topk_bf16_workspace_bytes).
 * Other arguments, requirements and ordering as csa_indexer_topk. */
size_t csa_indexer_topk_bf16_workspace_bytes(int B, int L, int Nc, int HI, int topk, int scores_given);
cslc_status csa_indexer_topk_bf16(const cslc_bf16* q_idx, const cslc_bf16* w,
                                  const cslc_bf16* k_idx, int B, int L, int Nc, int HI,
                                  int dI, int m, int q_pos0, int topk, cslc_bf16* scores,
                                  int32_t* idx, void* ws, size_t ws_bytes,
                                  cslc_stream_t stream);
/* csa_topk on given bf16 scores [B, L, Nc]. */
cslc_status csa_topk_bf16(const cslc_bf16* scores, int B, int L, int Nc, int m, int q_pos0,
                          int topk, int32_t* idx, cslc_stream_t stream);

/* FP8 indexer operands (first page §1.4: a low-precision lightning indexer).
 *
 * cslc_quantize_rows_e4m3: rows x [rows, d] bf16 -> codes [rows, d] uint8
 * (e4m3) and scales [rows] fp32, per row s = amax(|x|) / 448 (1 for a zero
 * row) and codes = RNE-saturate(x / s), scale and quotient in fp32 (the rule
 * of cslc_quantize_kv_mixed). Requires d == 64 (the indexer's rows).
 *
 * csa_indexer_topk_fp8: csa_indexer_topk on e4m3 operands,
 *   S[b,t,i] = sum_h w[b,t,h] * max(0, qd[b,t,h,:] . kd[b,i,:]),
 *   qd = e4m3(q8) * q_scale[b,t,h],  kd = e4m3(k8) * k_scale[b,i],
 * with the code products accumulated in fp32 on the tensor cores, the scales
 * applied afterwards (they are positive: S = k_scale * sum_h w q_scale
 * max(0, q8 . k8)), and the scores stored fp32; idx is their exact top-k
 * under the rule of csa_indexer_topk.
 *   q8 [B, L, H_I, 64] uint8, q_scale [B, L, H_I] fp32, w [B, L, H_I] bf16,
 *   k8 [B, Nc, 64] uint8, k_scale [B, Nc] fp32 (scales > 0, as produced by
 *   cslc_quantize_rows_e4m3), q8 and k8 16-byte aligned;
 *   scores, idx, ws and ordering as csa_indexer_topk, workspace
 *   csa_indexer_topk_workspace_bytes().
 * Requires the limits of csa_indexer_topk.
 */
cslc_status cslc_quantize_rows_e4m3(const cslc_bf16* x, int64_t rows, int d, uint8_t* codes, float* scales,
                                    cslc_stream_t stream);
cslc_status csa_indexer_topk_fp8(const uint8_t* q8, const float* q_scale, const cslc_bf16* w,
                                 const uint8_t* k8, const float* k_scale, int B, int L, int Nc, int HI,
                                 int dI, int m, int q_pos0, int topk, float* scores, int32_t* idx,
                                 void* ws, size_t ws_bytes, cslc_stream_t stream);

/* ------------------------------------------------------------------------ */
/* CSA core attention ("读完这篇…" §三 注意力计算: ordinary attention over the
 * selected entries, KV shared by the heads)
 *
 *   o[b,t,h,:] = sum_{i in idx[b,t]} softmax_i(scale * q[b,t,h,:] . kv[b,i,:]) kv[b,i,:]
 * with K = V = the compressed entry; slots holding -1 are skipped; a row with
 * no valid slot outputs 0 and lse = -inf. fp32 accumulation, bf16 output.
 *
 *   q   [B, L, H, D] bf16    kv [B, Nc, D] bf16    idx [B, L, topk] int32
 *   out [B, L, H, D] bf16    lse [B, L, H] fp32 natural-log sum-exp of the
 *                            scaled logits, or NULL.
 * Indices must lie in [-1, Nc); others are treated as -1.
 */
cslc_status csa_sparse_attn(const cslc_bf16* q, const cslc_bf16* kv, const int32_t* idx,
                            int B, int L, int H, int D, int Nc, int topk, float scale,
                            cslc_bf16* out, float* lse, cslc_stream_t stream);

/* HCA core attention (first page §1.2: dense attention over all compressed
 * entries), causal: query row t (absolute position q_pos0 + t) sees entries
 * 0 .. n_vis-1 with n_vis = min(Nc, floor((q_pos0+t+1)/m')).
 * Shapes as csa_sparse_attn without idx. */
cslc_status hca_dense_attn(const cslc_bf16* q, const cslc_bf16* kv, int B, int L, int H,
                           int D, int Nc, int m_prime, int q_pos0, float scale,
                           cslc_bf16* out, float* lse, cslc_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Mixed decode KV layout (first page §1.4 存储格式混)
 *
 * Splits entries kv [B, N, 128] bf16 into
 *   nope  [B, N, 64] uint8  e4m3 codes of dims 0..63 divided by the entry scale
 *   rope  [B, N, 64] bf16   dims 64..127 unchanged
 *   scale [B, N] fp32       amax(|dims 0..63|) / 448 (1 when amax = 0)
 * Scale and quotient are computed in fp32 (IEEE division); codes round to
 * nearest even and saturate to +-448. 196 bytes per entry instead of 256.
 */
cslc_status cslc_quantize_kv_mixed(const cslc_bf16* kv, int B, int N, uint8_t* nope,
                                   cslc_bf16* rope, float* scale, cslc_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Decode: one new query token per sequence, all n_entries[b] entries visible.
 *
 * A CSA layer runs the indexer over the sequence's indexer keys, selects the
 * top-k entries exactly (ties to the smaller index) and attends to them; an
 * HCA layer attends densely to all entries. The KV is read in the mixed
 * layout above and dequantised as e4m3 value * scale (rounded to bf16 for the
 * tensor-core products).
 */
typedef struct {
  int kind;                  /* 0 = CSA (indexer + top-k + sparse), 1 = HCA (dense) */
  const cslc_bf16* q;        /* [B, H, 128] bf16 query heads */
  const cslc_bf16* q_idx;    /* [B, H_I, 64] bf16 indexer query (CSA only) */
  const cslc_bf16* w;        /* [B, H_I] bf16 indexer head weights (CSA only) */
  const cslc_bf16* k_idx;    /* [B, n_max, 64] bf16 indexer keys (CSA only) */
  const uint8_t* nope;       /* [B, n_max, 64] e4m3 */
  const cslc_bf16* rope;     /* [B, n_max, 64] bf16 */
  const float* kv_scale;     /* [B, n_max] fp32 */
  const int32_t* n_entries;  /* [B] int32 device array, 0 <= n_entries[b] <= n_max */
  int n_max;                 /* row stride (entries) of the per-sequence arrays */
  int topk;                  /* CSA: entries kept per sequence, 1..2048 */
  float scale;               /* softmax scale */
  cslc_bf16* out;            /* [B, H, 128] bf16 */
  int32_t* idx_out;          /* [B, topk] int32 selected entries (CSA), or NULL */
  float* scores_out;         /* [B, n_max] fp32 indexer scores (CSA), or NULL */
} cslc_decode_layer;

/* Workspace for cslc_decode_step over these layers: the sum of the layers'
 * needs (the layers run concurrently, each on its own slice). */
size_t cslc_decode_workspace_bytes(const cslc_decode_layer* layers, int n_layers, int B,
                                   int H, int HI);

/* Runs the layers (the hybrid C,H,C,H decode step is four layers, at most
 * 16 per call). The layers are independent and run concurrently: layer 0 on
 * `stream`, the others on internal streams (one set per host thread and
 * device) that are forked from `stream` and joined back into it, so work
 * queued on `stream` before the call happens before every layer and work
 * queued after it happens after all of them (also under stream capture).
 * Requires D == 128, d_I == 64, H a multiple of 16 <= 128, 1 <= H_I <= 16. */
cslc_status cslc_decode_step(const cslc_decode_layer* layers, int n_layers, int B, int H,
                             int D, int HI, int dI, void* ws, size_t ws_bytes,
                             cslc_stream_t stream);

/* Decode-time incremental compression ("读完这篇…" §三 压缩机制; first page
 * §1.1 工程细节): appends one token per sequence and, when that token completes
 * a window, one compressed entry to the layer's decode cache.
 *
 * For sequence b with pos[b] = p >= 0 (the new token's absolute position;
 * p < 0 skips the sequence): the token's c, z (and key candidate k_c, k_z) go
 * to ring slot p mod W, W = 2m with overlap (CSA), W = m without (HCA). When
 * (p + 1) mod m == 0, entry i = (p + 1)/m - 1 is compressed from the window of
 * csa_compress / hca_compress (C^b = tokens (i-1)m .. im-1, C^a = im .. im+m-1;
 * the first CSA entry has no C^b), computed by the same code as a prefill
 * pass (bit-identical entries), stored in the mixed layout of
 * cslc_quantize_kv_mixed at index i (bit-identical codes), its indexer key
 * compressed the same way from the 64-dim key candidates into k_idx[b, i], and
 * n_entries[b] = i + 1. A window completing at i >= n_max is not stored and
 * n_entries[b] is left as it was.
 *
 *   c, z          [B, 128] bf16  the new token's candidate and logits
 *   k_c, k_z      [B, 64]  bf16  its indexer-key candidate and logits, or NULL
 *   pos_bias      [W, 128] bf16; k_pos_bias [W, 64] bf16 (NULL without keys)
 *   pos           [B] int32 device array
 *   ring_c/ring_z [B, W, 128], ring_kc/ring_kz [B, W, 64] bf16: caller-owned
 *                 state; slot t mod W holds token t. Before the call it must
 *                 hold the tokens of the window that p completes (positions
 *                 p-W+1 .. p-1), e.g. filled by earlier appends or copied from
 *                 a prefill's last W tokens.
 *   nope [B, n_max, 64] u8, rope [B, n_max, 64] bf16, kv_scale [B, n_max] fp32,
 *   k_idx [B, n_max, 64] bf16 (NULL without keys), n_entries [B] int32: the
 *                 decode cache of cslc_decode_layer, updated in place.
 * Requires m a power of two <= 128, overlap 0 or 1; the key arguments all
 * given or all NULL. One launch of B blocks; no workspace.
 */
cslc_status cslc_decode_append(const cslc_bf16* c, const cslc_bf16* z, const cslc_bf16* k_c,
                               const cslc_bf16* k_z, const cslc_bf16* pos_bias,
                               const cslc_bf16* k_pos_bias, const int32_t* pos, int B, int m,
                               int overlap, cslc_bf16* ring_c, cslc_bf16* ring_z,
                               cslc_bf16* ring_kc, cslc_bf16* ring_kz, uint8_t* nope,
                               cslc_bf16* rope, float* kv_scale, cslc_bf16* k_idx, int n_max,
                               int32_t* n_entries, cslc_stream_t stream);

/* The decode top-k stage alone on given scores [B, n_max] fp32: idx [B, topk]
 * = the min(topk, n_entries[b]) largest of the first n_entries[b] scores
 * (ties to the smaller index), ascending, -1 padded. */
size_t cslc_decode_topk_workspace_bytes(int B, int n_max, int topk);
cslc_status cslc_decode_topk(const float* scores, const int32_t* n_entries, int B, int n_max,
                             int topk, int32_t* idx, void* ws, size_t ws_bytes,
                             cslc_stream_t stream);

/* ------------------------------------------------------------------------ */
/* The decode top-k without a caller workspace (the source pages have no
 * counterpart: this is a deployment convenience of the library).
 *
 * For callers that cannot call cudaMalloc -- e.g. a serving process whose
 * device memory is fully planned at start-up, code where an allocation would
 * synchronise the device, or a C caller with no device allocator. Same
 * arguments, selection rule and result as cslc_decode_topk, but the scratch
 * comes from one static device array of 16 MiB inside the library, held by
 * every GPU that loads the library until the process exits. The call
 * allocates nothing.
 *   - Requires cslc_decode_topk_workspace_bytes(B, n_max, topk) <= 16 MiB
 *     (16,777,216 bytes): e.g. B = 8 with n_max up to 259,068, or B = 64 with
 *     n_max up to 29,695; larger calls return CSLC_ERR_WORKSPACE without
 *     launching anything. The 1M-context shape B = 8 x 262,144 entries is over
 *     the limit: use cslc_decode_topk with a workspace for it.
 *   - The first call on a device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *     After the device's context is replaced (cudaDeviceReset) the next call
 *     looks the address up again, so it too must come before any capture.
 *   - Every call shares the array and it keeps the last call's contents (the
 *     parts that must start at zero are cleared on the stream by each call);
 *     calls whose work overlaps on the GPU (e.g. on two streams at once) race.
 */
cslc_status cslc_decode_topk_noalloc(const float* scores, const int32_t* n_entries, int B, int n_max,
                                     int topk, int32_t* idx, cslc_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* CSLC_H_ */
