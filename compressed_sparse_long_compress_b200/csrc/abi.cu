// C ABI of libcslc: argument validation, workspace carving and dispatch.
// Every entry point validates before launching anything and never throws.

#include <stdarg.h>
#include <stdio.h>

#include "common.cuh"

namespace cslc {

static thread_local char g_err[512] = "";

cslc_status set_error(cslc_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

cslc_status check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(CSLC_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return CSLC_OK;
}

// kernels (defined in the other translation units)
cslc_status launch_compress(const uint16_t*, const uint16_t*, const uint16_t*, const uint16_t*,
                            const uint16_t*, int, int, int, int, int, uint16_t*, cudaStream_t);
cslc_status launch_decode_append(const uint16_t*, const uint16_t*, const uint16_t*, const uint16_t*, const uint16_t*,
                                 const uint16_t*, const int32_t*, int, int, int, uint16_t*, uint16_t*, uint16_t*,
                                 uint16_t*, uint8_t*, uint16_t*, float*, uint16_t*, int, int32_t*, cudaStream_t);
cslc_status launch_quantize_kv(const uint16_t*, long long, uint8_t*, uint16_t*, float*, cudaStream_t);
cslc_status launch_quantize_rows64(const uint16_t*, long long, uint8_t*, float*, cudaStream_t);
cslc_status launch_indexer_scores_fp8(const uint8_t*, const float*, const uint16_t*, const uint8_t*, const float*, int,
                                      int, int, int, int, int, int, int, float*, int, cudaStream_t);
cslc_status launch_indexer_scores(const uint16_t*, const uint16_t*, const uint16_t*, int, int, int, int,
                                  int, int, int, int, void*, bool, int, cudaStream_t);
cslc_status launch_topk_rows(const void*, bool, int, int, int, int, int, int, int, int, int, int32_t*,
                             cudaStream_t);
cslc_status launch_sparse_attn_sm100(const uint16_t*, const uint16_t*, const int32_t*, int, int, int, int, int,
                                     float, uint16_t*, float*, cudaStream_t);
cslc_status launch_dense_attn_sm100(const uint16_t*, const uint16_t*, int, int, int, int, int, int, float,
                                    uint16_t*, float*, cudaStream_t);
size_t decode_workspace_bytes(const cslc_decode_layer*, int, int, int);
int sparse_attn_sm100_read_error();
int dense_attn_sm100_read_error();
int indexer_sm100_read_error();
int front_end_sm100_read_error();
cudaError_t sparse_attn_sm100_set_wait_limits(uint64_t, uint32_t);
cudaError_t dense_attn_sm100_set_wait_limits(uint64_t, uint32_t);
cudaError_t indexer_sm100_set_wait_limits(uint64_t, uint32_t);
cudaError_t front_end_sm100_set_wait_limits(uint64_t, uint32_t);
cslc_status launch_front_end(const uint16_t*, const uint16_t*, const uint16_t*, int, int, int, int, int, uint16_t*,
                             cudaStream_t);
size_t decode_topk_workspace_bytes(int, int, int);
cslc_status run_decode_step(const cslc_decode_layer*, int, int, int, int, void*, size_t, cudaStream_t);
cslc_status run_decode_topk(const float*, const int32_t*, int, int, int, int32_t*, void*, cudaStream_t);

constexpr int kMaxTopk = 2048;
constexpr int kMaxPrefillTopkNc = 786432;   // a row's selection masks (Nc / 4 bytes) fit in shared memory

static bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

#define REQUIRE(cond, st, ...) \
  do {                          \
    if (!(cond)) return set_error(st, __VA_ARGS__); \
  } while (0)

#define REQUIRE_PTR(p)                                                                 \
  do {                                                                                 \
    REQUIRE((p) != nullptr, CSLC_ERR_NULL, "%s: %s is NULL", __func__, #p);            \
    REQUIRE(aligned16(p), CSLC_ERR_ALIGN, "%s: %s is not 16-byte aligned", __func__, #p); \
  } while (0)

// When the caller does not keep the scores they are produced in blocks of
// this many rows (up to 4 GiB of scores), two blocks in flight when there are
// more: the top-k of one block runs on an auxiliary stream beside the indexer
// of the next. Large blocks measured faster than small ones (fewer launch
// tails), and one block, where it fits, faster than two side by side.
static int score_block_rows(int Nc, int score_bytes = 4) {
  const long long budget = 4096ll << 20;   // bytes of scores per block
  long long rows = budget / ((long long)Nc * score_bytes);
  rows = rows < 64 ? 64 : rows;
  rows = (rows / 64) * 64;
  return (int)rows;
}

// The auxiliary stream and its events, one set per host thread and device
// (created on first use, kept for the life of the process).
struct BlockOverlap {
  cudaStream_t aux = nullptr;
  cudaEvent_t ready[2] = {nullptr, nullptr};   // scores of the block in buffer j written
  cudaEvent_t freed[2] = {nullptr, nullptr};   // buffer j read by its top-k
};

static cslc_status block_overlap(BlockOverlap** out) {
  constexpr int kMaxDevices = 64;
  thread_local BlockOverlap sets[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return set_error(CSLC_ERR_CUDA, "csa_indexer_topk: no usable current device");
  BlockOverlap& o = sets[dev];
  if (!o.aux) {
    e = cudaStreamCreateWithFlags(&o.aux, cudaStreamNonBlocking);
    for (int j = 0; j < 2 && e == cudaSuccess; ++j) {
      e = cudaEventCreateWithFlags(&o.ready[j], cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&o.freed[j], cudaEventDisableTiming);
    }
    if (e != cudaSuccess) {
      o.aux = nullptr;
      return set_error(CSLC_ERR_CUDA, "csa_indexer_topk: stream/event creation: %s", cudaGetErrorString(e));
    }
  }
  *out = &o;
  return CSLC_OK;
}

}  // namespace cslc

using namespace cslc;

extern "C" {

int cslc_abi_version(void) { return CSLC_ABI_VERSION; }

const char* cslc_last_error(void) { return g_err; }

cslc_status cslc_sync_status(cslc_stream_t stream) {
  const cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return set_error(CSLC_ERR_CUDA, "cslc_sync_status: %s", cudaGetErrorString(e));
  const int code = sparse_attn_sm100_read_error();
  if (code != 0)
    return set_error(CSLC_ERR_DEVICE_CHECK, "csa_sparse_attn: a pipeline wait timed out (code %d)", code);
  const int code2 = dense_attn_sm100_read_error();
  if (code2 != 0)
    return set_error(CSLC_ERR_DEVICE_CHECK, "hca_dense_attn: a pipeline wait timed out (code %d)", code2);
  const int code3 = indexer_sm100_read_error();
  if (code3 != 0)
    return set_error(CSLC_ERR_DEVICE_CHECK, "csa_indexer_topk: a pipeline wait timed out (code %d)", code3);
  const int code4 = front_end_sm100_read_error();
  if (code4 != 0)
    return set_error(CSLC_ERR_DEVICE_CHECK, "compressor front end: a pipeline wait timed out (code %d)", code4);
  return CSLC_OK;
}

cslc_status cslc_testing_set_wait_limits(uint64_t limit_ns, uint32_t sleep_ns) {
  cudaError_t e = sparse_attn_sm100_set_wait_limits(limit_ns, sleep_ns);
  if (e == cudaSuccess) e = dense_attn_sm100_set_wait_limits(limit_ns, sleep_ns);
  if (e == cudaSuccess) e = indexer_sm100_set_wait_limits(limit_ns, sleep_ns);
  if (e == cudaSuccess) e = front_end_sm100_set_wait_limits(limit_ns, sleep_ns);
  if (e != cudaSuccess) return set_error(CSLC_ERR_CUDA, "cslc_testing_set_wait_limits: %s", cudaGetErrorString(e));
  return CSLC_OK;
}

cslc_status csa_compress(const cslc_bf16* c, const cslc_bf16* z, const cslc_bf16* c_b,
                         const cslc_bf16* z_b, const cslc_bf16* pos_bias, int B, int L, int D, int m,
                         cslc_bf16* out, cslc_stream_t stream) {
  REQUIRE(B >= 0 && L >= 0, CSLC_ERR_SHAPE, "csa_compress: negative size");
  REQUIRE(D == kD || D == kDI, CSLC_ERR_UNSUPPORTED, "csa_compress: D must be 128 or 64 (got %d)", D);
  REQUIRE(is_pow2(m) && m <= 128, CSLC_ERR_UNSUPPORTED, "csa_compress: m must be a power of two <= 128");
  REQUIRE((c_b == nullptr) == (z_b == nullptr), CSLC_ERR_NULL, "csa_compress: give both c_b and z_b or neither");
  if ((long long)B * (L / m) == 0) return CSLC_OK;
  REQUIRE_PTR(c); REQUIRE_PTR(z); REQUIRE_PTR(pos_bias); REQUIRE_PTR(out);
  if (c_b) { REQUIRE_PTR(c_b); REQUIRE_PTR(z_b); }
  return launch_compress(c, z, c_b, z_b, pos_bias, B, L, D, m, 1, out, stream);
}

cslc_status hca_compress(const cslc_bf16* c, const cslc_bf16* z, const cslc_bf16* pos_bias, int B, int L,
                         int D, int m_prime, cslc_bf16* out, cslc_stream_t stream) {
  REQUIRE(B >= 0 && L >= 0, CSLC_ERR_SHAPE, "hca_compress: negative size");
  REQUIRE(D == kD || D == kDI, CSLC_ERR_UNSUPPORTED, "hca_compress: D must be 128 or 64 (got %d)", D);
  REQUIRE(is_pow2(m_prime) && m_prime <= 128, CSLC_ERR_UNSUPPORTED,
          "hca_compress: m' must be a power of two <= 128");
  if ((long long)B * (L / m_prime) == 0) return CSLC_OK;
  REQUIRE_PTR(c); REQUIRE_PTR(z); REQUIRE_PTR(pos_bias); REQUIRE_PTR(out);
  return launch_compress(c, z, nullptr, nullptr, pos_bias, B, L, D, m_prime, 0, out, stream);
}

static cslc_status front_end_common(const char* fn, const cslc_bf16* h, const cslc_bf16* W,
                                    const cslc_bf16* pos_bias, int B, int L, int d_model, cslc_bf16* out) {
  REQUIRE(B >= 0 && L >= 0 && d_model >= 0, CSLC_ERR_SHAPE, "%s: negative size", fn);
  REQUIRE(d_model >= 64 && d_model % 64 == 0 && d_model <= 65536, CSLC_ERR_UNSUPPORTED,
          "%s: d_model must be a multiple of 64 in [64, 65536]", fn);
  REQUIRE((long long)B * L < (1ll << 31), CSLC_ERR_UNSUPPORTED, "%s: B * L must be below 2^31", fn);
  REQUIRE_PTR(h); REQUIRE_PTR(W); REQUIRE_PTR(pos_bias); REQUIRE_PTR(out);
  return CSLC_OK;
}

cslc_status csa_compress_front_end(const cslc_bf16* h, const cslc_bf16* W, const cslc_bf16* pos_bias, int B, int L,
                                   int d_model, int m, cslc_bf16* out, cslc_stream_t stream) {
  REQUIRE(is_pow2(m) && m <= 64, CSLC_ERR_UNSUPPORTED, "csa_compress_front_end: m must be a power of two <= 64");
  if (B >= 0 && L >= 0 && (long long)B * (L / m) == 0) return CSLC_OK;
  const cslc_status st = front_end_common("csa_compress_front_end", h, W, pos_bias, B, L, d_model, out);
  if (st != CSLC_OK) return st;
  return launch_front_end(h, W, pos_bias, B, L, d_model, m, 1, out, stream);
}

cslc_status hca_compress_front_end(const cslc_bf16* h, const cslc_bf16* W, const cslc_bf16* pos_bias, int B, int L,
                                   int d_model, int m_prime, cslc_bf16* out, cslc_stream_t stream) {
  REQUIRE(m_prime == 128, CSLC_ERR_UNSUPPORTED, "hca_compress_front_end: m' must be 128");
  if (B >= 0 && L >= 0 && (long long)B * (L / m_prime) == 0) return CSLC_OK;
  const cslc_status st = front_end_common("hca_compress_front_end", h, W, pos_bias, B, L, d_model, out);
  if (st != CSLC_OK) return st;
  return launch_front_end(h, W, pos_bias, B, L, d_model, m_prime, 0, out, stream);
}

static size_t indexer_ws_bytes(int B, int L, int Nc, int score_bytes, int scores_given) {
  if (scores_given || B <= 0 || L <= 0 || Nc <= 0) return 0;
  const int rows = score_block_rows(Nc, score_bytes);
  const int R = L < rows ? L : rows;
  const int n_buf = L > R ? 2 : 1;
  return (size_t)n_buf * B * R * Nc * score_bytes;
}

// The indexer's operands: bf16 q_I / k_I, or e4m3 codes with per-row scales.
struct IndexerOperands {
  const void* q;
  const cslc_bf16* w;
  const void* k;
  const float* q_scale;
  const float* k_scale;
  bool fp8;
};

// Scores of rows [r0, r1) into buf ([B][R][Nc]; fp32, or bf16 when bf16).
static cslc_status launch_scores(const IndexerOperands& op, int B, int L, int Nc, int HI, int m, int q_pos0, int r0,
                                 int r1, void* buf, bool bf16, int R, cudaStream_t stream) {
  if (op.fp8)
    return launch_indexer_scores_fp8(static_cast<const uint8_t*>(op.q), op.q_scale, op.w,
                                     static_cast<const uint8_t*>(op.k), op.k_scale, B, L, Nc, HI, m, q_pos0, r0, r1,
                                     static_cast<float*>(buf), R, stream);
  return launch_indexer_scores(static_cast<const uint16_t*>(op.q), op.w, static_cast<const uint16_t*>(op.k), B, L,
                               Nc, HI, m, q_pos0, r0, r1, buf, bf16, R, stream);
}

// The indexer and the top-k, with fp32 or bf16 scores (bf16: each fp32 score
// rounded to nearest even before it is stored and selected on).
static cslc_status indexer_topk_impl(const char* fn, const IndexerOperands& op, int B, int L, int Nc, int HI, int dI,
                                     int m, int q_pos0, int topk, void* scores, bool bf16, int32_t* idx, void* ws,
                                     size_t ws_bytes, cudaStream_t stream) {
  REQUIRE(B >= 0 && L >= 0 && Nc >= 0 && q_pos0 >= 0 && m >= 1, CSLC_ERR_SHAPE, "%s: negative size / m < 1", fn);
  REQUIRE(dI == kDI, CSLC_ERR_UNSUPPORTED, "%s: d_I must be 64 (got %d)", fn, dI);
  REQUIRE(HI >= 1 && HI <= 16, CSLC_ERR_UNSUPPORTED, "%s: H_I must be in [1, 16]", fn);
  REQUIRE(topk >= 1 && topk <= kMaxTopk, CSLC_ERR_UNSUPPORTED, "%s: topk must be in [1, 2048]", fn);
  REQUIRE(Nc <= kMaxPrefillTopkNc, CSLC_ERR_UNSUPPORTED, "%s: Nc must be <= %d", fn, kMaxPrefillTopkNc);
  if ((long long)B * L == 0) return CSLC_OK;
  REQUIRE_PTR(idx);
  if (Nc > 0) {
    const void* q_idx = op.q;
    const void* k_idx = op.k;
    const cslc_bf16* w = op.w;
    REQUIRE_PTR(q_idx); REQUIRE_PTR(w); REQUIRE_PTR(k_idx);
    if (op.fp8) {
      const float* q_scale = op.q_scale;
      const float* k_scale = op.k_scale;
      REQUIRE_PTR(q_scale); REQUIRE_PTR(k_scale);
    }
  }
  if (scores) REQUIRE_PTR(scores);
  const int sb = bf16 ? 2 : 4;
  const size_t need = indexer_ws_bytes(B, L, Nc, sb, scores != nullptr);
  if (need) {
    REQUIRE(ws != nullptr && ws_bytes >= need, CSLC_ERR_WORKSPACE, "%s: workspace of %zu bytes needed", fn, need);
    REQUIRE(aligned16(ws), CSLC_ERR_ALIGN, "%s: ws is not 16-byte aligned", fn);
  }
  cslc_status st;
  if (scores) {
    st = launch_scores(op, B, L, Nc, HI, m, q_pos0, 0, L, scores, bf16, L, stream);
    if (st != CSLC_OK) return st;
    return launch_topk_rows(scores, bf16, L, 0, L, B, L, Nc, m, q_pos0, topk, idx, stream);
  }
  const int rows = score_block_rows(Nc, sb);
  const int R = L < rows ? L : rows;
  uint8_t* buf = static_cast<uint8_t*>(ws);
  if (L <= R || Nc == 0) {
    if (Nc > 0) {
      st = launch_scores(op, B, L, Nc, HI, m, q_pos0, 0, L, buf, bf16, R, stream);
      if (st != CSLC_OK) return st;
    }
    return launch_topk_rows(buf, bf16, R, 0, L, B, L, Nc, m, q_pos0, topk, idx, stream);
  }
  BlockOverlap* o = nullptr;
  st = block_overlap(&o);
  if (st != CSLC_OK) return st;
  const size_t block_bytes = (size_t)B * R * Nc * sb;
  int last = 0;
  for (int i = 0, r0 = 0; r0 < L; ++i, r0 += R) {
    const int r1 = r0 + R < L ? r0 + R : L;
    const int j = i & 1;
    uint8_t* bj = buf + j * block_bytes;
    cudaError_t e = i >= 2 ? cudaStreamWaitEvent(stream, o->freed[j], 0) : cudaSuccess;
    if (e != cudaSuccess) return set_error(CSLC_ERR_CUDA, "%s: %s", fn, cudaGetErrorString(e));
    st = launch_scores(op, B, L, Nc, HI, m, q_pos0, r0, r1, bj, bf16, R, stream);
    if (st != CSLC_OK) return st;
    e = cudaEventRecord(o->ready[j], stream);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(o->aux, o->ready[j], 0);
    if (e != cudaSuccess) return set_error(CSLC_ERR_CUDA, "%s: %s", fn, cudaGetErrorString(e));
    st = launch_topk_rows(bj, bf16, R, r0, r1, B, L, Nc, m, q_pos0, topk, idx, o->aux);
    if (st != CSLC_OK) return st;
    e = cudaEventRecord(o->freed[j], o->aux);
    if (e != cudaSuccess) return set_error(CSLC_ERR_CUDA, "%s: %s", fn, cudaGetErrorString(e));
    last = j;
  }
  // join: `stream` continues after the last top-k (the auxiliary stream runs in order)
  const cudaError_t e = cudaStreamWaitEvent(stream, o->freed[last], 0);
  if (e != cudaSuccess) return set_error(CSLC_ERR_CUDA, "%s: %s", fn, cudaGetErrorString(e));
  return CSLC_OK;
}

static cslc_status topk_impl(const char* fn, const void* scores, bool bf16, int B, int L, int Nc, int m, int q_pos0,
                             int topk, int32_t* idx, cudaStream_t stream) {
  REQUIRE(B >= 0 && L >= 0 && Nc >= 0 && q_pos0 >= 0 && m >= 1, CSLC_ERR_SHAPE, "%s: bad size", fn);
  REQUIRE(topk >= 1 && topk <= kMaxTopk, CSLC_ERR_UNSUPPORTED, "%s: topk must be in [1, 2048]", fn);
  REQUIRE(Nc <= kMaxPrefillTopkNc, CSLC_ERR_UNSUPPORTED, "%s: Nc must be <= %d", fn, kMaxPrefillTopkNc);
  if ((long long)B * L == 0) return CSLC_OK;
  REQUIRE_PTR(idx);
  if (Nc > 0) REQUIRE_PTR(scores);
  return launch_topk_rows(scores, bf16, L, 0, L, B, L, Nc, m, q_pos0, topk, idx, stream);
}

size_t csa_indexer_topk_workspace_bytes(int B, int L, int Nc, int HI, int topk, int scores_given) {
  (void)HI; (void)topk;
  return indexer_ws_bytes(B, L, Nc, 4, scores_given);
}

cslc_status csa_indexer_topk(const cslc_bf16* q_idx, const cslc_bf16* w, const cslc_bf16* k_idx, int B,
                             int L, int Nc, int HI, int dI, int m, int q_pos0, int topk, float* scores,
                             int32_t* idx, void* ws, size_t ws_bytes, cslc_stream_t stream) {
  const IndexerOperands op{q_idx, w, k_idx, nullptr, nullptr, false};
  return indexer_topk_impl("csa_indexer_topk", op, B, L, Nc, HI, dI, m, q_pos0, topk, scores, false, idx, ws, ws_bytes,
                           stream);
}

size_t csa_indexer_topk_bf16_workspace_bytes(int B, int L, int Nc, int HI, int topk, int scores_given) {
  (void)HI; (void)topk;
  return indexer_ws_bytes(B, L, Nc, 2, scores_given);
}

cslc_status csa_indexer_topk_bf16(const cslc_bf16* q_idx, const cslc_bf16* w, const cslc_bf16* k_idx, int B,
                                  int L, int Nc, int HI, int dI, int m, int q_pos0, int topk, cslc_bf16* scores,
                                  int32_t* idx, void* ws, size_t ws_bytes, cslc_stream_t stream) {
  const IndexerOperands op{q_idx, w, k_idx, nullptr, nullptr, false};
  return indexer_topk_impl("csa_indexer_topk_bf16", op, B, L, Nc, HI, dI, m, q_pos0, topk, scores, true, idx, ws,
                           ws_bytes, stream);
}

cslc_status csa_indexer_topk_fp8(const uint8_t* q8, const float* q_scale, const cslc_bf16* w, const uint8_t* k8,
                                 const float* k_scale, int B, int L, int Nc, int HI, int dI, int m, int q_pos0,
                                 int topk, float* scores, int32_t* idx, void* ws, size_t ws_bytes,
                                 cslc_stream_t stream) {
  const IndexerOperands op{q8, w, k8, q_scale, k_scale, true};
  return indexer_topk_impl("csa_indexer_topk_fp8", op, B, L, Nc, HI, dI, m, q_pos0, topk, scores, false, idx, ws,
                           ws_bytes, stream);
}

cslc_status cslc_quantize_rows_e4m3(const cslc_bf16* x, int64_t rows, int d, uint8_t* codes, float* scales,
                                    cslc_stream_t stream) {
  REQUIRE(rows >= 0, CSLC_ERR_SHAPE, "cslc_quantize_rows_e4m3: negative size");
  REQUIRE(d == 64, CSLC_ERR_UNSUPPORTED, "cslc_quantize_rows_e4m3: d must be 64 (got %d)", d);
  REQUIRE(rows <= (1ll << 34), CSLC_ERR_UNSUPPORTED, "cslc_quantize_rows_e4m3: at most 2^34 rows");
  if (rows == 0) return CSLC_OK;
  REQUIRE_PTR(x); REQUIRE_PTR(codes); REQUIRE_PTR(scales);
  return launch_quantize_rows64(x, rows, codes, scales, stream);
}

cslc_status csa_topk(const float* scores, int B, int L, int Nc, int m, int q_pos0, int topk, int32_t* idx,
                     cslc_stream_t stream) {
  return topk_impl("csa_topk", scores, false, B, L, Nc, m, q_pos0, topk, idx, stream);
}

cslc_status csa_topk_bf16(const cslc_bf16* scores, int B, int L, int Nc, int m, int q_pos0, int topk, int32_t* idx,
                          cslc_stream_t stream) {
  return topk_impl("csa_topk_bf16", scores, true, B, L, Nc, m, q_pos0, topk, idx, stream);
}

cslc_status csa_sparse_attn(const cslc_bf16* q, const cslc_bf16* kv, const int32_t* idx, int B, int L, int H,
                            int D, int Nc, int topk, float scale, cslc_bf16* out, float* lse,
                            cslc_stream_t stream) {
  REQUIRE(B >= 0 && L >= 0 && Nc >= 0, CSLC_ERR_SHAPE, "csa_sparse_attn: negative size");
  REQUIRE(D == kD, CSLC_ERR_UNSUPPORTED, "csa_sparse_attn: D must be 128");
  REQUIRE(H >= 16 && H <= 128 && H % 16 == 0, CSLC_ERR_UNSUPPORTED,
          "csa_sparse_attn: H must be a multiple of 16 in [16, 128]");
  REQUIRE(topk >= 1 && topk <= kMaxTopk, CSLC_ERR_UNSUPPORTED, "csa_sparse_attn: topk must be in [1, 2048]");
  if ((long long)B * L == 0) return CSLC_OK;
  REQUIRE_PTR(q); REQUIRE_PTR(idx); REQUIRE_PTR(out);
  if (Nc > 0) REQUIRE_PTR(kv);
  if (lse) REQUIRE_PTR(lse);
  return launch_sparse_attn_sm100(q, kv, idx, B, L, H, Nc, topk, scale, out, lse, stream);
}

cslc_status hca_dense_attn(const cslc_bf16* q, const cslc_bf16* kv, int B, int L, int H, int D, int Nc,
                           int m_prime, int q_pos0, float scale, cslc_bf16* out, float* lse,
                           cslc_stream_t stream) {
  REQUIRE(B >= 0 && L >= 0 && Nc >= 0 && q_pos0 >= 0 && m_prime >= 1, CSLC_ERR_SHAPE,
          "hca_dense_attn: bad size");
  REQUIRE(D == kD, CSLC_ERR_UNSUPPORTED, "hca_dense_attn: D must be 128");
  REQUIRE(H >= 16 && H <= 128 && H % 16 == 0, CSLC_ERR_UNSUPPORTED,
          "hca_dense_attn: H must be a multiple of 16 in [16, 128]");
  if ((long long)B * L == 0) return CSLC_OK;
  REQUIRE_PTR(q); REQUIRE_PTR(out);
  if (Nc > 0) REQUIRE_PTR(kv);
  if (lse) REQUIRE_PTR(lse);
  return launch_dense_attn_sm100(q, kv, B, L, H, Nc, m_prime, q_pos0, scale, out, lse, stream);
}

cslc_status cslc_quantize_kv_mixed(const cslc_bf16* kv, int B, int N, uint8_t* nope, cslc_bf16* rope,
                                   float* scale, cslc_stream_t stream) {
  REQUIRE(B >= 0 && N >= 0, CSLC_ERR_SHAPE, "cslc_quantize_kv_mixed: negative size");
  if ((long long)B * N == 0) return CSLC_OK;
  REQUIRE_PTR(kv); REQUIRE_PTR(nope); REQUIRE_PTR(rope); REQUIRE_PTR(scale);
  return launch_quantize_kv(kv, (long long)B * N, nope, rope, scale, stream);
}

size_t cslc_decode_workspace_bytes(const cslc_decode_layer* layers, int n_layers, int B, int H, int HI) {
  (void)HI;
  if (layers == nullptr || n_layers <= 0 || B <= 0 || H <= 0) return 0;
  return decode_workspace_bytes(layers, n_layers, B, H);
}

cslc_status cslc_decode_step(const cslc_decode_layer* layers, int n_layers, int B, int H, int D, int HI,
                             int dI, void* ws, size_t ws_bytes, cslc_stream_t stream) {
  REQUIRE(layers != nullptr || n_layers == 0, CSLC_ERR_NULL, "cslc_decode_step: layers is NULL");
  REQUIRE(n_layers >= 0 && B >= 0, CSLC_ERR_SHAPE, "cslc_decode_step: negative size");
  REQUIRE(D == kD && dI == kDI, CSLC_ERR_UNSUPPORTED, "cslc_decode_step: D must be 128 and d_I 64");
  REQUIRE(H >= 16 && H <= 128 && H % 16 == 0, CSLC_ERR_UNSUPPORTED,
          "cslc_decode_step: H must be a multiple of 16 in [16, 128]");
  REQUIRE(HI >= 1 && HI <= 16, CSLC_ERR_UNSUPPORTED, "cslc_decode_step: H_I must be in [1, 16]");
  if (n_layers == 0 || B == 0) return CSLC_OK;
  for (int i = 0; i < n_layers; ++i) {
    const cslc_decode_layer& l = layers[i];
    REQUIRE(l.kind == 0 || l.kind == 1, CSLC_ERR_UNSUPPORTED, "cslc_decode_step: layer %d kind must be 0 or 1", i);
    REQUIRE(l.n_max >= 0, CSLC_ERR_SHAPE, "cslc_decode_step: layer %d n_max < 0", i);
    REQUIRE_PTR(l.q); REQUIRE_PTR(l.out); REQUIRE_PTR(l.n_entries);
    if (l.n_max > 0) { REQUIRE_PTR(l.nope); REQUIRE_PTR(l.rope); REQUIRE_PTR(l.kv_scale); }
    if (l.kind == 0) {
      REQUIRE(l.topk >= 1 && l.topk <= kMaxTopk, CSLC_ERR_UNSUPPORTED, "cslc_decode_step: layer %d topk", i);
      if (l.n_max > 0) { REQUIRE_PTR(l.q_idx); REQUIRE_PTR(l.w); REQUIRE_PTR(l.k_idx); }
      if (l.idx_out) REQUIRE_PTR(l.idx_out);
      if (l.scores_out) REQUIRE_PTR(l.scores_out);
    }
  }
  const size_t need = decode_workspace_bytes(layers, n_layers, B, H);
  REQUIRE(ws != nullptr && ws_bytes >= need, CSLC_ERR_WORKSPACE,
          "cslc_decode_step: workspace of %zu bytes needed", need);
  REQUIRE(aligned16(ws), CSLC_ERR_ALIGN, "cslc_decode_step: ws is not 16-byte aligned");
  return run_decode_step(layers, n_layers, B, H, HI, ws, ws_bytes, stream);
}

cslc_status cslc_decode_append(const cslc_bf16* c, const cslc_bf16* z, const cslc_bf16* k_c, const cslc_bf16* k_z,
                               const cslc_bf16* pos_bias, const cslc_bf16* k_pos_bias, const int32_t* pos, int B,
                               int m, int overlap, cslc_bf16* ring_c, cslc_bf16* ring_z, cslc_bf16* ring_kc,
                               cslc_bf16* ring_kz, uint8_t* nope, cslc_bf16* rope, float* kv_scale, cslc_bf16* k_idx,
                               int n_max, int32_t* n_entries, cslc_stream_t stream) {
  REQUIRE(B >= 0 && n_max >= 0, CSLC_ERR_SHAPE, "cslc_decode_append: negative size");
  REQUIRE(is_pow2(m) && m <= 128, CSLC_ERR_UNSUPPORTED, "cslc_decode_append: m must be a power of two <= 128");
  REQUIRE(overlap == 0 || overlap == 1, CSLC_ERR_UNSUPPORTED, "cslc_decode_append: overlap must be 0 or 1");
  REQUIRE((k_c == nullptr) == (k_z == nullptr) && (k_c == nullptr) == (k_pos_bias == nullptr) &&
              (k_c == nullptr) == (ring_kc == nullptr) && (k_c == nullptr) == (ring_kz == nullptr) &&
              (k_c == nullptr) == (k_idx == nullptr),
          CSLC_ERR_NULL, "cslc_decode_append: give all of k_c, k_z, k_pos_bias, ring_kc, ring_kz, k_idx or none");
  if (B == 0) return CSLC_OK;
  REQUIRE_PTR(c); REQUIRE_PTR(z); REQUIRE_PTR(pos_bias); REQUIRE_PTR(pos); REQUIRE_PTR(ring_c); REQUIRE_PTR(ring_z);
  REQUIRE_PTR(n_entries);
  if (n_max > 0) { REQUIRE_PTR(nope); REQUIRE_PTR(rope); REQUIRE_PTR(kv_scale); }
  if (k_c) {
    REQUIRE_PTR(k_c); REQUIRE_PTR(k_z); REQUIRE_PTR(k_pos_bias); REQUIRE_PTR(ring_kc); REQUIRE_PTR(ring_kz);
    if (n_max > 0) REQUIRE_PTR(k_idx);
  }
  return launch_decode_append(c, z, k_c, k_z, pos_bias, k_pos_bias, pos, B, m, overlap, ring_c, ring_z, ring_kc,
                              ring_kz, nope, rope, kv_scale, k_idx, n_max, n_entries, stream);
}

size_t cslc_decode_topk_workspace_bytes(int B, int n_max, int topk) {
  if (B <= 0 || n_max < 0 || topk <= 0) return 0;
  return decode_topk_workspace_bytes(B, n_max, topk);
}

cslc_status cslc_decode_topk(const float* scores, const int32_t* n_entries, int B, int n_max, int topk,
                             int32_t* idx, void* ws, size_t ws_bytes, cslc_stream_t stream) {
  REQUIRE(B >= 0 && n_max >= 0, CSLC_ERR_SHAPE, "cslc_decode_topk: negative size");
  REQUIRE(topk >= 1 && topk <= kMaxTopk, CSLC_ERR_UNSUPPORTED, "cslc_decode_topk: topk must be in [1, 2048]");
  if (B == 0) return CSLC_OK;
  REQUIRE_PTR(n_entries); REQUIRE_PTR(idx);
  if (n_max > 0) REQUIRE_PTR(scores);
  const size_t need = decode_topk_workspace_bytes(B, n_max, topk);
  REQUIRE(ws != nullptr && ws_bytes >= need, CSLC_ERR_WORKSPACE,
          "cslc_decode_topk: workspace of %zu bytes needed", need);
  REQUIRE(aligned16(ws), CSLC_ERR_ALIGN, "cslc_decode_topk: ws is not 16-byte aligned");
  return run_decode_topk(scores, n_entries, B, n_max, topk, idx, ws, stream);
}

}  // extern "C"
