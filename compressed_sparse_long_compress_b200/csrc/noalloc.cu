// Allocation-free variant of the decode top-k (cslc_decode_topk_noalloc).
//
// Some callers cannot call cudaMalloc: for example a serving process whose
// device memory is fully planned at start-up, a code path where an
// allocation would synchronise the device and stall other work, or a plain C
// caller with no device allocator of its own. This entry point gives them the
// decode top-k without a caller workspace: its scratch (histogram, counters,
// selected list, candidate buffer) lives in one file-scope device array of
// fixed size that every GPU loading the library holds until the process exits.
//
// Host code must not pass the array's name to a kernel: on the host it is only
// a stand-in symbol. The device address is looked up once per device (with
// that device current) through cudaGetSymbolAddress and cached together with
// the id of the context it belongs to; when the device's context has been
// replaced (cudaDeviceReset, or the primary context released and created
// again) the module is loaded anew and the address is looked up again.

#include <cuda.h>

#include <mutex>

#include "common.cuh"

namespace cslc {

constexpr size_t kNoAllocScratchBytes = 16u << 20;   // 16 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

size_t decode_topk_workspace_bytes(int, int, int);
cslc_status run_decode_topk(const float*, const int32_t*, int, int, int, int32_t*, void*, cudaStream_t);

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {nullptr};
unsigned long long g_noalloc_ctx[kMaxDevices] = {0};   // id of the context the address belongs to

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context (0 when there is none or
// the driver cannot report it). Driver symbols are looked up once.
unsigned long long current_ctx_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  }
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}
}  // namespace

// Device address of the static scratch on the current device (set-up on first
// use, and again whenever the device's context has changed since).
static cslc_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_error(CSLC_ERR_CUDA, "cslc_decode_topk_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return set_error(CSLC_ERR_UNSUPPORTED, "cslc_decode_topk_noalloc: device %d", dev);
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  const unsigned long long ctx = current_ctx_id();
  if (g_noalloc_ptr[dev] == nullptr || ctx == 0 || ctx != g_noalloc_ctx[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);   // also makes the device's primary context current
    if (e != cudaSuccess || p == nullptr)
      return set_error(CSLC_ERR_CUDA, "cslc_decode_topk_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    g_noalloc_ptr[dev] = p;
    g_noalloc_ctx[dev] = current_ctx_id();
  }
  *out = g_noalloc_ptr[dev];
  return CSLC_OK;
}

}  // namespace cslc

using namespace cslc;

extern "C" cslc_status cslc_decode_topk_noalloc(const float* scores, const int32_t* n_entries, int B, int n_max,
                                                int topk, int32_t* idx, cslc_stream_t stream) {
  if (B < 0 || n_max < 0) return set_error(CSLC_ERR_SHAPE, "cslc_decode_topk_noalloc: negative size");
  if (topk < 1 || topk > 2048) return set_error(CSLC_ERR_UNSUPPORTED, "cslc_decode_topk_noalloc: topk must be in [1, 2048]");
  if (B == 0) return CSLC_OK;
  if (n_entries == nullptr || idx == nullptr || (n_max > 0 && scores == nullptr))
    return set_error(CSLC_ERR_NULL, "cslc_decode_topk_noalloc: NULL pointer");
  if (!aligned16(n_entries) || !aligned16(idx) || (scores && !aligned16(scores)))
    return set_error(CSLC_ERR_ALIGN, "cslc_decode_topk_noalloc: pointers must be 16-byte aligned");
  const size_t need = decode_topk_workspace_bytes(B, n_max, topk);
  if (need > kNoAllocScratchBytes)
    return set_error(CSLC_ERR_WORKSPACE,
                     "cslc_decode_topk_noalloc: B=%d, n_max=%d need %zu bytes of scratch; the static scratch holds "
                     "%zu bytes (use cslc_decode_topk with a workspace)",
                     B, n_max, need, kNoAllocScratchBytes);
  void* ws = nullptr;
  const cslc_status st = noalloc_scratch(&ws);
  if (st != CSLC_OK) return st;
  return run_decode_topk(scores, n_entries, B, n_max, topk, idx, ws, stream);
}
