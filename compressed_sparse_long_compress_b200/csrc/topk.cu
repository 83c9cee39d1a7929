// Exact per-row top-k selection for prefill (first page §1.1: each query keeps
// k = 1024 compressed entries; "读完这篇你就搞懂 DeepSeek v4 了", §三 闪电索引: keep
// the top-k by indexer score).
//
// Rule: the min(k, n_vis) visible entries with the largest fp32 score, ties
// to the smaller entry index, emitted in ascending index order, -1 padded.
//
// One CTA per query row. The row's visible scores are mapped to
// order-preserving uint32 keys in shared memory, the k-th largest key is found
// by a most-significant-digit radix select (8-bit digits, per-warp histograms
// with warp-aggregated shared-memory atomics; it stops early once every key
// sharing the chosen prefix is known to be selected), and the selection is
// compacted in index order with warp ballots: one pass counts per warp
// segment, one writes. Ties at the threshold take the smallest indices.

#include "common.cuh"

namespace cslc {

constexpr int TOPK_THREADS = 512;
constexpr int TOPK_WARPS = TOPK_THREADS / 32;

struct RadixResult {
  uint32_t prefix, mask;
  int remaining;   // how many keys equal to the prefix (under mask) are still to take
  int take_all;    // every key matching the prefix is selected
};

// Block-wide radix select of the `k`-th largest key among keys[0..n).
// Requires blockDim.x == TOPK_THREADS and k <= n. hist: TOPK_WARPS * 256 words.
__device__ RadixResult radix_select(const uint32_t* keys, int n, int k, uint32_t* hist,
                                    int* bcast) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  RadixResult r{0u, 0u, k, 0};
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int x = tid; x < TOPK_WARPS * 256; x += TOPK_THREADS) hist[x] = 0;
    if (tid == 0) { bcast[0] = 0; bcast[1] = 0; bcast[2] = 0; }
    __syncthreads();
    uint32_t* hw = hist + warp * 256;
    for (int i = tid; i < n; i += TOPK_THREADS) {
      const uint32_t key = keys[i];
      if ((key & r.mask) == r.prefix) {
        const uint32_t d = (key >> shift) & 255u;
        const unsigned peers = __match_any_sync(__activemask(), d);
        if (lane == __ffs(peers) - 1) atomicAdd(&hw[d], (uint32_t)__popc(peers));
      }
    }
    __syncthreads();
    if (tid < 256) {
      uint32_t s = 0;
      for (int w = 0; w < TOPK_WARPS; ++w) s += hist[w * 256 + tid];
      hist[tid] = s;   // warp 0's copy becomes the total (read below only after the sync)
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns digits 255-8l .. 248-8l (descending)
      uint32_t cnt[8], lane_sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) { cnt[j] = hist[255 - 8 * lane - j]; lane_sum += cnt[j]; }
      uint32_t incl = lane_sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const uint32_t excl = incl - lane_sum;
      const uint32_t need = (uint32_t)r.remaining;
      if (excl < need && incl >= need) {
        uint32_t above = excl;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (above + cnt[j] >= need) {
            bcast[0] = 255 - 8 * lane - j;
            bcast[1] = (int)above;
            bcast[2] = (int)cnt[j];
            break;
          }
          above += cnt[j];
        }
      }
    }
    __syncthreads();
    const uint32_t d = (uint32_t)bcast[0];
    const int above = bcast[1], cnt_d = bcast[2];
    __syncthreads();
    r.remaining -= above;
    r.prefix |= d << shift;
    r.mask |= 255u << shift;
    if (cnt_d == r.remaining) { r.take_all = 1; break; }
  }
  return r;
}

// Compacts the selected indices of keys[0..n) into out[] in ascending index
// order (exactly k of them). wsum: 2 * TOPK_WARPS ints of shared memory.
__device__ void emit_selection(const uint32_t* keys, int n, const RadixResult& r, int32_t* out,
                               int k, int* wsum) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int seg = ((n + TOPK_WARPS - 1) / TOPK_WARPS + 31) & ~31;
  const int lo = warp * seg, hi = min(n, lo + seg);
  const unsigned lt = (1u << lane) - 1u;
  // pass 1: per-warp counts of "equal" keys (for the tie rank) and "greater" keys
  int n_eq = 0, n_gt = 0;
  for (int base = lo; base < hi; base += 32) {
    const int i = base + lane;
    const uint32_t key = i < hi ? (keys[i] & r.mask) : 0u;
    const bool valid = i < hi;
    n_eq += __popc(__ballot_sync(0xffffffffu, valid && key == r.prefix));
    n_gt += __popc(__ballot_sync(0xffffffffu, valid && key > r.prefix));
  }
  if (lane == 0) { wsum[warp] = n_eq; wsum[TOPK_WARPS + warp] = n_gt; }
  __syncthreads();
  int eq_before = 0, sel_before = 0;
  {
    int eq_acc = 0;
    for (int w = 0; w < TOPK_WARPS; ++w) {
      const int e = wsum[w], g = wsum[TOPK_WARPS + w];
      const int take_eq = r.take_all ? e : max(0, min(e, r.remaining - eq_acc));
      if (w < warp) { eq_before += e; sel_before += g + take_eq; }
      eq_acc += e;
    }
  }
  __syncthreads();
  // pass 2: write
  int eq_run = eq_before, sel_run = sel_before;
  for (int base = lo; base < hi; base += 32) {
    const int i = base + lane;
    const bool valid = i < hi;
    const uint32_t key = valid ? (keys[i] & r.mask) : 0u;
    const bool is_eq = valid && key == r.prefix;
    const unsigned eq_mask = __ballot_sync(0xffffffffu, is_eq);
    const int eq_rank = eq_run + __popc(eq_mask & lt);
    const bool sel = valid && (key > r.prefix || (is_eq && (r.take_all || eq_rank < r.remaining)));
    const unsigned sel_mask = __ballot_sync(0xffffffffu, sel);
    const int pos = sel_run + __popc(sel_mask & lt);
    if (sel && pos < k) out[pos] = i;
    eq_run += __popc(eq_mask);
    sel_run += __popc(sel_mask);
  }
}

constexpr int TK_BINS = 4096;   // value-range histogram bins (shares storage with the radix histogram)
constexpr int TK_CAND = 2048;   // threshold-bin candidates handled in shared memory

// Compacts the indices i in [0, n) with pred(i) into out[] in ascending order
// (at most k are written): per-warp counts over contiguous segments, then a
// second pass writes. wsum: TOPK_WARPS ints.
template <class Pred>
__device__ void emit_where(Pred pred, int n, int32_t* out, int k, int* wsum) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int seg = ((n + TOPK_WARPS - 1) / TOPK_WARPS + 31) & ~31;
  const int lo = warp * seg, hi = min(n, lo + seg);
  const unsigned lt = (1u << lane) - 1u;
  int cnt = 0;
  for (int base = lo; base < hi; base += 32) {
    const int i = base + lane;
    cnt += __popc(__ballot_sync(0xffffffffu, i < hi && pred(i)));
  }
  if (lane == 0) wsum[warp] = cnt;
  __syncthreads();
  int run = 0;
  for (int w = 0; w < warp; ++w) run += wsum[w];
  for (int base = lo; base < hi; base += 32) {
    const int i = base + lane;
    const bool sel = i < hi && pred(i);
    const unsigned m = __ballot_sync(0xffffffffu, sel);
    const int pos = run + __popc(m & lt);
    if (sel && pos < k) out[pos] = i;
    run += __popc(m);
  }
}

__device__ __forceinline__ uint64_t composite(float v, int i) {
  return ((uint64_t)float_key(v) << 32) | (uint64_t)(0xffffffffu - (uint32_t)i);
}

// One CTA per query row. Fast path: the row's min / max define 4096 equal
// value bins; the bin holding the k-th largest score is found from a
// histogram, every score in a higher bin is selected, and the remaining
// slots go to the candidates of that bin ranked by (score desc, index asc).
// Rows where that bin is too crowded (or the range is degenerate) take the
// exact 8-bit radix select over order-preserving keys.
__global__ void __launch_bounds__(TOPK_THREADS) topk_rows_kernel(
    const float* __restrict__ scores, int rows_in_buf, int row_begin, int L, int Nc, int m,
    int q_pos0, int topk, int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) float vals[];
  __shared__ uint32_t hist[TK_BINS];
  __shared__ uint64_t cand[TK_CAND];
  __shared__ float red[2][TOPK_WARPS];
  __shared__ uint32_t wtot[TOPK_WARPS];
  __shared__ int bcast[4];
  __shared__ int wsum[2 * TOPK_WARPS];
  __shared__ int n_cand;
  __shared__ uint64_t thr_comp;
  const int r = row_begin + blockIdx.x;
  const int b = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nv = n_visible((long long)q_pos0 + r, m, Nc);
  int32_t* out = idx + ((size_t)b * L + r) * topk;
  if (nv <= topk) {
    for (int j = tid; j < topk; j += TOPK_THREADS) out[j] = j < nv ? j : -1;
    return;
  }
  for (int x = tid; x < TK_BINS; x += TOPK_THREADS) hist[x] = 0;
  if (tid == 0) n_cand = 0;
  // load the visible scores, tracking min / max
  const float* srow = scores + ((size_t)b * rows_in_buf + (r - row_begin)) * (size_t)Nc;
  float vmin = INFINITY, vmax = -INFINITY;
  int done = 0;
  if ((Nc & 3) == 0) {
    const int n4 = nv >> 2;
    for (int j = tid; j < n4; j += TOPK_THREADS) {
      const float4 v = __ldcs(reinterpret_cast<const float4*>(srow) + j);
      reinterpret_cast<float4*>(vals)[j] = v;
      vmin = fminf(fminf(vmin, v.x), fminf(fminf(v.y, v.z), v.w));
      vmax = fmaxf(fmaxf(vmax, v.x), fmaxf(fmaxf(v.y, v.z), v.w));
    }
    done = n4 << 2;
  }
  for (int j = done + tid; j < nv; j += TOPK_THREADS) {
    const float v = __ldcs(srow + j);
    vals[j] = v;
    vmin = fminf(vmin, v);
    vmax = fmaxf(vmax, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, o));
    vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
  }
  if (lane == 0) { red[0][warp] = vmin; red[1][warp] = vmax; }
  __syncthreads();
  float lo = red[0][0], hi = red[1][0];
  for (int w = 1; w < TOPK_WARPS; ++w) { lo = fminf(lo, red[0][w]); hi = fmaxf(hi, red[1][w]); }
  const float span = hi - lo;
  bool fast = span > 0.f && isfinite(span);
  const float bscale = fast ? ((float)TK_BINS - 0.5f) / span : 0.f;
  auto bin_of = [&](float v) { return min(TK_BINS - 1, (int)((v - lo) * bscale)); };
  int T = 0, remaining = 0;
  if (fast) {
    for (int j = tid; j < nv; j += TOPK_THREADS) atomicAdd(&hist[bin_of(vals[j])], 1u);
    __syncthreads();
    // thread t owns bins 4095 - 8t .. 4088 - 8t (descending); find the bin holding the k-th largest
    uint32_t c[8], s = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) { c[j] = hist[TK_BINS - 1 - 8 * tid - j]; s += c[j]; }
    uint32_t incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) wtot[warp] = incl;
    __syncthreads();
    uint32_t before = 0;
    for (int w = 0; w < warp; ++w) before += wtot[w];
    incl += before;
    const uint32_t excl = incl - s;
    if (excl < (uint32_t)topk && incl >= (uint32_t)topk) {
      uint32_t above = excl;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (above + c[j] >= (uint32_t)topk) {
          bcast[0] = TK_BINS - 1 - 8 * tid - j;
          bcast[1] = (int)above;
          bcast[2] = (int)c[j];
          break;
        }
        above += c[j];
      }
    }
    __syncthreads();
    T = bcast[0];
    remaining = topk - bcast[1];
    const int cntT = bcast[2];
    if (cntT == remaining) {
      emit_where([&](int i) { return bin_of(vals[i]) >= T; }, nv, out, topk, wsum);
      return;
    }
    if (cntT > TK_CAND) fast = false;
  }
  if (fast) {
    // candidates of bin T, then the remaining-th largest (score desc, index asc)
    for (int j = tid; j < nv; j += TOPK_THREADS) {
      const float v = vals[j];
      if (bin_of(v) == T) cand[atomicAdd(&n_cand, 1)] = composite(v, j);
    }
    __syncthreads();
    const int C = n_cand;
    if (C <= TOPK_THREADS) {
      if (tid < C) {
        const uint64_t me = cand[tid];
        int rank = 0;
        for (int j = 0; j < C; ++j) rank += cand[j] > me;
        if (rank == remaining - 1) thr_comp = me;
      }
    } else {
      int P = 1;
      while (P < C) P <<= 1;
      for (int j = C + tid; j < P; j += TOPK_THREADS) cand[j] = 0ull;
      __syncthreads();
      for (int size = 2; size <= P; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
          for (int i = tid; i < P; i += TOPK_THREADS) {
            const int jx = i ^ stride;
            if (jx > i) {
              const bool desc = (i & size) == 0;
              const uint64_t a = cand[i], c2 = cand[jx];
              if ((a < c2) == desc) { cand[i] = c2; cand[jx] = a; }
            }
          }
          __syncthreads();
        }
      }
      if (tid == 0) thr_comp = cand[remaining - 1];
    }
    __syncthreads();
    const uint64_t tc = thr_comp;
    emit_where([&](int i) {
      const float v = vals[i];
      const int bi = bin_of(v);
      return bi > T || (bi == T && composite(v, i) >= tc);
    }, nv, out, topk, wsum);
    return;
  }
  // exact radix select over order-preserving keys (degenerate value ranges)
  __syncthreads();
  uint32_t* keys = reinterpret_cast<uint32_t*>(vals);
  for (int j = tid; j < nv; j += TOPK_THREADS) keys[j] = float_key(vals[j]);
  __syncthreads();
  const RadixResult rr = radix_select(keys, nv, topk, hist, bcast);
  emit_selection(keys, nv, rr, out, topk, wsum);
}

cslc_status launch_topk_rows(const float* scores, int rows_in_buf, int row_begin, int row_end,
                             int B, int L, int Nc, int m, int q_pos0, int topk, int32_t* idx,
                             cudaStream_t stream) {
  if (row_end <= row_begin || B == 0) return CSLC_OK;
  const size_t smem = (size_t)Nc * 4;
  static int configured_for = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_for != dev) {
    cudaFuncSetAttribute(topk_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         192 * 1024);
    configured_for = dev;
  }
  dim3 grid(row_end - row_begin, B);
  topk_rows_kernel<<<grid, TOPK_THREADS, smem, stream>>>(scores, rows_in_buf, row_begin, L, Nc, m,
                                                         q_pos0, topk, idx);
  return check_launch("topk_rows_kernel");
}

}  // namespace cslc
