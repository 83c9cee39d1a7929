// Exact per-row top-k selection for prefill (first page §1.1: each query keeps
// k = 1024 compressed entries; "读完这篇你就搞懂 DeepSeek v4 了", §三 闪电索引: keep
// the top-k by indexer score).
//
// Rule: the min(k, n_vis) visible entries with the largest fp32 score, ties
// to the smaller entry index, emitted in ascending index order, -1 padded.
//
// Each row is selected by one small CTA. The fast path (below, at
// topk_rows_kernel) bins the scores into a value-range histogram, ranks only
// the scores near the bin that holds the k-th largest one, and compacts the
// selection in index order. Rows it cannot take map their scores to
// order-preserving uint32 keys and find the k-th largest key by a
// most-significant-digit radix select (8-bit digits, per-warp histograms; it
// stops early once every key sharing the chosen prefix is known to be
// selected); the selection is then compacted in index order with warp
// ballots. Ties at the threshold take the smallest indices.

#include "common.cuh"

namespace cslc {

constexpr int TOPK_THREADS = 128;
constexpr int TOPK_WARPS = TOPK_THREADS / 32;

struct RadixResult {
  uint32_t prefix, mask;
  int remaining;   // how many keys equal to the prefix (under mask) are still to take
  int take_all;    // every key matching the prefix is selected
};

// Block-wide radix select of the `k`-th largest key among key_of(0..n-1).
// Requires blockDim.x == TOPK_THREADS and k <= n. hist: TOPK_WARPS * 256 words.
template <class KeyFn>
__device__ RadixResult radix_select(KeyFn key_of, int n, int k, uint32_t* hist, int* bcast) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  RadixResult r{0u, 0u, k, 0};
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int x = tid; x < TOPK_WARPS * 256; x += TOPK_THREADS) hist[x] = 0;
    if (tid == 0) { bcast[0] = 0; bcast[1] = 0; bcast[2] = 0; }
    __syncthreads();
    uint32_t* hw = hist + warp * 256;
    for (int i = tid; i < n; i += TOPK_THREADS) {
      const uint32_t key = key_of(i);
      if ((key & r.mask) == r.prefix) {
        const uint32_t d = (key >> shift) & 255u;
        const unsigned peers = __match_any_sync(__activemask(), d);
        if (lane == __ffs(peers) - 1) atomicAdd(&hw[d], (uint32_t)__popc(peers));
      }
    }
    __syncthreads();
    for (int d = tid; d < 256; d += TOPK_THREADS) {
      uint32_t s = 0;
      for (int w = 0; w < TOPK_WARPS; ++w) s += hist[w * 256 + d];
      hist[d] = s;   // warp 0's copy becomes the total (read below only after the sync)
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

// Compacts the selected indices of key_of(0..n-1) into out[] in ascending index
// order (exactly k of them). wsum: 2 * TOPK_WARPS ints of shared memory.
template <class KeyFn>
__device__ void emit_selection(KeyFn key_of, int n, const RadixResult& r, int32_t* out, int k,
                               int* wsum) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int seg = ((n + TOPK_WARPS - 1) / TOPK_WARPS + 31) & ~31;
  const int lo = warp * seg, hi = min(n, lo + seg);
  const unsigned lt = (1u << lane) - 1u;
  // pass 1: per-warp counts of "equal" keys (for the tie rank) and "greater" keys
  int n_eq = 0, n_gt = 0;
  for (int base = lo; base < hi; base += 32) {
    const int i = base + lane;
    const uint32_t key = i < hi ? (key_of(i) & r.mask) : 0u;
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
    const uint32_t key = valid ? (key_of(i) & r.mask) : 0u;
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

constexpr int TK_SLICE = 4 * TOPK_THREADS;   // entries per slice
constexpr int TK_BATCH = 8;                  // 16-byte loads per thread in flight
constexpr int TK_BINS = 2048;                // value-range histogram bins
constexpr int TK_CAND = 512;                 // keys near the threshold ranked in shared memory
constexpr float TK_MAGIC = 12582912.f;       // 1.5 * 2^23: adding it leaves round(x) in the low mantissa bits
static_assert(TK_BINS >= TOPK_WARPS * 256, "the value histogram doubles as the radix histograms");
static_assert(TK_BINS == 16 * TOPK_THREADS, "the threshold scan gives each thread 16 bins");

__device__ __forceinline__ uint64_t composite(float v, int i) {
  return ((uint64_t)float_key(v) << 32) | (uint64_t)(0xffffffffu - (uint32_t)i);
}

__device__ __forceinline__ int tk_bin(float v, float lo, float bscale) {
  const float t = fminf(fmaxf(fmaf(v - lo, bscale, TK_MAGIC), TK_MAGIC), TK_MAGIC + (float)(TK_BINS - 1));
  return (int)(__float_as_uint(t) & (uint32_t)(TK_BINS - 1));
}

// Block-wide exclusive scan of one int per thread; also returns the total.
__device__ __forceinline__ int tk_block_excl_scan(int v, int* wtot, int& total) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) wtot[warp] = incl;
  __syncthreads();
  int before = 0;
  total = 0;
#pragma unroll
  for (int w = 0; w < TOPK_WARPS; ++w) {
    const int t = wtot[w];
    before += w < warp ? t : 0;
    total += t;
  }
  return before + incl - v;
}

// One CTA of TOPK_THREADS threads per query row; many rows per SM run side by
// side. The row is read in slices of TK_SLICE entries (thread t reads entries
// 4t..4t+3 of each slice with one 16-byte load); entries past n_vis read NaN.
// Fast path:
//   A. one pass counts every score in a 2048-bin histogram over a value range
//      [lo, hi] taken from one score per thread of the first loads (scores
//      outside clamp to the edge bins, so the binning stays monotone);
//   B. a block scan of the histogram finds the bin T holding the k-th largest
//      score; fp32 bounds lo_T < hi_T are put one and a half bins either side
//      of T. A second pass (the row is still in L2) marks every score above
//      hi_T in a 4-bit mask per four entries (shared memory), counts them
//      exactly and collects the (score, index) keys in (lo_T, hi_T]. With fewer
//      than k above hi_T and at least k above lo_T, the k-th key is among the
//      collected ones: ranking them by (score desc, index asc) picks the
//      remaining ones, whose bits are then set;
//   C. the mask words are counted per thread, scanned across the block, and
//      each thread writes the indices of its set bits in ascending order.
// Rows for which a check fails (degenerate sampled range, too many collected
// keys, bounds that miss the k-th score, e.g. through NaN scores) take the
// exact 8-bit radix select over order-preserving keys read from the row.
// Score rows are fp32, or bf16 (the half-size score path; a bf16 score
// converts to fp32 exactly, so the selection below is the same code).
__device__ __forceinline__ float score_at(const float* p) { return __ldg(p); }
__device__ __forceinline__ float score_at(const uint16_t* p) { return bf16_to_f(__ldg(p)); }
__device__ __forceinline__ float4 score4(const float* p, bool last_use) {
  const float4* v = reinterpret_cast<const float4*>(p);
  return last_use ? __ldcs(v) : __ldg(v);
}
__device__ __forceinline__ float4 score4(const uint16_t* p, bool last_use) {
  const uint2* v = reinterpret_cast<const uint2*>(p);
  const uint2 u = last_use ? __ldcs(v) : __ldg(v);
  return make_float4(bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y));
}

template <typename ScoreT>
__global__ void __launch_bounds__(TOPK_THREADS, 8) topk_rows_kernel(
    const ScoreT* __restrict__ scores, int rows_in_buf, int row_begin, int L, int Nc, int m,
    int q_pos0, int topk, int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) uint32_t nibw[];   // 4-bit masks: entries 16w..16w+15 in word w
  uint8_t* nib = reinterpret_cast<uint8_t*>(nibw);
  __shared__ __align__(16) uint32_t hist[TK_BINS];
  __shared__ uint64_t cand[TK_CAND];
  __shared__ float red[2][TOPK_WARPS];
  __shared__ int wtot[TOPK_WARPS];
  __shared__ int bcast[4];
  __shared__ int wsum[2 * TOPK_WARPS];
  __shared__ int n_cand;
  // rows in decreasing order: the causally heaviest rows start first, so that
  // the last wave holds the light ones
  const int r = row_begin + (int)(gridDim.x - 1 - blockIdx.x);
  const int b = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nv = n_visible((long long)q_pos0 + r, m, Nc);
  int32_t* out = idx + ((size_t)b * L + r) * topk;
  if (nv <= topk) {
    for (int j = tid; j < topk; j += TOPK_THREADS) out[j] = j < nv ? j : -1;
    return;
  }
  const ScoreT* srow = scores + ((size_t)b * rows_in_buf + (r - row_begin)) * (size_t)Nc;
  const int n_sl = (nv + TK_SLICE - 1) / TK_SLICE;
#pragma unroll
  for (int j = 0; j < TK_BINS / (4 * TOPK_THREADS); ++j)
    reinterpret_cast<uint4*>(hist)[j * TOPK_THREADS + tid] = make_uint4(0u, 0u, 0u, 0u);
  if (tid == 0) n_cand = 0;
  const bool vec = (Nc & 3) == 0;   // rows start 16-byte (fp32) / 8-byte (bf16) aligned
  auto load4 = [&](int e, bool last_use) -> float4 {   // entries e..e+3, NaN past the row
    if (vec && e + 4 <= nv) return score4(srow + e, last_use);
    const float qnan = __int_as_float(0x7fc00000);
    float4 f;
    f.x = e + 0 < nv ? score_at(srow + e + 0) : qnan;
    f.y = e + 1 < nv ? score_at(srow + e + 1) : qnan;
    f.z = e + 2 < nv ? score_at(srow + e + 2) : qnan;
    f.w = e + 3 < nv ? score_at(srow + e + 3) : qnan;
    return f;
  };
  // A. histogram
  bool fast = true;
  float lo = 0.f, bscale = 0.f;
  for (int s0 = 0; s0 < n_sl; s0 += TK_BATCH) {
    float4 rv[TK_BATCH];
#pragma unroll
    for (int i = 0; i < TK_BATCH; ++i)
      rv[i] = s0 + i < n_sl ? load4((s0 + i) * TK_SLICE + 4 * tid, false) : make_float4(0.f, 0.f, 0.f, 0.f);
    if (s0 == 0) {
      // value range from one score per thread (fminf / fmaxf skip the NaN past the row)
      const int si = tid & (TK_BATCH - 1);
      float v = rv[0].x;
#pragma unroll
      for (int i = 1; i < TK_BATCH; ++i) v = (i == si && i < n_sl) ? rv[i].x : v;
      float vmin = v, vmax = v;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, o));
        vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
      }
      if (lane == 0) { red[0][warp] = vmin; red[1][warp] = vmax; }
      __syncthreads();
      lo = red[0][0];
      float hi = red[1][0];
#pragma unroll
      for (int w = 1; w < TOPK_WARPS; ++w) { lo = fminf(lo, red[0][w]); hi = fmaxf(hi, red[1][w]); }
      const float span = hi - lo;
      bscale = (float)(TK_BINS - 1) / span;
      fast = span > 0.f && isfinite(span) && isfinite(bscale);
    }
    if (fast) {
#pragma unroll
      for (int i = 0; i < TK_BATCH; ++i) {
        const int e = (s0 + i) * TK_SLICE + 4 * tid;
        if (e + 4 <= nv) {
          atomicAdd(&hist[tk_bin(rv[i].x, lo, bscale)], 1u);
          atomicAdd(&hist[tk_bin(rv[i].y, lo, bscale)], 1u);
          atomicAdd(&hist[tk_bin(rv[i].z, lo, bscale)], 1u);
          atomicAdd(&hist[tk_bin(rv[i].w, lo, bscale)], 1u);
        } else if (e < nv) {
          atomicAdd(&hist[tk_bin(rv[i].x, lo, bscale)], 1u);
          if (e + 1 < nv) atomicAdd(&hist[tk_bin(rv[i].y, lo, bscale)], 1u);
          if (e + 2 < nv) atomicAdd(&hist[tk_bin(rv[i].z, lo, bscale)], 1u);
        }
      }
    }
  }
  __syncthreads();
  if (fast) {
    // B1. threshold bin: thread t owns bins 2047 - 16t .. 2032 - 16t (descending)
    uint32_t c[16], sum = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint4 h = reinterpret_cast<const uint4*>(hist)[(TK_BINS - 16 * (tid + 1)) / 4 + 3 - j];
      c[4 * j + 0] = h.w; c[4 * j + 1] = h.z; c[4 * j + 2] = h.y; c[4 * j + 3] = h.x;
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) sum += c[j];
    int tot_unused;
    const uint32_t excl = (uint32_t)tk_block_excl_scan((int)sum, wtot, tot_unused);
    if (excl < (uint32_t)topk && excl + sum >= (uint32_t)topk) {
      uint32_t above = excl;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (above + c[j] >= (uint32_t)topk) { bcast[0] = TK_BINS - 1 - 16 * tid - j; break; }
        above += c[j];
      }
    }
    __syncthreads();
    const int T = bcast[0];
    const float lo_T = T == 0 ? -INFINITY : lo + ((float)T - 1.5f) / bscale;
    const float hi_T = T == TK_BINS - 1 ? INFINITY : lo + ((float)T + 1.5f) / bscale;
    // B2. masks of the scores above hi_T; keys in (lo_T, hi_T]
    int above = 0;
    for (int s0 = 0; s0 < n_sl; s0 += TK_BATCH) {
      // all of the batch's loads in flight before any is used
      float4 rv[TK_BATCH];
#pragma unroll
      for (int i = 0; i < TK_BATCH; ++i)
        rv[i] = s0 + i < n_sl ? load4((s0 + i) * TK_SLICE + 4 * tid, true)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int i = 0; i < TK_BATCH; ++i) {
        const int sl = s0 + i;
        if (sl >= n_sl) break;
        const int e = sl * TK_SLICE + 4 * tid;
        const float4 f = rv[i];
        const uint32_t mh = (uint32_t)(f.x > hi_T) | ((uint32_t)(f.y > hi_T) << 1) |
                            ((uint32_t)(f.z > hi_T) << 2) | ((uint32_t)(f.w > hi_T) << 3);
        const uint32_t ml = (uint32_t)(f.x > lo_T) | ((uint32_t)(f.y > lo_T) << 1) |
                            ((uint32_t)(f.z > lo_T) << 2) | ((uint32_t)(f.w > lo_T) << 3);
        nib[sl * TOPK_THREADS + tid] = (uint8_t)mh;
        above += __popc(mh);
        if (ml != mh) {
          const float fv[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (((ml ^ mh) >> q) & 1u) {
              const int slot = atomicAdd(&n_cand, 1);
              if (slot < TK_CAND) cand[slot] = composite(fv[q], e + q);
            }
          }
        }
      }
    }
    above = __reduce_add_sync(0xffffffffu, above);
    if (lane == 0) wsum[warp] = above;
    __syncthreads();
    above = 0;
#pragma unroll
    for (int w = 0; w < TOPK_WARPS; ++w) above += wsum[w];
    const int C = n_cand;
    const int remaining = topk - above;
    fast = above < topk && C >= remaining && C <= TK_CAND;
    if (fast) {
      // B3. the remaining largest collected keys join the selection
      if (C <= TOPK_THREADS) {
        if (tid < C) {
          const uint64_t me = cand[tid];
          int rank = 0;
          for (int j = 0; j < C; ++j) rank += cand[j] > me;
          if (rank < remaining) {
            const int e = (int)(0xffffffffu - (uint32_t)me);
            atomicOr(&nibw[e >> 4], 1u << (8 * ((e >> 2) & 3) + (e & 3)));
          }
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
        for (int j = tid; j < remaining; j += TOPK_THREADS) {
          const int e = (int)(0xffffffffu - (uint32_t)cand[j]);
          atomicOr(&nibw[e >> 4], 1u << (8 * ((e >> 2) & 3) + (e & 3)));
        }
      }
      __syncthreads();
      // C. write the set bits in ascending index order (16 entries per word)
      const int n_words = n_sl * (TK_SLICE / 16);
      const int wpt = (n_words + TOPK_THREADS - 1) / TOPK_THREADS;
      const int w0 = min(tid * wpt, n_words), w1 = min(w0 + wpt, n_words);
      int cnt = 0;
      for (int w = w0; w < w1; ++w) cnt += __popc(nibw[w]);
      int tot;
      int pos = tk_block_excl_scan(cnt, wtot, tot);
      for (int w = w0; w < w1; ++w) {
        uint32_t x = nibw[w];
        while (x) {
          const int bit = __ffs(x) - 1;
          if (pos < topk) out[pos] = 16 * w + 4 * (bit >> 3) + (bit & 7);
          ++pos;
          x &= x - 1;
        }
      }
      return;
    }
  }
  // exact radix select over order-preserving keys read from the row
  __syncthreads();
  auto key_of = [&](int i) { return float_key(score_at(srow + i)); };
  const RadixResult rr = radix_select(key_of, nv, topk, hist, bcast);
  emit_selection(key_of, nv, rr, out, topk, wsum);
}

// Largest row (entries) the top-k takes: its 4-bit selection masks (Nc / 4
// bytes of dynamic shared memory) beside the kernel's 12.5 KB of static
// shared memory stay within the per-CTA limit.
constexpr int kMaxTopkRow = 786432;

// scores: fp32 [rows][Nc], or bf16 when bf16_scores
cslc_status launch_topk_rows(const void* scores, bool bf16_scores, int rows_in_buf, int row_begin, int row_end,
                             int B, int L, int Nc, int m, int q_pos0, int topk, int32_t* idx,
                             cudaStream_t stream) {
  if (row_end <= row_begin || B == 0) return CSLC_OK;
  static int configured_for = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_for != dev) {
    const int max_dyn = kMaxTopkRow / 4;   // rows above 196,608 entries need more than the default 48 KB
    cudaFuncSetAttribute(topk_rows_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_dyn);
    cudaFuncSetAttribute(topk_rows_kernel<uint16_t>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_dyn);
    configured_for = dev;
  }
  // mask storage for the launch's longest row (rows see more entries as t grows)
  const int nv_max = n_visible((long long)q_pos0 + row_end - 1, m, Nc);
  const size_t smem = (size_t)((nv_max + TK_SLICE - 1) / TK_SLICE) * (TK_SLICE / 4);
  dim3 grid(row_end - row_begin, B);
  if (bf16_scores)
    topk_rows_kernel<uint16_t><<<grid, TOPK_THREADS, smem, stream>>>(static_cast<const uint16_t*>(scores), rows_in_buf,
                                                                     row_begin, L, Nc, m, q_pos0, topk, idx);
  else
    topk_rows_kernel<float><<<grid, TOPK_THREADS, smem, stream>>>(static_cast<const float*>(scores), rows_in_buf,
                                                                  row_begin, L, Nc, m, q_pos0, topk, idx);
  return check_launch("topk_rows_kernel");
}

}  // namespace cslc
