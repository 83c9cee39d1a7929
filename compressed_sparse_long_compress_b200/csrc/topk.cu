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

__device__ __forceinline__ uint64_t composite(float v, int i) {
  return ((uint64_t)float_key(v) << 32) | (uint64_t)(0xffffffffu - (uint32_t)i);
}

// One CTA per query row.
// Fast path (touches each score a few times with cheap work):
//   1. each thread loads its scores with all loads in flight; one of them per
//      thread, spread over the row, fixes a value range [lo, hi];
//   2. one pass over those registers bins every score into 4096 equal
//      bins of that range (scores outside clamp to the edge bins, which keeps
//      the binning monotone), adds it to a shared histogram and keeps its
//      16-bit bin in shared memory;
//   3. the bin T holding the k-th largest score is found by a block scan; all
//      scores in higher bins are selected; when bin T must be split, its
//      scores are re-read and ranked exactly by (score desc, index asc) and the
//      chosen ones are marked in a bitmap;
//   4. two passes over the 16-bit bins (eight per 16-byte read) count the
//      selection per warp segment and then write the indices in ascending order.
// Rows whose sampled range is degenerate, or whose threshold bin is too
// crowded, take the exact 8-bit radix select over order-preserving keys.
constexpr int TK_MAXN = 45056;   // longest row (entries) the shared memory holds
constexpr int TK_REG = 8;        // float4 loads per thread held in registers (power of two)

__global__ void __launch_bounds__(TOPK_THREADS) topk_rows_kernel(
    const float* __restrict__ scores, int rows_in_buf, int row_begin, int L, int Nc, int m,
    int q_pos0, int topk, int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) uint32_t dyn[];          // n words: bins (fast) or keys (fallback)
  __shared__ uint32_t hist[TK_BINS];
  __shared__ uint64_t cand[TK_CAND];
  __shared__ uint32_t selbits[TK_MAXN / 32];
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
  const float* srow = scores + ((size_t)b * rows_in_buf + (r - row_begin)) * (size_t)Nc;
  uint16_t* bins = reinterpret_cast<uint16_t*>(dyn);
  for (int x = tid; x < TK_BINS; x += TOPK_THREADS) hist[x] = 0;
  for (int x = tid; x < (nv + 31) / 32; x += TOPK_THREADS) selbits[x] = 0;
  if (tid == 0) n_cand = 0;
  // 1. the row's first TK_REG * 4 * TOPK_THREADS scores go to registers with all
  //    loads in flight at once; one of them per thread (spread over the row)
  //    samples the value range
  const bool vec = (Nc & 3) == 0;
  const int n4 = vec ? (nv >> 2) : 0;
  float4 rv[TK_REG];
#pragma unroll
  for (int i = 0; i < TK_REG; ++i) {
    const int j = tid + i * TOPK_THREADS;
    rv[i] = j < n4 ? __ldcs(reinterpret_cast<const float4*>(srow) + j) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  {
    const int si = tid & (TK_REG - 1);
    const int sj = tid + si * TOPK_THREADS;
    float v;
    if (vec && sj < n4) {
      v = rv[0].x;
#pragma unroll
      for (int i = 1; i < TK_REG; ++i) if (i == si) v = rv[i].x;
    } else {
      v = __ldg(srow + (int)(((long long)tid * nv) / TOPK_THREADS));
    }
    float vmin = v, vmax = v;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, o));
      vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    }
    if (lane == 0) { red[0][warp] = vmin; red[1][warp] = vmax; }
  }
  __syncthreads();
  float lo = red[0][0], hi = red[1][0];
  for (int w = 1; w < TOPK_WARPS; ++w) { lo = fminf(lo, red[0][w]); hi = fmaxf(hi, red[1][w]); }
  const float span = hi - lo;
  bool fast = span > 0.f && isfinite(span) && nv <= TK_MAXN;
  const float bscale = fast ? ((float)TK_BINS - 0.5f) / span : 0.f;
  auto bin_of = [&](float v) { return min(TK_BINS - 1, max(0, (int)((v - lo) * bscale))); };
  int T = 0, remaining = 0;
  bool take_all = false;
  if (fast) {
    // 2. bin every score (registers / global -> histogram + 16-bit bins)
#pragma unroll
    for (int i = 0; i < TK_REG; ++i) {
      const int j = tid + i * TOPK_THREADS;
      if (j < n4) {
        const float4 v = rv[i];
        const int b0 = bin_of(v.x), b1 = bin_of(v.y), b2 = bin_of(v.z), b3 = bin_of(v.w);
        atomicAdd(&hist[b0], 1u); atomicAdd(&hist[b1], 1u); atomicAdd(&hist[b2], 1u); atomicAdd(&hist[b3], 1u);
        reinterpret_cast<uint2*>(bins)[j] = make_uint2((uint32_t)b0 | ((uint32_t)b1 << 16), (uint32_t)b2 | ((uint32_t)b3 << 16));
      }
    }
    for (int j = tid + TK_REG * TOPK_THREADS; j < n4; j += TOPK_THREADS) {
      const float4 v = __ldcs(reinterpret_cast<const float4*>(srow) + j);
      const int b0 = bin_of(v.x), b1 = bin_of(v.y), b2 = bin_of(v.z), b3 = bin_of(v.w);
      atomicAdd(&hist[b0], 1u); atomicAdd(&hist[b1], 1u); atomicAdd(&hist[b2], 1u); atomicAdd(&hist[b3], 1u);
      reinterpret_cast<uint2*>(bins)[j] = make_uint2((uint32_t)b0 | ((uint32_t)b1 << 16), (uint32_t)b2 | ((uint32_t)b3 << 16));
    }
    for (int j = (n4 << 2) + tid; j < nv; j += TOPK_THREADS) {
      const int bb = bin_of(__ldcs(srow + j));
      atomicAdd(&hist[bb], 1u);
      bins[j] = (uint16_t)bb;
    }
    __syncthreads();
    // 3. threshold bin: thread t owns bins 4095 - 8t .. 4088 - 8t (descending)
    uint32_t c[8], sum = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) { c[j] = hist[TK_BINS - 1 - 8 * tid - j]; sum += c[j]; }
    uint32_t incl = sum;
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
    const uint32_t excl = incl - sum;
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
    take_all = (cntT == remaining);
    if (!take_all && cntT > TK_CAND) fast = false;
    if (fast && !take_all) {
      // candidates of bin T (re-read from global), ranked by (score desc, index asc)
      const int n8 = (nv + 7) >> 3;
      for (int j8 = tid; j8 < n8; j8 += TOPK_THREADS) {
        const uint4 bv = reinterpret_cast<const uint4*>(bins)[j8];
        const uint32_t wds[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int i = 8 * j8 + q;
          const uint32_t bi = (wds[q >> 1] >> (16 * (q & 1))) & 0xffffu;
          if (i < nv && (int)bi == T) cand[atomicAdd(&n_cand, 1)] = composite(__ldg(srow + i), i);
        }
      }
      __syncthreads();
      const int C = n_cand;
      if (C <= TOPK_THREADS) {
        if (tid < C) {
          const uint64_t me = cand[tid];
          int rank = 0;
          for (int j = 0; j < C; ++j) rank += cand[j] > me;
          if (rank < remaining) {
            const int i = (int)(0xffffffffu - (uint32_t)me);
            atomicOr(&selbits[i >> 5], 1u << (i & 31));
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
          const int i = (int)(0xffffffffu - (uint32_t)cand[j]);
          atomicOr(&selbits[i >> 5], 1u << (i & 31));
        }
      }
      __syncthreads();
    }
  }
  if (fast) {
    // 4. count per warp segment, then write in ascending index order (8 bins per lane per step)
    const int seg = ((nv + TOPK_WARPS - 1) / TOPK_WARPS + 255) & ~255;
    const int lo_i = warp * seg, hi_i = min(nv, lo_i + seg);
    auto sel_mask = [&](int base) -> uint32_t {   // 8-bit selection mask of elements base .. base+7
      if (base >= hi_i) return 0u;
      const uint4 bv = reinterpret_cast<const uint4*>(bins)[base >> 3];
      const uint32_t wds[4] = {bv.x, bv.y, bv.z, bv.w};
      uint32_t msk = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int i = base + q;
        const int bi = (int)((wds[q >> 1] >> (16 * (q & 1))) & 0xffffu);
        bool sel = bi > T || (bi == T && (take_all || ((selbits[i >> 5] >> (i & 31)) & 1u)));
        if (i >= hi_i) sel = false;
        msk |= (uint32_t)sel << q;
      }
      return msk;
    };
    int cnt = 0;
    for (int base = lo_i; base < hi_i; base += 256) cnt += __popc(sel_mask(base + 8 * lane));
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (lane == 0) wsum[warp] = cnt;
    __syncthreads();
    int run = 0;
    for (int w = 0; w < warp; ++w) run += wsum[w];
    for (int base = lo_i; base < hi_i; base += 256) {
      uint32_t msk = sel_mask(base + 8 * lane);
      const int c8 = __popc(msk);
      int incl2 = c8;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl2, o);
        if (lane >= o) incl2 += v;
      }
      int pos = run + incl2 - c8;
      while (msk) {
        const int q = __ffs(msk) - 1;
        if (pos < topk) out[pos] = base + 8 * lane + q;
        ++pos;
        msk &= msk - 1;
      }
      run += __shfl_sync(0xffffffffu, incl2, 31);
    }
    return;
  }
  // exact radix select over order-preserving keys (degenerate value ranges / crowded bins)
  __syncthreads();
  uint32_t* keys = dyn;
  for (int j = tid; j < nv; j += TOPK_THREADS) keys[j] = float_key(__ldcs(srow + j));
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
                         TK_MAXN * 4);
    configured_for = dev;
  }
  dim3 grid(row_end - row_begin, B);
  topk_rows_kernel<<<grid, TOPK_THREADS, smem, stream>>>(scores, rows_in_buf, row_begin, L, Nc, m,
                                                         q_pos0, topk, idx);
  return check_launch("topk_rows_kernel");
}

}  // namespace cslc
