// Decode step over the mixed BF16-RoPE / FP8 KV cache.
//
// "读完这篇你就搞懂 DeepSeek v4 了", §三: in decode every new token re-reads the
// compressed KV from HBM, so cost grows with the context; CSA adds the
// lightning indexer over all entries and attends to the top-k; HCA attends to
// all entries. First page §1.4 存储格式混: RoPE dims stay BF16, the rest FP8.
//
// Kernels (one CSA layer = 1 memset + 5 launches, one HCA layer = 2):
//   decode_scores_kernel   indexer scores of every entry (tensor-core m16n8k16
//                          with k_I tiles as A and the 8 indexer heads as N=8),
//                          ReLU-weighted head sum, fp32 store, and a 4096-bin
//                          histogram of the score keys (top 12 bits)
//   decode_select_kernel   finds the histogram bin holding the k-th largest
//                          score; entries above it are selected, entries in it
//                          become candidates (a block scan places them; one
//                          atomic per counter and CTA)
//   decode_finalize_kernel exact choice among the candidates (64-bit radix
//                          select on score key ++ reversed index, so ties go to
//                          the smaller index), then the k indices in ascending
//                          order through a bitmap of the context and a block
//                          scan (a bitonic sort above 262,144 entries)
//   decode_attn_kernel     split-K attention: each CTA takes one or more chunks
//                          of 128 entries (about two CTAs per SM over the
//                          layer); a chunk's stored entries are staged with
//                          one batch of cp.async while the previous chunk is
//                          computed, dequantised (e4m3 * scale -> bf16, RoPE
//                          half copied) into shared memory, and QK^T / softmax
//                          / PV run for all heads
//   decode_combine_kernel  merges the splits with their max / sum statistics
//                          (two thread groups, each over half of the splits)
//   decode_tail_kernel     for large batches, select + finalize + attention +
//                          combine of a CSA layer in one launch of one
//                          thread-block cluster per sequence (see its comment)
// The layers of a step are independent: layer 0 runs on the caller's stream,
// the others on internal streams forked from it and joined back with events,
// each with its own workspace slice. Inside a layer the kernels after the
// first are launched as programmatic dependents: each may be scheduled while
// its predecessor finishes and waits (griddepcontrol.wait) before it reads
// what the predecessor wrote.

#include <algorithm>

#include "common.cuh"

namespace cslc {

constexpr int DEC_CHUNK = 4096;      // entries per scores / select CTA
constexpr int DEC_THREADS = 256;
constexpr int HIST_BINS = 4096;      // top 12 bits of the score key
constexpr int HIST_SHIFT = 20;
constexpr int SPLIT = 128;           // entries per attention chunk (a CTA takes one or more)
constexpr int ATTN_CTAS = 296;       // attention CTAs aimed at per layer: two per SM on 148 SMs
constexpr int DTILE = 64;            // entries per attention tile
constexpr int FIN_THREADS = 1024;
constexpr int MAX_TOPK = 2048;

// Programmatic dependent launch: wait for the preceding kernel's results (a
// no-op when the kernel was not launched as a dependent), and let the next
// kernel be scheduled once every CTA of this one has reached this point.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

struct DecodeWs {
  float* scores;          // [B, n_max]
  uint32_t* hist;         // [B, HIST_BINS]
  int32_t* counters;      // [B, 2]: selected-above, candidates
  int32_t* sel;           // [B, MAX_TOPK]
  uint2* cand;            // [B, n_max] (key, index)
  int32_t* idx;           // [B, topk]
  float* part_o;          // [B, splits, H, 128]
  float* part_ml;         // [B, splits, H, 2]
};

// ------------------------------------------------------------ scores + hist

template <int NT>  // indexer heads padded to NT * 8
__global__ void __launch_bounds__(DEC_THREADS) decode_scores_kernel(
    const uint16_t* __restrict__ q_idx, const uint16_t* __restrict__ w,
    const uint16_t* __restrict__ k_idx, const int32_t* __restrict__ n_entries, int n_max, int HI,
    float* __restrict__ scores, uint32_t* __restrict__ ghist) {
  __shared__ uint32_t hist[HIST_BINS];
  const int b = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tq = lane & 3;
  const int n = min(n_entries[b], n_max);
  const int c0 = blockIdx.x * DEC_CHUNK;
  if (c0 >= n) return;   // whole CTA exits together: no barrier reached
  for (int x = tid; x < HIST_BINS; x += DEC_THREADS) hist[x] = 0;

  // B fragments: q_I of head nt*8+g, physical dims 16*tq .. 16*tq+15 (see the
  // dims permutation note below); weights of heads nt*8 + 2*tq, +1.
  uint32_t qb[NT][8];
  float wv[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int h = nt * 8 + g;
    if (h < HI) {
      const uint4* src = reinterpret_cast<const uint4*>(q_idx + ((size_t)b * HI + h) * kDI + 16 * tq);
      const uint4 v0 = __ldg(src), v1 = __ldg(src + 1);
      qb[nt][0] = v0.x; qb[nt][1] = v0.y; qb[nt][2] = v0.z; qb[nt][3] = v0.w;
      qb[nt][4] = v1.x; qb[nt][5] = v1.y; qb[nt][6] = v1.z; qb[nt][7] = v1.w;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) qb[nt][j] = 0u;
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int hw = nt * 8 + 2 * tq + j;
      wv[nt][j] = hw < HI ? bf16_to_f(w[(size_t)b * HI + hw]) : 0.f;
    }
  }
  __syncthreads();

  // Dims permutation: the product runs over the 64 dims in any order as long
  // as A and B agree. Thread (g, tq) loads physical dims [16tq, 16tq+16) of
  // rows g and g+8; in k-step s its fragment registers hold physical pairs
  // 16tq+4s (+0,+1) and 16tq+4s+2 (+2,+3) -- the same pairs its B registers hold.
  const int c1 = min(n, c0 + DEC_CHUNK);
  const uint16_t* kbase = k_idx + (size_t)b * n_max * kDI;
  // the key rows of a warp's group of 16 entries (clamped to the last entry);
  // the next group's loads are issued before this group is used, so that two
  // groups per warp are in flight
  auto load_group = [&](int e0, uint4 (&v)[4]) {
    const uint4* pa = reinterpret_cast<const uint4*>(kbase + (size_t)min(e0 + g, n - 1) * kDI + 16 * tq);
    const uint4* pb = reinterpret_cast<const uint4*>(kbase + (size_t)min(e0 + g + 8, n - 1) * kDI + 16 * tq);
    v[0] = __ldcs(pa); v[1] = __ldcs(pa + 1); v[2] = __ldcs(pb); v[3] = __ldcs(pb + 1);
  };
  constexpr int GROUP_STRIDE = 16 * (DEC_THREADS / 32);
  uint4 nxt[4];
  if (c0 + warp * 16 < c1) load_group(c0 + warp * 16, nxt);
  for (int e0 = c0 + warp * 16; e0 < c1; e0 += GROUP_STRIDE) {
    const int ea = e0 + g, eb = ea + 8;
    uint32_t ra[8], rb[8];
    {
      const uint4 a0 = nxt[0], a1 = nxt[1], b0 = nxt[2], b1 = nxt[3];
      if (e0 + GROUP_STRIDE < c1) load_group(e0 + GROUP_STRIDE, nxt);
      ra[0] = a0.x; ra[1] = a0.y; ra[2] = a0.z; ra[3] = a0.w; ra[4] = a1.x; ra[5] = a1.y; ra[6] = a1.z; ra[7] = a1.w;
      rb[0] = b0.x; rb[1] = b0.y; rb[2] = b0.z; rb[3] = b0.w; rb[4] = b1.x; rb[5] = b1.y; rb[6] = b1.z; rb[7] = b1.w;
    }
    float sa = 0.f, sb = 0.f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const uint32_t af[4] = {ra[2 * s], rb[2 * s], ra[2 * s + 1], rb[2 * s + 1]};
        mma_bf16_16816(d, af, qb[nt][2 * s], qb[nt][2 * s + 1]);
      }
      sa = fmaf(wv[nt][0], fmaxf(d[0], 0.f), sa);
      sa = fmaf(wv[nt][1], fmaxf(d[1], 0.f), sa);
      sb = fmaf(wv[nt][0], fmaxf(d[2], 0.f), sb);
      sb = fmaf(wv[nt][1], fmaxf(d[3], 0.f), sb);
    }
    sa += __shfl_xor_sync(0xffffffffu, sa, 1);
    sa += __shfl_xor_sync(0xffffffffu, sa, 2);
    sb += __shfl_xor_sync(0xffffffffu, sb, 1);
    sb += __shfl_xor_sync(0xffffffffu, sb, 2);
    // lane tq==0 owns row g, lane tq==1 owns row g+8
    const int e = tq == 0 ? ea : eb;
    const float v = tq == 0 ? sa : sb;
    const bool mine = tq < 2 && e < c1;
    if (mine) scores[(size_t)b * n_max + e] = v;
    if (mine) {
      const uint32_t bin = float_key(v) >> HIST_SHIFT;
      const unsigned peers = __match_any_sync(__activemask(), bin);
      if (lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
    }
  }
  __syncthreads();
  uint32_t* gh = ghist + (size_t)b * HIST_BINS;
  for (int x = tid; x < HIST_BINS; x += DEC_THREADS) {
    const uint32_t v = hist[x];
    if (v) atomicAdd(&gh[x], v);
  }
  pdl_trigger();
}

// Histogram only (for the stand-alone top-k entry on given scores).
__global__ void __launch_bounds__(DEC_THREADS) decode_hist_kernel(const float* __restrict__ scores,
                                                                  const int32_t* __restrict__ n_entries,
                                                                  int n_max, uint32_t* __restrict__ ghist) {
  __shared__ uint32_t hist[HIST_BINS];
  const int b = blockIdx.y, tid = threadIdx.x, lane = tid & 31;
  const int n = min(n_entries[b], n_max);
  const int c0 = blockIdx.x * DEC_CHUNK;
  if (c0 >= n) return;
  for (int x = tid; x < HIST_BINS; x += DEC_THREADS) hist[x] = 0;
  __syncthreads();
  const int c1 = min(n, c0 + DEC_CHUNK);
  for (int e = c0 + tid; e < c1; e += DEC_THREADS) {
    const uint32_t bin = float_key(scores[(size_t)b * n_max + e]) >> HIST_SHIFT;
    const unsigned peers = __match_any_sync(__activemask(), bin);
    if (lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
  }
  __syncthreads();
  for (int x = tid; x < HIST_BINS; x += DEC_THREADS) {
    const uint32_t v = hist[x];
    if (v) atomicAdd(&ghist[(size_t)b * HIST_BINS + x], v);
  }
}

// -------------------------------------------------------------- selection

// Finds bin T with count(bins > T) < k <= count(bins >= T). Block-wide, DEC_THREADS.
__device__ void find_threshold_bin(const uint32_t* gh, int k, int* out_bin, int* out_above) {
  __shared__ uint32_t wsum[DEC_THREADS / 32];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // thread t owns bins 4095-16t .. 4080-16t
  uint32_t cnt[16], s = 0;
#pragma unroll
  for (int j = 0; j < 16; ++j) { cnt[j] = gh[HIST_BINS - 1 - 16 * tid - j]; s += cnt[j]; }
  // inclusive scan over threads: warp shuffles, then the warps' totals
  uint32_t incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  for (int w = 0; w < warp; ++w) incl += wsum[w];
  const uint32_t excl = incl - s;
  if (excl < (uint32_t)k && incl >= (uint32_t)k) {
    uint32_t above = excl;
    for (int j = 0; j < 16; ++j) {
      if (above + cnt[j] >= (uint32_t)k) {
        *out_bin = HIST_BINS - 1 - 16 * tid - j;
        *out_above = (int)above;
        break;
      }
      above += cnt[j];
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(DEC_THREADS) decode_select_kernel(
    const float* __restrict__ scores, const int32_t* __restrict__ n_entries, int n_max, int topk,
    const uint32_t* __restrict__ ghist, int32_t* __restrict__ counters, int32_t* __restrict__ sel,
    uint2* __restrict__ cand) {
  __shared__ int thr[2];
  const int b = blockIdx.y, tid = threadIdx.x, lane = tid & 31;
  pdl_wait();
  if (tid == 0) { thr[0] = HIST_BINS; thr[1] = 0; }   // "nothing above" if no bin is found
  const int n = min(n_entries[b], n_max);
  const int c0 = blockIdx.x * DEC_CHUNK;
  if (n <= topk || c0 >= n) return;
  const int c1 = min(n, c0 + DEC_CHUNK);
  // this thread's scores of the chunk: all loads in flight before any is used,
  // and issued before the threshold scan so that the two latencies overlap
  constexpr int PER_THREAD = DEC_CHUNK / DEC_THREADS;
  static_assert(PER_THREAD <= 16, "per-thread flags fit 16 bits");
  float sv[PER_THREAD];
#pragma unroll
  for (int i = 0; i < PER_THREAD; ++i) {
    const int e = c0 + i * DEC_THREADS + tid;
    sv[i] = e < c1 ? scores[(size_t)b * n_max + e] : 0.f;
  }
  find_threshold_bin(ghist + (size_t)b * HIST_BINS, topk, &thr[0], &thr[1]);
  const uint32_t T = (uint32_t)thr[0];
  uint32_t fa = 0u, fc = 0u;   // bit i: score i is above / inside the threshold bin
#pragma unroll
  for (int i = 0; i < PER_THREAD; ++i) {
    const int e = c0 + i * DEC_THREADS + tid;
    const uint32_t bin = float_key(sv[i]) >> HIST_SHIFT;
    if (e < c1 && bin > T) fa |= 1u << i;
    if (e < c1 && bin == T) fc |= 1u << i;
  }
  // block exclusive scan of (above count << 16 | candidate count); one atomic
  // per counter and CTA reserves the CTA's output ranges
  __shared__ uint32_t wtot[DEC_THREADS / 32];
  __shared__ int base[2];
  const int warp = tid >> 5;
  const uint32_t mine = ((uint32_t)__popc(fa) << 16) | (uint32_t)__popc(fc);
  uint32_t incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wtot[warp] = incl;
  __syncthreads();
  uint32_t before = 0u, total = 0u;
#pragma unroll
  for (int w = 0; w < DEC_THREADS / 32; ++w) {
    const uint32_t t = wtot[w];
    if (w < warp) before += t;
    total += t;
  }
  if (tid == 0) {
    base[0] = (total >> 16) ? atomicAdd(&counters[2 * b], (int)(total >> 16)) : 0;
    base[1] = (total & 0xffffu) ? atomicAdd(&counters[2 * b + 1], (int)(total & 0xffffu)) : 0;
  }
  __syncthreads();
  const uint32_t excl = before + incl - mine;
  int pa = base[0] + (int)(excl >> 16), pc = base[1] + (int)(excl & 0xffffu);
#pragma unroll
  for (int i = 0; i < PER_THREAD; ++i) {
    const int e = c0 + i * DEC_THREADS + tid;
    if ((fa >> i) & 1u) {
      if (pa < MAX_TOPK) sel[(size_t)b * MAX_TOPK + pa] = e;
      ++pa;
    }
    if ((fc >> i) & 1u) {
      if (pc < n_max) cand[(size_t)b * n_max + pc] = make_uint2(float_key(sv[i]), (uint32_t)e);
      ++pc;
    }
  }
  pdl_trigger();
}

// 64-bit composite of a candidate: score key, then reversed index, so that a
// larger composite means a larger score or an equal score at a smaller index.
__device__ __forceinline__ uint64_t cand_key(uint2 c) {
  return ((uint64_t)c.x << 32) | (uint64_t)(0xffffffffu - c.y);
}

__global__ void __launch_bounds__(FIN_THREADS) decode_finalize_kernel(
    const int32_t* __restrict__ n_entries, int n_max, int topk, const int32_t* __restrict__ counters,
    const int32_t* __restrict__ sel, const uint2* __restrict__ cand, int32_t* __restrict__ idx) {
  __shared__ int32_t list[MAX_TOPK];
  __shared__ uint32_t hist[FIN_THREADS / 32][256];
  __shared__ int bc[4];
  __shared__ int fill;
  const int b = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_wait();
  pdl_trigger();   // the attention's CTAs may be scheduled meanwhile (they wait for this grid)
  const int n = min(n_entries[b], n_max);
  int32_t* out = idx + (size_t)b * topk;
  if (n <= topk) {
    for (int j = tid; j < topk; j += FIN_THREADS) out[j] = j < n ? j : -1;
    return;
  }
  const int n_above = min(counters[2 * b], topk);
  const int C = min(counters[2 * b + 1], n_max);
  const int need = topk - n_above;
  const uint2* cb = cand + (size_t)b * n_max;
  for (int j = tid; j < n_above; j += FIN_THREADS) list[j] = sel[(size_t)b * MAX_TOPK + j];
  if (tid == 0) fill = n_above;
  __syncthreads();

  // radix select of the need-th largest composite key among the C candidates;
  // they all share the top HIST_BITS key bits (the threshold bin), so the
  // digits start below those (8-bit digits, a last 4-bit one)
  constexpr int FIXED = 64 - (32 - HIST_SHIFT);   // bits 63 .. FIXED are the bin
  uint64_t prefix = C > 0 ? (cand_key(cb[0]) >> FIXED) << FIXED : 0ull;
  uint64_t mask = ~0ull << FIXED;
  int remaining = need;
  bool take_all = (C == need);
  for (int shift = FIXED - 8; shift > -8 && !take_all; shift -= 8) {
    const int sh = shift < 0 ? 0 : shift;                  // the last digit is narrower
    const uint32_t dmask = shift < 0 ? (0xffu >> -shift) : 0xffu;
    for (int x = tid; x < (FIN_THREADS / 32) * 256; x += FIN_THREADS) (&hist[0][0])[x] = 0;
    if (tid == 0) { bc[0] = 0; bc[1] = 0; bc[2] = 0; }
    __syncthreads();
    for (int i = tid; i < C; i += FIN_THREADS) {
      const uint64_t k = cand_key(cb[i]);
      if ((k & mask) == prefix) {
        const uint32_t d = (uint32_t)(k >> sh) & dmask;
        const unsigned peers = __match_any_sync(__activemask(), d);
        if (lane == __ffs(peers) - 1) atomicAdd(&hist[warp][d], (uint32_t)__popc(peers));
      }
    }
    __syncthreads();
    if (tid < 256) {
      uint32_t s = 0;
      for (int w = 0; w < FIN_THREADS / 32; ++w) s += hist[w][tid];
      hist[0][tid] = s;
    }
    __syncthreads();
    if (warp == 0) {
      uint32_t cnt[8], ls = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) { cnt[j] = hist[0][255 - 8 * lane - j]; ls += cnt[j]; }
      uint32_t incl = ls;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const uint32_t excl = incl - ls;
      if (excl < (uint32_t)remaining && incl >= (uint32_t)remaining) {
        uint32_t above = excl;
        for (int j = 0; j < 8; ++j) {
          if (above + cnt[j] >= (uint32_t)remaining) {
            bc[0] = 255 - 8 * lane - j; bc[1] = (int)above; bc[2] = (int)cnt[j];
            break;
          }
          above += cnt[j];
        }
      }
    }
    __syncthreads();
    const uint64_t d = (uint64_t)bc[0];
    const int above = bc[1], cnt_d = bc[2];
    __syncthreads();
    remaining -= above;
    prefix |= d << sh;
    mask |= (uint64_t)dmask << sh;
    if (cnt_d == remaining) take_all = true;
  }
  // composite keys are unique, so after the last digit exactly `remaining` match
  for (int i = tid; i < C; i += FIN_THREADS) {
    const uint2 c = cb[i];
    const uint64_t k = cand_key(c);
    const bool s = take_all ? ((k & mask) >= prefix) : ((k & mask) > prefix || (k & mask) == prefix);
    if (s) {
      const int pos = atomicAdd(&fill, 1);
      if (pos < topk) list[pos] = (int32_t)c.y;
    }
  }
  __syncthreads();
  if (n <= FIN_THREADS * 8 * 32) {
    // ascending order through a bitmap of the context (the radix histogram's
    // 8192 words): each thread owns 8 words, a block scan of their bit counts
    // gives every thread its first output position
    uint32_t* bm = &hist[0][0];
    for (int x = tid; x < FIN_THREADS * 8; x += FIN_THREADS) bm[x] = 0u;
    __syncthreads();
    const int n_sel = min(fill, topk);
    for (int j = tid; j < n_sel; j += FIN_THREADS) atomicOr(&bm[list[j] >> 5], 1u << (list[j] & 31));
    __syncthreads();
    uint32_t wv[8];
    int cnt = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      wv[k] = bm[tid * 8 + k];
      cnt += __popc(wv[k]);
    }
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    __shared__ int wsum[FIN_THREADS / 32];
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int t = wsum[lane];
      int ti = t;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, ti, o);
        if (lane >= o) ti += v;
      }
      wsum[lane] = ti - t;   // exclusive prefix of the warp totals
    }
    __syncthreads();
    int pos = wsum[warp] + incl - cnt;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      uint32_t w = wv[k];
      while (w) {
        const int bit = __ffs(w) - 1;
        out[pos++] = (tid * 8 + k) * 32 + bit;
        w &= w - 1;
      }
    }
    for (int j = n_sel + tid; j < topk; j += FIN_THREADS) out[j] = -1;
    return;
  }
  // larger contexts: bitonic sort of list[0..topk) ascending, padded to a power of two
  int P = 1;
  while (P < topk) P <<= 1;
  for (int j = topk + tid; j < P; j += FIN_THREADS) list[j] = 0x7fffffff;
  __syncthreads();
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < P; i += FIN_THREADS) {
        const int jx = i ^ stride;
        if (jx > i) {
          const bool up = (i & size) == 0;
          const int a = list[i], c = list[jx];
          if ((a > c) == up) { list[i] = c; list[jx] = a; }
        }
      }
      __syncthreads();
    }
  }
  for (int j = tid; j < topk; j += FIN_THREADS) out[j] = list[j];
}

// -------------------------------------------------------------- attention

// 2^x on the SFU (approximate; -inf gives +0, subnormal results flush to zero)
__device__ __forceinline__ float dec_ex2(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(r) : "f"(x));
  return r;
}

template <bool SPARSE>
__global__ void __launch_bounds__(256) decode_attn_kernel(
    const uint16_t* __restrict__ q, const uint8_t* __restrict__ nope, const uint16_t* __restrict__ rope,
    const float* __restrict__ kv_scale, const int32_t* __restrict__ n_entries, int n_max,
    const int32_t* __restrict__ idx, int topk, int H, float scale_log2, int splits, int chunks,
    float* __restrict__ part_o, float* __restrict__ part_ml) {
  constexpr int ST_BYTES = SPLIT * (kNope + kRope * 2 + 4);   // one chunk as stored
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* q_s = smem;                               // [H][256 B]
  uint8_t* kv_s = smem + H * 256;                    // [SPLIT][256 B] dequantised entries
  uint8_t* st_base = kv_s + SPLIT * 256;             // [2] x (FP8 codes [SPLIT][64 B], RoPE dims
                                                     //        [SPLIT][128 B], scales [SPLIT])
  __shared__ int32_t ent_buf[2][SPLIT];
  const int b = blockIdx.y, sp = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nthreads = (H / 16) * 32;
  pdl_wait();
  const int g = lane >> 2, tq = lane & 3;
  const int n = min(n_entries[b], n_max);
  const int n_slots = SPARSE ? topk : n;
  const int slot0 = sp * chunks * SPLIT;
  // chunks of this CTA that hold a slot (the rest of the split is past the end)
  const int n_chunks = slot0 >= n_slots ? 0 : min(chunks, (n_slots - slot0 + SPLIT - 1) / SPLIT);

  // the entries of chunk c (-1 for empty slots) into ent_buf[c & 1]
  auto fill_ent = [&](int c) {
    for (int j = tid; j < SPLIT; j += nthreads) {
      const int slot = slot0 + c * SPLIT + j;
      int e = -1;
      if (slot < n_slots) e = SPARSE ? idx[(size_t)b * topk + slot] : slot;
      if (e >= n) e = -1;
      ent_buf[c & 1][j] = e;
    }
  };
  // the stored entries of chunk c, all copies in flight at once; empty slots read as zeros
  constexpr int PIECES = kNope / 16 + (kRope * 2) / 16 + 1;   // 16-byte pieces + the scale
  auto stage_chunk = [&](int c) {
    uint8_t* st_nope = st_base + (c & 1) * ST_BYTES;
    uint8_t* st_rope = st_nope + SPLIT * kNope;
    float* st_scale = reinterpret_cast<float*>(st_rope + SPLIT * kRope * 2);
    const int32_t* ent = ent_buf[c & 1];
    for (int x = tid; x < SPLIT * PIECES; x += nthreads) {
      const int row = x / PIECES, pc = x - row * PIECES;
      const int e = ent[row];
      const size_t er = (size_t)b * n_max + (e < 0 ? 0 : e);
      if (pc < kNope / 16)
        cp_async16(smem_u32(st_nope + row * kNope + pc * 16), nope + er * kNope + pc * 16, e >= 0);
      else if (pc < PIECES - 1)
        cp_async16(smem_u32(st_rope + row * (kRope * 2) + (pc - kNope / 16) * 16),
                   reinterpret_cast<const uint8_t*>(rope + er * kRope) + (pc - kNope / 16) * 16, e >= 0);
      else
        cp_async4(smem_u32(st_scale + row), kv_scale + er, e >= 0);
    }
    cp_async_commit();
  };
  if (n_chunks > 0) fill_ent(0);
  __syncthreads();
  if (n_chunks > 0) {
    // the queries travel in the first chunk's group of copies
    for (int x = tid; x < H * 16; x += nthreads) {
      const int chunk = x & 15, row = x >> 4;
      cp_async16(smem_u32(q_s + swz(row, chunk, 256)), q + ((size_t)b * H + row) * kD + chunk * 8, true);
    }
    stage_chunk(0);
  }
  uint32_t qf[8][4];
  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) o[i][j] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};

  for (int c = 0; c < n_chunks; ++c) {
    // the next chunk's copies go out before this chunk is waited for
    if (c + 1 < n_chunks) {
      fill_ent(c + 1);
      __syncthreads();
      stage_chunk(c + 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (c == 0) {
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const int row = warp * 16 + (lane & 15);
        const int chunk = ks * 2 + (lane >> 4);
        ldsm_x4(smem_u32(q_s + swz(row, chunk, 256)), qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3]);
      }
    }
    const int32_t* ent = ent_buf[c & 1];
    const int s0 = slot0 + c * SPLIT;
    {
      // dequantise into the MMA layout: chunks 0..7 = FP8 dims x scale, 8..15 = RoPE dims
      const uint8_t* st_nope = st_base + (c & 1) * ST_BYTES;
      const uint8_t* st_rope = st_nope + SPLIT * kNope;
      const float* st_scale = reinterpret_cast<const float*>(st_rope + SPLIT * kRope * 2);
      for (int x = tid; x < SPLIT * 16; x += nthreads) {
        const int chunk = x & 15, row = x >> 4;
        uint4 v;
        if (chunk < 8) {
          const uint2 c8 = *reinterpret_cast<const uint2*>(st_nope + row * kNope + chunk * 8);
          const float sc = st_scale[row];
          const uint32_t cw[2] = {c8.x, c8.y};
          uint32_t ow[4];
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const __half2_raw h01 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(cw[k] & 0xffffu), __NV_E4M3);
            const __half2_raw h23 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(cw[k] >> 16), __NV_E4M3);
            const float2 f01 = __half22float2(*reinterpret_cast<const __half2*>(&h01));
            const float2 f23 = __half22float2(*reinterpret_cast<const __half2*>(&h23));
            ow[2 * k] = pack_bf16x2(f01.x * sc, f01.y * sc);
            ow[2 * k + 1] = pack_bf16x2(f23.x * sc, f23.y * sc);
          }
          v = make_uint4(ow[0], ow[1], ow[2], ow[3]);
        } else {
          v = *reinterpret_cast<const uint4*>(st_rope + row * (kRope * 2) + (chunk - 8) * 16);
        }
        *reinterpret_cast<uint4*>(kv_s + swz(row, chunk, 256)) = v;
      }
    }
    __syncthreads();

    for (int t0 = 0; t0 < SPLIT; t0 += DTILE) {
      if (s0 + t0 >= n_slots) break;
      const uint8_t* kv_t = kv_s + t0 * 256;   // this tile's 64 entries
      float s[8][4];
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) s[i][j] = 0.f;
#pragma unroll
      for (int np = 0; np < 4; ++np) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          uint32_t b0, b1, b2, b3;
          const int row = np * 16 + (lane & 7) + ((lane >> 4) << 3);
          const int chunk = ks * 2 + ((lane >> 3) & 1);
          ldsm_x4(smem_u32(kv_t + swz(row, chunk, 256)), b0, b1, b2, b3);
          mma_bf16_16816(s[2 * np], qf[ks], b0, b1);
          mma_bf16_16816(s[2 * np + 1], qf[ks], b2, b3);
        }
      }
      float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int slot = t0 + nt * 8 + 2 * tq + j;   // within the chunk
          const bool valid = SPARSE ? ent[slot] >= 0 : s0 + slot < n_slots;
          const float v0 = valid ? s[nt][j] * scale_log2 : -INFINITY;
          const float v1 = valid ? s[nt][2 + j] * scale_log2 : -INFINITY;
          s[nt][j] = v0;
          s[nt][2 + j] = v1;
          tmax[0] = fmaxf(tmax[0], v0);
          tmax[1] = fmaxf(tmax[1], v1);
        }
      }
      float alpha[2], mnew[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        tmax[r] = fmaxf(tmax[r], __shfl_xor_sync(0xffffffffu, tmax[r], 1));
        tmax[r] = fmaxf(tmax[r], __shfl_xor_sync(0xffffffffu, tmax[r], 2));
        mnew[r] = fmaxf(mrow[r], tmax[r]);
        alpha[r] = mrow[r] == -INFINITY ? 0.f : dec_ex2(mrow[r] - mnew[r]);
        mrow[r] = mnew[r];
      }
      float psum[2] = {0.f, 0.f};
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int r = j >> 1;
          const float p = mnew[r] == -INFINITY ? 0.f : dec_ex2(s[nt][j] - mnew[r]);
          s[nt][j] = p;
          psum[r] += p;
        }
      }
      lrow[0] = lrow[0] * alpha[0] + psum[0];
      lrow[1] = lrow[1] * alpha[1] + psum[1];
#pragma unroll
      for (int dn = 0; dn < 16; ++dn) {
        o[dn][0] *= alpha[0]; o[dn][1] *= alpha[0];
        o[dn][2] *= alpha[1]; o[dn][3] *= alpha[1];
      }
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        uint32_t pa[4];
        pa[0] = pack_bf16x2(s[2 * ks][0], s[2 * ks][1]);
        pa[1] = pack_bf16x2(s[2 * ks][2], s[2 * ks][3]);
        pa[2] = pack_bf16x2(s[2 * ks + 1][0], s[2 * ks + 1][1]);
        pa[3] = pack_bf16x2(s[2 * ks + 1][2], s[2 * ks + 1][3]);
#pragma unroll
        for (int dp = 0; dp < 8; ++dp) {
          uint32_t b0, b1, b2, b3;
          const int row = ks * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
          const int chunk = dp * 2 + (lane >> 4);
          ldsm_x4_t(smem_u32(kv_t + swz(row, chunk, 256)), b0, b1, b2, b3);
          mma_bf16_16816(o[2 * dp], pa, b0, b1);
          mma_bf16_16816(o[2 * dp + 1], pa, b2, b3);
        }
      }
      __syncthreads();
    }
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 1);
    lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 2);
  }
  const int h0 = warp * 16 + g, h1 = h0 + 8;
  float* po = part_o + (((size_t)b * splits + sp) * H) * kD;
#pragma unroll
  for (int dn = 0; dn < 16; ++dn) {
    const int col = dn * 8 + 2 * tq;
    *reinterpret_cast<float2*>(po + (size_t)h0 * kD + col) = make_float2(o[dn][0], o[dn][1]);
    *reinterpret_cast<float2*>(po + (size_t)h1 * kD + col) = make_float2(o[dn][2], o[dn][3]);
  }
  if (tq == 0) {
    float* pm = part_ml + (((size_t)b * splits + sp) * H) * 2;
    pm[2 * h0] = mrow[0]; pm[2 * h0 + 1] = lrow[0];
    pm[2 * h1] = mrow[1]; pm[2 * h1 + 1] = lrow[1];
  }
  pdl_trigger();
}

__global__ void __launch_bounds__(2 * kD) decode_combine_kernel(const float* __restrict__ part_o,
                                                                const float* __restrict__ part_ml,
                                                                const int32_t* __restrict__ n_entries,
                                                                int n_max, int topk, int sparse, int H,
                                                                int splits, int split_slots,
                                                                uint16_t* __restrict__ out) {
  __shared__ float xm[kD], xn[kD], xd[kD];
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x & (kD - 1), grp = threadIdx.x / kD;
  pdl_wait();
  const int n = min(n_entries[b], n_max);
  const int slots = sparse ? min(topk, n) : n;
  const int used = min(splits, (slots + split_slots - 1) / split_slots);
  const float* pm = part_ml + (size_t)b * splits * H * 2;
  const float* po = part_o + ((size_t)b * splits * H + h) * kD + d;
  // each group takes every other split, one pass with a running maximum; the
  // loads of 8 splits are issued together
  float M = -INFINITY, num = 0.f, den = 0.f;
  for (int s0 = 0; s0 < used; s0 += 16) {
    float ms[8], ls[8], os[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int sp = s0 + 2 * i + grp;
      ms[i] = sp < used ? pm[((size_t)sp * H + h) * 2] : -INFINITY;
      ls[i] = sp < used ? pm[((size_t)sp * H + h) * 2 + 1] : 0.f;
      os[i] = sp < used ? po[(size_t)sp * H * kD] : 0.f;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (ms[i] == -INFINITY) continue;
      if (ms[i] > M) {
        const float a = M == -INFINITY ? 0.f : exp2f(M - ms[i]);
        num *= a;
        den *= a;
        M = ms[i];
      }
      const float f = exp2f(ms[i] - M);
      den = fmaf(f, ls[i], den);
      num = fmaf(f, os[i], num);
    }
  }
  if (grp == 1) {
    xm[d] = M;
    xn[d] = num;
    xd[d] = den;
  }
  __syncthreads();
  if (grp == 0) {
    const float Mo = xm[d];
    if (Mo != -INFINITY) {
      const float Mn = fmaxf(M, Mo);
      const float a = M == -INFINITY ? 0.f : exp2f(M - Mn), c = exp2f(Mo - Mn);
      num = num * a + xn[d] * c;
      den = den * a + xd[d] * c;
    }
    const float r = den > 0.f ? num / den : 0.f;
    out[((size_t)b * H + h) * kD + d] = __bfloat16_as_ushort(__float2bfloat16_rn(r));
  }
}

// ------------------------------------------------- fused layer tail (clusters)
//
// One thread-block cluster of CL CTAs per sequence runs everything after the
// index scan of a CSA layer (and the whole of an HCA layer) in one launch,
// exchanging through distributed shared memory instead of global round trips:
//   selection  every CTA finds the threshold bin from the scan's histogram
//              and classifies its 1/CL of the scores: above the bin =
//              selected (kept in its shared memory), inside = candidate
//              (kept in its own slice of the candidate buffer);
//   choice     exact radix select among all candidates by 8-bit digits of
//              (score key, reversed index): each CTA histograms its own
//              candidates and sums all CTAs' histograms, so every CTA takes
//              the same digit with no further exchange;
//   order      each CTA marks its selected entries in a bitmap of its range;
//              a cluster scan of the counts places them, ascending, in the
//              index list held in CTA 0's shared memory (and idx_out);
//   attention  CTA r takes slots [r*S, (r+1)*S) of the list, as
//              decode_attn_kernel does per chunk; with H <= 64 two warp groups
//              take alternate 64-entry tiles and merge before publishing;
//   combine    every CTA's partial (max, sum, O) stays in its shared memory;
//              CTA r merges heads [r*H/CL, (r+1)*H/CL) over the cluster.
// Every CTA passes the same cluster barriers in the same order: each branch
// around one depends on per-sequence values or on sums every CTA computes
// identically. The CTAs of a cluster are co-scheduled by the hardware.

constexpr int TAIL_THREADS = 256;
constexpr int TAIL_BM_WORDS = 4096;   // bitmap words per CTA: ranges up to 131,072 entries

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire;\n" ::: "memory");
}
// the address of the same shared-memory location in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t dsmem_addr(const void* local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(r) : "r"(smem_u32(local)), "r"(rank));
  return r;
}
__device__ __forceinline__ uint32_t dsmem_ld_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];\n" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ float dsmem_ld_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];\n" : "=f"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ float4 dsmem_ld_f32x4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];\n"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ void dsmem_st_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;\n" ::"r"(addr), "r"(v) : "memory");
}

// Dynamic shared memory of the tail kernel: the index list (CTA 0's is the
// cluster's), then one region used in turn by the selection, the attention
// and the combine.
__host__ __device__ constexpr size_t tail_sel_bytes() { return 2 * 256 * 4 + MAX_TOPK * 4 + TAIL_BM_WORDS * 4; }
constexpr int TAIL_NBUF = 4;          // chunks of stored entries in flight per CTA
__host__ __device__ constexpr size_t tail_attn_bytes(int H) {
  return (size_t)H * 256 + SPLIT * 256 + TAIL_NBUF * (size_t)SPLIT * (kNope + kRope * 2 + 4);
}
__host__ __device__ constexpr size_t tail_smem_bytes(int H) {
  return MAX_TOPK * 4 + (tail_sel_bytes() > tail_attn_bytes(H) ? tail_sel_bytes() : tail_attn_bytes(H));
}

template <bool SPARSE, int CL>
__global__ void __launch_bounds__(TAIL_THREADS) decode_tail_kernel(
    const uint16_t* __restrict__ q, const uint8_t* __restrict__ nope, const uint16_t* __restrict__ rope,
    const float* __restrict__ kv_scale, const int32_t* __restrict__ n_entries, int n_max,
    const float* __restrict__ scores, const uint32_t* __restrict__ ghist, uint2* __restrict__ cand, int topk,
    int H, float scale_log2, int32_t* __restrict__ idx_out, uint16_t* __restrict__ out) {
  constexpr int ST_BYTES = SPLIT * (kNope + kRope * 2 + 4);
  extern __shared__ __align__(128) uint8_t smem[];
  int32_t* list = reinterpret_cast<int32_t*>(smem);   // [MAX_TOPK], read from CTA 0 by all
  uint8_t* work = smem + MAX_TOPK * 4;
  __shared__ uint32_t pub[4];                          // read by the other CTAs
  __shared__ int s_thr[2], s_nab, s_ncand, s_base, s_tot[2], bc[3];
  __shared__ uint32_t htot[256];
  __shared__ uint32_t wtot[TAIL_THREADS / 32];
  __shared__ int32_t ent_buf[2 * TAIL_NBUF][SPLIT];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();
  const int b = blockIdx.y;
  pdl_wait();
  const int n = max(0, min(n_entries[b], n_max));
  const bool select = SPARSE && n > topk;
  const int k_eff = SPARSE ? min(topk, n) : n;

  if (SPARSE && !select && idx_out != nullptr)
    for (int j = (int)rank * TAIL_THREADS + tid; j < topk; j += CL * TAIL_THREADS)
      idx_out[(size_t)b * topk + j] = j < n ? j : -1;

  if (select) {
    const int R = ((n + CL - 1) / CL + 31) & ~31;     // entries per CTA (multiple of 32)
    const int e_lo = (int)rank * R, e_hi = min(n, e_lo + R);
    uint32_t* hist2 = reinterpret_cast<uint32_t*>(work);                            // [2][256]
    int32_t* above_l = reinterpret_cast<int32_t*>(work + 2 * 256 * 4);                // [MAX_TOPK]
    uint32_t* bm = reinterpret_cast<uint32_t*>(work + 2 * 256 * 4 + MAX_TOPK * 4);    // [R / 32]
    if (tid == 0) { s_nab = 0; s_ncand = 0; s_thr[0] = HIST_BINS; s_thr[1] = 0; }
    find_threshold_bin(ghist + (size_t)b * HIST_BINS, topk, &s_thr[0], &s_thr[1]);
    const uint32_t T = (uint32_t)s_thr[0];
    uint2* my_cand = cand + (size_t)b * n_max + e_lo;
    const float* srow = scores + (size_t)b * n_max;
    // rounds of 32 scores per thread: flag masks (above the bin / in it),
    // one block scan of the counts, then each thread writes its scores' entry
    // numbers (above: this CTA's list; in the bin: its candidate slice)
    const bool vec = (n_max & 3) == 0 && (reinterpret_cast<uintptr_t>(scores) & 15) == 0;
    // element k of this thread in the round at `base` (16-byte loads: 4 consecutive per load)
    auto e_of = [&](int base, int k) {
      return vec ? base + 4 * ((k >> 2) * TAIL_THREADS + tid) + (k & 3) : base + k * TAIL_THREADS + tid;
    };
    int run_above = 0, run_cand = 0;   // this CTA's counts so far (the same in every thread)
    for (int base = e_lo; base < e_hi; base += TAIL_THREADS * 32) {
      float val[32];
      if (vec) {
        const float4* s4 = reinterpret_cast<const float4*>(srow);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int e = e_of(base, 4 * i);
          // rows are 16-byte aligned and e is a multiple of 4, so a load that
          // starts before e_hi stays inside the row (n_max is a multiple of 4)
          const float4 v = e < e_hi ? s4[e >> 2] : make_float4(0.f, 0.f, 0.f, 0.f);
          val[4 * i] = v.x; val[4 * i + 1] = v.y; val[4 * i + 2] = v.z; val[4 * i + 3] = v.w;
        }
      } else {
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const int e = e_of(base, k);
          val[k] = e < e_hi ? srow[e] : 0.f;
        }
      }
      uint32_t fa = 0u, fc = 0u;
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const uint32_t bin = float_key(val[k]) >> HIST_SHIFT;
        const bool in = e_of(base, k) < e_hi;
        if (in && bin > T) fa |= 1u << k;
        if (in && bin == T) fc |= 1u << k;
      }
      const uint32_t mine = ((uint32_t)__popc(fa) << 16) | (uint32_t)__popc(fc);
      uint32_t incl = mine;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (lane == 31) wtot[warp] = incl;
      __syncthreads();
      uint32_t before = 0u, total = 0u;
#pragma unroll
      for (int w = 0; w < TAIL_THREADS / 32; ++w) {
        const uint32_t t = wtot[w];
        if (w < warp) before += t;
        total += t;
      }
      const uint32_t excl = before + incl - mine;
      int pa = run_above + (int)(excl >> 16), pc = run_cand + (int)(excl & 0xffffu);
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        if ((fa >> k) & 1u) {
          if (pa < MAX_TOPK) above_l[pa] = e_of(base, k);
          ++pa;
        }
        if ((fc >> k) & 1u) my_cand[pc++] = make_uint2(float_key(val[k]), (uint32_t)e_of(base, k));
      }
      run_above += (int)(total >> 16);
      run_cand += (int)(total & 0xffffu);
      __syncthreads();   // wtot is rewritten by the next round
    }
    if (tid == 0) { s_nab = run_above; s_ncand = run_cand; }
    __syncthreads();
    if (tid == 0) { pub[0] = (uint32_t)s_nab; pub[1] = (uint32_t)s_ncand; }
    cluster_sync_all();   // counts published
    if (warp == 0) {
      uint32_t a = 0u, c = 0u;
      if (lane < CL) {
        a = dsmem_ld_u32(dsmem_addr(&pub[0], lane));
        c = dsmem_ld_u32(dsmem_addr(&pub[1], lane));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        a += __shfl_xor_sync(0xffffffffu, a, o);
        c += __shfl_xor_sync(0xffffffffu, c, o);
      }
      if (lane == 0) { s_tot[0] = (int)a; s_tot[1] = (int)c; }
    }
    __syncthreads();
    const int nc = s_ncand;

    // exact choice among the candidates: they share the bin's key bits, so the
    // digits start below them (8-bit digits, a last 4-bit one)
    constexpr int FIXED = 64 - (32 - HIST_SHIFT);
    uint64_t prefix = (uint64_t)T << FIXED, mask = ~0ull << FIXED;
    int remaining = topk - s_tot[0];
    bool take_all = (s_tot[1] == remaining);
    int pass = 0;
    for (int shift = FIXED - 8; shift > -8 && !take_all; shift -= 8, ++pass) {
      const int sh = shift < 0 ? 0 : shift;
      const uint32_t dmask = shift < 0 ? (0xffu >> -shift) : 0xffu;
      uint32_t* h = hist2 + (pass & 1) * 256;
      h[tid] = 0u;   // TAIL_THREADS == 256 digits
      __syncthreads();
      for (int i = tid; i < nc; i += TAIL_THREADS) {
        const uint64_t k = cand_key(my_cand[i]);
        if ((k & mask) == prefix) atomicAdd(&h[(uint32_t)(k >> sh) & dmask], 1u);
      }
      __syncthreads();
      cluster_sync_all();   // every CTA's histogram of this digit is complete
      uint32_t sum = 0u;
      for (int r = 0; r < CL; ++r) sum += dsmem_ld_u32(dsmem_addr(&h[tid], r));
      htot[tid] = sum;
      __syncthreads();
      if (warp == 0) {
        // a default every CTA shares, so that the pass count stays the same
        // across the cluster even if no digit were found
        if (lane == 0) { bc[0] = 0; bc[1] = 0; bc[2] = -1; }
        __syncwarp();
        uint32_t cnt[8], ls = 0u;
#pragma unroll
        for (int j = 0; j < 8; ++j) { cnt[j] = htot[255 - 8 * lane - j]; ls += cnt[j]; }
        uint32_t incl = ls;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        const uint32_t excl = incl - ls;
        if (excl < (uint32_t)remaining && incl >= (uint32_t)remaining) {
          uint32_t above = excl;
          for (int j = 0; j < 8; ++j) {
            if (above + cnt[j] >= (uint32_t)remaining) {
              bc[0] = 255 - 8 * lane - j; bc[1] = (int)above; bc[2] = (int)cnt[j];
              break;
            }
            above += cnt[j];
          }
        }
      }
      __syncthreads();
      remaining -= bc[1];
      prefix |= (uint64_t)bc[0] << sh;
      mask |= (uint64_t)dmask << sh;
      if (bc[2] == remaining) take_all = true;
      __syncthreads();   // bc and htot are rewritten by the next pass
    }

    // this CTA's selected entries, in ascending order, into CTA 0's list
    const int words = R >> 5;
    for (int x = tid; x < words; x += TAIL_THREADS) bm[x] = 0u;
    __syncthreads();
    const int nab = min(s_nab, MAX_TOPK);
    for (int j = tid; j < nab; j += TAIL_THREADS) {
      const int e = above_l[j] - e_lo;
      atomicOr(&bm[e >> 5], 1u << (e & 31));
    }
    for (int i = tid; i < nc; i += TAIL_THREADS) {
      const uint2 c = my_cand[i];
      if ((cand_key(c) & mask) >= prefix) {
        const int e = (int)c.y - e_lo;
        atomicOr(&bm[e >> 5], 1u << (e & 31));
      }
    }
    __syncthreads();
    const int wpt = (words + TAIL_THREADS - 1) / TAIL_THREADS;   // words per thread
    int cnt = 0;
    for (int k = 0; k < wpt; ++k) {
      const int x = tid * wpt + k;
      if (x < words) cnt += __popc(bm[x]);
    }
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) wtot[warp] = (uint32_t)incl;
    __syncthreads();
    int before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < TAIL_THREADS / 32; ++w) {
      const int t = (int)wtot[w];
      if (w < warp) before += t;
      total += t;
    }
    if (tid == 0) pub[2] = (uint32_t)total;
    cluster_sync_all();   // selected counts published
    if (warp == 0) {
      int c = (lane < (int)rank) ? (int)dsmem_ld_u32(dsmem_addr(&pub[2], lane)) : 0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
      if (lane == 0) s_base = c;
    }
    __syncthreads();
    int pos = s_base + before + incl - cnt;
    const uint32_t list0 = dsmem_addr(list, 0);
    for (int k = 0; k < wpt; ++k) {
      const int x = tid * wpt + k;
      uint32_t wv = x < words ? bm[x] : 0u;
      while (wv) {
        const int e = e_lo + x * 32 + (__ffs(wv) - 1);
        if (pos < topk) {
          dsmem_st_u32(list0 + 4u * (uint32_t)pos, (uint32_t)e);
          if (idx_out != nullptr) idx_out[(size_t)b * topk + pos] = e;
        }
        ++pos;
        wv &= wv - 1u;
      }
    }
  }
  cluster_sync_all();   // the list is complete; the selection's scratch is free

  // ---- attention over this CTA's slots
  uint8_t* q_s = work;                 // [H][256 B]
  uint8_t* kv_s = work + H * 256;      // [SPLIT][256 B] dequantised entries
  uint8_t* st_base = kv_s + SPLIT * 256;
  const int S = ((k_eff + CL - 1) / CL + DTILE - 1) / DTILE * DTILE;
  const int slot0 = (int)rank * S;
  const int slot_end = min(k_eff, slot0 + S);
  const int n_chunks = slot_end > slot0 ? (slot_end - slot0 + SPLIT - 1) / SPLIT : 0;
  const uint32_t list0 = dsmem_addr(list, 0);
  const int wpg = H / 16;              // warps per group; a warp owns 16 heads
  const int G = H <= 64 ? 2 : 1;       // groups taking alternate tiles
  const int grp = warp / wpg, lw = warp - grp * wpg;
  const bool mma_warp = grp < G;
  const int g = lane >> 2, tq = lane & 3;

  // chunk c's entry indices go to ent_buf[c % (2 NBUF)] and its stored
  // entries to staging buffer c % NBUF; NBUF chunks are in flight at once
  auto fill_ent = [&](int c) {
    for (int j = tid; j < SPLIT; j += TAIL_THREADS) {
      const int slot = slot0 + c * SPLIT + j;
      int e = -1;
      if (slot < slot_end) e = select ? (int)dsmem_ld_u32(list0 + 4u * (uint32_t)slot) : slot;
      if (e >= n) e = -1;
      ent_buf[c % (2 * TAIL_NBUF)][j] = e;
    }
  };
  constexpr int PIECES = kNope / 16 + (kRope * 2) / 16 + 1;
  auto stage_chunk = [&](int c) {
    uint8_t* st_nope = st_base + (c % TAIL_NBUF) * ST_BYTES;
    uint8_t* st_rope = st_nope + SPLIT * kNope;
    float* st_scale = reinterpret_cast<float*>(st_rope + SPLIT * kRope * 2);
    const int32_t* ent = ent_buf[c % (2 * TAIL_NBUF)];
    for (int x = tid; x < SPLIT * PIECES; x += TAIL_THREADS) {
      const int row = x / PIECES, pc = x - row * PIECES;
      const int e = ent[row];
      const size_t er = (size_t)b * n_max + (e < 0 ? 0 : e);
      if (pc < kNope / 16)
        cp_async16(smem_u32(st_nope + row * kNope + pc * 16), nope + er * kNope + pc * 16, e >= 0);
      else if (pc < PIECES - 1)
        cp_async16(smem_u32(st_rope + row * (kRope * 2) + (pc - kNope / 16) * 16),
                   reinterpret_cast<const uint8_t*>(rope + er * kRope) + (pc - kNope / 16) * 16, e >= 0);
      else
        cp_async4(smem_u32(st_scale + row), kv_scale + er, e >= 0);
    }
    cp_async_commit();
  };
  const int n_pre = min(n_chunks, TAIL_NBUF);
  for (int c = 0; c < n_pre; ++c) fill_ent(c);
  __syncthreads();
  for (int c = 0; c < n_pre; ++c) {
    if (c == 0)   // the queries travel in the first chunk's group of copies
      for (int x = tid; x < H * 16; x += TAIL_THREADS) {
        const int chunk = x & 15, row = x >> 4;
        cp_async16(smem_u32(q_s + swz(row, chunk, 256)), q + ((size_t)b * H + row) * kD + chunk * 8, true);
      }
    stage_chunk(c);
  }
  uint32_t qf[8][4];
  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) o[i][j] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};

  for (int c = 0; c < n_chunks; ++c) {
    // groups committed so far: chunks 0 .. min(n_chunks, c + NBUF) - 1; chunk c's must be complete
    const int pending = min(n_chunks, c + TAIL_NBUF) - c - 1;
    if (pending >= 3) cp_async_wait<3>();
    else if (pending == 2) cp_async_wait<2>();
    else if (pending == 1) cp_async_wait<1>();
    else cp_async_wait<0>();
    if (c + TAIL_NBUF < n_chunks) fill_ent(c + TAIL_NBUF);   // its ent slot was last used by chunk c - NBUF
    __syncthreads();
    if (c == 0 && mma_warp) {
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const int row = lw * 16 + (lane & 15);
        const int chunk = ks * 2 + (lane >> 4);
        ldsm_x4(smem_u32(q_s + swz(row, chunk, 256)), qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3]);
      }
    }
    const int32_t* ent = ent_buf[c % (2 * TAIL_NBUF)];
    const int s0 = slot0 + c * SPLIT;
    {
      const uint8_t* st_nope = st_base + (c % TAIL_NBUF) * ST_BYTES;
      const uint8_t* st_rope = st_nope + SPLIT * kNope;
      const float* st_scale = reinterpret_cast<const float*>(st_rope + SPLIT * kRope * 2);
      for (int x = tid; x < SPLIT * 16; x += TAIL_THREADS) {
        const int chunk = x & 15, row = x >> 4;
        uint4 v;
        if (chunk < 8) {
          const uint2 c8 = *reinterpret_cast<const uint2*>(st_nope + row * kNope + chunk * 8);
          const float sc = st_scale[row];
          const uint32_t cw[2] = {c8.x, c8.y};
          uint32_t ow[4];
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const __half2_raw h01 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(cw[k] & 0xffffu), __NV_E4M3);
            const __half2_raw h23 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(cw[k] >> 16), __NV_E4M3);
            const float2 f01 = __half22float2(*reinterpret_cast<const __half2*>(&h01));
            const float2 f23 = __half22float2(*reinterpret_cast<const __half2*>(&h23));
            ow[2 * k] = pack_bf16x2(f01.x * sc, f01.y * sc);
            ow[2 * k + 1] = pack_bf16x2(f23.x * sc, f23.y * sc);
          }
          v = make_uint4(ow[0], ow[1], ow[2], ow[3]);
        } else {
          v = *reinterpret_cast<const uint4*>(st_rope + row * (kRope * 2) + (chunk - 8) * 16);
        }
        *reinterpret_cast<uint4*>(kv_s + swz(row, chunk, 256)) = v;
      }
    }
    __syncthreads();
    if (c + TAIL_NBUF < n_chunks) stage_chunk(c + TAIL_NBUF);   // into the buffer just dequantised
    if (mma_warp) {
      for (int tile = grp; tile < SPLIT / DTILE; tile += G) {
        const int t0 = tile * DTILE;
        if (s0 + t0 >= slot_end) break;
        const uint8_t* kv_t = kv_s + t0 * 256;
        float sc[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) sc[i][j] = 0.f;
#pragma unroll
        for (int np = 0; np < 4; ++np) {
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            uint32_t b0, b1, b2, b3;
            const int row = np * 16 + (lane & 7) + ((lane >> 4) << 3);
            const int chunk = ks * 2 + ((lane >> 3) & 1);
            ldsm_x4(smem_u32(kv_t + swz(row, chunk, 256)), b0, b1, b2, b3);
            mma_bf16_16816(sc[2 * np], qf[ks], b0, b1);
            mma_bf16_16816(sc[2 * np + 1], qf[ks], b2, b3);
          }
        }
        float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const bool valid = ent[t0 + nt * 8 + 2 * tq + j] >= 0;
            const float v0 = valid ? sc[nt][j] * scale_log2 : -INFINITY;
            const float v1 = valid ? sc[nt][2 + j] * scale_log2 : -INFINITY;
            sc[nt][j] = v0;
            sc[nt][2 + j] = v1;
            tmax[0] = fmaxf(tmax[0], v0);
            tmax[1] = fmaxf(tmax[1], v1);
          }
        }
        float alpha[2], mnew[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          tmax[r] = fmaxf(tmax[r], __shfl_xor_sync(0xffffffffu, tmax[r], 1));
          tmax[r] = fmaxf(tmax[r], __shfl_xor_sync(0xffffffffu, tmax[r], 2));
          mnew[r] = fmaxf(mrow[r], tmax[r]);
          alpha[r] = mrow[r] == -INFINITY ? 0.f : dec_ex2(mrow[r] - mnew[r]);
          mrow[r] = mnew[r];
        }
        float psum[2] = {0.f, 0.f};
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int r = j >> 1;
            const float p = mnew[r] == -INFINITY ? 0.f : dec_ex2(sc[nt][j] - mnew[r]);
            sc[nt][j] = p;
            psum[r] += p;
          }
        }
        lrow[0] = lrow[0] * alpha[0] + psum[0];
        lrow[1] = lrow[1] * alpha[1] + psum[1];
#pragma unroll
        for (int dn = 0; dn < 16; ++dn) {
          o[dn][0] *= alpha[0]; o[dn][1] *= alpha[0];
          o[dn][2] *= alpha[1]; o[dn][3] *= alpha[1];
        }
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          uint32_t pa[4];
          pa[0] = pack_bf16x2(sc[2 * ks][0], sc[2 * ks][1]);
          pa[1] = pack_bf16x2(sc[2 * ks][2], sc[2 * ks][3]);
          pa[2] = pack_bf16x2(sc[2 * ks + 1][0], sc[2 * ks + 1][1]);
          pa[3] = pack_bf16x2(sc[2 * ks + 1][2], sc[2 * ks + 1][3]);
#pragma unroll
          for (int dp = 0; dp < 8; ++dp) {
            uint32_t b0, b1, b2, b3;
            const int row = ks * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
            const int chunk = dp * 2 + (lane >> 4);
            ldsm_x4_t(smem_u32(kv_t + swz(row, chunk, 256)), b0, b1, b2, b3);
            mma_bf16_16816(o[2 * dp], pa, b0, b1);
            mma_bf16_16816(o[2 * dp + 1], pa, b2, b3);
          }
        }
      }
    }
    __syncthreads();   // kv_s and ent_buf are rewritten for the next chunk
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 1);
    lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 2);
  }

  // ---- this CTA's partial: group 1 hands its rows to group 0, which merges
  float* po_s = reinterpret_cast<float*>(work);   // [H][kD]
  float* ml_s = po_s + (size_t)H * kD;            // [H][2]
  const int h0 = lw * 16 + g, h1 = h0 + 8;
  __syncthreads();   // the attention's shared memory is free
  if (mma_warp && grp == 1) {
#pragma unroll
    for (int dn = 0; dn < 16; ++dn) {
      const int col = dn * 8 + 2 * tq;
      *reinterpret_cast<float2*>(po_s + (size_t)h0 * kD + col) = make_float2(o[dn][0], o[dn][1]);
      *reinterpret_cast<float2*>(po_s + (size_t)h1 * kD + col) = make_float2(o[dn][2], o[dn][3]);
    }
    if (tq == 0) {
      ml_s[2 * h0] = mrow[0]; ml_s[2 * h0 + 1] = lrow[0];
      ml_s[2 * h1] = mrow[1]; ml_s[2 * h1 + 1] = lrow[1];
    }
  }
  __syncthreads();
  if (mma_warp && grp == 0) {
    if (G == 2) {
      const float m1[2] = {ml_s[2 * h0], ml_s[2 * h1]}, l1[2] = {ml_s[2 * h0 + 1], ml_s[2 * h1 + 1]};
      float a0[2], a1[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const float M = fmaxf(mrow[r], m1[r]);
        a0[r] = mrow[r] == -INFINITY ? 0.f : exp2f(mrow[r] - M);
        a1[r] = m1[r] == -INFINITY ? 0.f : exp2f(m1[r] - M);
        lrow[r] = lrow[r] * a0[r] + l1[r] * a1[r];
        mrow[r] = M;
      }
#pragma unroll
      for (int dn = 0; dn < 16; ++dn) {
        const int col = dn * 8 + 2 * tq;
        const float2 p0 = *reinterpret_cast<const float2*>(po_s + (size_t)h0 * kD + col);
        const float2 p1 = *reinterpret_cast<const float2*>(po_s + (size_t)h1 * kD + col);
        o[dn][0] = o[dn][0] * a0[0] + p0.x * a1[0];
        o[dn][1] = o[dn][1] * a0[0] + p0.y * a1[0];
        o[dn][2] = o[dn][2] * a0[1] + p1.x * a1[1];
        o[dn][3] = o[dn][3] * a0[1] + p1.y * a1[1];
      }
      __syncwarp();   // every lane has read its twin's (max, sum) before lane tq == 0 rewrites them
    }
#pragma unroll
    for (int dn = 0; dn < 16; ++dn) {
      const int col = dn * 8 + 2 * tq;
      *reinterpret_cast<float2*>(po_s + (size_t)h0 * kD + col) = make_float2(o[dn][0], o[dn][1]);
      *reinterpret_cast<float2*>(po_s + (size_t)h1 * kD + col) = make_float2(o[dn][2], o[dn][3]);
    }
    if (tq == 0) {
      ml_s[2 * h0] = mrow[0]; ml_s[2 * h0 + 1] = lrow[0];
      ml_s[2 * h1] = mrow[1]; ml_s[2 * h1 + 1] = lrow[1];
    }
  }
  cluster_sync_all();   // every CTA's partial is in its shared memory

  // ---- combine: CTA r writes heads [r*H/CL, (r+1)*H/CL), four dims per item
  const int hpc = H / CL;
  for (int x = tid; x < hpc * (kD / 4); x += TAIL_THREADS) {
    const int h = (int)rank * hpc + x / (kD / 4), d4 = (x % (kD / 4)) * 4;
    float ms[CL], ls[CL];
    float4 os[CL];
#pragma unroll
    for (int r = 0; r < CL; ++r) {
      ms[r] = dsmem_ld_f32(dsmem_addr(ml_s + 2 * h, r));
      ls[r] = dsmem_ld_f32(dsmem_addr(ml_s + 2 * h + 1, r));
      os[r] = dsmem_ld_f32x4(dsmem_addr(po_s + (size_t)h * kD + d4, r));
    }
    float M = -INFINITY;
#pragma unroll
    for (int r = 0; r < CL; ++r) M = fmaxf(M, ms[r]);
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
    float den = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int r = 0; r < CL; ++r) {
        if (ms[r] == -INFINITY) continue;
        const float f = exp2f(ms[r] - M);
        den = fmaf(f, ls[r], den);
        num.x = fmaf(f, os[r].x, num.x);
        num.y = fmaf(f, os[r].y, num.y);
        num.z = fmaf(f, os[r].z, num.z);
        num.w = fmaf(f, os[r].w, num.w);
      }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    uint2 packed;
    packed.x = pack_bf16x2(num.x * inv, num.y * inv);
    packed.y = pack_bf16x2(num.z * inv, num.w * inv);
    *reinterpret_cast<uint2*>(out + ((size_t)b * H + h) * kD + d4) = packed;
  }
  cluster_sync_all();   // no CTA leaves while its partial may still be read
}

// -------------------------------------------------------------- host side

static size_t align_up(size_t x) { return (x + 255) & ~(size_t)255; }

// Launches `kernel` as a programmatic dependent of the work before it on `stream`.
template <typename... KArgs, typename... Args>
static cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                    cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

struct DecodeWsSizes {
  size_t scores, hist, counters, sel, cand, idx, part_o, part_ml;
  size_t total() const { return scores + hist + counters + sel + cand + idx + part_o + part_ml; }
};

// chunks of SPLIT entries per attention CTA: about ATTN_CTAS CTAs over the layer
static int layer_chunks(const cslc_decode_layer& l, int B) {
  const int slots = l.kind == 0 ? l.topk : l.n_max;
  const long long total = slots > 0 ? (long long)B * ((slots + SPLIT - 1) / SPLIT) : 0;
  return (int)std::max<long long>(1, (total + ATTN_CTAS - 1) / ATTN_CTAS);
}
static int layer_splits(const cslc_decode_layer& l, int B) {
  const int slots = l.kind == 0 ? l.topk : l.n_max;
  const int per = SPLIT * layer_chunks(l, B);
  return slots > 0 ? (slots + per - 1) / per : 1;
}

static DecodeWsSizes ws_sizes(int B, int n_max, int topk, int splits, int H) {
  DecodeWsSizes s;
  s.scores = align_up((size_t)B * n_max * 4);
  s.hist = align_up((size_t)B * HIST_BINS * 4);
  s.counters = align_up((size_t)B * 2 * 4);
  s.sel = align_up((size_t)B * MAX_TOPK * 4);
  s.cand = align_up((size_t)B * n_max * 8);
  s.idx = align_up((size_t)B * (topk > 0 ? topk : 1) * 4);
  s.part_o = align_up((size_t)B * splits * H * kD * 4);
  s.part_ml = align_up((size_t)B * splits * H * 2 * 4);
  return s;
}

static DecodeWsSizes layer_ws_sizes(const cslc_decode_layer& l, int B, int H) {
  DecodeWsSizes s = ws_sizes(B, l.n_max, l.kind == 0 ? l.topk : 1, layer_splits(l, B), H);
  if (l.kind != 0) s.scores = s.hist = s.counters = s.sel = s.cand = s.idx = 0;
  return s;
}

// The layers run concurrently, so each has its own slice; the histograms and
// counters of all layers come first, so that one memset clears them.
size_t decode_workspace_bytes(const cslc_decode_layer* layers, int n_layers, int B, int H) {
  size_t total = 0;
  for (int i = 0; i < n_layers; ++i) total += layer_ws_sizes(layers[i], B, H).total();
  return total;
}

size_t decode_topk_workspace_bytes(int B, int n_max, int topk) {
  DecodeWsSizes s = ws_sizes(B, n_max, topk, 1, 16);
  return s.hist + s.counters + s.sel + s.cand;
}

static void carve(uint8_t* base, const DecodeWsSizes& s, DecodeWs& w) {
  uint8_t* p = base;
  w.hist = reinterpret_cast<uint32_t*>(p); p += s.hist;
  w.counters = reinterpret_cast<int32_t*>(p); p += s.counters;
  w.scores = reinterpret_cast<float*>(p); p += s.scores;
  w.sel = reinterpret_cast<int32_t*>(p); p += s.sel;
  w.cand = reinterpret_cast<uint2*>(p); p += s.cand;
  w.idx = reinterpret_cast<int32_t*>(p); p += s.idx;
  w.part_o = reinterpret_cast<float*>(p); p += s.part_o;
  w.part_ml = reinterpret_cast<float*>(p); p += s.part_ml;
}

static cslc_status run_topk_stages(const float* scores, const int32_t* n_entries, int B, int n_max,
                                   int topk, DecodeWs& w, int32_t* idx, cudaStream_t stream) {
  const dim3 grid((n_max + DEC_CHUNK - 1) / DEC_CHUNK, B);
  cudaError_t e = cudaSuccess;
  if (n_max > 0)
    e = launch_dependent(decode_select_kernel, grid, dim3(DEC_THREADS), 0, stream, scores, n_entries, n_max, topk,
                         w.hist, w.counters, w.sel, w.cand);
  if (e == cudaSuccess)
    e = launch_dependent(decode_finalize_kernel, dim3(B), dim3(FIN_THREADS), 0, stream, n_entries, n_max, topk,
                         w.counters, w.sel, w.cand, idx);
  if (e != cudaSuccess) return set_error(CSLC_ERR_CUDA, "decode top-k launch: %s", cudaGetErrorString(e));
  return check_launch("decode_finalize_kernel");
}

static cslc_status run_attention(const cslc_decode_layer& l, int B, int H, const int32_t* idx,
                                 DecodeWs& w, cudaStream_t stream) {
  const int chunks = layer_chunks(l, B), splits = layer_splits(l, B);
  const size_t smem = (size_t)H * 256 + SPLIT * 256 + 2 * SPLIT * (kNope + kRope * 2 + 4);
  static int configured_for = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_for != dev) {
    const int max_smem = 128 * 256 + SPLIT * 256 + 2 * SPLIT * (kNope + kRope * 2 + 4);
    cudaFuncSetAttribute(decode_attn_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
    cudaFuncSetAttribute(decode_attn_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
    configured_for = dev;
  }
  const dim3 grid(splits, B);
  const float sl2 = l.scale * kLog2e;
  cudaError_t e;
  if (l.kind == 0)   // after the top-k: a programmatic dependent of its finalize pass
    e = launch_dependent(decode_attn_kernel<true>, grid, dim3((H / 16) * 32), smem, stream, l.q, l.nope, l.rope,
                         l.kv_scale, l.n_entries, l.n_max, idx, l.topk, H, sl2, splits, chunks, w.part_o, w.part_ml);
  else {             // the first kernel of an HCA layer: an ordinary launch
    decode_attn_kernel<false><<<grid, (H / 16) * 32, smem, stream>>>(
        l.q, l.nope, l.rope, l.kv_scale, l.n_entries, l.n_max, nullptr, 0, H, sl2, splits, chunks, w.part_o,
        w.part_ml);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess)
    e = launch_dependent(decode_combine_kernel, dim3(H, B), dim3(2 * kD), 0, stream, w.part_o, w.part_ml,
                         l.n_entries, l.n_max, l.topk, (int)(l.kind == 0), H, splits, SPLIT * chunks, l.out);
  if (e != cudaSuccess) return set_error(CSLC_ERR_CUDA, "decode attention launch: %s", cudaGetErrorString(e));
  return CSLC_OK;
}

// Internal streams and events for the layers after the first, one set per
// host thread and device (created on first use, kept for the process).
constexpr int kMaxLayerStreams = 15;
struct LayerStreams {
  cudaStream_t s[kMaxLayerStreams] = {};
  cudaEvent_t fork = nullptr;
  cudaEvent_t done[kMaxLayerStreams] = {};
};

static cslc_status layer_streams(LayerStreams** out) {
  constexpr int kMaxDevices = 64;
  thread_local LayerStreams sets[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return set_error(CSLC_ERR_CUDA, "cslc_decode_step: no usable current device");
  LayerStreams& o = sets[dev];
  if (!o.fork) {
    e = cudaEventCreateWithFlags(&o.fork, cudaEventDisableTiming);
    for (int j = 0; j < kMaxLayerStreams && e == cudaSuccess; ++j) {
      e = cudaStreamCreateWithFlags(&o.s[j], cudaStreamNonBlocking);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&o.done[j], cudaEventDisableTiming);
    }
    if (e != cudaSuccess) {
      o.fork = nullptr;
      return set_error(CSLC_ERR_CUDA, "cslc_decode_step: stream/event creation: %s", cudaGetErrorString(e));
    }
  }
  *out = &o;
  return CSLC_OK;
}

static cslc_status run_layer(const cslc_decode_layer& l, int B, int H, int HI, DecodeWs& w, cudaStream_t stream);

cslc_status run_decode_step(const cslc_decode_layer* layers, int n_layers, int B, int H, int HI,
                            void* ws, size_t ws_bytes, cudaStream_t stream) {
  (void)ws_bytes;
  if (n_layers > 1 + kMaxLayerStreams)
    return set_error(CSLC_ERR_UNSUPPORTED, "cslc_decode_step: at most %d layers per call", 1 + kMaxLayerStreams);
  // carve: every layer's histogram + counters, then each layer's other buffers
  uint8_t* base = static_cast<uint8_t*>(ws);
  size_t zero_bytes = 0;
  for (int i = 0; i < n_layers; ++i) {
    const DecodeWsSizes s = layer_ws_sizes(layers[i], B, H);
    zero_bytes += s.hist + s.counters;
  }
  uint8_t* zp = base;
  uint8_t* rp = base + zero_bytes;
  DecodeWs w[1 + kMaxLayerStreams];
  for (int i = 0; i < n_layers; ++i) {
    const DecodeWsSizes s = layer_ws_sizes(layers[i], B, H);
    w[i].hist = reinterpret_cast<uint32_t*>(zp); zp += s.hist;
    w[i].counters = reinterpret_cast<int32_t*>(zp); zp += s.counters;
    w[i].scores = reinterpret_cast<float*>(rp); rp += s.scores;
    w[i].sel = reinterpret_cast<int32_t*>(rp); rp += s.sel;
    w[i].cand = reinterpret_cast<uint2*>(rp); rp += s.cand;
    w[i].idx = reinterpret_cast<int32_t*>(rp); rp += s.idx;
    w[i].part_o = reinterpret_cast<float*>(rp); rp += s.part_o;
    w[i].part_ml = reinterpret_cast<float*>(rp); rp += s.part_ml;
  }
  if (zero_bytes && cudaMemsetAsync(base, 0, zero_bytes, stream) != cudaSuccess)
    return set_error(CSLC_ERR_CUDA, "cudaMemsetAsync failed");
  if (n_layers == 1) return run_layer(layers[0], B, H, HI, w[0], stream);
  LayerStreams* ls = nullptr;
  cslc_status st = layer_streams(&ls);
  if (st != CSLC_OK) return st;
  cudaError_t e = cudaEventRecord(ls->fork, stream);
  for (int i = 1; i < n_layers && e == cudaSuccess; ++i) e = cudaStreamWaitEvent(ls->s[i - 1], ls->fork, 0);
  if (e != cudaSuccess) return set_error(CSLC_ERR_CUDA, "cslc_decode_step: %s", cudaGetErrorString(e));
  for (int i = 0; i < n_layers; ++i) {
    st = run_layer(layers[i], B, H, HI, w[i], i == 0 ? stream : ls->s[i - 1]);
    if (st != CSLC_OK) return st;
  }
  // join: `stream` continues after every layer
  for (int i = 1; i < n_layers && e == cudaSuccess; ++i) {
    e = cudaEventRecord(ls->done[i - 1], ls->s[i - 1]);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, ls->done[i - 1], 0);
  }
  if (e != cudaSuccess) return set_error(CSLC_ERR_CUDA, "cslc_decode_step: %s", cudaGetErrorString(e));
  return CSLC_OK;
}

// ---- fused tail: one cluster of CL CTAs per sequence (CL a power of two <= 16)
template <bool SPARSE, int CL>
static cudaError_t launch_tail(const cslc_decode_layer& l, int B, int H, const float* scores, const DecodeWs& w,
                               bool dependent, cudaStream_t stream) {
  static int configured_for = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_for != dev) {
    cudaFuncSetAttribute(decode_tail_kernel<SPARSE, CL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)tail_smem_bytes(128));
    if (CL > 8) cudaFuncSetAttribute(decode_tail_kernel<SPARSE, CL>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    configured_for = dev;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CL, B);
  cfg.blockDim = dim3(TAIL_THREADS);
  cfg.dynamicSmemBytes = tail_smem_bytes(H);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeClusterDimension;
  attr[na].val.clusterDim.x = CL;
  attr[na].val.clusterDim.y = 1;
  attr[na].val.clusterDim.z = 1;
  ++na;
  if (dependent) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, decode_tail_kernel<SPARSE, CL>, l.q, l.nope, l.rope, l.kv_scale, l.n_entries,
                            l.n_max, scores, (const uint32_t*)w.hist, w.cand, SPARSE ? l.topk : 0, H,
                            l.scale * kLog2e, SPARSE ? l.idx_out : (int32_t*)nullptr, l.out);
}

template <bool SPARSE>
static cudaError_t launch_tail_cl(int CL, const cslc_decode_layer& l, int B, int H, const float* scores,
                                  const DecodeWs& w, bool dependent, cudaStream_t stream) {
  switch (CL) {
    case 1: return launch_tail<SPARSE, 1>(l, B, H, scores, w, dependent, stream);
    case 2: return launch_tail<SPARSE, 2>(l, B, H, scores, w, dependent, stream);
    case 4: return launch_tail<SPARSE, 4>(l, B, H, scores, w, dependent, stream);
    case 8: return launch_tail<SPARSE, 8>(l, B, H, scores, w, dependent, stream);
    default: return launch_tail<SPARSE, 16>(l, B, H, scores, w, dependent, stream);
  }
}

// Per device, once: the SM count and whether 16-CTA clusters of the tail
// kernel fit (a non-portable size).
struct TailDevice {
  int sms = 0;
  bool cl16 = false;
};
static bool tail_device(TailDevice* out) {
  constexpr int kMaxDevices = 64;
  static TailDevice info[kMaxDevices];
  static bool known[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  if (!known[dev]) {
    TailDevice t;
    if (cudaDeviceGetAttribute(&t.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return false;
    }
    cudaFuncSetAttribute(decode_tail_kernel<true, 16>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    cudaFuncSetAttribute(decode_tail_kernel<true, 16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)tail_smem_bytes(128));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(16, 1);
    cfg.blockDim = dim3(TAIL_THREADS);
    cfg.dynamicSmemBytes = tail_smem_bytes(128);
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 16;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    const cudaError_t e = cudaOccupancyMaxActiveClusters(&n, decode_tail_kernel<true, 16>, &cfg);
    if (e != cudaSuccess) cudaGetLastError();
    t.cl16 = e == cudaSuccess && n > 0;
    info[dev] = t;
    known[dev] = true;
  }
  *out = info[dev];
  return true;
}

// The tail of a CSA layer as one cluster launch when it fits: the cluster
// size aims at one CTA per SM over the batch (a CTA of this kernel takes a
// whole SM), and a cluster must cover the context with its bitmaps (131,072
// entries per CTA). HCA layers keep the split attention + combine kernels.
// Returns false to use the separate kernels.
static bool run_tail_fused(const cslc_decode_layer& l, int B, int H, const float* scores, const DecodeWs& w,
                           bool dependent, cudaStream_t stream, cslc_status* st) {
  TailDevice dv;
  if (!tail_device(&dv)) return false;
  // a CTA takes a whole SM, so 16-CTA clusters only fit a few GPCs at a time:
  // 16 only when a context needs it
  const int cl_max = dv.cl16 ? 16 : 8;
  int CL = 1;
  while (CL < 8 && (long long)B * CL * 2 <= dv.sms) CL *= 2;
  // small batches (B x 4 < SMs) keep the separate kernels: their clusters
  // would hold whole SMs that the other layers' concurrent kernels need
  // (measured: hybrid 1M step, B = 8, 189 us split vs 204 us fused; CSA
  // 64 x 32,768, 120 us split vs 103 us fused)
  if (l.kind != 0 || (long long)B * 4 < dv.sms) return false;
  while (CL < cl_max && (long long)l.n_max > (long long)CL * TAIL_BM_WORDS * 32) CL *= 2;
  if ((long long)l.n_max > (long long)CL * TAIL_BM_WORDS * 32) return false;
  const cudaError_t e = launch_tail_cl<true>(CL, l, B, H, scores, w, dependent, stream);
  *st = e == cudaSuccess ? CSLC_OK : set_error(CSLC_ERR_CUDA, "decode tail launch: %s", cudaGetErrorString(e));
  return true;
}

static cslc_status run_layer(const cslc_decode_layer& l, int B, int H, int HI, DecodeWs& w, cudaStream_t stream) {
  {
    cslc_status st;
    if (l.kind == 0) {
      float* scores = l.scores_out ? l.scores_out : w.scores;
      int32_t* idx = l.idx_out ? l.idx_out : w.idx;
      if (l.n_max > 0) {
        const dim3 grid((l.n_max + DEC_CHUNK - 1) / DEC_CHUNK, B);
        if (HI <= 8)
          decode_scores_kernel<1><<<grid, DEC_THREADS, 0, stream>>>(l.q_idx, l.w, l.k_idx, l.n_entries,
                                                                    l.n_max, HI, scores, w.hist);
        else
          decode_scores_kernel<2><<<grid, DEC_THREADS, 0, stream>>>(l.q_idx, l.w, l.k_idx, l.n_entries,
                                                                    l.n_max, HI, scores, w.hist);
        st = check_launch("decode_scores_kernel");
        if (st != CSLC_OK) return st;
      }
      if (B > 0 && run_tail_fused(l, B, H, scores, w, l.n_max > 0, stream, &st)) return st;
      st = run_topk_stages(scores, l.n_entries, B, l.n_max, l.topk, w, idx, stream);
      if (st != CSLC_OK) return st;
      st = run_attention(l, B, H, idx, w, stream);
    } else {
      st = run_attention(l, B, H, nullptr, w, stream);
    }
    return st;
  }
}

cslc_status run_decode_topk(const float* scores, const int32_t* n_entries, int B, int n_max, int topk,
                            int32_t* idx, void* ws, cudaStream_t stream) {
  DecodeWsSizes s = ws_sizes(B, n_max, topk, 1, 16);
  s.scores = s.idx = s.part_o = s.part_ml = 0;
  DecodeWs w;
  carve(static_cast<uint8_t*>(ws), s, w);
  if (cudaMemsetAsync(w.hist, 0, s.hist + s.counters, stream) != cudaSuccess)
    return set_error(CSLC_ERR_CUDA, "cudaMemsetAsync failed");
  if (n_max > 0) {
    const dim3 grid((n_max + DEC_CHUNK - 1) / DEC_CHUNK, B);
    decode_hist_kernel<<<grid, DEC_THREADS, 0, stream>>>(scores, n_entries, n_max, w.hist);
    cslc_status st = check_launch("decode_hist_kernel");
    if (st != CSLC_OK) return st;
  }
  return run_topk_stages(scores, n_entries, B, n_max, topk, w, idx, stream);
}

}  // namespace cslc
