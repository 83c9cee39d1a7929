// Lightning-indexer scores for prefill on the 5th-generation tensor cores
// (tcgen05 + TMEM). "读完这篇你就搞懂 DeepSeek v4 了", §三 闪电索引: every query
// token is scored against every visible compressed entry,
//   S[t, i] = sum_h w[t, h] * max(0, q_I[t, h, :] . k_I[i, :]),
// fp32 accumulation of bf16 products; the ReLU acts per head before the sum.
//
// One MMA tile is D = K_I E^T with
//   A = 128 consecutive entries of k_I           (128 x d_I, K-major, TMA)
//   B = 256 (token, head) rows of q_I: 256 / HP tokens x HP heads, where HP is
//       H_I rounded up to a power of two (a 3-D TMA over tokens x heads x
//       dims fills the heads past H_I with zeros; their weights are zero)
// so D (fp32, in TMEM) holds entry i in lane i and pair (t, h) in column
// t*HP + h: the weighted ReLU head sum of a score is a sum over HP adjacent
// columns inside one thread, and a warp's 32 lanes store 32 consecutive
// entries of one score row (128-byte stores). Boxes reaching past the end of
// q_I or k_I read zeros, so any size runs on this kernel.
//
// CTA roles (persistent, one CTA per SM; work items = a query-row tile and a
// chunk of 16 key tiles, heavy rows first, dealt to the CTAs in a snake so that
// every CTA gets a similar load):
//   warp 0     producer: per row tile the Q tile (TMA) and the weights (fp32
//              in shared memory), then the visible key tiles (TMA, 4 stages);
//   warp 1     TMEM allocation and the single MMA-issuing thread (4 MMAs of
//              K = 16 per tile, M = 128, N = 256);
//   warps 2-17 epilogue: warp w reads TMEM lanes 32*(w%4).. (its entries) and
//              one quarter of the columns, forms the scores of its rows and
//              stores those of visible entries.
// TMEM: two accumulators of 256 columns (tile j+1 is computed while tile j is
// read out). All waits are time-bounded (abort + device error word).
//
// FP8 variant (first page §1.4: a low-precision lightning indexer): q_I and
// k_I arrive as e4m3 codes with one fp32 scale per (token, head) row and per
// entry. The tiles are 64-byte rows in the 64-byte swizzle, the products are
// kind::f8f6f4 (K = 32, two per tile) with fp32 accumulation, and since the
// scales are positive, S[t, i] = k_scale[i] * sum_h (w[t, h] q_scale[t, h]) *
// max(0, q8[t, h] . k8[i]): the producer folds q_scale into the head weights
// and the epilogue multiplies by k_scale.

#include "sm100.cuh"

namespace cslc {

using namespace sm100;

__device__ int g_indexer_err = 0;

namespace {

constexpr int IX_THREADS = 576;
constexpr int IX_PROD_WARP = 0;
constexpr int IX_MMA_WARP = 1;
constexpr int IX_EPI_WARP0 = 2;
constexpr int IX_EPI_WARPS = 16;
constexpr int IX_ET = 128;                       // entries per key tile (MMA M)
constexpr int IX_NP = 256;                       // (token, head) pairs per query tile (MMA N)
constexpr int IX_EPI_COLS = IX_NP / (IX_EPI_WARPS / 4);   // accumulator columns per epilogue warp
constexpr int IX_KSTAGES = 4;
constexpr int IX_CHUNK = 16;                     // key tiles per work item (2048 entries)
constexpr int IX_K_BYTES = IX_ET * 128;          // 16 KB: 128 entries x 64 bf16
constexpr int IX_Q_BYTES = IX_NP * 128;          // 32 KB: 256 pairs x 64 bf16

enum { ERR_Q_EMPTY = 1, ERR_K_EMPTY, ERR_Q_FULL, ERR_K_FULL, ERR_D_EMPTY, ERR_D_FULL, ERR_FINAL };

struct __align__(8) IxBars {
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[IX_KSTAGES], k_empty[IX_KSTAGES];
  uint64_t d_full[2], d_empty[2];
  uint64_t final_bar;
};

struct IxSmall {
  IxBars bars;
  uint32_t tmem_base;
  int abort_flag;
};

// Waits for a phase regardless of the abort flag (used only to let copies in
// flight land before an aborted CTA exits); bounded like every other wait.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_ns();
  while (!mbar_test(bar, parity) && global_ns() - t0 < kWaitLimitNs) {}
}

}  // namespace

// Score store: fp32, or bf16 (round to nearest even) for the half-size score path.
__device__ __forceinline__ void store_score(float* p, float v) { *p = v; }
__device__ __forceinline__ void store_score(uint16_t* p, float v) { *p = __bfloat16_as_ushort(__float2bfloat16_rn(v)); }

template <int HI, typename OutT, bool FP8>   // HI: heads per token in a tile (H_I rounded up to a power of two)
__global__ void __launch_bounds__(IX_THREADS, 1) indexer_sm100_kernel(
    const uint16_t* __restrict__ w, const float* __restrict__ q_scale, const float* __restrict__ k_scale, int B,
    int L, int Nc, int HI_act, int m, int q_pos0, int row_begin, int row_end, OutT* __restrict__ scores,
    int rows_in_buf, const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k) {
  constexpr int RT = IX_NP / HI;                 // query rows per tile
  // bytes of a loaded tile (the shared-memory slots are sized for bf16)
  constexpr uint32_t Q_TX = FP8 ? IX_NP * 64 : IX_Q_BYTES, K_TX = FP8 ? IX_ET * 64 : IX_K_BYTES;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_s = smem;                                        // [2][256 pairs][128 B]
  uint8_t* k_s = q_s + 2 * IX_Q_BYTES;                        // [KSTAGES][128 entries][128 B]
  float* w_s = reinterpret_cast<float*>(k_s + IX_KSTAGES * IX_K_BYTES);   // [2][256] weights per pair
  int* nv_s = reinterpret_cast<int*>(w_s + 2 * IX_NP);                     // [2][256] visible entries per row
  IxSmall* sm = reinterpret_cast<IxSmall*>(nv_s + 2 * IX_NP);
  IxBars& bars = sm->bars;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  const int rt_per_b = (row_end - row_begin + RT - 1) / RT;
  // work items: (query-row tile, chunk of IX_CHUNK key tiles), so that a block
  // of rows with fewer row tiles than SMs still fills the GPU
  const int et_max = (n_visible((long long)q_pos0 + row_end - 1, m, Nc) + IX_ET - 1) / IX_ET;
  const int n_ch = max(1, (et_max + IX_CHUNK - 1) / IX_CHUNK);
  const int n_items = B * rt_per_b * n_ch;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.q_full[i], 1);
      mbar_init(&bars.q_empty[i], 1 + IX_EPI_WARPS);
      mbar_init(&bars.d_full[i], 1);
      mbar_init(&bars.d_empty[i], IX_EPI_WARPS);
    }
    for (int s = 0; s < IX_KSTAGES; ++s) { mbar_init(&bars.k_full[s], 1); mbar_init(&bars.k_empty[s], 1); }
    mbar_init(&bars.final_bar, 1);
    sm->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == IX_MMA_WARP) tmem_alloc(&sm->tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;
  volatile int* abortp = &sm->abort_flag;
  int* errp = &g_indexer_err;

  // j-th work item of this CTA (snake over rounds of gridDim.x) -> batch,
  // first row, first key tile and number of key tiles (0: nothing visible in
  // this chunk); false when the CTA has no more items
  auto tile_of = [&](int j, int& b, int& t0, int& et0, int& n_et) -> bool {
    const int G = gridDim.x;
    const int i = j * G + ((j & 1) ? G - 1 - (int)blockIdx.x : (int)blockIdx.x);
    if (i >= n_items) return false;
    const int rb = i / n_ch;
    const int rt = rt_per_b - 1 - rb / B;          // heavy (late) rows first
    b = rb % B;
    t0 = row_begin + rt * RT;
    const int t_last = min(t0 + RT, row_end) - 1;
    const int n_all = (n_visible((long long)q_pos0 + t_last, m, Nc) + IX_ET - 1) / IX_ET;
    et0 = (i % n_ch) * IX_CHUNK;
    n_et = max(0, min(IX_CHUNK, n_all - et0));
    return true;
  };

  if (warp == IX_PROD_WARP) {
    // ------------------------------------------------------------ producer
    if (lane == 0) { tma_prefetch_map(&tm_q); tma_prefetch_map(&tm_k); }
    int rq = 0, kt = 0;
    bool ok = true;
    int b, t0, et0, n_et;
    for (int j = 0; ok && tile_of(j, b, t0, et0, n_et); ++j) {
      if (n_et == 0) continue;
      const int qs = rq & 1;
      bool w_ok = true;
      if (lane == 0 && rq >= 2)
        w_ok = mbar_wait(&bars.q_empty[qs], (uint32_t)(((rq >> 1) - 1) & 1), abortp, errp, ERR_Q_EMPTY);
      if (!__shfl_sync(0xffffffffu, (int)w_ok, 0)) break;
#pragma unroll
      for (int x = 0; x < IX_NP / 32; ++x) {
        const int j = x * 32 + lane, t = t0 + j / HI, h = j % HI;   // pair j of the tile
        const bool real = h < HI_act && t < L;                     // padding heads and rows past L weigh 0
        const long long p = ((long long)b * L + t) * HI_act + h;
        float wv = real ? bf16_to_f(w[p]) : 0.f;
        if constexpr (FP8) wv *= real ? q_scale[p] : 0.f;
        w_s[qs * IX_NP + x * 32 + lane] = wv;
      }
      for (int r = lane; r < RT; r += 32)
        nv_s[qs * IX_NP + r] = t0 + r < row_end ? n_visible((long long)q_pos0 + t0 + r, m, Nc) : 0;
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(&bars.q_full[qs], Q_TX);
        tma_load_3d(q_s + qs * IX_Q_BYTES, &tm_q, 0, 0, b * L + t0, &bars.q_full[qs]);
        for (int et = et0; et < et0 + n_et; ++et, ++kt) {
          const int ks = kt % IX_KSTAGES;
          if (kt >= IX_KSTAGES &&
              !mbar_wait(&bars.k_empty[ks], (uint32_t)((kt / IX_KSTAGES - 1) & 1), abortp, errp, ERR_K_EMPTY)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars.k_full[ks], K_TX);
          tma_load_2d(k_s + ks * IX_K_BYTES, &tm_k, 0, b * Nc + et * IX_ET, &bars.k_full[ks]);
        }
      }
      ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
      ++rq;
    }
    if (lane == 0 && *abortp) {
      // let the copies still in flight land before the CTA exits
      for (int i = max(0, kt - IX_KSTAGES); i < kt; ++i)
        drain_wait(&bars.k_full[i % IX_KSTAGES], (uint32_t)((i / IX_KSTAGES) & 1));
      for (int i = max(0, rq - 2); i < rq; ++i) drain_wait(&bars.q_full[i & 1], (uint32_t)((i >> 1) & 1));
    }
    __syncwarp();
  } else if (warp == IX_MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID = FP8 ? idesc_e4m3(IX_ET, IX_NP) : idesc_bf16(IX_ET, IX_NP, false, false);
      int rq = 0, kt = 0;
      bool ok = true;
      int b, t0, et0, n_et;
      for (int j = 0; ok && tile_of(j, b, t0, et0, n_et); ++j) {
        if (n_et == 0) continue;
        const int qs = rq & 1;
        if (!mbar_wait(&bars.q_full[qs], (uint32_t)((rq >> 1) & 1), abortp, errp, ERR_Q_FULL)) break;
        const uint32_t q0 = smem_u32(q_s + qs * IX_Q_BYTES);
        for (int et = et0; et < et0 + n_et; ++et, ++kt) {
          const int ks = kt % IX_KSTAGES, ds = kt & 1;
          if (!mbar_wait(&bars.k_full[ks], (uint32_t)((kt / IX_KSTAGES) & 1), abortp, errp, ERR_K_FULL) ||
              (kt >= 2 && !mbar_wait(&bars.d_empty[ds], (uint32_t)(((kt >> 1) - 1) & 1), abortp, errp, ERR_D_EMPTY))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t k0 = smem_u32(k_s + ks * IX_K_BYTES);
          if constexpr (FP8) {
#pragma unroll
            for (int k = 0; k < 2; ++k)   // K = 32 e4m3 per product: 32 bytes along the 64-byte rows
              mma_e4m3(tmem + ds * IX_NP, smem_desc_sw64(k0 + k * 32, 16, 512),
                       smem_desc_sw64(q0 + k * 32, 16, 512), ID, k > 0 ? 1u : 0u);
          } else {
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_bf16(tmem + ds * IX_NP, smem_desc_sw128(k0 + k * 32, 16, 1024),
                       smem_desc_sw128(q0 + k * 32, 16, 1024), ID, k > 0 ? 1u : 0u);
          }
          mma_commit(&bars.k_empty[ks]);
          mma_commit(&bars.d_full[ds]);
        }
        if (!ok) break;
        mma_commit(&bars.q_empty[qs]);
        ++rq;
      }
      mma_commit(&bars.final_bar);
      mbar_wait_done(&bars.final_bar, 0, errp, ERR_FINAL);   // also after an abort: the products finish on their own
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;                        // TMEM lanes 32*quad .. 32*quad+31
    const int part = (warp - IX_EPI_WARP0) >> 2;      // columns IX_EPI_COLS*part ..
    constexpr int RH = IX_EPI_COLS / HI;              // rows per part
    static_assert(32 % HI == 0, "a 32-column chunk holds whole rows");
    int rq = 0, kt = 0;
    bool ok = true;
    int b, t0, et0, n_et;
    for (int j = 0; ok && tile_of(j, b, t0, et0, n_et); ++j) {
      if (n_et == 0) continue;
      const int qs = rq & 1;
      bool w_ok = true;
      if (lane == 0) w_ok = mbar_wait(&bars.q_full[qs], (uint32_t)((rq >> 1) & 1), abortp, errp, ERR_Q_FULL);
      if (!__shfl_sync(0xffffffffu, (int)w_ok, 0)) break;
      const float4* wr = reinterpret_cast<const float4*>(w_s + qs * IX_NP + part * IX_EPI_COLS);
      const int* nvr = nv_s + qs * IX_NP + part * RH;
      const int r0 = t0 + part * RH;                  // first row of this warp's part
      OutT* out0 = scores + ((size_t)b * rows_in_buf + (r0 - row_begin)) * (size_t)Nc;
      for (int et = et0; et < et0 + n_et; ++et, ++kt) {
        const int ds = kt & 1;
        bool d_ok = true;
        if (lane == 0) d_ok = mbar_wait(&bars.d_full[ds], (uint32_t)((kt >> 1) & 1), abortp, errp, ERR_D_FULL);
        if (!__shfl_sync(0xffffffffu, (int)d_ok, 0)) { ok = false; break; }
        tc_fence_after();
        const int e = et * IX_ET + quad * 32 + lane;
        float ksc = 1.f;
        if constexpr (FP8) ksc = e < Nc ? k_scale[(size_t)b * Nc + e] : 0.f;
        const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + ds * IX_NP + part * IX_EPI_COLS;
        // one 32-column chunk per TMEM wait; each score's head sum runs as two
        // independent FMA chains
#pragma unroll
        for (int c = 0; c < IX_EPI_COLS / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(taddr + c * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int rr = 0; rr < 32 / HI; ++rr) {
            const int r = c * (32 / HI) + rr;
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int h4 = 0; h4 < (HI + 3) / 4; ++h4) {
              const int p = rr * HI + 4 * h4;          // first pair of this group of 4 heads
              float wq[4];
              if (HI >= 4) {
                const float4 f = wr[(c * 32 + p) / 4];
                wq[0] = f.x; wq[1] = f.y; wq[2] = f.z; wq[3] = f.w;
              } else {
#pragma unroll
                for (int q = 0; q < HI; ++q) wq[q] = reinterpret_cast<const float*>(wr)[c * 32 + p + q];
              }
#pragma unroll
              for (int q = 0; q < (HI < 4 ? HI : 4); ++q) {
                const float x = fmaxf(__uint_as_float(v[p + q]), 0.f);
                if (q & 1) s1 = fmaf(wq[q], x, s1); else s0 = fmaf(wq[q], x, s0);
              }
            }
            if constexpr (FP8) {
              if (e < nvr[r]) store_score(out0 + (size_t)r * Nc + e, ksc * (s0 + s1));
            } else {
              if (e < nvr[r]) store_score(out0 + (size_t)r * Nc + e, s0 + s1);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.d_empty[ds]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.q_empty[qs]);
      ++rq;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == IX_MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <typename OutT, bool FP8>
static cslc_status launch_indexer_sm100_t(const void* q_idx, const uint16_t* w, const void* k_idx,
                                          const float* q_scale, const float* k_scale, int B, int L, int Nc, int HI,
                                          int m, int q_pos0, int row_begin, int row_end, OutT* scores,
                                          int rows_in_buf, cudaStream_t stream) {
  static int configured_for = -1;
  static int n_sm = 148;
  int dev = 0;
  cudaGetDevice(&dev);
  const size_t smem = 1024 + 2 * IX_Q_BYTES + IX_KSTAGES * IX_K_BYTES + 2 * IX_NP * (sizeof(float) + sizeof(int)) +
                      sizeof(IxSmall);
  if (configured_for != dev) {
    cudaFuncSetAttribute(indexer_sm100_kernel<1, OutT, FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(indexer_sm100_kernel<2, OutT, FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(indexer_sm100_kernel<4, OutT, FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(indexer_sm100_kernel<8, OutT, FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(indexer_sm100_kernel<16, OutT, FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    configured_for = dev;
  }
  const int HP = HI <= 1 ? 1 : HI <= 2 ? 2 : HI <= 4 ? 4 : HI <= 8 ? 8 : 16;
  const int RT = IX_NP / HP;
  const int et_max = (n_visible((long long)q_pos0 + row_end - 1, m, Nc) + IX_ET - 1) / IX_ET;
  const int n_ch = et_max > IX_CHUNK ? (et_max + IX_CHUNK - 1) / IX_CHUNK : 1;
  const int n_items = B * ((row_end - row_begin + RT - 1) / RT) * n_ch;
  const int grid = n_items < n_sm ? n_items : n_sm;
  CUtensorMap tm_q, tm_k;
  const int eb = FP8 ? 1 : 2;   // bytes per element; a row is 64 elements
  const bool maps_ok =
      make_tmap_rows3d(&tm_q, q_idx, eb, (uint64_t)HI, (uint64_t)B * L, (uint32_t)HP, (uint32_t)RT) &&
      (FP8 ? make_tmap_u8_rows64(&tm_k, k_idx, (uint64_t)B * Nc, IX_ET)
           : make_tmap_bf16_2d(&tm_k, k_idx, (uint64_t)B * Nc, kDI, kDI * 2, IX_ET, 64));
  if (!maps_ok) return set_error(CSLC_ERR_CUDA, "csa_indexer_topk: tensor map encoding failed");
  switch (HP) {
    case 1: indexer_sm100_kernel<1, OutT, FP8><<<grid, IX_THREADS, smem, stream>>>(w, q_scale, k_scale, B, L, Nc, HI, m, q_pos0, row_begin, row_end, scores, rows_in_buf, tm_q, tm_k); break;
    case 2: indexer_sm100_kernel<2, OutT, FP8><<<grid, IX_THREADS, smem, stream>>>(w, q_scale, k_scale, B, L, Nc, HI, m, q_pos0, row_begin, row_end, scores, rows_in_buf, tm_q, tm_k); break;
    case 4: indexer_sm100_kernel<4, OutT, FP8><<<grid, IX_THREADS, smem, stream>>>(w, q_scale, k_scale, B, L, Nc, HI, m, q_pos0, row_begin, row_end, scores, rows_in_buf, tm_q, tm_k); break;
    case 8: indexer_sm100_kernel<8, OutT, FP8><<<grid, IX_THREADS, smem, stream>>>(w, q_scale, k_scale, B, L, Nc, HI, m, q_pos0, row_begin, row_end, scores, rows_in_buf, tm_q, tm_k); break;
    default: indexer_sm100_kernel<16, OutT, FP8><<<grid, IX_THREADS, smem, stream>>>(w, q_scale, k_scale, B, L, Nc, HI, m, q_pos0, row_begin, row_end, scores, rows_in_buf, tm_q, tm_k); break;
  }
  return check_launch("indexer_sm100_kernel");
}

// scores: fp32 [rows][Nc], or bf16 when bf16_out
cslc_status launch_indexer_sm100(const uint16_t* q_idx, const uint16_t* w, const uint16_t* k_idx, int B,
                                 int L, int Nc, int HI, int m, int q_pos0, int row_begin, int row_end,
                                 void* scores, bool bf16_out, int rows_in_buf, cudaStream_t stream) {
  if (bf16_out)
    return launch_indexer_sm100_t<uint16_t, false>(q_idx, w, k_idx, nullptr, nullptr, B, L, Nc, HI, m, q_pos0,
                                                   row_begin, row_end, static_cast<uint16_t*>(scores), rows_in_buf,
                                                   stream);
  return launch_indexer_sm100_t<float, false>(q_idx, w, k_idx, nullptr, nullptr, B, L, Nc, HI, m, q_pos0, row_begin,
                                              row_end, static_cast<float*>(scores), rows_in_buf, stream);
}

// e4m3 operands with per-row scales; fp32 scores [rows][Nc]
cslc_status launch_indexer_sm100_fp8(const uint8_t* q8, const float* q_scale, const uint16_t* w, const uint8_t* k8,
                                     const float* k_scale, int B, int L, int Nc, int HI, int m, int q_pos0,
                                     int row_begin, int row_end, float* scores, int rows_in_buf, cudaStream_t stream) {
  return launch_indexer_sm100_t<float, true>(q8, w, k8, q_scale, k_scale, B, L, Nc, HI, m, q_pos0, row_begin,
                                             row_end, scores, rows_in_buf, stream);
}

int indexer_sm100_read_error() {
  int v = 0, zero = 0;
  cudaMemcpyFromSymbol(&v, g_indexer_err, sizeof(int));
  if (v) cudaMemcpyToSymbol(g_indexer_err, &zero, sizeof(int));
  return v;
}

CSLC_DEFINE_WAIT_LIMIT_SETTER(indexer_sm100_set_wait_limits)

}  // namespace cslc
