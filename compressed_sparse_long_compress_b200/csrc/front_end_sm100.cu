// Compressor front end on the 5th-generation tensor cores: the learned
// projections of the hidden states and the window compression in one kernel.
//
// "读完这篇你就搞懂 DeepSeek v4 了", §三 压缩机制: the compressor has 4 learnable W
// matrices and 2 learnable B matrices. Read as: c^a = h W^{a,KV}, c^b = h
// W^{b,KV}, z^a = h W^{a,Z}, z^b = h W^{b,Z} (per token), and entry i, channel
// j = sum over the overlapped 2m-token window of softmax_t(z_t[j] + B[slot][j])
// c_t[j], where the C^b half (tokens (i-1)m .. im-1) uses (c^b, z^b, B^b) and
// the C^a half (tokens im .. im+m-1) uses (c^a, z^a, B^a). HCA (first page
// §1.2): W^{KV}, W^{Z} and one B over non-overlapping m'-token windows.
//
// Work item: 128 consecutive token rows (the MMA M) x 256 accumulator
// columns. CSA: one of two 64-channel halves, columns [c^a | c^b | z^a | z^b]
// of those channels; a tile starts m tokens early so that its first entry's
// C^b group is inside it, and yields (128 - m) / m entries. HCA (m' = 128):
// columns [c | z] of all 128 channels, one entry per tile. The K loop runs
// over d_model in 64-element stages (TMA, 128-byte swizzle, 4-stage ring);
// products accumulate in fp32 in TMEM (two 256-column accumulators, so that
// the epilogue of one item overlaps the products of the next). The epilogue
// moves 16 channels at a time from TMEM through shared memory and computes
// the window softmax in fp32 from the unrounded projections.
//
// CTA roles (persistent, one CTA per SM): warp 0 TMA producer, warp 1 TMEM
// allocation and the single MMA-issuing thread, warps 2-5 epilogue (TMEM lane
// quadrant = warp & 3). Every wait is time-bounded; a timeout raises a
// CTA-wide abort and records a code read by cslc_sync_status.

#include "sm100.cuh"

namespace cslc {

using namespace sm100;

__device__ int g_front_end_err = 0;

namespace {

constexpr int FE_THREADS = 192;
constexpr int FE_EPI_WARP0 = 2;
constexpr int FE_NEPI = 128;
constexpr int FE_ROWS = 128;
constexpr int FE_N = 256;
constexpr int FE_KB = 64;
constexpr int FE_STAGES = 4;
constexpr int FE_A_BYTES = FE_ROWS * 128;             // 16 KB
constexpr int FE_B_BYTES = FE_N * 128;                // 32 KB
constexpr int FE_STAGE_BYTES = FE_A_BYTES + FE_B_BYTES;
constexpr int FE_CH = 16;                             // channels per epilogue block
constexpr int FE_STAGE_F = 4 * FE_CH * FE_ROWS;       // floats of epilogue staging (32 KB)

enum { FE_ERR_FULL = 1, FE_ERR_EMPTY, FE_ERR_ACC_FULL, FE_ERR_ACC_EMPTY, FE_ERR_FINAL };

struct __align__(8) FeBars {
  uint64_t full[FE_STAGES], empty[FE_STAGES];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t final_bar;
};

struct FeSmall {
  FeBars bars;
  uint32_t tmem_base;
  int abort_flag;
};

struct FeShape {
  int B, L, d_model, m, n_c, per_tile, n_tiles, n_items;
};

__device__ __forceinline__ void fe_item(const FeShape& sh, bool overlap, long long it, int& b, int& t, int& hc) {
  if (overlap) {
    hc = (int)(it & 1);
    const long long bt = it >> 1;
    b = (int)(bt / sh.n_tiles);
    t = (int)(bt - (long long)b * sh.n_tiles);
  } else {
    hc = 0;
    b = (int)(it / sh.n_tiles);
    t = (int)(it - (long long)b * sh.n_tiles);
  }
}

}  // namespace

template <bool OVERLAP>
__global__ void __launch_bounds__(FE_THREADS, 1) front_end_sm100_kernel(
    FeShape sh, const uint16_t* __restrict__ pos_bias, uint16_t* __restrict__ out,
    const __grid_constant__ CUtensorMap tm_h, const __grid_constant__ CUtensorMap tm_w) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;                                                   // [STAGES][A 16 KB | B 32 KB]
  float* stage_f = reinterpret_cast<float*>(smem + FE_STAGES * FE_STAGE_BYTES);   // [4][16][128]
  FeSmall* sm = reinterpret_cast<FeSmall*>(stage_f + FE_STAGE_F);
  FeBars& bars = sm->bars;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kblocks = sh.d_model / FE_KB;

  if (tid == 0) {
    for (int s = 0; s < FE_STAGES; ++s) { mbar_init(&bars.full[s], 1); mbar_init(&bars.empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&bars.acc_full[a], 1); mbar_init(&bars.acc_empty[a], FE_NEPI / 32); }
    mbar_init(&bars.final_bar, 1);
    sm->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 1) tmem_alloc(&sm->tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;
  volatile int* abortp = &sm->abort_flag;
  int* errp = &g_front_end_err;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_map(&tm_h);
      tma_prefetch_map(&tm_w);
      int kv = 0;
      bool ok = true;
      for (long long it = blockIdx.x; it < sh.n_items && ok; it += gridDim.x) {
        int b, t, hc;
        fe_item(sh, OVERLAP, it, b, t, hc);
        const int T = OVERLAP ? t * sh.per_tile * sh.m - sh.m : t * FE_ROWS;
        const int row = b * sh.L + T;   // a negative first tile reads the fill value (never used)
        for (int kb = 0; kb < kblocks; ++kb, ++kv) {
          const int s = kv % FE_STAGES;
          if (kv >= FE_STAGES &&
              !mbar_wait(&bars.empty[s], (uint32_t)((kv / FE_STAGES - 1) & 1), abortp, errp, FE_ERR_EMPTY)) {
            ok = false;
            break;
          }
          uint8_t* a_s = stages + s * FE_STAGE_BYTES;
          uint8_t* b_s = a_s + FE_A_BYTES;
          mbar_arrive_expect_tx(&bars.full[s], (uint32_t)FE_STAGE_BYTES);
          tma_load_2d(a_s, &tm_h, kb * FE_KB, row, &bars.full[s]);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            // CSA: stream k's 64 channels of half hc; HCA: rows 64k .. 64k+63 of [W^KV; W^Z]
            const int wrow = OVERLAP ? k * 128 + hc * 64 : k * 64;
            tma_load_2d(b_s + k * 64 * 128, &tm_w, kb * FE_KB, wrow, &bars.full[s]);
          }
        }
      }
      // copies in flight after an abort land before the CTA leaves
      for (int d = 1; d <= FE_STAGES && kv - d >= 0; ++d) {
        const int k2 = kv - d;
        mbar_wait_done(&bars.full[k2 % FE_STAGES], (uint32_t)((k2 / FE_STAGES) & 1), errp, FE_ERR_FULL);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID = idesc_bf16(FE_ROWS, FE_N, false, false);
      int kv = 0, n = 0;
      bool ok = true;
      for (long long it = blockIdx.x; it < sh.n_items && ok; it += gridDim.x, ++n) {
        const int acc = n & 1;
        if (n >= 2 && !mbar_wait(&bars.acc_empty[acc], (uint32_t)(((n >> 1) - 1) & 1), abortp, errp, FE_ERR_ACC_EMPTY))
          break;
        tc_fence_after();
        for (int kb = 0; kb < kblocks; ++kb, ++kv) {
          const int s = kv % FE_STAGES;
          if (!mbar_wait(&bars.full[s], (uint32_t)((kv / FE_STAGES) & 1), abortp, errp, FE_ERR_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(stages + s * FE_STAGE_BYTES);
          const uint32_t b0 = a0 + FE_A_BYTES;
#pragma unroll
          for (int k = 0; k < FE_KB / 16; ++k)
            mma_bf16(tmem + acc * FE_N, smem_desc_sw128(a0 + k * 32, 16, 1024), smem_desc_sw128(b0 + k * 32, 16, 1024),
                     ID, (kb > 0 || k > 0) ? 1u : 0u);
          mma_commit(&bars.empty[s]);
        }
        if (!ok) break;
        mma_commit(&bars.acc_full[acc]);
      }
      mma_commit(&bars.final_bar);
      mbar_wait_done(&bars.final_bar, 0, errp, FE_ERR_FINAL);   // also after an abort
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int e = tid - FE_EPI_WARP0 * 32;   // 0..127
    const int qd = warp & 3;
    const int r = qd * 32 + lane;            // token row of the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    const int m = sh.m;
    int n = 0;
    bool ok = true;
    for (long long it = blockIdx.x; it < sh.n_items && ok; it += gridDim.x, ++n) {
      int b, t, hc;
      fe_item(sh, OVERLAP, it, b, t, hc);
      const int acc = n & 1;
      {
        bool w = true;
        if (e == 0) w = mbar_wait(&bars.acc_full[acc], (uint32_t)((n >> 1) & 1), abortp, errp, FE_ERR_ACC_FULL);
        ok = !named_bar_or(1, FE_NEPI, !w);
      }
      if (!ok) break;
      tc_fence_after();
      constexpr int NBLK = OVERLAP ? 64 / FE_CH : 128 / FE_CH;
      for (int q = 0; q < NBLK; ++q) {
        // this row's values of the block's 16 channels, per stream
        constexpr int NS = OVERLAP ? 4 : 2;
#pragma unroll
        for (int st = 0; st < NS; ++st) {
          uint32_t v[16];
          const int col = OVERLAP ? st * 64 + q * FE_CH : st * 128 + q * FE_CH;
          tmem_ld16(tmem + lane_off + acc * FE_N + col, v);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < FE_CH; ++c) stage_f[(st * FE_CH + c) * FE_ROWS + r] = __uint_as_float(v[c]);
        }
        if (q == NBLK - 1) {
          // the accumulator is free for the item two ahead
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars.acc_empty[acc]);
        }
        named_bar(1, FE_NEPI);
        if (OVERLAP) {
          // entries of the tile x 16 channels; window rows: C^b j*m .. j*m+m-1,
          // C^a j*m+m .. j*m+2m-1 (the first entry of the sequence has no C^b)
          const int i0 = t * sh.per_tile;
          for (int o = e; o < sh.per_tile * FE_CH; o += FE_NEPI) {
            const int j = o / FE_CH, c = o - j * FE_CH;
            const int i = i0 + j;
            if (i >= sh.n_c) continue;
            const int gc = hc * 64 + q * FE_CH + c;
            float mx = -INFINITY, sum = 0.f, accv = 0.f;
            for (int s2 = (i == 0 ? m : 0); s2 < 2 * m; ++s2) {
              const bool prev = s2 < m;
              const int rr = j * m + s2;
              const float z = stage_f[((prev ? 3 : 2) * FE_CH + c) * FE_ROWS + rr];
              const float cv = stage_f[((prev ? 1 : 0) * FE_CH + c) * FE_ROWS + rr];
              const float a = (z + bf16_to_f(pos_bias[(size_t)s2 * kD + gc])) * kLog2e;
              if (a > mx) {
                const float f = exp2f(mx - a);
                sum = sum * f + 1.f;
                accv = accv * f + cv;
                mx = a;
              } else {
                const float p = exp2f(a - mx);
                sum += p;
                accv = fmaf(p, cv, accv);
              }
            }
            out[((size_t)b * sh.n_c + i) * kD + gc] = __bfloat16_as_ushort(__float2bfloat16_rn(accv / sum));
          }
        } else {
          // one entry (the tile's 128 rows) x 16 channels: 8 threads per channel,
          // 16 rows each, merged with shuffles
          const int c = e >> 3, part = e & 7;
          const int gc = q * FE_CH + c;
          float mx = -INFINITY, sum = 0.f, accv = 0.f;
          for (int rr = part * 16; rr < part * 16 + 16; ++rr) {
            const float z = stage_f[(1 * FE_CH + c) * FE_ROWS + rr];
            const float cv = stage_f[(0 * FE_CH + c) * FE_ROWS + rr];
            const float a = (z + bf16_to_f(pos_bias[(size_t)rr * kD + gc])) * kLog2e;
            if (a > mx) {
              const float f = exp2f(mx - a);
              sum = sum * f + 1.f;
              accv = accv * f + cv;
              mx = a;
            } else {
              const float p = exp2f(a - mx);
              sum += p;
              accv = fmaf(p, cv, accv);
            }
          }
#pragma unroll
          for (int o = 1; o < 8; o <<= 1) {
            const float omx = __shfl_xor_sync(0xffffffffu, mx, o);
            const float osum = __shfl_xor_sync(0xffffffffu, sum, o);
            const float oacc = __shfl_xor_sync(0xffffffffu, accv, o);
            const float M = fmaxf(mx, omx);
            const float f1 = exp2f(mx - M), f2 = exp2f(omx - M);
            sum = sum * f1 + osum * f2;
            accv = accv * f1 + oacc * f2;
            mx = M;
          }
          if (part == 0 && t < sh.n_c)
            out[((size_t)b * sh.n_c + t) * kD + gc] = __bfloat16_as_ushort(__float2bfloat16_rn(accv / sum));
        }
        named_bar(1, FE_NEPI);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

namespace {
constexpr size_t fe_smem_bytes() {
  return 1024 + (size_t)FE_STAGES * FE_STAGE_BYTES + (size_t)FE_STAGE_F * 4 + sizeof(FeSmall);
}
}  // namespace

cslc_status launch_front_end(const uint16_t* h, const uint16_t* W, const uint16_t* pos_bias, int B, int L,
                             int d_model, int m, int overlap, uint16_t* out, cudaStream_t stream) {
  static int configured_for = -1;
  static int n_sm = 148;
  int dev = 0;
  cudaGetDevice(&dev);
  const size_t smem = fe_smem_bytes();
  if (configured_for != dev) {
    cudaFuncSetAttribute(front_end_sm100_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(front_end_sm100_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    configured_for = dev;
  }
  FeShape sh;
  sh.B = B; sh.L = L; sh.d_model = d_model; sh.m = m; sh.n_c = L / m;
  sh.per_tile = overlap ? (FE_ROWS - m) / m : 1;
  sh.n_tiles = (sh.n_c + sh.per_tile - 1) / sh.per_tile;
  sh.n_items = B * sh.n_tiles * (overlap ? 2 : 1);
  if (sh.n_items == 0) return CSLC_OK;
  CUtensorMap tm_h, tm_w;
  if (!sm100::make_tmap_bf16_2d(&tm_h, h, (uint64_t)B * L, (uint64_t)d_model, (uint64_t)d_model * 2, FE_ROWS, FE_KB) ||
      !sm100::make_tmap_bf16_2d(&tm_w, W, (uint64_t)(overlap ? 4 : 2) * kD, (uint64_t)d_model, (uint64_t)d_model * 2,
                                64, FE_KB))
    return set_error(CSLC_ERR_CUDA, "compressor front end: tensor map encoding failed");
  const int grid = sh.n_items < n_sm ? sh.n_items : n_sm;
  if (overlap)
    front_end_sm100_kernel<true><<<grid, FE_THREADS, smem, stream>>>(sh, pos_bias, out, tm_h, tm_w);
  else
    front_end_sm100_kernel<false><<<grid, FE_THREADS, smem, stream>>>(sh, pos_bias, out, tm_h, tm_w);
  return check_launch("front_end_sm100_kernel");
}

int front_end_sm100_read_error() {
  int v = 0, zero = 0;
  cudaMemcpyFromSymbol(&v, g_front_end_err, sizeof(int));
  if (v) cudaMemcpyToSymbol(g_front_end_err, &zero, sizeof(int));
  return v;
}

CSLC_DEFINE_WAIT_LIMIT_SETTER(front_end_sm100_set_wait_limits)

}  // namespace cslc
