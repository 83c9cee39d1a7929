// Lightning-indexer scores for prefill ("读完这篇你就搞懂 DeepSeek v4 了", §三 闪电索引:
// every query token is scored against every compressed entry, per-head scores
// are weighted and summed, then the top-k are kept; the same mechanism as the
// V3.2 DSA indexer):
//   S[t, i] = sum_h w[t, h] * max(0, q_I[t, h, :] . k_I[i, :])
//
// CTA = 64 query rows (4 warps x 16 rows) x up to 1024 entries, all H_I heads. The CTA's
// queries (64 rows x H_I heads x 64 dims, bf16) stay in shared memory; key
// tiles of 64 entries x 64 dims stream through a two-stage cp.async ring. Per
// key tile each warp keeps the tile's B fragments in registers and runs, for
// every head, a 16x64x64 tensor-core product whose ReLU-weighted result is
// accumulated in fp32 registers, so the ReLU is applied per head before the
// head sum as the formula requires. Only tiles that hold a visible entry for
// some row of the CTA are computed.

#include "common.cuh"

namespace cslc {

constexpr int IDX_ROWS = 64;     // query rows per CTA
constexpr int IDX_TILE = 64;     // entries per key tile
constexpr int IDX_THREADS = 128;
constexpr int IDX_SPLIT_TILES = 16;   // key tiles (1024 entries) per CTA

// Score stores: fp32, or bf16 (round to nearest even) for the half-size score path.
__device__ __forceinline__ void put1(float* p, float v) { *p = v; }
__device__ __forceinline__ void put1(uint16_t* p, float v) { *p = __bfloat16_as_ushort(__float2bfloat16_rn(v)); }
__device__ __forceinline__ void put2(float* p, float a, float b) { *reinterpret_cast<float2*>(p) = make_float2(a, b); }
__device__ __forceinline__ void put2(uint16_t* p, float a, float b) {
  *reinterpret_cast<uint32_t*>(p) = pack_bf16x2(a, b);
}

template <typename OutT>
__global__ void __launch_bounds__(IDX_THREADS, 2) indexer_scores_kernel(
    const uint16_t* __restrict__ q_idx, const uint16_t* __restrict__ w,
    const uint16_t* __restrict__ k_idx, int L, int Nc, int HI, int m, int q_pos0,
    int row_begin, int row_end, OutT* __restrict__ scores, int rows_in_buf) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* q_s = smem;                                        // [HI][64 rows][128 B]
  uint8_t* k_s = smem + HI * IDX_ROWS * 128;                  // [2][64 entries][128 B]
  float* w_s = reinterpret_cast<float*>(k_s + 2 * IDX_TILE * 128);   // [64 rows][HI]

  const int b = blockIdx.y;
  // blockIdx.x enumerates (entry split, row block); row blocks run heavy (late) rows first
  const int n_rb = (row_end - row_begin + IDX_ROWS - 1) / IDX_ROWS;
  const int rblk = n_rb - 1 - (int)(blockIdx.x % n_rb);
  const int split = (int)(blockIdx.x / n_rb);
  const int r0 = row_begin + rblk * IDX_ROWS;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tq = lane & 3;

  const int last_row = min(r0 + IDX_ROWS, row_end) - 1;
  const int nv_max = n_visible((long long)q_pos0 + last_row, m, Nc);
  const int tile_lo = split * IDX_SPLIT_TILES;
  const int tile_hi = min((nv_max + IDX_TILE - 1) / IDX_TILE, tile_lo + IDX_SPLIT_TILES);
  if (tile_lo >= tile_hi) return;   // uniform: this split holds no visible entry of the block
  const int n_tiles = tile_hi - tile_lo;

  // queries -> smem (16-byte chunks, swizzled per 128-byte row)
  for (int x = tid; x < HI * IDX_ROWS * 8; x += IDX_THREADS) {
    const int chunk = x & 7, row = (x >> 3) % IDX_ROWS, h = (x >> 3) / IDX_ROWS;
    const int r = r0 + row;
    const bool ok = r < row_end;
    const uint16_t* src = q_idx + (((size_t)b * L + (ok ? r : 0)) * HI + h) * kDI + chunk * 8;
    cp_async16(smem_u32(q_s + h * IDX_ROWS * 128 + swz(row, chunk, 128)), src, ok);
  }
  for (int x = tid; x < IDX_ROWS * HI; x += IDX_THREADS) {
    const int row = x / HI, h = x - row * HI;
    const int r = r0 + row;
    w_s[x] = r < row_end ? bf16_to_f(w[((size_t)b * L + r) * HI + h]) : 0.f;
  }
  auto load_tile = [&](int tile, int stage) {
    const int e0 = (tile_lo + tile) * IDX_TILE;
    for (int x = tid; x < IDX_TILE * 8; x += IDX_THREADS) {
      const int chunk = x & 7, row = x >> 3;
      const int e = e0 + row;
      const bool ok = e < Nc;
      const uint16_t* src = k_idx + ((size_t)b * Nc + (ok ? e : 0)) * kDI + chunk * 8;
      cp_async16(smem_u32(k_s + stage * IDX_TILE * 128 + swz(row, chunk, 128)), src, ok);
    }
  };
  if (n_tiles > 0) load_tile(0, 0);
  cp_async_commit();

  // rows of this thread: warp*16 + g and warp*16 + g + 8
  const int ra = r0 + warp * 16 + g, rb = ra + 8;
  const int nva = ra < row_end ? n_visible((long long)q_pos0 + ra, m, Nc) : 0;
  const int nvb = rb < row_end ? n_visible((long long)q_pos0 + rb, m, Nc) : 0;
  const int warp_nv = max(nva, nvb);
  // the warp's largest visible count (rows grow with the lane index)
  const int warp_nv_max = __reduce_max_sync(0xffffffffu, warp_nv);

  for (int tile = 0; tile < n_tiles; ++tile) {
    const int stage = tile & 1;
    if (tile + 1 < n_tiles) load_tile(tile + 1, stage ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();

    const int e0 = (tile_lo + tile) * IDX_TILE;
    if (e0 < warp_nv_max) {
      // B fragments of the key tile: b[nt][ks][2] for 8 n-tiles of 8 entries and 4 k-steps
      uint32_t bf[8][4][2];
      const uint8_t* kt = k_s + stage * IDX_TILE * 128;
#pragma unroll
      for (int np = 0; np < 4; ++np) {
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const int row = np * 16 + (lane & 7) + ((lane >> 4) << 3);
          const int chunk = ks * 2 + ((lane >> 3) & 1);
          ldsm_x4(smem_u32(kt + swz(row, chunk, 128)), bf[2 * np][ks][0], bf[2 * np][ks][1],
                  bf[2 * np + 1][ks][0], bf[2 * np + 1][ks][1]);
        }
      }
      float acc[8][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[nt][j] = 0.f;

      for (int h = 0; h < HI; ++h) {
        uint32_t af[4][4];
        const uint8_t* qh = q_s + h * IDX_ROWS * 128;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const int row = warp * 16 + (lane & 15);
          const int chunk = ks * 2 + (lane >> 4);
          ldsm_x4(smem_u32(qh + swz(row, chunk, 128)), af[ks][0], af[ks][1], af[ks][2], af[ks][3]);
        }
        const float wa = w_s[(warp * 16 + g) * HI + h];
        const float wb = w_s[(warp * 16 + g + 8) * HI + h];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) mma_bf16_16816(d, af[ks], bf[nt][ks][0], bf[nt][ks][1]);
          acc[nt][0] = fmaf(wa, fmaxf(d[0], 0.f), acc[nt][0]);
          acc[nt][1] = fmaf(wa, fmaxf(d[1], 0.f), acc[nt][1]);
          acc[nt][2] = fmaf(wb, fmaxf(d[2], 0.f), acc[nt][2]);
          acc[nt][3] = fmaf(wb, fmaxf(d[3], 0.f), acc[nt][3]);
        }
      }
      // store: entries past n_vis inside this tile get -inf; never past Nc. Pairs
      // go out as one 8-byte store only when every row starts 8-byte aligned.
      const bool pair_ok = (Nc & 1) == 0;
      OutT* sa = scores + ((size_t)b * rows_in_buf + (ra - row_begin)) * (size_t)Nc;
      OutT* sb = scores + ((size_t)b * rows_in_buf + (rb - row_begin)) * (size_t)Nc;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const int col = e0 + nt * 8 + 2 * tq;
        if (ra < row_end && e0 < nva) {
          if (pair_ok && col + 1 < Nc) {
            put2(sa + col, col < nva ? acc[nt][0] : -INFINITY, col + 1 < nva ? acc[nt][1] : -INFINITY);
          } else {
            if (col < Nc) put1(sa + col, col < nva ? acc[nt][0] : -INFINITY);
            if (col + 1 < Nc) put1(sa + col + 1, col + 1 < nva ? acc[nt][1] : -INFINITY);
          }
        }
        if (rb < row_end && e0 < nvb) {
          if (pair_ok && col + 1 < Nc) {
            put2(sb + col, col < nvb ? acc[nt][2] : -INFINITY, col + 1 < nvb ? acc[nt][3] : -INFINITY);
          } else {
            if (col < Nc) put1(sb + col, col < nvb ? acc[nt][2] : -INFINITY);
            if (col + 1 < Nc) put1(sb + col + 1, col + 1 < nvb ? acc[nt][3] : -INFINITY);
          }
        }
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();
}

size_t indexer_smem_bytes(int HI) {
  return (size_t)HI * IDX_ROWS * 128 + 2 * IDX_TILE * 128 + (size_t)IDX_ROWS * HI * 4;
}

bool indexer_sm100_supported(int HI);
cslc_status launch_indexer_sm100(const uint16_t* q_idx, const uint16_t* w, const uint16_t* k_idx, int B,
                                 int L, int Nc, int HI, int m, int q_pos0, int row_begin, int row_end,
                                 void* scores, bool bf16_out, int rows_in_buf, cudaStream_t stream);

cslc_status launch_indexer_sm100_fp8(const uint8_t* q8, const float* q_scale, const uint16_t* w, const uint8_t* k8,
                                     const float* k_scale, int B, int L, int Nc, int HI, int m, int q_pos0,
                                     int row_begin, int row_end, float* scores, int rows_in_buf, cudaStream_t stream);

// FP8 operands on the CUDA cores, for inputs smaller than one tensor-core
// tile (fewer than 256 (token, head) rows or 128 entries): one thread per
// (row, entry), the code products summed in fp32 and the scales applied as
// the tensor-core kernel applies them.
__global__ void __launch_bounds__(256) indexer_fp8_small_kernel(
    const uint8_t* __restrict__ q8, const float* __restrict__ q_scale, const uint16_t* __restrict__ w,
    const uint8_t* __restrict__ k8, const float* __restrict__ k_scale, int B, int L, int Nc, int HI, int m,
    int q_pos0, int row_begin, int row_end, float* __restrict__ scores, int rows_in_buf) {
  const int R = row_end - row_begin;
  const long long id = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= (long long)B * R * Nc) return;
  const int i = (int)(id % Nc);
  const long long br = id / Nc;
  const int r = (int)(br % R), b = (int)(br / R);
  const int t = row_begin + r;
  if (i >= n_visible((long long)q_pos0 + t, m, Nc)) return;
  const uint16_t* kr = reinterpret_cast<const uint16_t*>(k8 + ((size_t)b * Nc + i) * 64);
  float acc = 0.f;
  for (int h = 0; h < HI; ++h) {
    const size_t p = ((size_t)b * L + t) * HI + h;
    const uint16_t* qr = reinterpret_cast<const uint16_t*>(q8 + p * 64);
    float dot = 0.f;
    for (int d = 0; d < 32; ++d) {
      const __half2_raw qh = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)qr[d], __NV_E4M3);
      const __half2_raw kh = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)kr[d], __NV_E4M3);
      const float2 qf = __half22float2(*reinterpret_cast<const __half2*>(&qh));
      const float2 kf = __half22float2(*reinterpret_cast<const __half2*>(&kh));
      dot = fmaf(qf.x, kf.x, dot);
      dot = fmaf(qf.y, kf.y, dot);
    }
    acc = fmaf(bf16_to_f(w[p]) * q_scale[p], fmaxf(dot, 0.f), acc);
  }
  scores[((size_t)b * rows_in_buf + r) * Nc + i] = k_scale[(size_t)b * Nc + i] * acc;
}

cslc_status launch_indexer_scores_fp8(const uint8_t* q8, const float* q_scale, const uint16_t* w, const uint8_t* k8,
                                      const float* k_scale, int B, int L, int Nc, int HI, int m, int q_pos0,
                                      int row_begin, int row_end, float* scores, int rows_in_buf,
                                      cudaStream_t stream) {
  if (row_end <= row_begin || B == 0 || Nc == 0) return CSLC_OK;
  if ((long long)B * L * HI >= 256 && (long long)B * Nc >= 128)
    return launch_indexer_sm100_fp8(q8, q_scale, w, k8, k_scale, B, L, Nc, HI, m, q_pos0, row_begin, row_end, scores,
                                    rows_in_buf, stream);
  const long long n = (long long)B * (row_end - row_begin) * Nc;
  indexer_fp8_small_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(
      q8, q_scale, w, k8, k_scale, B, L, Nc, HI, m, q_pos0, row_begin, row_end, scores, rows_in_buf);
  return check_launch("indexer_fp8_small_kernel");
}

// scores: fp32 [rows][Nc], or bf16 when bf16_out
cslc_status launch_indexer_scores(const uint16_t* q_idx, const uint16_t* w, const uint16_t* k_idx,
                                  int B, int L, int Nc, int HI, int m, int q_pos0, int row_begin,
                                  int row_end, void* scores, bool bf16_out, int rows_in_buf, cudaStream_t stream) {
  if (row_end <= row_begin || B == 0) return CSLC_OK;
  // tensor-core path when whole TMA boxes fit the operands (256 query pairs,
  // 128 entries); the mma.sync kernel below takes the rest
  if (indexer_sm100_supported(HI) && (long long)B * L * HI >= 256 && (long long)B * Nc >= 128)
    return launch_indexer_sm100(q_idx, w, k_idx, B, L, Nc, HI, m, q_pos0, row_begin, row_end, scores, bf16_out,
                                rows_in_buf, stream);
  const size_t smem = indexer_smem_bytes(HI);
  static int configured_for = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_for != dev) {
    cudaFuncSetAttribute(indexer_scores_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)indexer_smem_bytes(16));
    cudaFuncSetAttribute(indexer_scores_kernel<uint16_t>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)indexer_smem_bytes(16));
    configured_for = dev;
  }
  const int n_rb = (row_end - row_begin + IDX_ROWS - 1) / IDX_ROWS;
  const int nv_max = n_visible((long long)q_pos0 + row_end - 1, m, Nc);
  const int n_split = ((nv_max + IDX_TILE - 1) / IDX_TILE + IDX_SPLIT_TILES - 1) / IDX_SPLIT_TILES;
  if (n_split == 0) return CSLC_OK;
  dim3 grid(n_rb * n_split, B);
  if (bf16_out)
    indexer_scores_kernel<uint16_t><<<grid, IDX_THREADS, smem, stream>>>(
        q_idx, w, k_idx, L, Nc, HI, m, q_pos0, row_begin, row_end, static_cast<uint16_t*>(scores), rows_in_buf);
  else
    indexer_scores_kernel<float><<<grid, IDX_THREADS, smem, stream>>>(
        q_idx, w, k_idx, L, Nc, HI, m, q_pos0, row_begin, row_end, static_cast<float*>(scores), rows_in_buf);
  return check_launch("indexer_scores_kernel");
}

}  // namespace cslc
