// Prefill attention over compressed entries, K = V = entry (one KV head
// shared by all query heads).
//   CSA ("读完这篇你就搞懂 DeepSeek v4 了", §三 注意力计算): each query token attends
//       to its top-k selected entries (gathered by index).
//   HCA (first page §1.2): dense causal attention over all visible entries.
//
// CTA = TOK query tokens x H heads; warp = 16 heads of one token. Entry tiles
// of 64 x 128 bf16 (16 KB) are copied to shared memory with cp.async (row
// gather through the index list for CSA, contiguous rows for HCA) in a
// two-stage ring; each warp computes S = Q K^T and O += P V on the tensor cores
// (mma.sync m16n8k16, fp32 accumulation) with an online softmax kept in
// registers (exp2 with the scale folded into the exponent). Output rows are
// normalised once at the end; lse is the natural-log sum of exp(scale*q.k).

#include "common.cuh"

namespace cslc {

constexpr int ATT_TILE = 64;                 // entries per tile
constexpr int ATT_ROW_BYTES = kD * 2;        // 256 B per entry row

template <bool SPARSE, int TOK>
__global__ void __launch_bounds__(256) attention_kernel(
    const uint16_t* __restrict__ q, const uint16_t* __restrict__ kv,
    const int32_t* __restrict__ idx, int L, int H, int Nc, int topk, int m, int q_pos0,
    float scale_log2, uint16_t* __restrict__ out, float* __restrict__ lse) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int HG = H >> 4;                         // 16-head groups per token
  const int nthreads = TOK * HG * 32;
  uint8_t* q_s = smem;                           // [TOK*H rows][256 B]
  uint8_t* kv_s = smem + TOK * H * ATT_ROW_BYTES;    // [2][64][256 B]
  int32_t* idx_s = reinterpret_cast<int32_t*>(kv_s + 2 * ATT_TILE * ATT_ROW_BYTES);   // [topk]

  const int b = blockIdx.y;
  const int t0 = SPARSE ? blockIdx.x * TOK : (gridDim.x - 1 - blockIdx.x) * TOK;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tq = lane & 3;
  const int tk = warp / HG, hg = warp - tk * HG;
  const int t = t0 + tk;
  const bool row_ok = t < L;

  // queries -> smem
  for (int x = tid; x < TOK * H * 16; x += nthreads) {
    const int chunk = x & 15, row = x >> 4;
    const int tt = t0 + row / H, h = row % H;
    const bool ok = tt < L;
    const uint16_t* src = q + (((size_t)b * L + (ok ? tt : 0)) * H + h) * kD + chunk * 8;
    cp_async16(smem_u32(q_s + swz(row, chunk, ATT_ROW_BYTES)), src, ok);
  }
  int n_ent;   // entries (CSA: index slots) to walk for the CTA
  int nv_row;  // HCA: visible entries of this warp's token
  if (SPARSE) {
    const int32_t* irow = idx + ((size_t)b * L + t0) * topk;
    for (int j = tid; j < topk; j += nthreads) idx_s[j] = t0 < L ? irow[j] : -1;
    n_ent = topk;
    nv_row = 0;
  } else {
    const int t_last = min(t0 + TOK, L) - 1;
    n_ent = n_visible((long long)q_pos0 + t_last, m, Nc);
    nv_row = row_ok ? n_visible((long long)q_pos0 + t, m, Nc) : 0;
  }
  cp_async_commit();
  __syncthreads();   // idx_s visible to the loader

  auto load_tile = [&](int tile, int stage) {
    const int e0 = tile * ATT_TILE;
    uint8_t* dst = kv_s + stage * ATT_TILE * ATT_ROW_BYTES;
    for (int x = tid; x < ATT_TILE * 16; x += nthreads) {
      const int chunk = x & 15, row = x >> 4;
      const int slot = e0 + row;
      int e;
      if (SPARSE) {
        e = slot < n_ent ? idx_s[slot] : -1;
        if (e >= Nc) e = -1;
      } else {
        e = slot < n_ent ? slot : -1;
      }
      const bool ok = e >= 0;
      const uint16_t* src = kv + ((size_t)b * Nc + (ok ? e : 0)) * kD + chunk * 8;
      cp_async16(smem_u32(dst + swz(row, chunk, ATT_ROW_BYTES)), src, ok);
    }
  };
  const int n_tiles = (n_ent + ATT_TILE - 1) / ATT_TILE;
  if (n_tiles > 0) load_tile(0, 0);
  cp_async_commit();

  cp_async_wait<1>();   // queries landed
  __syncthreads();
  uint32_t qf[8][4];
  {
    const int rbase = tk * H + hg * 16;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int row = rbase + (lane & 15);
      const int chunk = ks * 2 + (lane >> 4);
      ldsm_x4(smem_u32(q_s + swz(row, chunk, ATT_ROW_BYTES)), qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3]);
    }
  }

  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) o[i][j] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};

  for (int tile = 0; tile < n_tiles; ++tile) {
    const int stage = tile & 1;
    if (tile + 1 < n_tiles) load_tile(tile + 1, stage ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint8_t* kt = kv_s + stage * ATT_TILE * ATT_ROW_BYTES;
    const int e0 = tile * ATT_TILE;
    const bool warp_active = SPARSE ? row_ok : (e0 < nv_row);
    if (warp_active) {
      // S = Q K^T for 64 entries: 8 n-tiles of 8 entries
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
          ldsm_x4(smem_u32(kt + swz(row, chunk, ATT_ROW_BYTES)), b0, b1, b2, b3);
          mma_bf16_16816(s[2 * np], qf[ks], b0, b1);
          mma_bf16_16816(s[2 * np + 1], qf[ks], b2, b3);
        }
      }
      // mask + scale (log2 units)
      float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int slot = e0 + nt * 8 + 2 * tq + j;
          bool valid;
          if (SPARSE) {
            const int e = slot < n_ent ? idx_s[slot] : -1;
            valid = e >= 0 && e < Nc;
          } else {
            valid = slot < nv_row;
          }
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
        alpha[r] = mrow[r] == -INFINITY ? 0.f : exp2f(mrow[r] - mnew[r]);
        mrow[r] = mnew[r];
      }
      float psum[2] = {0.f, 0.f};
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int r = j >> 1;
          const float p = mnew[r] == -INFINITY ? 0.f : exp2f(s[nt][j] - mnew[r]);
          s[nt][j] = p;
          psum[r] += p;
        }
      }
      lrow[0] = lrow[0] * alpha[0] + psum[0];
      lrow[1] = lrow[1] * alpha[1] + psum[1];
#pragma unroll
      for (int dn = 0; dn < 16; ++dn) {
        o[dn][0] *= alpha[0];
        o[dn][1] *= alpha[0];
        o[dn][2] *= alpha[1];
        o[dn][3] *= alpha[1];
      }
      // O += P V: 4 k-steps of 16 entries, 16 n-tiles of 8 dims
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
          ldsm_x4_t(smem_u32(kt + swz(row, chunk, ATT_ROW_BYTES)), b0, b1, b2, b3);
          mma_bf16_16816(o[2 * dp], pa, b0, b1);
          mma_bf16_16816(o[2 * dp + 1], pa, b2, b3);
        }
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  if (!row_ok) return;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 1);
    lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 2);
  }
  const float inv0 = lrow[0] > 0.f ? 1.f / lrow[0] : 0.f;
  const float inv1 = lrow[1] > 0.f ? 1.f / lrow[1] : 0.f;
  const int h0 = hg * 16 + g, h1 = h0 + 8;
  uint16_t* o0 = out + (((size_t)b * L + t) * H + h0) * kD;
  uint16_t* o1 = out + (((size_t)b * L + t) * H + h1) * kD;
#pragma unroll
  for (int dn = 0; dn < 16; ++dn) {
    const int col = dn * 8 + 2 * tq;
    *reinterpret_cast<uint32_t*>(o0 + col) = pack_bf16x2(o[dn][0] * inv0, o[dn][1] * inv0);
    *reinterpret_cast<uint32_t*>(o1 + col) = pack_bf16x2(o[dn][2] * inv1, o[dn][3] * inv1);
  }
  if (lse != nullptr && tq == 0) {
    float* l = lse + ((size_t)b * L + t) * H;
    l[h0] = lrow[0] > 0.f ? (mrow[0] + log2f(lrow[0])) * kLn2 : -INFINITY;
    l[h1] = lrow[1] > 0.f ? (mrow[1] + log2f(lrow[1])) * kLn2 : -INFINITY;
  }
}

template <bool SPARSE, int TOK>
static size_t attn_smem(int H, int topk) {
  return (size_t)TOK * H * ATT_ROW_BYTES + 2 * ATT_TILE * ATT_ROW_BYTES + (SPARSE ? (size_t)topk * 4 : 0);
}

template <bool SPARSE, int TOK>
static void attn_configure() {
  static int configured_for = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_for != dev) {
    cudaFuncSetAttribute(attention_kernel<SPARSE, TOK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)attn_smem<SPARSE, TOK>(128, 2048));
    configured_for = dev;
  }
}

bool sparse_attn_sm100_supported(int H);
cslc_status launch_sparse_attn_sm100(const uint16_t*, const uint16_t*, const int32_t*, int, int, int, int, int,
                                     float, uint16_t*, float*, cudaStream_t);

cslc_status launch_sparse_attn(const uint16_t* q, const uint16_t* kv, const int32_t* idx, int B, int L,
                               int H, int Nc, int topk, float scale, uint16_t* out, float* lse,
                               cudaStream_t stream) {
  if (B == 0 || L == 0) return CSLC_OK;
  // tcgen05 kernel for up to 64 heads; more heads take the warp-level MMA kernel below
  if (sparse_attn_sm100_supported(H))
    return launch_sparse_attn_sm100(q, kv, idx, B, L, H, Nc, topk, scale, out, lse, stream);
  attn_configure<true, 1>();
  dim3 grid(L, B);
  attention_kernel<true, 1><<<grid, (H / 16) * 32, attn_smem<true, 1>(H, topk), stream>>>(
      q, kv, idx, L, H, Nc, topk, 1, 0, scale * kLog2e, out, lse);
  return check_launch("attention_kernel<sparse>");
}

bool dense_attn_sm100_supported(int H);
cslc_status launch_dense_attn_sm100(const uint16_t*, const uint16_t*, int, int, int, int, int, int, float,
                                    uint16_t*, float*, cudaStream_t);

cslc_status launch_dense_attn(const uint16_t* q, const uint16_t* kv, int B, int L, int H, int Nc,
                              int m, int q_pos0, float scale, uint16_t* out, float* lse,
                              cudaStream_t stream) {
  if (B == 0 || L == 0) return CSLC_OK;
  // tcgen05 kernel when 128 rows hold whole tokens (H divides 128); other head counts below
  if (dense_attn_sm100_supported(H))
    return launch_dense_attn_sm100(q, kv, B, L, H, Nc, m, q_pos0, scale, out, lse, stream);
  if (H <= 64) {
    attn_configure<false, 2>();
    // 2 tokens per CTA when H <= 64 (<= 8 warps)
    dim3 grid((L + 1) / 2, B);
    attention_kernel<false, 2><<<grid, 2 * (H / 16) * 32, attn_smem<false, 2>(H, 0), stream>>>(
        q, kv, nullptr, L, H, Nc, 0, m, q_pos0, scale * kLog2e, out, lse);
  } else {
    attn_configure<false, 1>();
    dim3 grid(L, B);
    attention_kernel<false, 1><<<grid, (H / 16) * 32, attn_smem<false, 1>(H, 0), stream>>>(
        q, kv, nullptr, L, H, Nc, 0, m, q_pos0, scale * kLog2e, out, lse);
  }
  return check_launch("attention_kernel<dense>");
}

}  // namespace cslc
