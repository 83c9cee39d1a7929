// HCA dense causal attention on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// First page §1.2 (HCA): every m' = 128 tokens become one entry and attention
// over the short compressed sequence is dense; query t sees the entries whose
// window has ended, n_vis(t) = min(Nc, floor((t+1)/m')). K = V = the entry.
//
// Rows of the MMA are (token, head) pairs: a Q tile is 128 consecutive rows of
// q viewed as [B*L tokens][H heads][128] (128/H tokens), loaded with one 3-D TMA per 64-dim
// half. KV tiles are 128 consecutive entries (2-D TMA); the same shared tile is
// K (K-major) for S = Q K^T and V (MN-major) for O += P V.
//
// CTA roles (persistent, one CTA per SM, Q tiles in decreasing-work order):
//   warps 0-3  softmax + epilogue, thread = row = TMEM lane. The row's
//              reference m is the exact maximum of its first visible tile and
//              then stays put: a later tile is redone against its exact
//              maximum (O in TMEM and the row sum rescaled) only when its
//              probabilities sum above 2^64, so the steady state needs no
//              per-tile maximum (fp32 sums and bf16 P keep their relative
//              precision at any magnitude). P goes to 128-byte-swizzled
//              shared memory (double buffered). At the end O / l is stored.
//   warp 4     producer: Q tile and KV tiles (TMA, STAGES-deep ring).
//   warp 5     TMEM allocation and the single MMA-issuing thread.
// TMEM: S double buffer (2 x 128 columns) + O (128 columns).
// All waits are time-bounded (abort + device error word, as elsewhere).

#include "sm100.cuh"

namespace cslc {

using namespace sm100;

__device__ int g_dense_attn_err = 0;

namespace {

constexpr int DA_THREADS = 192;
constexpr int DA_PROD_WARP = 4;
constexpr int DA_MMA_WARP = 5;
constexpr int DA_ROWS = 128;
constexpr int DA_TILE = 128;                  // entries per KV tile
constexpr int DA_STAGES = 3;
constexpr int DA_TILE_BYTES = DA_TILE * 256;  // 32 KB (also the Q tile and a P tile)
constexpr float DA_SUM_MAX = 1.8446744e19f;   // 2^64: a tile whose probabilities sum above this is redone

enum { ERR_Q_EMPTY = 1, ERR_KV_EMPTY, ERR_Q_FULL, ERR_O_FREE, ERR_KV_FULL, ERR_P_FULL, ERR_S_FULL, ERR_PV_DONE,
       ERR_O_FULL, ERR_FINAL };

struct __align__(8) DaBars {
  uint64_t q_full, q_empty;
  uint64_t kv_full[DA_STAGES], kv_empty[DA_STAGES];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t pv_done;
  uint64_t o_full, o_free;
  uint64_t final_bar;
};

struct DaSmall {
  DaBars bars;
  uint32_t tmem_base;
  int abort_flag;
};

}  // namespace

__global__ void __launch_bounds__(DA_THREADS, 1) dense_attn_sm100_kernel(
    int B, int L, int H, int Nc, int m, int q_pos0, float scale_log2, uint16_t* __restrict__ out,
    float* __restrict__ lse, int h_stride, int h_off, const __grid_constant__ CUtensorMap tm_q,
    const __grid_constant__ CUtensorMap tm_kv) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_s = smem;                                   // [2 kb][128][128 B]
  uint8_t* kv_s = q_s + DA_TILE_BYTES;                   // [STAGES][2 kb][128][128 B]
  uint8_t* p_s = kv_s + DA_STAGES * DA_TILE_BYTES;       // [2][2 kb][128][128 B]
  DaSmall* sm = reinterpret_cast<DaSmall*>(p_s + 2 * DA_TILE_BYTES);
  DaBars& bars = sm->bars;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  const int tpt = DA_ROWS / H;                           // tokens per Q tile
  const int qt_per_b = (L + tpt - 1) / tpt;
  const long long n_qt = (long long)B * qt_per_b;

  if (tid == 0) {
    mbar_init(&bars.q_full, 1); mbar_init(&bars.q_empty, 1);
    for (int s = 0; s < DA_STAGES; ++s) { mbar_init(&bars.kv_full[s], 1); mbar_init(&bars.kv_empty[s], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&bars.s_full[i], 1); mbar_init(&bars.p_full[i], 4); }
    mbar_init(&bars.pv_done, 1);
    mbar_init(&bars.o_full, 1); mbar_init(&bars.o_free, 4);
    mbar_init(&bars.final_bar, 1);
    sm->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == DA_MMA_WARP) tmem_alloc(&sm->tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;
  volatile int* abortp = &sm->abort_flag;
  int* errp = &g_dense_attn_err;

  // tile k of this CTA -> (batch, first token, number of KV tiles); heavy tiles first
  auto tile_of = [&](long long g, int& b, int& t0, int& nkv) {
    b = (int)(g / qt_per_b);
    const int qt = qt_per_b - 1 - (int)(g - (long long)b * qt_per_b);
    t0 = qt * tpt;
    const int t_last = min(t0 + tpt, L) - 1;
    nkv = (n_visible((long long)q_pos0 + t_last, m, Nc) + DA_TILE - 1) / DA_TILE;
  };

  if (warp == DA_PROD_WARP) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_map(&tm_q);
      tma_prefetch_map(&tm_kv);
      int kv_it = 0;
      long long tk = 0, q_last = -1;   // last tile whose Q load was issued
      bool ok = true;
      for (long long g = blockIdx.x; g < n_qt && ok; g += gridDim.x, ++tk) {
        int b, t0, nkv;
        tile_of(g, b, t0, nkv);
        if (tk >= 1 && !mbar_wait(&bars.q_empty, (uint32_t)((tk - 1) & 1), abortp, errp, ERR_Q_EMPTY)) break;
        q_last = tk;
        mbar_arrive_expect_tx(&bars.q_full, DA_TILE_BYTES);
        // heads h_off .. h_off+H-1 of tokens t0 .. t0+128/H-1 (rows token-major)
        const int tok0 = (int)((long long)b * L + t0);
        tma_load_3d(q_s, &tm_q, 0, h_off, tok0, &bars.q_full);
        tma_load_3d(q_s + DA_TILE * 128, &tm_q, 64, h_off, tok0, &bars.q_full);
        for (int j = 0; j < nkv; ++j) {
          const int stage = kv_it % DA_STAGES;
          if (kv_it >= DA_STAGES &&
              !mbar_wait(&bars.kv_empty[stage], (uint32_t)((kv_it / DA_STAGES - 1) & 1), abortp, errp, ERR_KV_EMPTY)) {
            ok = false;
            break;
          }
          uint8_t* dst = kv_s + stage * DA_TILE_BYTES;
          mbar_arrive_expect_tx(&bars.kv_full[stage], DA_TILE_BYTES);
          const int krow = b * Nc + j * DA_TILE;
          tma_load_2d(dst, &tm_kv, 0, krow, &bars.kv_full[stage]);
          tma_load_2d(dst + DA_TILE * 128, &tm_kv, 64, krow, &bars.kv_full[stage]);
          ++kv_it;
        }
      }
      // loads in flight after an abort land before the CTA leaves (the last
      // load into each barrier is its latest phase)
      if (q_last >= 0) mbar_wait_done(&bars.q_full, (uint32_t)(q_last & 1), errp, ERR_Q_FULL);
      for (int d = 1; d <= DA_STAGES && kv_it - d >= 0; ++d) {
        const int k2 = kv_it - d;
        mbar_wait_done(&bars.kv_full[k2 % DA_STAGES], (uint32_t)((k2 / DA_STAGES) & 1), errp, ERR_KV_FULL);
      }
    }
    __syncwarp();
  } else if (warp == DA_MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID_S = idesc_bf16(128, 128, false, false);
      constexpr uint32_t ID_O = idesc_bf16(128, 128, false, true);
      int kv_it = 0, s_it = 0, p_it = 0;
      long long tk = 0;
      bool ok = true;
      const uint32_t q0 = smem_u32(q_s);
      auto issue_pv = [&](int stage, bool first) -> bool {
        const int pb = p_it & 1;
        if (!mbar_wait(&bars.p_full[pb], (uint32_t)((p_it >> 1) & 1), abortp, errp, ERR_P_FULL)) return false;
        tc_fence_after();
        const uint32_t p0 = smem_u32(p_s + pb * DA_TILE_BYTES), v0 = smem_u32(kv_s + stage * DA_TILE_BYTES);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t ad = smem_desc_sw128(p0 + (k >> 2) * (DA_ROWS * 128) + (k & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(v0 + k * 2048, DA_TILE * 128, 1024);
          mma_bf16(tmem + 256, ad, bd, ID_O, (!first || k > 0) ? 1u : 0u);
        }
        mma_commit(&bars.kv_empty[stage]);
        mma_commit(&bars.pv_done);
        ++p_it;
        return true;
      };
      for (long long g = blockIdx.x; g < n_qt && ok; g += gridDim.x, ++tk) {
        int b, t0, nkv;
        tile_of(g, b, t0, nkv);
        if (!mbar_wait(&bars.q_full, (uint32_t)(tk & 1), abortp, errp, ERR_Q_FULL)) break;
        if (tk >= 1 && !mbar_wait(&bars.o_free, (uint32_t)((tk - 1) & 1), abortp, errp, ERR_O_FREE)) break;
        int stage_prev = 0;
        for (int j = 0; j < nkv; ++j) {
          const int stage = kv_it % DA_STAGES, sb = s_it & 1;
          if (!mbar_wait(&bars.kv_full[stage], (uint32_t)((kv_it / DA_STAGES) & 1), abortp, errp, ERR_KV_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t k0 = smem_u32(kv_s + stage * DA_TILE_BYTES);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint64_t ad = smem_desc_sw128(q0 + (k >> 2) * (DA_ROWS * 128) + (k & 3) * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(k0 + (k >> 2) * (DA_TILE * 128) + (k & 3) * 32, 16, 1024);
            mma_bf16(tmem + sb * 128, ad, bd, ID_S, k > 0 ? 1u : 0u);
          }
          mma_commit(&bars.s_full[sb]);
          ++s_it;
          if (j > 0 && !issue_pv(stage_prev, j == 1)) { ok = false; break; }
          stage_prev = stage;
          ++kv_it;
        }
        if (!ok) break;
        mma_commit(&bars.q_empty);     // every S of this tile has read Q
        if (nkv > 0 && !issue_pv(stage_prev, nkv == 1)) break;
        mma_commit(&bars.o_full);
      }
      mma_commit(&bars.final_bar);
      mbar_wait_done(&bars.final_bar, 0, errp, ERR_FINAL);   // also after an abort: the products finish on their own
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------ softmax + epilogue
    const int row = tid;                                   // 0..127 = TMEM lane
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    int s_it = 0, p_it = 0;
    long long tk = 0;
    bool ok = true;
    for (long long g = blockIdx.x; g < n_qt && ok; g += gridDim.x, ++tk) {
      int b, t0, nkv;
      tile_of(g, b, t0, nkv);
      const int tok = t0 + row / H;
      const bool row_ok = tok < L;
      const int nv = row_ok ? n_visible((long long)q_pos0 + tok, m, Nc) : 0;
      float mrow = -INFINITY, lrow = 0.f;
      for (int j = 0; j < nkv; ++j) {
        const int sb = s_it & 1, pb = p_it & 1;
        // each warp waits for S on its own; a failed wait is acted on at the
        // tile's single vote below (reading TMEM is harmless meanwhile)
        bool w = true;
        if (lane == 0) w = mbar_wait(&bars.s_full[sb], (uint32_t)((s_it >> 1) & 1), abortp, errp, ERR_S_FULL);
        w = __shfl_sync(0xffffffffu, (int)w, 0) != 0;
        tc_fence_after();
        // the tile's 128 scores of this row: all four TMEM loads before one wait
        uint32_t sr[DA_TILE / 32][32];
#pragma unroll
        for (int c0 = 0; c0 < DA_TILE / 32; ++c0) tmem_ld32(tmem + lane_off + sb * 128 + c0 * 32, sr[c0]);
        tmem_wait_ld();
        float s[DA_TILE];
#pragma unroll
        for (int c = 0; c < DA_TILE; ++c) s[c] = __uint_as_float(sr[c >> 5][c & 31]);
        const int lim = nv - j * DA_TILE;                   // entries of this tile the row sees
        if (lim < DA_TILE) {
#pragma unroll
          for (int c = 0; c < DA_TILE; ++c) s[c] = c < lim ? s[c] : -INFINITY;
        }
        // exact row maximum (scaled, log2 units); 8 independent chains
        auto row_max = [&]() -> float {
          float mx8[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) mx8[q] = s[q];
#pragma unroll
          for (int c = 8; c < DA_TILE; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], s[c]);
          return fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                       fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) * scale_log2;
        };
        // the row's first visible tile sets the reference (nothing to rescale yet)
        if (mrow == -INFINITY) mrow = row_max();
        // P = 2^(c*s - m): bf16, row-major (K-major A operand) in two 64-entry halves
        uint8_t* prow = p_s + pb * DA_TILE_BYTES;
        auto write_p = [&](float mneg) -> float {
          float ps8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};   // 8 independent partial sums
#pragma unroll
          for (int c8 = 0; c8 < 16; ++c8) {
            uint32_t pk[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float a = ex2_approx(fmaf(s[8 * c8 + 2 * k], scale_log2, mneg));
              const float bq = ex2_approx(fmaf(s[8 * c8 + 2 * k + 1], scale_log2, mneg));
              ps8[2 * k] += a;
              ps8[2 * k + 1] += bq;
              pk[k] = pack_bf16x2(a, bq);
            }
            *reinterpret_cast<uint4*>(prow + (c8 >> 3) * (DA_ROWS * 128) + sw128(row, c8 & 7)) =
                make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
          return ((ps8[0] + ps8[1]) + (ps8[2] + ps8[3])) + ((ps8[4] + ps8[5]) + (ps8[6] + ps8[7]));
        };
        float tsum = write_p(mrow == -INFINITY ? 0.f : -mrow);
        // a stale reference: redo the tile against its exact maximum and rescale
        // O (after the previous PV) and l
        const bool over = !(tsum <= DA_SUM_MAX);
        if (__any_sync(0xffffffffu, over)) {
          float alpha = 1.f;
          if (over) {
            const float mx = row_max();
            alpha = ex2_approx(mrow - mx);
            mrow = mx;
            lrow *= alpha;
            tsum = write_p(-mrow);
          }
          if (j > 0 && w) {
            if (lane == 0) w = mbar_wait(&bars.pv_done, (uint32_t)((p_it - 1) & 1), abortp, errp, ERR_PV_DONE);
            w = __shfl_sync(0xffffffffu, (int)w, 0) != 0;
            if (w) {
              tc_fence_after();
#pragma unroll
              for (int c0 = 0; c0 < 128; c0 += 32) {
                uint32_t r[32];
                tmem_ld32(tmem + lane_off + 256 + c0, r);
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * alpha);
                tmem_st32(tmem + lane_off + 256 + c0, r);
              }
              tmem_wait_st();
            }
          }
        }
        ok = !named_bar_or(1, 128, !w || *abortp != 0);
        if (!ok) break;
        lrow += tsum;
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.p_full[pb]);
        ++s_it;
        ++p_it;
      }
      if (!ok) break;
      // ---- epilogue
      {
        bool w = true;
        if (tid == 0) w = mbar_wait(&bars.o_full, (uint32_t)(tk & 1), abortp, errp, ERR_O_FULL);
        ok = !named_bar_or(1, 128, !w);
      }
      if (!ok) break;
      tc_fence_after();
      const float inv = lrow > 0.f ? 1.f / lrow : 0.f;
      const long long orow = ((long long)b * L + t0 + row / H) * h_stride + h_off + row % H;
#pragma unroll
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t r[32];
        if (nkv > 0) {
          tmem_ld32(tmem + lane_off + 256 + c0, r);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) r[k] = 0u;
        }
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(out + orow * kD + c0);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            dst[k] = make_uint4(pack_bf16x2(__uint_as_float(r[8 * k]) * inv, __uint_as_float(r[8 * k + 1]) * inv),
                                pack_bf16x2(__uint_as_float(r[8 * k + 2]) * inv, __uint_as_float(r[8 * k + 3]) * inv),
                                pack_bf16x2(__uint_as_float(r[8 * k + 4]) * inv, __uint_as_float(r[8 * k + 5]) * inv),
                                pack_bf16x2(__uint_as_float(r[8 * k + 6]) * inv, __uint_as_float(r[8 * k + 7]) * inv));
        }
      }
      if (row_ok && lse != nullptr) lse[orow] = lrow > 0.f ? (mrow + log2f(lrow)) * kLn2 : -INFINITY;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.o_free);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == DA_MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Any multiple of 16 up to 128 heads: groups of 128, 64, 32 and 16 heads (a
// group's 128-row tiles hold whole tokens), one launch each on the group's
// heads of q / out / lse.
bool dense_attn_sm100_supported(int H) { return H >= 16 && H <= 128 && H % 16 == 0; }

cslc_status launch_dense_attn_sm100(const uint16_t* q, const uint16_t* kv, int B, int L, int H, int Nc, int m,
                                    int q_pos0, float scale, uint16_t* out, float* lse, cudaStream_t stream) {
  static int configured_for = -1;
  static int n_sm = 148;
  int dev = 0;
  cudaGetDevice(&dev);
  const size_t smem = 1024 + (size_t)(1 + DA_STAGES + 2) * DA_TILE_BYTES + sizeof(DaSmall);
  if (configured_for != dev) {
    cudaFuncSetAttribute(dense_attn_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    configured_for = dev;
  }
  const void* kv_base = Nc > 0 ? (const void*)kv : (const void*)q;
  CUtensorMap tm_kv;
  if (!sm100::make_tmap_bf16_2d(&tm_kv, kv_base, (uint64_t)B * (Nc > 0 ? Nc : 1), kD, kD * 2, DA_TILE, 64))
    return set_error(CSLC_ERR_CUDA, "hca_dense_attn: tensor map encoding failed");
  for (int h0 = 0; h0 < H;) {
    const int rem = H - h0;
    const int hg = rem >= 128 ? 128 : rem >= 64 ? 64 : rem >= 32 ? 32 : 16;
    const int tpt = DA_ROWS / hg;
    const long long n_qt = (long long)B * ((L + tpt - 1) / tpt);
    const int grid = (int)(n_qt < n_sm ? n_qt : n_sm);
    CUtensorMap tm_q;   // q as [B*L tokens][H heads][128]; a box is 64 dims x hg heads x 128/hg tokens
    if (!sm100::make_tmap_bf16_3d(&tm_q, q, (uint64_t)H, (uint64_t)B * L, (uint32_t)hg, (uint32_t)tpt))
      return set_error(CSLC_ERR_CUDA, "hca_dense_attn: tensor map encoding failed");
    dense_attn_sm100_kernel<<<grid, DA_THREADS, smem, stream>>>(B, L, hg, Nc, m, q_pos0, scale * kLog2e, out, lse, H,
                                                                h0, tm_q, tm_kv);
    const cslc_status st = check_launch("dense_attn_sm100_kernel");
    if (st != CSLC_OK) return st;
    h0 += hg;
  }
  return CSLC_OK;
}

int dense_attn_sm100_read_error() {
  int v = 0, zero = 0;
  cudaMemcpyFromSymbol(&v, g_dense_attn_err, sizeof(int));
  if (v) cudaMemcpyToSymbol(g_dense_attn_err, &zero, sizeof(int));
  return v;
}

CSLC_DEFINE_WAIT_LIMIT_SETTER(dense_attn_sm100_set_wait_limits)

}  // namespace cslc
