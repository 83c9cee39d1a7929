// CSA sparse attention on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// "读完这篇你就搞懂 DeepSeek v4 了", §三 注意力计算: every query token attends with
// all its heads to the k entries the indexer selected; K = V = the compressed
// entry (one KV head shared by the query heads).
//
// Formulation (per query token t, entries gathered in tiles of 128):
//   S^T[e, h] = E[e, :] . Q_t[h, :]          (M = 128 entries, N = H heads, K = 128)
//   P^T[e, h] = exp2(scale*log2e*S^T - m[h]) (softmax over e, per head h)
//   O^T[d, h] += sum_e E[e, d] P^T[e, h]      (M = 128 dims, N = 64, K = 128 entries)
// Putting the 128 gathered entries on the MMA's M side keeps M = 128 (full
// rate) although a token has only 64 heads, and lets both products read the
// same shared-memory tile of entries (K-major for S^T, MN-major for O^T).
//
// CTA roles (persistent CTAs, one per SM, loop over tokens):
//   warps 0-3  softmax + epilogue: thread = TMEM lane = entry of the tile; the
//              per-head running max m[h] is shared by the CTA and only updated
//              (exact tile max, O^T rescale) when a score exceeds it by more
//              than 2^8 -- always on a token's first tile, rarely after; P^T
//              rows go to swizzled shared memory; at the token's end the head
//              sums are reduced, O^T is read from TMEM, normalised, transposed
//              through shared memory and stored
//   warps 4-6  producer: per token the index row and Q_t (cp.async), then the
//              gathered entry tiles (cp.async, 16 B chunks, 128-byte swizzle)
//              into a STAGES-deep ring
//   warp 7     TMEM allocation and the single MMA-issuing thread
// (8 warps = 2 per SM sub-partition, so each thread may use up to 255 registers)
// TMEM: S^T double buffer (2 x 64 columns) + O^T double buffer (2 x 64).
// Every wait is time-bounded; a timeout raises a CTA-wide abort, records an
// error code in a device word read by cslc_sync_status, and all roles leave.

#include "sm100.cuh"

namespace cslc {

using namespace sm100;

__device__ int g_sparse_attn_err = 0;

namespace {

constexpr int SA_THREADS = 256;
constexpr int SA_NPROD = 96;             // producer threads (warps 4-6)
constexpr int SA_TILE = 128;              // entries per tile (MMA M)
constexpr int SA_NP = 64;                 // padded head count of P^T / O^T
constexpr int SA_STAGES = 4;
constexpr int SA_E_BYTES = SA_TILE * 256; // 32 KB per entry tile
constexpr int SA_P_BYTES = SA_TILE * 128; // 16 KB per P^T tile (64 heads bf16)
constexpr int SA_Q_BYTES = SA_NP * 256;   // 16 KB (also the output staging)
constexpr int SA_MAXK = 2048;

enum { ERR_KV_EMPTY = 1, ERR_TOK_FULL, ERR_KV_FULL, ERR_S_FREE, ERR_P_FULL, ERR_O_FREE, ERR_S_FULL,
       ERR_PV_DONE, ERR_O_FULL, ERR_Q_EMPTY, ERR_FINAL };

struct __align__(8) SaBars {
  uint64_t kv_full[SA_STAGES], kv_empty[SA_STAGES];
  uint64_t tok_full[2], q_empty[2];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full[2];
  uint64_t pv_done;
  uint64_t o_full[2], o_free[2];
  uint64_t final_bar;
};

struct SaSmall {
  SaBars bars;
  uint32_t tmem_base;
  int abort_flag;
  int n_tiles[2];
  int max_slot[2];
  int any_rescale;
  float mref[SA_NP];       // running max per head (log2 units)
  float alpha[SA_NP];
  float inv_l[SA_NP];
  float red[4][SA_NP];     // per-warp partials
};

}  // namespace

template <int H>
__global__ void __launch_bounds__(SA_THREADS, 1) sparse_attn_sm100_kernel(
    const uint16_t* __restrict__ q, const uint16_t* __restrict__ kv, const int32_t* __restrict__ idx,
    int B, int L, int Nc, int topk, float scale_log2, uint16_t* __restrict__ out, float* __restrict__ lse) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* e_s = smem;                                       // [STAGES][2 kb][128][128 B]
  uint8_t* p_s = e_s + SA_STAGES * SA_E_BYTES;               // [2][128][128 B]
  uint8_t* q_s = p_s + 2 * SA_P_BYTES;                       // [2][2 kb][64][128 B]
  int32_t* idx_s = reinterpret_cast<int32_t*>(q_s + 2 * SA_Q_BYTES);   // [2][SA_MAXK]
  SaSmall* sm = reinterpret_cast<SaSmall*>(idx_s + 2 * SA_MAXK);
  SaBars& bars = sm->bars;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long n_tok = (long long)B * L;

  if (tid == 0) {
    for (int s = 0; s < SA_STAGES; ++s) { mbar_init(&bars.kv_full[s], SA_NPROD); mbar_init(&bars.kv_empty[s], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.tok_full[i], SA_NPROD); mbar_init(&bars.q_empty[i], 128);
      mbar_init(&bars.s_full[i], 1); mbar_init(&bars.s_free[i], 128);
      mbar_init(&bars.p_full[i], 128);
      mbar_init(&bars.o_full[i], 1); mbar_init(&bars.o_free[i], 128);
    }
    mbar_init(&bars.pv_done, 1);
    mbar_init(&bars.final_bar, 1);
    sm->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 7) tmem_alloc(&sm->tmem_base, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;
  volatile int* abortp = &sm->abort_flag;
  int* errp = &g_sparse_attn_err;

  if (warp >= 4 && warp < 7) {
    // ------------------------------------------------------------ producer
    const int p = tid - 128;           // 0..95
    int kv_it = 0;
    bool ok = true;
    long long tk = 0;
    for (long long g = blockIdx.x; g < n_tok && ok; g += gridDim.x, ++tk) {
      const int qb = (int)(tk & 1);
      if (tk >= 2) {
        bool w = true;
        if (p == 0) w = mbar_wait(&bars.q_empty[qb], (uint32_t)(((tk >> 1) - 1) & 1), abortp, errp, ERR_Q_EMPTY);
        ok = !named_bar_or(1, SA_NPROD, !w);
        if (!ok) break;
      }
      // index row -> smem, last valid slot
      const int32_t* irow = idx + g * (long long)topk;
      int32_t* is = idx_s + qb * SA_MAXK;
      int last = 0;
      for (int s = p; s < topk; s += SA_NPROD) {
        int e = __ldg(irow + s);
        if (e < 0 || e >= Nc) e = -1;
        is[s] = e;
        if (e >= 0) last = s + 1;
      }
      last = __reduce_max_sync(0xffffffffu, last);
      if (p == 0) sm->max_slot[qb] = 0;
      named_bar(1, SA_NPROD);
      if (lane == 0) atomicMax(&sm->max_slot[qb], last);
      // Q_t: H rows x 256 B -> [2 kb][64][128 B] (rows >= H stay unused)
      uint8_t* qd = q_s + qb * SA_Q_BYTES;
      const uint16_t* qsrc = q + g * (long long)H * kD;
      for (int x = p; x < H * 16; x += SA_NPROD) {
        const int r = x >> 4, c = x & 15;
        cp_async16(smem_u32(qd + (c >> 3) * (SA_NP * 128) + sw128(r, c & 7)), qsrc + r * kD + c * 8, true);
      }
      cp_async_commit();
      cp_async_wait<0>();
      fence_proxy_async_smem();
      named_bar(1, SA_NPROD);
      const int nt = (sm->max_slot[qb] + SA_TILE - 1) / SA_TILE;
      if (p == 0) sm->n_tiles[qb] = nt;
      mbar_arrive(&bars.tok_full[qb]);
      // entry tiles: 128 rows x 16 chunks of 16 B, chunk x -> row x >> 4, chunk x & 15
      const uint16_t* kvb = kv + (g / L) * (long long)Nc * kD;
      int issued = 0;
      for (int j = 0; j < nt; ++j) {
        const int stage = kv_it % SA_STAGES;
        if (kv_it >= SA_STAGES) {
          bool w = true;
          if (p == 0) w = mbar_wait(&bars.kv_empty[stage], (uint32_t)((kv_it / SA_STAGES - 1) & 1), abortp, errp, ERR_KV_EMPTY);
          ok = !named_bar_or(1, SA_NPROD, !w);
          if (!ok) break;
        }
        uint8_t* ed = e_s + stage * SA_E_BYTES;
        for (int x = p; x < SA_TILE * 16; x += SA_NPROD) {
          const int r = x >> 4, c = x & 15;
          const int slot = j * SA_TILE + r;
          const int e = slot < topk ? is[slot] : -1;
          cp_async16(smem_u32(ed + (c >> 3) * (SA_TILE * 128) + sw128(r, c & 7)),
                     kvb + (long long)(e < 0 ? 0 : e) * kD + c * 8, e >= 0);
        }
        cp_async_commit();
        ++issued;
        if (issued >= SA_STAGES - 1) {
          cp_async_wait<SA_STAGES - 2>();
          fence_proxy_async_smem();
          mbar_arrive(&bars.kv_full[(kv_it - (SA_STAGES - 2)) % SA_STAGES]);
          --issued;
        }
        ++kv_it;
      }
      cp_async_wait<0>();
      fence_proxy_async_smem();
      for (int k = issued; k > 0; --k) mbar_arrive(&bars.kv_full[(kv_it - k) % SA_STAGES]);
    }
    cp_async_wait<0>();
  } else if (warp < 4) {
    // ------------------------------------------------------ softmax + epilogue
    const int s_lane = tid;                // 0..127 = TMEM lane = entry row / output dim
    const int wq = warp;                   // TMEM lane quadrant
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    int s_it = 0, p_it = 0;
    bool ok = true;
    long long tk = 0;
    for (long long g = blockIdx.x; g < n_tok && ok; g += gridDim.x, ++tk) {
      const int qb = (int)(tk & 1), ob = qb;
      bool w = true;
      if (s_lane == 0) w = mbar_wait(&bars.tok_full[qb], (uint32_t)((tk >> 1) & 1), abortp, errp, ERR_TOK_FULL);
      ok = !named_bar_or(2, 128, !w);
      const int nt = sm->n_tiles[qb];
      if (s_lane < SA_NP) sm->mref[s_lane] = -INFINITY;
      named_bar(2, 128);
      if (!ok) break;
      const int32_t* is = idx_s + qb * SA_MAXK;
      float lpart[H];
#pragma unroll
      for (int h = 0; h < H; ++h) lpart[h] = 0.f;

      for (int j = 0; j < nt; ++j) {
        const int sb = s_it & 1, pb = p_it & 1;
        bool w = true;
        if (s_lane == 0) w = mbar_wait(&bars.s_full[sb], (uint32_t)((s_it >> 1) & 1), abortp, errp, ERR_S_FULL);
        ok = !named_bar_or(2, 128, !w);
        if (!ok) break;
        tc_fence_after();
        float sv[H];
        {
          uint32_t r[32];
#pragma unroll
          for (int c0 = 0; c0 < H; c0 += 32) {
            tmem_ld32(tmem + lane_off + sb * 64 + c0, r);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k)
              if (c0 + k < H) sv[c0 + k] = __uint_as_float(r[k]);
          }
        }
        tc_fence_before();
        mbar_arrive(&bars.s_free[sb]);
        const int slot = j * SA_TILE + s_lane;
        const bool valid = slot < topk && is[slot] >= 0;
        bool exceed = false;
#pragma unroll
        for (int h = 0; h < H; ++h) {
          sv[h] = valid ? sv[h] * scale_log2 : -INFINITY;
          exceed |= sv[h] > sm->mref[h] + 8.f;
        }
        if (j == 0 || named_bar_or(3, 128, exceed)) {
          // exact per-head maximum of this tile, then the new running max
#pragma unroll
          for (int h = 0; h < H; ++h) {
            const float mx = warp_max(sv[h]);
            if (lane == 0) sm->red[wq][h] = mx;
          }
          if (s_lane == 0) sm->any_rescale = 0;
          named_bar(2, 128);
          if (s_lane < H) {
            const float old = sm->mref[s_lane];
            const float tmx = fmaxf(fmaxf(sm->red[0][s_lane], sm->red[1][s_lane]), fmaxf(sm->red[2][s_lane], sm->red[3][s_lane]));
            const float nm = fmaxf(old, tmx);
            float a = 1.f;
            if (old != -INFINITY && nm != old) a = exp2f(old - nm);
            else if (old == -INFINITY) a = 0.f;
            sm->alpha[s_lane] = a;
            sm->mref[s_lane] = nm;
            if (a != 1.f && j > 0) sm->any_rescale = 1;
          }
          named_bar(2, 128);
#pragma unroll
          for (int h = 0; h < H; ++h) lpart[h] *= sm->alpha[h];
          if (sm->any_rescale) {
            // O^T must be stable: the previous tile's PV has to be complete
            bool w2 = true;
            if (s_lane == 0) w2 = mbar_wait(&bars.pv_done, (uint32_t)((p_it - 1) & 1), abortp, errp, ERR_PV_DONE);
            ok = !named_bar_or(2, 128, !w2);
            if (!ok) break;
            tc_fence_after();
            uint32_t r[32];
#pragma unroll
            for (int c0 = 0; c0 < SA_NP; c0 += 32) {
              tmem_ld32(tmem + lane_off + 128 + ob * 64 + c0, r);
              tmem_wait_ld();
#pragma unroll
              for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * (c0 + k < H ? sm->alpha[c0 + k] : 1.f));
              tmem_st32(tmem + lane_off + 128 + ob * 64 + c0, r);
            }
            tmem_wait_st();
          }
        }
        // P^T row of this entry: 64 bf16 (heads >= H are zero)
        uint32_t pk[SA_NP / 2];
#pragma unroll
        for (int h2 = 0; h2 < SA_NP / 2; ++h2) {
          float a = 0.f, b = 0.f;
          if (2 * h2 < H) {
            const float m0 = sm->mref[2 * h2], m1 = sm->mref[2 * h2 + 1];
            a = valid ? exp2f(sv[2 * h2] - m0) : 0.f;
            b = valid ? exp2f(sv[2 * h2 + 1] - m1) : 0.f;
            lpart[2 * h2] += a;
            lpart[2 * h2 + 1] += b;
          }
          pk[h2] = pack_bf16x2(a, b);
        }
        uint8_t* prow = p_s + pb * SA_P_BYTES;
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8)
          *reinterpret_cast<uint4*>(prow + sw128(s_lane, c8)) =
              make_uint4(pk[4 * c8], pk[4 * c8 + 1], pk[4 * c8 + 2], pk[4 * c8 + 3]);
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars.p_full[pb]);
        ++s_it;
        ++p_it;
      }
      if (!ok) break;
      // ---- epilogue: head sums, normalise O^T, transpose through smem, store
#pragma unroll
      for (int h = 0; h < H; ++h) {
        const float sm_h = warp_sum(lpart[h]);
        if (lane == 0) sm->red[wq][h] = sm_h;
      }
      named_bar(2, 128);
      if (s_lane < H) {
        const float l = sm->red[0][s_lane] + sm->red[1][s_lane] + sm->red[2][s_lane] + sm->red[3][s_lane];
        sm->inv_l[s_lane] = l > 0.f ? 1.f / l : 0.f;
        if (lse != nullptr)
          lse[g * H + s_lane] = l > 0.f ? (sm->mref[s_lane] + log2f(l)) * kLn2 : -INFINITY;
      }
      bool wo = true;
      if (s_lane == 0) wo = mbar_wait(&bars.o_full[ob], (uint32_t)((tk >> 1) & 1), abortp, errp, ERR_O_FULL);
      ok = !named_bar_or(2, 128, !wo);
      if (!ok) break;
      tc_fence_after();
      uint16_t* stage_out = reinterpret_cast<uint16_t*>(q_s + qb * SA_Q_BYTES);   // [H][128] bf16
      {
        uint32_t r[32];
#pragma unroll
        for (int c0 = 0; c0 < H; c0 += 32) {
          if (nt > 0) {
            tmem_ld32(tmem + lane_off + 128 + ob * 64 + c0, r);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int k = 0; k < 32; ++k) r[k] = 0u;
          }
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            if (c0 + k < H) {
              const float v = __uint_as_float(r[k]) * sm->inv_l[c0 + k];
              stage_out[(c0 + k) * kD + s_lane] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bars.o_free[ob]);
      named_bar(2, 128);
      uint4* dst = reinterpret_cast<uint4*>(out + g * (long long)H * kD);
      const uint4* src = reinterpret_cast<const uint4*>(stage_out);
      for (int x = s_lane; x < H * 16; x += 128) dst[x] = src[x];
      named_bar(2, 128);
      mbar_arrive(&bars.q_empty[qb]);
    }
  } else {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID_S = idesc_bf16(128, H, false, false);
      constexpr uint32_t ID_O = idesc_bf16(128, SA_NP, true, true);
      int kv_it = 0, s_it = 0, p_it = 0;
      bool ok = true;
      long long tk = 0;
      auto issue_pv = [&](int stage_prev, int j_prev, int ob) -> bool {
        const int pb = p_it & 1;
        if (!mbar_wait(&bars.p_full[pb], (uint32_t)((p_it >> 1) & 1), abortp, errp, ERR_P_FULL)) return false;
        tc_fence_after();
        const uint32_t e0 = smem_u32(e_s + stage_prev * SA_E_BYTES);
        const uint32_t p0 = smem_u32(p_s + pb * SA_P_BYTES);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t ad = smem_desc_sw128(e0 + k * 2048, SA_TILE * 128, 1024);
          const uint64_t bd = smem_desc_sw128(p0 + k * 2048, SA_TILE * 128, 1024);
          mma_bf16(tmem + 128 + ob * 64, ad, bd, ID_O, (j_prev > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(&bars.kv_empty[stage_prev]);
        mma_commit(&bars.pv_done);
        ++p_it;
        return true;
      };
      for (long long g = blockIdx.x; g < n_tok && ok; g += gridDim.x, ++tk) {
        const int qb = (int)(tk & 1), ob = qb;
        if (!mbar_wait(&bars.tok_full[qb], (uint32_t)((tk >> 1) & 1), abortp, errp, ERR_TOK_FULL)) { ok = false; break; }
        const int nt = sm->n_tiles[qb];
        if (tk >= 2 && nt > 0) {
          // (waited only when this token writes O^T[ob])
        }
        if (tk >= 2) {
          if (!mbar_wait(&bars.o_free[ob], (uint32_t)(((tk >> 1) - 1) & 1), abortp, errp, ERR_O_FREE)) { ok = false; break; }
        }
        const uint32_t q0 = smem_u32(q_s + qb * SA_Q_BYTES);
        int stage_prev = 0;
        for (int j = 0; j < nt; ++j) {
          const int stage = kv_it % SA_STAGES, sb = s_it & 1;
          if (!mbar_wait(&bars.kv_full[stage], (uint32_t)((kv_it / SA_STAGES) & 1), abortp, errp, ERR_KV_FULL)) { ok = false; break; }
          if (s_it >= 2 && !mbar_wait(&bars.s_free[sb], (uint32_t)(((s_it >> 1) - 1) & 1), abortp, errp, ERR_S_FREE)) { ok = false; break; }
          tc_fence_after();
          const uint32_t e0 = smem_u32(e_s + stage * SA_E_BYTES);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint64_t ad = smem_desc_sw128(e0 + (k >> 2) * (SA_TILE * 128) + (k & 3) * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(q0 + (k >> 2) * (SA_NP * 128) + (k & 3) * 32, 16, 1024);
            mma_bf16(tmem + sb * 64, ad, bd, ID_S, k > 0 ? 1u : 0u);
          }
          mma_commit(&bars.s_full[sb]);
          ++s_it;
          if (j > 0 && !issue_pv(stage_prev, j - 1, ob)) { ok = false; break; }
          stage_prev = stage;
          ++kv_it;
        }
        if (!ok) break;
        if (nt > 0 && !issue_pv(stage_prev, nt - 1, ob)) { ok = false; break; }
        mma_commit(&bars.o_full[ob]);
      }
      // every MMA issued so far has completed before TMEM is released
      mma_commit(&bars.final_bar);
      mbar_wait(&bars.final_bar, 0, abortp, errp, ERR_FINAL);
    }
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 7) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

namespace {
constexpr size_t sa_smem_bytes() {
  return 1024 + (size_t)SA_STAGES * SA_E_BYTES + 2 * SA_P_BYTES + 2 * SA_Q_BYTES + 2 * SA_MAXK * 4 + sizeof(SaSmall);
}
}  // namespace

bool sparse_attn_sm100_supported(int H) { return H == 16 || H == 32 || H == 64; }

cslc_status launch_sparse_attn_sm100(const uint16_t* q, const uint16_t* kv, const int32_t* idx, int B, int L,
                                     int H, int Nc, int topk, float scale, uint16_t* out, float* lse,
                                     cudaStream_t stream) {
  static int configured_for = -1;
  static int n_sm = 148;
  int dev = 0;
  cudaGetDevice(&dev);
  const size_t smem = sa_smem_bytes();
  if (configured_for != dev) {
    cudaFuncSetAttribute(sparse_attn_sm100_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(sparse_attn_sm100_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(sparse_attn_sm100_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    configured_for = dev;
  }
  const long long n_tok = (long long)B * L;
  const int grid = (int)(n_tok < n_sm ? n_tok : n_sm);
  const float sl2 = scale * kLog2e;
  switch (H) {
    case 16: sparse_attn_sm100_kernel<16><<<grid, SA_THREADS, smem, stream>>>(q, kv, idx, B, L, Nc, topk, sl2, out, lse); break;
    case 32: sparse_attn_sm100_kernel<32><<<grid, SA_THREADS, smem, stream>>>(q, kv, idx, B, L, Nc, topk, sl2, out, lse); break;
    default: sparse_attn_sm100_kernel<64><<<grid, SA_THREADS, smem, stream>>>(q, kv, idx, B, L, Nc, topk, sl2, out, lse); break;
  }
  return check_launch("sparse_attn_sm100_kernel");
}

int sparse_attn_sm100_read_error() {
  int v = 0, zero = 0;
  cudaMemcpyFromSymbol(&v, g_sparse_attn_err, sizeof(int));
  if (v) cudaMemcpyToSymbol(g_sparse_attn_err, &zero, sizeof(int));
  return v;
}

}  // namespace cslc
