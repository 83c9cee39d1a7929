// CSA sparse attention on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// "读完这篇你就搞懂 DeepSeek v4 了", §三 注意力计算: every query token attends with
// all its heads to the k entries the indexer selected; K = V = the compressed
// entry (one KV head shared by the query heads).
//
// Formulation (per query token t, entries gathered in tiles of 128):
//   S^T[e, h] = E[e, :] . Q_t[h, :]          (M = 128 entries, N = H heads, K = 128)
//   P^T[e, h] = 2^(c*S^T[e,h] - m[h])        (c = scale*log2 e; softmax over e per head)
//   O^T[d, h] += sum_e E[e, d] P^T[e, h]      (M = 128 dims, N = 64, K = 128 entries)
// Putting the 128 gathered entries on the MMA's M side keeps M = 128 (full
// rate) although a token has only 64 heads, and both products read the same
// shared-memory tile of entries (K-major for S^T, MN-major for O^T).
//
// CTA roles (persistent CTAs, one per SM, loop over tokens):
//   warps 0-7   softmax + epilogue. Warp w owns TMEM lane quadrant w & 3 (32
//               entries of the tile, or 32 output dims) and head half w >> 2,
//               so two warps share each SM sub-partition. The per-head
//               reference m[h] is CTA-wide: on a token's first tile it is the
//               score of the token's first valid entry, and it only moves
//               (exact tile max by warp reduction, O^T rescale in TMEM) when a
//               probability would exceed 2^8. P^T rows go to 128-byte-swizzled shared memory.
//               At the token's end the head sums are reduced (butterfly
//               reduce-scatter), O^T is read from TMEM, normalised,
//               transposed through shared memory and stored.
//   warps 8-10  producer: per token the index row and Q_t (2-D TMA), then the
//               gathered entry tiles (cp.async 16 B chunks, 128-byte swizzle;
//               the copies arrive on the stage barrier as they land) into a
//               STAGES-deep ring. (Measured on B200: random 256-byte rows from
//               an L2-resident table gather at ~10 TB/s with cp.async but only
//               ~2 TB/s with TMA tile::gather4.)
//   warp 11     TMEM allocation and the single MMA-issuing thread.
// TMEM: S^T triple buffer (3 x 64 columns) + O^T double buffer (2 x 64); PV runs
// two tiles behind S^T so that the next S^T never waits for the softmax.
// Every wait is time-bounded; a timeout raises a CTA-wide abort, records an
// error code in a device word read by cslc_sync_status, and all roles leave.

#include "sm100.cuh"

namespace cslc {

using namespace sm100;

__device__ int g_sparse_attn_err = 0;

namespace {

constexpr int SA_THREADS = 384;
constexpr int SA_NSOFT = 256;             // softmax threads (warps 0-7)
constexpr int SA_PROD_WARP0 = 8;          // producer warps 8-10
constexpr int SA_NPROD = 96;
constexpr int SA_MMA_WARP = 11;
constexpr int SA_TILE = 128;              // entries per tile (MMA M)
constexpr int SA_ROWS_PER_PROD = (SA_TILE * 16 + SA_NPROD - 1) / SA_NPROD;   // 22 (6 rows per pass)
constexpr int SA_NP = 64;                 // padded head count of P^T / O^T
constexpr int SA_STAGES = 4;
constexpr int SA_E_BYTES = SA_TILE * 256; // 32 KB per entry tile
constexpr int SA_P_BYTES = SA_TILE * 128; // 16 KB per P^T tile (64 heads bf16)
constexpr int SA_Q_BYTES = SA_NP * 256;   // 16 KB (also the output staging)
constexpr int SA_MAXK = 2048;
constexpr float SA_OVERFLOW = 256.f;      // probabilities up to 2^8 are kept unrescaled
constexpr uint32_t SA_O_COL = 192;        // TMEM: S^T buffers at columns 0, 64, 128; O^T at 192 and 256

enum { ERR_KV_EMPTY = 1, ERR_TOK_FULL, ERR_KV_FULL, ERR_P_FULL, ERR_O_FREE, ERR_S_FULL,
       ERR_PV_DONE, ERR_O_FULL, ERR_Q_EMPTY, ERR_FINAL };

struct __align__(8) SaBars {
  uint64_t kv_full[SA_STAGES], kv_empty[SA_STAGES];
  uint64_t tok_full[2], q_empty[2];
  uint64_t s_full[3];
  uint64_t p_full[2];
  uint64_t pv_done[2];   // per P^T buffer: its PV has completed
  uint64_t o_full[2], o_free[2];
  uint64_t final_bar;
};

struct SaSmall {
  SaBars bars;
  uint32_t tmem_base;
  int abort_flag;
  int n_tiles[2];
  int last_w[2][4];
  int first_w[2][4];
  int ref_slot[2];     // first valid slot of the token (the softmax reference row), or SA_MAXK
  int any_rescale;
  __align__(16) float mref[SA_NP];   // running max per head (log2 units of c*S)
  __align__(16) float alpha[SA_NP];
  __align__(16) float inv_l[SA_NP];
  __align__(16) float red[4][SA_NP];  // per lane-quadrant partials
};

// Reduce-scatter of N per-lane values over the warp: returns, in every lane,
// the warp sum of value index rs_index<N>(lane).
template <int N, int OFF>
struct ReduceScatter {
  static __device__ __forceinline__ float run(const float* v, int lane) {
    float w[N / 2];
    const bool up = (lane & OFF) != 0;
#pragma unroll
    for (int i = 0; i < N / 2; ++i) {
      const float send = up ? v[i] : v[i + N / 2];
      const float keep = up ? v[i + N / 2] : v[i];
      w[i] = keep + __shfl_xor_sync(0xffffffffu, send, OFF);
    }
    return ReduceScatter<N / 2, OFF / 2>::run(w, lane);
  }
};
template <int OFF>
struct ReduceScatter<1, OFF> {
  static __device__ __forceinline__ float run(const float* v, int) {
    float x = v[0];
#pragma unroll
    for (int o = OFF; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
  }
};
template <int N>
__device__ __forceinline__ int rs_index(int lane) {
  int idx = 0, n = N;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    if (n > 1) {
      if (lane & off) idx += n / 2;
      n >>= 1;
    }
  }
  return idx;
}

}  // namespace

template <int H>
__global__ void __launch_bounds__(SA_THREADS, 1) sparse_attn_sm100_kernel(
    const uint16_t* __restrict__ q, const uint16_t* __restrict__ kv, const int32_t* __restrict__ idx,
    int B, int L, int Nc, int topk, float scale_log2, uint16_t* __restrict__ out, float* __restrict__ lse,
    int h_stride, int h_off, const __grid_constant__ CUtensorMap tm_q) {
  constexpr int HT = H / 2;           // heads per softmax thread
  static_assert(HT % 8 == 0 && HT <= 32, "H must be 16, 32 or 64");
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
      mbar_init(&bars.tok_full[i], 1); mbar_init(&bars.q_empty[i], SA_NSOFT / 32);
      mbar_init(&bars.p_full[i], SA_NSOFT / 32);
      mbar_init(&bars.o_full[i], 1); mbar_init(&bars.o_free[i], SA_NSOFT / 32);
    }
    for (int i = 0; i < 3; ++i) mbar_init(&bars.s_full[i], 1);
    for (int i = 0; i < 2; ++i) mbar_init(&bars.pv_done[i], 1);
    mbar_init(&bars.final_bar, 1);
    sm->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == SA_MMA_WARP) tmem_alloc(&sm->tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;
  volatile int* abortp = &sm->abort_flag;
  int* errp = &g_sparse_attn_err;

  if (warp >= SA_PROD_WARP0 && warp < SA_MMA_WARP) {
    // ------------------------------------------------------------ producer
    // Three warps. Per token: the index row (plain loads) and Q_t (2-D TMA,
    // completing on tok_full); per tile: 128 gathered rows x 16 chunks of
    // 16 B with cp.async into the 128-byte swizzled layout. Each thread's
    // copies arrive on the stage's barrier when they land (no waiting here).
    const int p = tid - SA_PROD_WARP0 * 32;   // 0..95
    const int pc = p & 15, pr0 = p >> 4;      // 16-byte column and first row of this thread
    int kv_it = 0;
    bool ok = true;
    long long tk = 0;
    long long q_issued0 = -1, q_issued1 = -1;   // last token whose Q load went to buffer 0 / 1
    if (p == 0) tma_prefetch_map(&tm_q);
    for (long long g = blockIdx.x; g < n_tok && ok; g += gridDim.x, ++tk) {
      const int qb = (int)(tk & 1);
      if (tk >= 2) {
        bool w = true;
        if (p == 0) w = mbar_wait(&bars.q_empty[qb], (uint32_t)(((tk >> 1) - 1) & 1), abortp, errp, ERR_Q_EMPTY);
        ok = !named_bar_or(1, SA_NPROD, !w);
        if (!ok) break;
      }
      // the index row: every element's copy in flight at once, then each
      // thread checks its own elements (out-of-range indices become -1)
      const int32_t* irow = idx + g * (long long)topk;
      int32_t* is = idx_s + qb * SA_MAXK;
      const uint32_t is_u = smem_u32(is);
      for (int s = p; s < topk; s += SA_NPROD) cp_async4(is_u + 4u * s, irow + s, true);
      cp_async_wait_all();
      int last = 0, first = SA_MAXK;
      for (int s = p; s < topk; s += SA_NPROD) {
        const int e = is[s];
        if (e < 0 || e >= Nc) {
          is[s] = -1;
        } else {
          last = s + 1;
          first = min(first, s);
        }
      }
      last = __reduce_max_sync(0xffffffffu, last);
      first = __reduce_min_sync(0xffffffffu, first);
      if (lane == 0) {
        sm->last_w[qb][p >> 5] = last;
        sm->first_w[qb][p >> 5] = first;
      }
      named_bar(1, SA_NPROD);
      const int nt = (max(max(sm->last_w[qb][0], sm->last_w[qb][1]), sm->last_w[qb][2]) + SA_TILE - 1) / SA_TILE;
      if (p == 0) {
        sm->n_tiles[qb] = nt;
        sm->ref_slot[qb] = min(min(sm->first_w[qb][0], sm->first_w[qb][1]), sm->first_w[qb][2]);
        uint8_t* qd = q_s + qb * SA_Q_BYTES;
        mbar_arrive_expect_tx(&bars.tok_full[qb], (uint32_t)(H * 256));
        const int qrow = (int)(g * h_stride + h_off);   // this token's first head of the group
        tma_load_2d(qd, &tm_q, 0, qrow, &bars.tok_full[qb]);
        tma_load_2d(qd + SA_NP * 128, &tm_q, 64, qrow, &bars.tok_full[qb]);
        if (qb == 0) q_issued0 = tk; else q_issued1 = tk;
      }
      const uint16_t* kvb = kv + (g / L) * (long long)Nc * kD;
      for (int j = 0; j < nt; ++j) {
        const int stage = kv_it % SA_STAGES;
        if (kv_it >= SA_STAGES) {
          bool w = true;
          if (p == 0) w = mbar_wait(&bars.kv_empty[stage], (uint32_t)((kv_it / SA_STAGES - 1) & 1), abortp, errp, ERR_KV_EMPTY);
          ok = !named_bar_or(1, SA_NPROD, !w);
          if (!ok) break;
        }
        // this thread always copies 16-byte column pc of rows pr0 + 6 i
        const uint32_t ed = smem_u32(e_s + stage * SA_E_BYTES) + (pc >> 3) * (SA_TILE * 128);
        int ev[SA_ROWS_PER_PROD];
#pragma unroll
        for (int i = 0; i < SA_ROWS_PER_PROD; ++i) {
          const int r = pr0 + 6 * i;
          const int slot = j * SA_TILE + r;
          ev[i] = (r < SA_TILE && slot < topk) ? is[slot] : -1;
        }
#pragma unroll
        for (int i = 0; i < SA_ROWS_PER_PROD; ++i) {
          const int r = pr0 + 6 * i;
          if (r < SA_TILE)
            cp_async16(ed + sw128(r, pc & 7), kvb + (long long)(ev[i] < 0 ? 0 : ev[i]) * kD + pc * 8, ev[i] >= 0);
        }
        cp_async_mbar_arrive(&bars.kv_full[stage]);
        ++kv_it;
      }
    }
    cp_async_wait<0>();
    // Q loads still in flight after an abort land before the CTA leaves (the
    // last load into each buffer is the latest phase of its barrier)
    if (p == 0) {
      if (q_issued0 >= 0) mbar_wait_done(&bars.tok_full[0], (uint32_t)((q_issued0 >> 1) & 1), errp, ERR_TOK_FULL);
      if (q_issued1 >= 0) mbar_wait_done(&bars.tok_full[1], (uint32_t)((q_issued1 >> 1) & 1), errp, ERR_TOK_FULL);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------ softmax + epilogue
    const int q4 = warp & 3, hh = warp >> 2;
    const int row = q4 * 32 + lane;         // TMEM lane = entry row of the tile / output dim
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const int h0 = hh * HT;                 // first head of this thread
    int s_it = 0, p_it = 0;
    bool ok = true;
    long long tk = 0;
    for (long long g = blockIdx.x; g < n_tok && ok; g += gridDim.x, ++tk) {
      const int qb = (int)(tk & 1), ob = qb;
      {
        bool w = true;
        if (tid == 0) w = mbar_wait(&bars.tok_full[qb], (uint32_t)((tk >> 1) & 1), abortp, errp, ERR_TOK_FULL);
        ok = !named_bar_or(2, SA_NSOFT, !w);
      }
      if (!ok) break;
      const int nt = sm->n_tiles[qb];
      if (tid < SA_NP) sm->mref[tid] = -INFINITY;
      named_bar(2, SA_NSOFT);
      const int32_t* is = idx_s + qb * SA_MAXK;
      float lpart[HT];
#pragma unroll
      for (int h = 0; h < HT; ++h) lpart[h] = 0.f;

      float negm[HT];                        // -m[h] (log2 units) of this thread's heads
#pragma unroll
      for (int h = 0; h < HT; ++h) negm[h] = INFINITY;
      for (int j = 0; j < nt; ++j) {
        const int sb = s_it % 3, pb = p_it & 1;
        // each warp waits for S on its own; a timeout anywhere raises the abort
        // flag, which every thread reads after the tile's CTA-wide barrier
        bool w = true;
        if (lane == 0) {
          w = mbar_wait(&bars.s_full[sb], (uint32_t)((s_it / 3) & 1), abortp, errp, ERR_S_FULL);
          // P^T buffer pb is free once the PV two tiles back has read it
          if (w && p_it >= 2) w = mbar_wait(&bars.pv_done[pb], (uint32_t)(((p_it >> 1) - 1) & 1), abortp, errp, ERR_PV_DONE);
        }
        w = __shfl_sync(0xffffffffu, (int)w, 0) != 0;
        const int slot = j * SA_TILE + row;
        const bool valid = slot < topk && is[slot] >= 0;
        // On a token's first tile the reference m[h] is the score of the
        // token's first valid entry (its probability is exactly 1, so nothing
        // underflows); a tile whose probabilities would exceed 2^8 against it
        // takes the exact-max path below. Without a valid entry in the first
        // tile the exact-max path runs directly.
        bool ref_ok = true;
        if (j == 0) {
          const int rs = sm->ref_slot[qb];
          ref_ok = rs < SA_TILE;
          if (w && ref_ok && q4 == (rs >> 5)) {   // the warps holding that row (warp-uniform)
            tc_fence_after();
            uint32_t rr[32];
            tmem_ld32(tmem + lane_off + sb * 64 + h0, rr);
            tmem_wait_ld();
            if (row == rs) {
#pragma unroll
              for (int h4 = 0; h4 < HT; h4 += 4)
                *reinterpret_cast<float4*>(&sm->mref[h0 + h4]) =
                    make_float4(__uint_as_float(rr[h4]) * scale_log2, __uint_as_float(rr[h4 + 1]) * scale_log2,
                                __uint_as_float(rr[h4 + 2]) * scale_log2, __uint_as_float(rr[h4 + 3]) * scale_log2);
            }
          }
          named_bar(2, SA_NSOFT);
          if (ref_ok) {
#pragma unroll
            for (int h4 = 0; h4 < HT; h4 += 4) {
              const float4 m4 = *reinterpret_cast<const float4*>(&sm->mref[h0 + h4]);
              negm[h4] = -m4.x; negm[h4 + 1] = -m4.y; negm[h4 + 2] = -m4.z; negm[h4 + 3] = -m4.w;
            }
          }
        }
        uint32_t r[32];
        if (w) {
          tc_fence_after();
          tmem_ld32(tmem + lane_off + sb * 64 + h0, r);
          tmem_wait_ld();
        }
        float v[HT];
        float pmax = 0.f;
        if (w && valid && ref_ok) {
#pragma unroll
          for (int h = 0; h < HT; ++h) {
            v[h] = ex2_approx(fmaf(__uint_as_float(r[h]), scale_log2, negm[h]));
            pmax = fmaxf(pmax, v[h]);
          }
        } else {
#pragma unroll
          for (int h = 0; h < HT; ++h) v[h] = 0.f;
        }
        // A raised abort flag joins the vote, so that all softmax warps leave
        // together (the named barriers stay matched).
        bool slow = false;
        if (named_bar_or(3, SA_NSOFT, !ref_ok || !(pmax <= SA_OVERFLOW) || !w || *abortp != 0)) {
          if (named_bar_or(3, SA_NSOFT, !w || *abortp != 0)) { ok = false; break; }
          slow = true;
        }
        if (slow) {
          // exact per-head maximum of this tile from S (still intact: the next
          // S into this buffer waits for this tile's p_full)
          uint32_t r[32];
          tmem_ld32(tmem + lane_off + sb * 64 + h0, r);
          tmem_wait_ld();
          float mx[HT];
#pragma unroll
          for (int h = 0; h < HT; ++h) mx[h] = warp_redux_max(valid ? __uint_as_float(r[h]) : -INFINITY);
          if (lane == 0) {
#pragma unroll
            for (int h4 = 0; h4 < HT; h4 += 4)
              *reinterpret_cast<float4*>(&sm->red[q4][h0 + h4]) = make_float4(mx[h4], mx[h4 + 1], mx[h4 + 2], mx[h4 + 3]);
          }
          if (tid == 0) sm->any_rescale = 0;
          named_bar(2, SA_NSOFT);
          if (tid < H) {
            const float old = sm->mref[tid];
            const float tmx = fmaxf(fmaxf(sm->red[0][tid], sm->red[1][tid]), fmaxf(sm->red[2][tid], sm->red[3][tid])) * scale_log2;
            const float nm = fmaxf(old, tmx);
            float a = 1.f;
            if (old == -INFINITY) a = 0.f;
            else if (nm != old) a = ex2_approx(old - nm);
            sm->alpha[tid] = a;
            sm->mref[tid] = nm;
            if (a != 1.f && j > 0) sm->any_rescale = 1;
          } else if (tid < SA_NP) {
            sm->alpha[tid] = 1.f;
          }
          named_bar(2, SA_NSOFT);
#pragma unroll
          for (int h4 = 0; h4 < HT; h4 += 4) {
            const float4 m4 = *reinterpret_cast<const float4*>(&sm->mref[h0 + h4]);
            const float4 a4 = *reinterpret_cast<const float4*>(&sm->alpha[h0 + h4]);
            negm[h4] = m4.x == -INFINITY ? INFINITY : -m4.x;
            negm[h4 + 1] = m4.y == -INFINITY ? INFINITY : -m4.y;
            negm[h4 + 2] = m4.z == -INFINITY ? INFINITY : -m4.z;
            negm[h4 + 3] = m4.w == -INFINITY ? INFINITY : -m4.w;
            lpart[h4] *= a4.x; lpart[h4 + 1] *= a4.y; lpart[h4 + 2] *= a4.z; lpart[h4 + 3] *= a4.w;
          }
          if (sm->any_rescale) {
            // O^T must be stable: the previous tile's PV has to be complete
            bool w2 = true;
            if (tid == 0)
              w2 = mbar_wait(&bars.pv_done[(p_it - 1) & 1], (uint32_t)(((p_it - 1) >> 1) & 1), abortp, errp, ERR_PV_DONE);
            ok = !named_bar_or(2, SA_NSOFT, !w2);
            if (!ok) break;
            tc_fence_after();
            uint32_t o[32];
            const uint32_t oc = tmem + lane_off + SA_O_COL + ob * 64 + hh * 32;
            tmem_ld32(oc, o);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * sm->alpha[hh * 32 + k]);
            tmem_st32(oc, o);
            tmem_wait_st();
          }
#pragma unroll
          for (int h = 0; h < HT; ++h) v[h] = valid ? ex2_approx(fmaf(__uint_as_float(r[h]), scale_log2, negm[h])) : 0.f;
        }
#pragma unroll
        for (int h = 0; h < HT; ++h) lpart[h] += v[h];
        // P^T row: this thread's heads h0 .. h0+HT-1 (chunks of 8 heads); the
        // second head half also zero-fills the padding heads H .. 63
        uint8_t* prow = p_s + pb * SA_P_BYTES;
#pragma unroll
        for (int c8 = 0; c8 < HT / 8; ++c8) {
          const uint4 pv = make_uint4(pack_bf16x2(v[8 * c8], v[8 * c8 + 1]), pack_bf16x2(v[8 * c8 + 2], v[8 * c8 + 3]),
                                      pack_bf16x2(v[8 * c8 + 4], v[8 * c8 + 5]), pack_bf16x2(v[8 * c8 + 6], v[8 * c8 + 7]));
          *reinterpret_cast<uint4*>(prow + sw128(row, h0 / 8 + c8)) = pv;
        }
        if (H < SA_NP && hh == 1) {
#pragma unroll
          for (int c8 = H / 8; c8 < 8; ++c8) *reinterpret_cast<uint4*>(prow + sw128(row, c8)) = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.p_full[pb]);
        ++s_it;
        ++p_it;
      }
      if (!ok) break;
      // ---- epilogue: head sums, normalise O^T, transpose through smem, store
      {
        const float part = ReduceScatter<HT, 16>::run(lpart, lane);
        if ((lane & (32 / HT - 1)) == 0) sm->red[q4][h0 + rs_index<HT>(lane)] = part;
      }
      named_bar(2, SA_NSOFT);
      if (tid < H) {
        const float l = sm->red[0][tid] + sm->red[1][tid] + sm->red[2][tid] + sm->red[3][tid];
        sm->inv_l[tid] = l > 0.f ? 1.f / l : 0.f;
        if (lse != nullptr) lse[g * h_stride + h_off + tid] = l > 0.f ? (sm->mref[tid] + log2f(l)) * kLn2 : -INFINITY;
      }
      {
        bool w = true;
        if (tid == 0) w = mbar_wait(&bars.o_full[ob], (uint32_t)((tk >> 1) & 1), abortp, errp, ERR_O_FULL);
        ok = !named_bar_or(2, SA_NSOFT, !w);
      }
      if (!ok) break;
      tc_fence_after();
      uint16_t* stage_out = reinterpret_cast<uint16_t*>(q_s + qb * SA_Q_BYTES);   // [H][128] bf16
      if (hh * 32 < H) {
        uint32_t r[32];
        if (nt > 0) {
          tmem_ld32(tmem + lane_off + SA_O_COL + ob * 64 + hh * 32, r);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) r[k] = 0u;
        }
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const int h = hh * 32 + k;
          if (h < H) stage_out[h * kD + row] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(r[k]) * sm->inv_l[h]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.o_free[ob]);
      named_bar(2, SA_NSOFT);
      uint4* dst = reinterpret_cast<uint4*>(out + (g * (long long)h_stride + h_off) * kD);
      const uint4* src = reinterpret_cast<const uint4*>(stage_out);
      for (int x = tid; x < H * 16; x += SA_NSOFT) dst[x] = src[x];
      named_bar(2, SA_NSOFT);
      if (lane == 0) mbar_arrive(&bars.q_empty[qb]);
    }
  } else {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID_S = idesc_bf16(128, H, false, false);
      constexpr uint32_t ID_O = idesc_bf16(128, SA_NP, true, true);
      int kv_it = 0, p_it = 0;
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
          mma_bf16(tmem + SA_O_COL + ob * 64, ad, bd, ID_O, (j_prev > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(&bars.kv_empty[stage_prev]);
        mma_commit(&bars.pv_done[pb]);
        ++p_it;
        return true;
      };
      // S^T[j+3] reuses S buffer j % 3; it is issued after PV(j), which waits
      // for p_full(j), so the softmax has finished reading S^T[j] by then.
      int s_cnt = 0;
      for (long long g = blockIdx.x; g < n_tok && ok; g += gridDim.x, ++tk) {
        const int qb = (int)(tk & 1), ob = qb;
        if (!mbar_wait(&bars.tok_full[qb], (uint32_t)((tk >> 1) & 1), abortp, errp, ERR_TOK_FULL)) { ok = false; break; }
        const int nt = sm->n_tiles[qb];
        if (tk >= 2 && !mbar_wait(&bars.o_free[ob], (uint32_t)(((tk >> 1) - 1) & 1), abortp, errp, ERR_O_FREE)) {
          ok = false;
          break;
        }
        const uint32_t q0 = smem_u32(q_s + qb * SA_Q_BYTES);
        int stage_1 = 0, stage_2 = 0;   // stages of tiles j-1 and j-2
        for (int j = 0; j < nt; ++j) {
          const int stage = kv_it % SA_STAGES, sb = s_cnt % 3;
          if (!mbar_wait(&bars.kv_full[stage], (uint32_t)((kv_it / SA_STAGES) & 1), abortp, errp, ERR_KV_FULL)) { ok = false; break; }
          fence_proxy_async_smem();   // cp.async (generic proxy) writes -> tensor-core reads
          tc_fence_after();
          const uint32_t e0 = smem_u32(e_s + stage * SA_E_BYTES);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint64_t ad = smem_desc_sw128(e0 + (k >> 2) * (SA_TILE * 128) + (k & 3) * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(q0 + (k >> 2) * (SA_NP * 128) + (k & 3) * 32, 16, 1024);
            mma_bf16(tmem + sb * 64, ad, bd, ID_S, k > 0 ? 1u : 0u);
          }
          mma_commit(&bars.s_full[sb]);
          ++s_cnt;
          // PV lags S by two tiles: S^T[j+1] needs only the gathered tile, not
          // the softmax of tile j-1
          if (j > 1 && !issue_pv(stage_2, j - 2, ob)) { ok = false; break; }
          stage_2 = stage_1;
          stage_1 = stage;
          ++kv_it;
        }
        if (!ok) break;
        if (nt > 1 && !issue_pv(stage_2, nt - 2, ob)) { ok = false; break; }
        if (nt > 0 && !issue_pv(stage_1, nt - 1, ob)) { ok = false; break; }
        mma_commit(&bars.o_full[ob]);
      }
      // every MMA issued so far has completed before TMEM is released, also
      // after an abort (the products finish on their own)
      mma_commit(&bars.final_bar);
      mbar_wait_done(&bars.final_bar, 0, errp, ERR_FINAL);
    }
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == SA_MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

namespace {
constexpr size_t sa_smem_bytes() {
  return 1024 + (size_t)SA_STAGES * SA_E_BYTES + 2 * SA_P_BYTES + 2 * SA_Q_BYTES + 2 * SA_MAXK * 4 + sizeof(SaSmall);
}
}  // namespace

// Any multiple of 16 up to 128 heads: groups of 64, 32 and 16 heads, one
// launch each on a view of q / out / lse that starts at the group's first
// head (the gathered entries are read again by every group, from L2).
bool sparse_attn_sm100_supported(int H) { return H >= 16 && H <= 128 && H % 16 == 0; }

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
  for (int h0 = 0; h0 < H;) {
    const int hg = H - h0 >= 64 ? 64 : (H - h0 >= 32 ? 32 : 16);
    CUtensorMap tm_q;   // q viewed as [B*L*H rows, 128] with a box of hg rows x 64 dims
    if (!sm100::make_tmap_bf16_2d(&tm_q, q, (uint64_t)n_tok * H, kD, kD * 2, (uint32_t)hg, 64))
      return set_error(CSLC_ERR_CUDA, "csa_sparse_attn: tensor map encoding failed");
    switch (hg) {
      case 16: sparse_attn_sm100_kernel<16><<<grid, SA_THREADS, smem, stream>>>(q, kv, idx, B, L, Nc, topk, sl2, out, lse, H, h0, tm_q); break;
      case 32: sparse_attn_sm100_kernel<32><<<grid, SA_THREADS, smem, stream>>>(q, kv, idx, B, L, Nc, topk, sl2, out, lse, H, h0, tm_q); break;
      default: sparse_attn_sm100_kernel<64><<<grid, SA_THREADS, smem, stream>>>(q, kv, idx, B, L, Nc, topk, sl2, out, lse, H, h0, tm_q); break;
    }
    const cslc_status st = check_launch("sparse_attn_sm100_kernel");
    if (st != CSLC_OK) return st;
    h0 += hg;
  }
  return CSLC_OK;
}

int sparse_attn_sm100_read_error() {
  int v = 0, zero = 0;
  cudaMemcpyFromSymbol(&v, g_sparse_attn_err, sizeof(int));
  if (v) cudaMemcpyToSymbol(g_sparse_attn_err, &zero, sizeof(int));
  return v;
}

CSLC_DEFINE_WAIT_LIMIT_SETTER(sparse_attn_sm100_set_wait_limits)

}  // namespace cslc
