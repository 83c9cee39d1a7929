// Token-window compression (CSA overlapped 2m windows, HCA m' windows).
//
// "读完这篇你就搞懂 DeepSeek v4 了", §三 压缩机制: tokens are grouped m at a time,
// each token's contribution is weighted per dimension, and two consecutive
// groups are joined for CSA; HCA 步骤简化: one group, no join. The weight form
// is the per-channel softmax over the window of (z_t + positional bias).
//
// Layout: one warp per compressed entry. Lane = split * 16 + chunk: `chunk`
// selects 8 channels (one 16-byte vector of c / z), `split` selects half of
// the window's tokens. Each lane keeps an fp32 online-softmax state per
// channel (running max, sum of weights, weighted sum of c) over its tokens;
// the two halves are merged with one shuffle. The pass streams c and z once
// (CSA reads each token twice, the second time from L2) with 16-byte loads.

#include "common.cuh"

namespace cslc {

struct SoftmaxAcc {
  float mx[8], sum[8], acc[8];
};

__device__ __forceinline__ void acc_init(SoftmaxAcc& s) {
#pragma unroll
  for (int j = 0; j < 8; ++j) { s.mx[j] = -INFINITY; s.sum[j] = 0.f; s.acc[j] = 0.f; }
}

// Adds one token: logit a (already in log2 units) and candidate value c.
__device__ __forceinline__ void acc_add(SoftmaxAcc& s, int j, float a, float c) {
  if (a > s.mx[j]) {
    float r = exp2f(s.mx[j] - a);   // 0 when the old max is -inf
    s.sum[j] = s.sum[j] * r + 1.f;
    s.acc[j] = s.acc[j] * r + c;
    s.mx[j] = a;
  } else {
    float p = exp2f(a - s.mx[j]);
    s.sum[j] += p;
    s.acc[j] = fmaf(p, c, s.acc[j]);
  }
}

// One compressed entry of D (128 or 64) channels, computed by one warp from
// its W window slots; `fetch(s, cv, zv)` loads the 16-byte chunk `chunk` of
// slot s's candidate and logit. Slots below s_begin are absent (the first CSA
// entry has no C^b half). Every caller runs this same code, so an entry is
// bit-identical whether it comes from a prefill pass or a decode append.
// Lanes whose chunk lies past D / 8 compute on a valid chunk and discard it.
template <int D, class Fetch>
__device__ __forceinline__ void window_entry(int W, int s_begin, const uint16_t* __restrict__ bias, int lane,
                                             Fetch fetch, float (&res)[8]) {
  const int chunk = (lane & 15) % (D / 8);
  const int split = lane >> 4;
  const int half = (W + 1) >> 1;
  const int s_lo = max(split * half, s_begin), s_hi = min(W, split * half + half);
  SoftmaxAcc st;
  acc_init(st);
  for (int s = s_lo; s < s_hi; ++s) {
    uint4 cv, zv;
    fetch(s, chunk, cv, zv);
    const uint4 bv = __ldg(reinterpret_cast<const uint4*>(bias + (size_t)s * D) + chunk);
    const uint32_t cw[4] = {cv.x, cv.y, cv.z, cv.w};
    const uint32_t zw[4] = {zv.x, zv.y, zv.z, zv.w};
    const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      acc_add(st, 2 * k, (bf16_lo(zw[k]) + bf16_lo(bw[k])) * kLog2e, bf16_lo(cw[k]));
      acc_add(st, 2 * k + 1, (bf16_hi(zw[k]) + bf16_hi(bw[k])) * kLog2e, bf16_hi(cw[k]));
    }
  }
  // merge the two halves (lanes chunk and chunk + 16)
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float omx = __shfl_xor_sync(0xffffffffu, st.mx[j], 16);
    const float osum = __shfl_xor_sync(0xffffffffu, st.sum[j], 16);
    const float oacc = __shfl_xor_sync(0xffffffffu, st.acc[j], 16);
    const float M = fmaxf(st.mx[j], omx);
    const float f1 = st.mx[j] == -INFINITY ? 0.f : exp2f(st.mx[j] - M);
    const float f2 = omx == -INFINITY ? 0.f : exp2f(omx - M);
    const float sum = st.sum[j] * f1 + osum * f2;
    const float acc = st.acc[j] * f1 + oacc * f2;
    res[j] = acc / sum;
  }
}

__device__ __forceinline__ uint4 pack_entry_chunk(const float (&res)[8]) {
  uint4 o;
  o.x = pack_bf16x2(res[0], res[1]);
  o.y = pack_bf16x2(res[2], res[3]);
  o.z = pack_bf16x2(res[4], res[5]);
  o.w = pack_bf16x2(res[6], res[7]);
  return o;
}

template <int D>
__global__ void __launch_bounds__(256) compress_kernel(
    const uint16_t* __restrict__ c, const uint16_t* __restrict__ z,
    const uint16_t* __restrict__ cb, const uint16_t* __restrict__ zb,
    const uint16_t* __restrict__ bias, int B, int L, int m, int overlap, int n_c,
    uint16_t* __restrict__ out) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= B * n_c) return;
  const int b = warp / n_c;
  const int i = warp - b * n_c;
  // Window: slots 0..W-1. CSA: slot s < m is token (i-1)m + s (C^b), slot
  // s >= m is token i*m + s - m (C^a). HCA: slot s is token i*m + s.
  const int W = overlap ? 2 * m : m;
  const size_t row0 = (size_t)b * L;
  auto fetch = [&](int s, int chunk, uint4& cv, uint4& zv) {
    const bool prev = overlap && s < m;
    const int t = overlap ? (i - 1) * m + s : i * m + s;
    cv = __ldg(reinterpret_cast<const uint4*>((prev ? cb : c) + (row0 + t) * D) + chunk);
    zv = __ldg(reinterpret_cast<const uint4*>((prev ? zb : z) + (row0 + t) * D) + chunk);
  };
  float res[8];
  window_entry<D>(W, overlap && i == 0 ? m : 0, bias, lane, fetch, res);
  if (lane < D / 8) reinterpret_cast<uint4*>(out + ((size_t)b * n_c + i) * D)[lane] = pack_entry_chunk(res);
}

cslc_status launch_compress(const uint16_t* c, const uint16_t* z, const uint16_t* cb,
                            const uint16_t* zb, const uint16_t* bias, int B, int L, int D, int m,
                            int overlap, uint16_t* out, cudaStream_t stream) {
  const int n_c = L / m;
  const long long warps = (long long)B * n_c;
  if (warps == 0) return CSLC_OK;
  const int threads = 256;
  const long long blocks = (warps * 32 + threads - 1) / threads;
  if (D == 64)
    compress_kernel<64><<<(unsigned)blocks, threads, 0, stream>>>(c, z, cb ? cb : c, zb ? zb : z, bias, B, L, m,
                                                                  overlap, n_c, out);
  else
    compress_kernel<128><<<(unsigned)blocks, threads, 0, stream>>>(c, z, cb ? cb : c, zb ? zb : z, bias, B, L, m,
                                                                   overlap, n_c, out);
  return check_launch("compress_kernel");
}

// ---------------------------------------------------------------------------
// Mixed decode KV layout (first page §1.4 存储格式混): dims 0..63 as e4m3 with
// one fp32 scale per entry, dims 64..127 kept bf16. One warp per entry; lane l
// owns dims 2l, 2l+1 of each half.

// One entry's row (lane l holds dims 2l, 2l+1 in `lo` and 64+2l, 64+2l+1 in
// `hi`) into the mixed layout; shared by the bulk quantiser and the decode
// append so that both produce identical codes.
// 64 bf16 values (lane l holds 2l, 2l+1 in `lo`) as e4m3 codes with one fp32
// scale: s = amax / 448 (1 for a zero row), codes = RNE-saturate(x / s), the
// division in fp32.
__device__ __forceinline__ void e4m3_row64(uint32_t lo, int lane, uint8_t* __restrict__ codes_row,
                                           float* __restrict__ scale_out) {
  const float x0 = bf16_lo(lo), x1 = bf16_hi(lo);
  const float amax = warp_max(fmaxf(fabsf(x0), fabsf(x1)));
  const float s = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  const float2 q = make_float2(__fdiv_rn(x0, s), __fdiv_rn(x1, s));
  const __nv_fp8x2_storage_t codes = __nv_cvt_float2_to_fp8x2(q, __NV_SATFINITE, __NV_E4M3);
  reinterpret_cast<uint16_t*>(codes_row)[lane] = codes;
  if (lane == 0) *scale_out = s;
}

__device__ __forceinline__ void quantize_row(uint32_t lo, uint32_t hi, int lane, uint8_t* __restrict__ nope_row,
                                             uint16_t* __restrict__ rope_row, float* __restrict__ scale_out) {
  e4m3_row64(lo, lane, nope_row, scale_out);
  reinterpret_cast<uint32_t*>(rope_row)[lane] = hi;
}

__global__ void __launch_bounds__(256) quantize_kv_kernel(const uint16_t* __restrict__ kv,
                                                          long long n_entries,
                                                          uint8_t* __restrict__ nope,
                                                          uint16_t* __restrict__ rope,
                                                          float* __restrict__ scale) {
  const long long e = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (e >= n_entries) return;
  const uint32_t* row = reinterpret_cast<const uint32_t*>(kv + e * kD);
  quantize_row(row[lane], row[32 + lane], lane, nope + e * kNope, rope + e * kRope, scale + e);
}

// Rows of 64 values (the indexer's q_I / k_I rows) as e4m3 codes + a scale each.
__global__ void __launch_bounds__(256) quantize_rows64_kernel(const uint16_t* __restrict__ x, long long rows,
                                                              uint8_t* __restrict__ codes,
                                                              float* __restrict__ scales) {
  const long long r = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  e4m3_row64(reinterpret_cast<const uint32_t*>(x + r * 64)[lane], lane, codes + r * 64, scales + r);
}

cslc_status launch_quantize_rows64(const uint16_t* x, long long rows, uint8_t* codes, float* scales,
                                   cudaStream_t stream) {
  if (rows == 0) return CSLC_OK;
  const long long blocks = (rows * 32 + 255) / 256;
  quantize_rows64_kernel<<<(unsigned)blocks, 256, 0, stream>>>(x, rows, codes, scales);
  return check_launch("quantize_rows64_kernel");
}

cslc_status launch_quantize_kv(const uint16_t* kv, long long n, uint8_t* nope, uint16_t* rope,
                               float* scale, cudaStream_t stream) {
  if (n == 0) return CSLC_OK;
  const long long blocks = (n * 32 + 255) / 256;
  quantize_kv_kernel<<<(unsigned)blocks, 256, 0, stream>>>(kv, n, nope, rope, scale);
  return check_launch("quantize_kv_kernel");
}

// ---------------------------------------------------------------------------
// Decode append ("读完这篇…" §三 压缩机制; first page §1.1 工程细节 for the
// overlapped window): when the new token p of a sequence completes a window,
// (p + 1) mod m == 0, entry i = (p + 1) / m - 1 is compressed from the last W
// tokens exactly as a prefill pass would compress it, stored in the mixed
// layout, and its indexer key is compressed the same way from the tokens'
// 64-dim key candidates. One block per sequence: warp 0 the entry, warp 1 the
// key. The ring holds token t in slot t mod W (W = 2m with overlap, else m).

template <int D>
__device__ __forceinline__ bool append_window(int b, int lane, int p, int m, int overlap,
                                              const uint16_t* __restrict__ cin, const uint16_t* __restrict__ zin,
                                              const uint16_t* __restrict__ bias, uint16_t* __restrict__ ring_c,
                                              uint16_t* __restrict__ ring_z, int& entry, float (&res)[8]) {
  const int W = overlap ? 2 * m : m;
  const uint4* c_new = reinterpret_cast<const uint4*>(cin + (size_t)b * D);
  const uint4* z_new = reinterpret_cast<const uint4*>(zin + (size_t)b * D);
  uint16_t* rc = ring_c + (size_t)b * W * D;
  uint16_t* rz = ring_z + (size_t)b * W * D;
  const bool completes = (p + 1) % m == 0;
  if (completes) {
    const int i = (p + 1) / m - 1;
    auto fetch = [&](int s, int chunk, uint4& cv, uint4& zv) {
      const int t = overlap ? (i - 1) * m + s : i * m + s;
      if (t == p) {   // the new token itself
        cv = __ldg(c_new + chunk);
        zv = __ldg(z_new + chunk);
      } else {        // an earlier token, from its ring slot
        const int slot = t % W;
        cv = __ldg(reinterpret_cast<const uint4*>(rc + (size_t)slot * D) + chunk);
        zv = __ldg(reinterpret_cast<const uint4*>(rz + (size_t)slot * D) + chunk);
      }
    };
    window_entry<D>(W, overlap && i == 0 ? m : 0, bias, lane, fetch, res);
    entry = i;
  }
  // the new token into its slot (it held token p - W, outside every window read here)
  if (lane < D / 8) {
    reinterpret_cast<uint4*>(rc + (size_t)(p % W) * D)[lane] = __ldg(c_new + lane);
    reinterpret_cast<uint4*>(rz + (size_t)(p % W) * D)[lane] = __ldg(z_new + lane);
  }
  return completes;
}

__global__ void __launch_bounds__(64) decode_append_kernel(
    const uint16_t* __restrict__ c, const uint16_t* __restrict__ z, const uint16_t* __restrict__ kc,
    const uint16_t* __restrict__ kz, const uint16_t* __restrict__ bias, const uint16_t* __restrict__ kbias,
    const int32_t* __restrict__ pos, int m, int overlap, uint16_t* __restrict__ ring_c,
    uint16_t* __restrict__ ring_z, uint16_t* __restrict__ ring_kc, uint16_t* __restrict__ ring_kz,
    uint8_t* __restrict__ nope, uint16_t* __restrict__ rope, float* __restrict__ kv_scale,
    uint16_t* __restrict__ k_idx, int n_max, int32_t* __restrict__ n_entries) {
  __shared__ uint4 row_s[kD / 8];
  const int b = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int p = pos[b];
  if (p < 0) return;   // no new token for this sequence (uniform over the block)
  float res[8];
  int i = -1;
  if (warp == 0) {
    if (append_window<kD>(b, lane, p, m, overlap, c, z, bias, ring_c, ring_z, i, res) && i < n_max) {
      if (lane < kD / 8) row_s[lane] = pack_entry_chunk(res);
      __syncwarp();
      const uint32_t* row = reinterpret_cast<const uint32_t*>(row_s);
      const size_t e = (size_t)b * n_max + i;
      quantize_row(row[lane], row[32 + lane], lane, nope + e * kNope, rope + e * kRope, kv_scale + e);
      if (lane == 0) n_entries[b] = i + 1;
    }
  } else if (kc != nullptr) {
    if (append_window<kDI>(b, lane, p, m, overlap, kc, kz, kbias, ring_kc, ring_kz, i, res) && i < n_max &&
        lane < kDI / 8)
      reinterpret_cast<uint4*>(k_idx + ((size_t)b * n_max + i) * kDI)[lane] = pack_entry_chunk(res);
  }
}

cslc_status launch_decode_append(const uint16_t* c, const uint16_t* z, const uint16_t* kc, const uint16_t* kz,
                                 const uint16_t* bias, const uint16_t* kbias, const int32_t* pos, int B, int m,
                                 int overlap, uint16_t* ring_c, uint16_t* ring_z, uint16_t* ring_kc,
                                 uint16_t* ring_kz, uint8_t* nope, uint16_t* rope, float* kv_scale,
                                 uint16_t* k_idx, int n_max, int32_t* n_entries, cudaStream_t stream) {
  if (B == 0) return CSLC_OK;
  decode_append_kernel<<<B, 64, 0, stream>>>(c, z, kc, kz, bias, kbias, pos, m, overlap, ring_c, ring_z, ring_kc,
                                             ring_kz, nope, rope, kv_scale, k_idx, n_max, n_entries);
  return check_launch("decode_append_kernel");
}

}  // namespace cslc
