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
  const int chunk = lane & 15;
  const int split = lane >> 4;

  // Window: slots 0..W-1. CSA: slot s < m is token (i-1)m + s (C^b), slot
  // s >= m is token i*m + s - m (C^a). HCA: slot s is token i*m + s.
  const int W = overlap ? 2 * m : m;
  const int half = (W + 1) >> 1;
  int s_lo = split * half, s_hi = min(W, s_lo + half);
  if (overlap && i == 0) s_lo = max(s_lo, m);   // entry 0 has no C^b half

  SoftmaxAcc st;
  acc_init(st);
  const size_t row0 = (size_t)b * L;
  for (int s = s_lo; s < s_hi; ++s) {
    const bool prev = overlap && s < m;
    const int t = overlap ? (i - 1) * m + s : i * m + s;
    const uint16_t* cs = prev ? cb : c;
    const uint16_t* zs = prev ? zb : z;
    const uint4 cv = __ldg(reinterpret_cast<const uint4*>(cs + (row0 + t) * kD) + chunk);
    const uint4 zv = __ldg(reinterpret_cast<const uint4*>(zs + (row0 + t) * kD) + chunk);
    const uint4 bv = __ldg(reinterpret_cast<const uint4*>(bias + (size_t)s * kD) + chunk);
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
  float res[8];
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
  if (split == 0) {
    uint4 o;
    o.x = pack_bf16x2(res[0], res[1]);
    o.y = pack_bf16x2(res[2], res[3]);
    o.z = pack_bf16x2(res[4], res[5]);
    o.w = pack_bf16x2(res[6], res[7]);
    reinterpret_cast<uint4*>(out + ((size_t)b * n_c + i) * kD)[chunk] = o;
  }
}

cslc_status launch_compress(const uint16_t* c, const uint16_t* z, const uint16_t* cb,
                            const uint16_t* zb, const uint16_t* bias, int B, int L, int m,
                            int overlap, uint16_t* out, cudaStream_t stream) {
  const int n_c = L / m;
  const long long warps = (long long)B * n_c;
  if (warps == 0) return CSLC_OK;
  const int threads = 256;
  const long long blocks = (warps * 32 + threads - 1) / threads;
  compress_kernel<<<(unsigned)blocks, threads, 0, stream>>>(c, z, cb ? cb : c, zb ? zb : z, bias,
                                                            B, L, m, overlap, n_c, out);
  return check_launch("compress_kernel");
}

// ---------------------------------------------------------------------------
// Mixed decode KV layout (first page §1.4 存储格式混): dims 0..63 as e4m3 with
// one fp32 scale per entry, dims 64..127 kept bf16. One warp per entry; lane l
// owns dims 2l, 2l+1 of each half.

__global__ void __launch_bounds__(256) quantize_kv_kernel(const uint16_t* __restrict__ kv,
                                                          long long n_entries,
                                                          uint8_t* __restrict__ nope,
                                                          uint16_t* __restrict__ rope,
                                                          float* __restrict__ scale) {
  const long long e = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (e >= n_entries) return;
  const uint32_t* row = reinterpret_cast<const uint32_t*>(kv + e * kD);
  const uint32_t lo = row[lane];        // dims 2l, 2l+1
  const uint32_t hi = row[32 + lane];   // dims 64+2l, 64+2l+1
  const float x0 = bf16_lo(lo), x1 = bf16_hi(lo);
  const float amax = warp_max(fmaxf(fabsf(x0), fabsf(x1)));
  const float s = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  const float2 q = make_float2(__fdiv_rn(x0, s), __fdiv_rn(x1, s));
  const __nv_fp8x2_storage_t codes = __nv_cvt_float2_to_fp8x2(q, __NV_SATFINITE, __NV_E4M3);
  reinterpret_cast<uint16_t*>(nope + e * kNope)[lane] = codes;
  reinterpret_cast<uint32_t*>(rope + e * kRope)[lane] = hi;
  if (lane == 0) scale[e] = s;
}

cslc_status launch_quantize_kv(const uint16_t* kv, long long n, uint8_t* nope, uint16_t* rope,
                               float* scale, cudaStream_t stream) {
  if (n == 0) return CSLC_OK;
  const long long blocks = (n * 32 + 255) / 256;
  quantize_kv_kernel<<<(unsigned)blocks, 256, 0, stream>>>(kv, n, nope, rope, scale);
  return check_launch("quantize_kv_kernel");
}

}  // namespace cslc
