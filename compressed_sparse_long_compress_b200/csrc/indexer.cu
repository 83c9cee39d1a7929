// Lightning-indexer score dispatch ("读完这篇你就搞懂 DeepSeek v4 了", §三 闪电索引):
//   S[t, i] = sum_h w[t, h] * max(0, q_I[t, h, :] . k_I[i, :])
// Every shape runs on the tcgen05 kernel of indexer_sm100.cu (bf16 operands,
// or e4m3 codes with per-row scales); this file only routes the calls.

#include "common.cuh"

namespace cslc {

cslc_status launch_indexer_sm100(const uint16_t* q_idx, const uint16_t* w, const uint16_t* k_idx, int B,
                                 int L, int Nc, int HI, int m, int q_pos0, int row_begin, int row_end,
                                 void* scores, bool bf16_out, int rows_in_buf, cudaStream_t stream);
cslc_status launch_indexer_sm100_fp8(const uint8_t* q8, const float* q_scale, const uint16_t* w, const uint8_t* k8,
                                     const float* k_scale, int B, int L, int Nc, int HI, int m, int q_pos0,
                                     int row_begin, int row_end, float* scores, int rows_in_buf, cudaStream_t stream);

// e4m3 operands: fp32 scores [B][rows_in_buf][Nc] of rows [row_begin, row_end)
cslc_status launch_indexer_scores_fp8(const uint8_t* q8, const float* q_scale, const uint16_t* w, const uint8_t* k8,
                                      const float* k_scale, int B, int L, int Nc, int HI, int m, int q_pos0,
                                      int row_begin, int row_end, float* scores, int rows_in_buf,
                                      cudaStream_t stream) {
  if (row_end <= row_begin || B == 0 || Nc == 0) return CSLC_OK;
  return launch_indexer_sm100_fp8(q8, q_scale, w, k8, k_scale, B, L, Nc, HI, m, q_pos0, row_begin, row_end, scores,
                                  rows_in_buf, stream);
}

// bf16 operands: scores fp32, or bf16 when bf16_out
cslc_status launch_indexer_scores(const uint16_t* q_idx, const uint16_t* w, const uint16_t* k_idx,
                                  int B, int L, int Nc, int HI, int m, int q_pos0, int row_begin,
                                  int row_end, void* scores, bool bf16_out, int rows_in_buf, cudaStream_t stream) {
  if (row_end <= row_begin || B == 0 || Nc == 0) return CSLC_OK;
  return launch_indexer_sm100(q_idx, w, k_idx, B, L, Nc, HI, m, q_pos0, row_begin, row_end, scores, bf16_out,
                              rows_in_buf, stream);
}

}  // namespace cslc
