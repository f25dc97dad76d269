// grouped.cu -- nslm_seed_grouped_gemm (tensor-core batched path).
#include "common.cuh"

extern "C" int32_t nslm_seed_grouped_gemm(const nslm_seed_matrix *W, int32_t E,
                                          const uint16_t *x_bf16, const int32_t *offsets,
                                          int32_t R, float *y, void *ws, size_t ws_bytes,
                                          nslm_stream_t stream) {
  (void)W; (void)E; (void)x_bf16; (void)offsets; (void)R; (void)y; (void)ws; (void)ws_bytes;
  (void)stream;
  nslm::g_launches = 0;
  return NSLM_ERR_UNSUPPORTED;
}
