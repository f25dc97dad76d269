// grouped.cuh -- internal declarations of the tensor-core batched path.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/nslm.h"
#include "moe.cuh"

namespace nslm {

// Workspace of the batched FFN (carved from the caller's buffer; base may be
// null to size it).
struct BatchedPlan {
  int32_t *status;    // 1 if a tensor-core wait timed out
  int32_t *offsets;   // [E + 1] sorted-pair offsets per expert
  int32_t *tiles_gu;  // [E + 1] gate/up tiles before expert e
  int32_t *tiles_dn;  // [E + 1] down tiles before expert e
  int32_t *row_of;    // [T*k] sorted pair -> token
  int32_t *pair_of;   // [T*k] sorted pair -> pair index t*k + q
  uint16_t *h;        // [T*k][inter] bf16 hidden activations, sorted order
  float *part;        // [T*k][hidden] weighted down outputs, by pair
  size_t bytes;
};
BatchedPlan batched_workspace(char *base, int T, int k, int E, int hidden, int inter);

int32_t launch_batched_ffn(const FfnDims &d, const nslm_seed_matrix *gate, const nslm_seed_matrix *up,
                           const nslm_seed_matrix *down, const uint16_t *x_bf16, const int32_t *ids,
                           const float *w, int T, int k, float *y, void *ws, cudaStream_t s,
                           int &launches);

size_t grouped_ws_bytes(int E);

}  // namespace nslm
