// hybrid.cu -- a MoE layer whose experts are packed with different P
// ("NanoSeedLM: LLM inference using pseudo-random numbers" news list: hybrid
// P3 / P4 seed packs, about 4.17 bits per weight, where each expert is packed
// with P = 3 or with P = 4).
//
// Experts 0 .. E3-1 are the P = 3 stack and E3 .. E3+E4-1 the P = 4 stack.  A
// small kernel splits the routed ids into each stack's ids (pairs of the other
// stack dropped), the routed FFN runs once per stack with the layer's usual
// kernels (the P = 3 output into the workspace, the P = 4 output into y), and
// a last kernel adds the two in a fixed order.  The device status word at
// the head of the shared workspace is copied aside after the P = 3 stack (the
// P = 4 stack's routing kernel resets it) and merged back by the last kernel,
// so that a wait that gave up in either stack is reported.
#include <algorithm>

#include "common.cuh"
#include "moe.cuh"

namespace nslm {
namespace {

__global__ void hybrid_split_kernel(const int32_t *ids, int n, int E3, int E4, int32_t *ids3, int32_t *ids4) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const int e = ids[i];
    ids3[i] = (e >= 0 && e < E3) ? e : -1;
    ids4[i] = (e >= E3 && e < E3 + E4) ? e - E3 : -1;
  }
}

__global__ void hybrid_add_kernel(float *y, const float *y3, int64_t n, int32_t *status,
                                  const int32_t *status3) {
  if (blockIdx.x == 0 && threadIdx.x == 0 && *status3 != 0) *status = *status3;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    y[i] = y[i] + y3[i];
}

size_t round256(size_t n) { return (n + 255) / 256 * 256; }

}  // namespace

size_t hybrid_extra_bytes(int T, int k, int hidden) {
  return 2 * round256((size_t)T * k * sizeof(int32_t)) + round256((size_t)T * hidden * sizeof(float)) +
         round256(sizeof(int32_t));
}

}  // namespace nslm

using namespace nslm;

extern "C" int32_t nslm_moe_seed_ffn_hybrid(const nslm_moe_layer *p3, int32_t E3, const nslm_moe_layer *p4,
                                            int32_t E4, const uint16_t *x_bf16, const int32_t *ids,
                                            const float *w, int32_t T, int32_t k, float *y, void *ws,
                                            size_t ws_bytes, nslm_stream_t stream) {
  g_launches = 0;
  if (!p3 || !p4 || !x_bf16 || !ids || !w || !y) return NSLM_ERR_ARG;
  if (E3 < 1 || E4 < 1 || k < 1 || k > kMaxK || T < 0) return NSLM_ERR_SHAPE;
  FfnDims d3{}, d4{};
  int32_t st = check_ffn_shapes(&p3->gate, &p3->up, &p3->down, E3, d3);
  if (st) return st;
  if ((st = check_ffn_shapes(&p4->gate, &p4->up, &p4->down, E4, d4))) return st;
  if (d3.P != 3 || d4.P != 4 || d3.hidden != d4.hidden || d3.inter != d4.inter) return NSLM_ERR_SHAPE;
  if (T == 0) return NSLM_OK;
  const size_t need = nslm_workspace_bytes(NSLM_OP_MOE_FFN_HYBRID, T, E3 + E4, d3.hidden, d3.inter, k, 0);
  if (!ws || ws_bytes < need) return NSLM_ERR_WORKSPACE;
  if (!aligned16(ws) || !aligned16(y) || !aligned16(x_bf16)) return NSLM_ERR_ALIGN;
  if ((st = check_device())) return st;
  // workspace: [the FFN's workspace (sized for E3 + E4 experts, enough for
  // either stack)][ids3 [T][k]][ids4 [T][k]][y3 [T][hidden]][status of the P = 3 stack]
  const size_t ffn_bytes = nslm_workspace_bytes(NSLM_OP_MOE_FFN, T, E3 + E4, d3.hidden, d3.inter, k, 0);
  const size_t ids_bytes = round256((size_t)T * k * sizeof(int32_t));
  char *base = static_cast<char *>(ws);
  int32_t *ids3 = reinterpret_cast<int32_t *>(base + ffn_bytes);
  int32_t *ids4 = reinterpret_cast<int32_t *>(base + ffn_bytes + ids_bytes);
  float *y3 = reinterpret_cast<float *>(base + ffn_bytes + 2 * ids_bytes);
  int32_t *status3 = reinterpret_cast<int32_t *>(base + ffn_bytes + 2 * ids_bytes +
                                                 round256((size_t)T * d3.hidden * sizeof(float)));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int n = T * k;
  hybrid_split_kernel<<<(n + 255) / 256, 256, 0, s>>>(ids, n, E3, E4, ids3, ids4);
  if ((st = launch_status())) return st;
  int launches = 1;
  // the two stacks one after the other on the stream, sharing the FFN workspace
  if ((st = nslm_moe_seed_ffn(&p3->gate, &p3->up, &p3->down, E3, x_bf16, ids3, w, T, k, y3, ws, ffn_bytes, stream)))
    return st;
  launches += nslm_last_launch_count();
  if ((st = cuda_status(cudaMemcpyAsync(status3, ws, sizeof(int32_t), cudaMemcpyDeviceToDevice, s)))) return st;
  if ((st = nslm_moe_seed_ffn(&p4->gate, &p4->up, &p4->down, E4, x_bf16, ids4, w, T, k, y, ws, ffn_bytes, stream)))
    return st;
  launches += nslm_last_launch_count();
  const int64_t ny = (int64_t)T * d3.hidden;
  hybrid_add_kernel<<<(int)std::min<int64_t>((ny + 255) / 256, 4 * num_sms()), 256, 0, s>>>(y, y3, ny, static_cast<int32_t *>(ws), status3);
  if ((st = launch_status())) return st;
  g_launches = launches + 1;
  return NSLM_OK;
}
