// decode1.cuh -- the one-token decode layer with persistent warps (internal).
#pragma once
#include "moe.cuh"

namespace nslm {

constexpr int kGateUp1Threads = 256;
constexpr int kGateUp1MaxCtasPerSm = 4;
// whole-chunk weight fields land in shared memory one step ahead (cp.async)
constexpr bool kAsyncFields = true;
constexpr int kDown1Threads = 512;
constexpr int kDown1CtasPerSm = 1;

size_t gate_up1_smem(const FfnDims &d);
size_t down1_smem(const FfnDims &d, int k);
// Shapes the one-token kernels take (index arithmetic and shared memory).
bool decode1_supported(const FfnDims &d, int k);

// Gate/up + SiLU, then down + weighted combine, for one token: two launches,
// each allowed to start while the kernel ahead of it drains (it waits for
// that kernel before touching anything the kernel writes or reads).
// h is [k][inter] scratch; y [hidden] is written in full.  plan_early: the
// plan was written two or more kernels back, so it may be read before the
// wait.
int32_t launch_decode1(const FfnDims &d, const nslm_seed_matrix *gate, const nslm_seed_matrix *up,
                       const nslm_seed_matrix *down, const SlotPlan *plan, const uint16_t *x_bf16,
                       const float *y_prev, int k, float *h, float *y, bool plan_early,
                       cudaStream_t s, int &launches);

}  // namespace nslm
