// stack1.cuh -- the one-token decode stack as one persistent cooperative
// kernel (internal).
#pragma once
#include "moe.cuh"

namespace nslm {

constexpr int kStack1MaxThreads = 640;  // up to 20 warps (>= 96 registers each): one CTA per SM
constexpr int kMaxFusedLayers = 64;     // layers per launch (kernel parameter space)
constexpr int kMaxStack1Ctas = kMaxNormParts;

// Whether the fused kernel takes this shape (shared memory, index ranges).
bool stack1_supported(const FfnDims &d, int k);

// All n layers of a one-token stack in cooperative launches of up to
// kMaxFusedLayers layers each: x0 (bf16 [hidden]) -> y_out (fp32 [hidden]).
// plans[l] are complete; sync[] and the tagged words ytag
// [hidden + kMaxStack1Ctas] (y rows and per-CTA sums of y^2 between layers)
// were zeroed after their last use, as the routing kernel does.
int32_t launch_stack1(const FfnDims &d, const nslm_moe_layer *layers, int n, const SlotPlan *plans,
                      const uint16_t *x0, int k, float *h, uint64_t *ytag, float *y_out, int32_t *sync,
                      cudaStream_t s, int &launches);

}  // namespace nslm
