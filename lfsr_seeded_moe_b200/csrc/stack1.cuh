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

// Layers l0 .. l0+n-1 of a one-token stack in one cooperative launch:
// x0 (bf16, may be null when y_in holds the fp32 output of layer l0-1) ->
// y_out.  plans[l] are complete; sync[] was zeroed after the last use.
// rms_part [kMaxStack1Ctas] holds per-CTA sums of squares of y between
// layers (when y_in is given it must come from the same kernel).
int32_t launch_stack1(const FfnDims &d, const nslm_moe_layer *layers, int n, const SlotPlan *plans,
                      const uint16_t *x0, const float *y_in, int k, float *h, float *y_mid,
                      float *y_out, int32_t *sync, float *rms_part, cudaStream_t s, int &launches);

}  // namespace nslm
