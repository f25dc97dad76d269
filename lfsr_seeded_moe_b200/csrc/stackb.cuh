// stackb.cuh -- the decode stack for 2..8 tokens as one persistent
// cooperative kernel (internal).
#pragma once
#include "moe.cuh"

namespace nslm {

constexpr int kStackBThreads = 512;  // 16 warps, up to 128 registers each: one CTA per SM
constexpr int kSlotTokens = 4;       // pairs per slot in the plans this kernel takes

// Whether the kernel takes this shape (64-weight chunks, shared memory,
// index ranges) for T tokens of k experts each.
bool stackb_supported(const FfnDims &d, int T, int k);

// Layers l0 .. l0+n-1 of a T-token stack (2 <= T <= 8) in cooperative
// launches of up to kMaxFusedLayers layers: x0 (bf16 [T][hidden], or null
// when y_in holds the fp32 output of layer l0-1 from this kernel) -> y_out
// [T][hidden].  plans[l] were made with at most kSlotTokens pairs per slot;
// sync[] was zeroed after the last use; rms_part holds [T][grid] per-CTA
// sums of squares of y between layers.
int32_t launch_stackb(const FfnDims &d, const nslm_moe_layer *layers, int n, const SlotPlan *plans,
                      const uint16_t *x0, const float *y_in, int T, int k, float *h, float *y_mid,
                      float *y_out, int32_t *sync, float *rms_part, cudaStream_t s, int &launches);

// Slots per expert group that the routing plan must use for T tokens: the
// persistent T > 1 kernel takes at most kSlotTokens pairs per slot.
int decode_slot_cap(const FfnDims &d, int T, int k);

// The decode path for L layers of T <= 8 tokens once the plans are made: the
// one-token or the T-token persistent kernel where the shape allows, else two
// launches per layer.
int32_t launch_decode_stack(const FfnDims &d, const nslm_moe_layer *layers, int L, const uint16_t *x0,
                            int T, int k, const FfnWorkspace &fw, float *y, cudaStream_t s, int &launches);

}  // namespace nslm
