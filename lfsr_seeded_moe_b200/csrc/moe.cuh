// moe.cuh -- internal declarations of the MoE decode path (not part of the ABI).
#pragma once
#include <cstddef>
#include <cstdint>
#include <algorithm>
#include <cuda_runtime.h>

#include "../../include/nslm.h"

namespace nslm {

constexpr int kMaxT = 8;                 // decode path: at most 8 tokens
constexpr int kMaxK = 8;                 // at most 8 experts per token
constexpr int kMaxPairs = kMaxT * kMaxK;

// One layer's routing grouped by expert.  A slot is one expert together with
// the (token, slot-in-token) pairs routed to it, at most slot_cap <= T pairs
// per slot (an expert with more pairs takes several slots).
struct SlotPlan {
  int32_t n_slots;
  int32_t n_pairs;
  int32_t expert[kMaxPairs];
  int32_t start[kMaxPairs + 1];  // pairs of slot s: pair[start[s] .. start[s+1])
  int32_t pair[kMaxPairs];       // pair index t * k + q, sorted by expert
  int32_t ids[kMaxPairs];        // routed expert ids [T][k]
  float w[kMaxPairs];            // routing weights [T][k]
};
constexpr size_t kPlanBytes = (sizeof(SlotPlan) + 255) / 256 * 256;

struct FfnDims {
  int32_t E, hidden, inter, P;
};

int32_t check_ffn_shapes(const nslm_seed_matrix *gate, const nslm_seed_matrix *up,
                         const nslm_seed_matrix *down, int32_t E, FfnDims &d);

// Workspace of the decode path, carved from the caller's buffer (base may be
// null to size it).  counters must be zero before the first down kernel; the
// routing kernel zeroes them and the down kernel leaves them zero.
// Device status words at the head of the decode workspace: [0] status (0 ok,
// 1 a grid barrier wait gave up), [1] barrier arrivals, [2] abort flag; the
// routing kernel zeroes them at the start of every call.
constexpr int kSyncWords = 4;

constexpr int kMaxNormParts = 1024;

struct FfnWorkspace {
  int32_t *sync;       // [kSyncWords], at offset 0
  float *rms_part;     // [T][kMaxNormParts] per-token, per-CTA sums of y^2 between fused layers
  SlotPlan *plans;     // [L]
  int32_t *counters;   // [hidden]
  float *h;            // [T*k][inter]
  float *y_part;       // [slot groups][T][hidden]
  float *y_mid;        // [T][hidden] (layer stack)
  // one-token layer stack: y rows, then the per-CTA norm partials, between
  // layers as 64-bit words (value bits low, 32-bit layer tag high), zeroed
  // by the routing kernel at the start of every one-token call of two or
  // more layers (a one-layer call does not read them)
  uint64_t *ytag;      // [hidden + kMaxNormParts]
  int32_t n_ytag;
  size_t bytes;
};
FfnWorkspace ffn_workspace(char *base, int T, int k, int hidden, int inter, int L);

// Workspace a hybrid P3/P4 layer needs beyond the FFN's: two id arrays and
// the P = 3 stack's output.
size_t hybrid_extra_bytes(int T, int k, int hidden);

int32_t launch_route_plan(const float *logits, const int32_t *ids, const float *w, int T, int E,
                          int k, int L, SlotPlan *plans, int32_t *ids_out, float *w_out,
                          int32_t *counters, int n_counters, int32_t *sync, int slot_cap,
                          uint64_t *tags, int n_tags, cudaStream_t s);
int32_t launch_decode_layer(const FfnDims &d, const nslm_seed_matrix *gate,
                            const nslm_seed_matrix *up, const nslm_seed_matrix *down,
                            const SlotPlan *plan, const uint16_t *x_bf16, const float *y_prev,
                            int T, int k, const FfnWorkspace &w, float *y, cudaStream_t s,
                            int &launches);

}  // namespace nslm
