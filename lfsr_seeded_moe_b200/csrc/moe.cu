// moe.cu -- routed MoE expert FFN on seed-packed experts, decode path (T <= 8).
//
// "NanoSeedLM: LLM inference using pseudo-random numbers", "Why K2-Horizon-MoVA":
// 100 routed FFN experts per layer, top 8; each expert is gate and up
// projections, SiLU, and a down projection, and the layer output is the
// routing-weighted sum.  Weights are regenerated inside the kernels
// ("What I changed: September 2026": never decompressed).
//
// Launch sequence of one layer:
//   1. route_plan_kernel   top-k + softmax (or the caller's ids/w), then the
//                          routed (token, slot) pairs grouped by expert
//   2. ffn_gate_up_kernel  per (expert, row group): g = Gate x, u = Up x for
//                          every token routed to the expert, h = SiLU(g) * u
//   3. ffn_down_kernel     per (output row group, group of experts):
//                          y[t] += w * Down h over the group's experts; the
//                          last CTA of a row group adds the groups' partial
//                          sums in a fixed order (deterministic, no float
//                          atomics)
// For a stack of layers the routing of all layers is one launch (the logits
// are inputs), and layer l+1's gate/up kernel normalises layer l's output
// itself (x = bf16(y / sqrt(mean(y^2) + 1e-6))), so a layer is two launches.
#include <algorithm>
#include <cfloat>
#include <climits>

#include "chunk.cuh"
#include "common.cuh"
#include "moe.cuh"

namespace nslm {

// ------------------------------------------------------------------ routing

// Top-k of one token's logits by one warp: k rounds of a warp arg-max
// (ties to the lower expert id), then the softmax of the selected logits.
__device__ void warp_topk(const float *__restrict__ logits, int E, int k, int32_t *ids_out,
                          float *w_out) {
  const int lane = threadIdx.x & 31;
  uint32_t taken = 0;  // bit j: entry j*32 + lane already selected
  float sel[kMaxK];
  int sid[kMaxK];
  for (int q = 0; q < k; ++q) {
    float bv = -FLT_MAX;
    int bi = INT_MAX;
    for (int j = 0; j * 32 + lane < E; ++j) {
      if ((taken >> j) & 1u) continue;
      const int e = j * 32 + lane;
      const float v = logits[e];
      if (bi == INT_MAX || v > bv || (v == bv && e < bi)) { bv = v; bi = e; }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      if (oi != INT_MAX && (bi == INT_MAX || ov > bv || (ov == bv && oi < bi))) { bv = ov; bi = oi; }
    }
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    sel[q] = bv;
    sid[q] = bi;
  }
  float den = 0.f;
  for (int q = 0; q < k; ++q) den += expf(sel[q] - sel[0]);
  if (lane == 0) {
    for (int q = 0; q < k; ++q) {
      ids_out[q] = sid[q];
      w_out[q] = expf(sel[q] - sel[0]) / den;
    }
  }
}

// One CTA per layer.  Either routes from logits [T][E] or takes the caller's
// ids/w [T][k]; then groups the T*k (token, slot) pairs by expert.  Pairs with
// an expert id outside [0, E) are dropped (they contribute nothing).
__global__ void __launch_bounds__(256) route_plan_kernel(const float *__restrict__ logits,
                                                         const int32_t *__restrict__ ids_in,
                                                         const float *__restrict__ w_in, int T,
                                                         int E, int k, SlotPlan *plans,
                                                         int32_t *ids_out, float *w_out,
                                                         int32_t *counters, int n_counters,
                                                         int32_t *sync, int slot_cap,
                                                         uint64_t *tags, int n_tags) {
  const int layer = blockIdx.x;
  if (counters && layer == 0)
    for (int i = threadIdx.x; i < n_counters; i += blockDim.x) counters[i] = 0;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_tags; i += gridDim.x * blockDim.x) tags[i] = 0;
  if (sync && layer == 0 && threadIdx.x < kSyncWords) sync[threadIdx.x] = 0;
  __shared__ int32_t s_ids[kMaxPairs];
  __shared__ float s_w[kMaxPairs];
  const int warp = threadIdx.x >> 5;
  if (logits) {
    for (int t = warp; t < T; t += blockDim.x >> 5)
      warp_topk(logits + ((size_t)layer * T + t) * E, E, k, s_ids + t * k, s_w + t * k);
  } else {
    for (int i = threadIdx.x; i < T * k; i += blockDim.x) {
      s_ids[i] = ids_in[i];
      s_w[i] = w_in[i];
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && ids_out) {
    const int n = T * k;
    for (int i = 0; i < n; ++i) {
      ids_out[(size_t)layer * n + i] = s_ids[i];
      w_out[(size_t)layer * n + i] = s_w[i];
    }
  }
  if (threadIdx.x == 0 && plans) {
    SlotPlan &pl = plans[layer];
    const int n = T * k;
    int order[kMaxPairs];
    int cnt = 0;
    for (int i = 0; i < n; ++i) {
      pl.ids[i] = s_ids[i];
      pl.w[i] = s_w[i];
      if (s_ids[i] < 0 || s_ids[i] >= E) continue;
      // insertion sort by (expert, pair index)
      int j = cnt++;
      while (j > 0 && s_ids[order[j - 1]] > s_ids[i]) { order[j] = order[j - 1]; --j; }
      order[j] = i;
    }
    // a new slot starts at a new expert, or after slot_cap pairs of the same
    // expert (slot_cap <= T: more only if a token lists an expert twice)
    int ns = 0, in_slot = 0;
    for (int i = 0; i < cnt; ++i) {
      if (i == 0 || s_ids[order[i]] != s_ids[order[i - 1]] || in_slot == slot_cap) {
        pl.expert[ns] = s_ids[order[i]];
        pl.start[ns] = i;
        ++ns;
        in_slot = 0;
      }
      ++in_slot;
      pl.pair[i] = order[i];
    }
    pl.start[ns] = cnt;
    pl.n_slots = ns;
    pl.n_pairs = cnt;
  }
}

// The codes stream of row `grow`: P = 4 packs two 4-bit codes per byte, the
// 5-bit P = 3 format 3 code bits per block (3 bytes per 8 blocks); P = 3 has
// none.
template <int P>
__device__ __forceinline__ const uint8_t *codes_row(const uint8_t *codes, size_t grow, int nb) {
  return P == 4 ? codes + grow * (nb / 2) : (P == kP3C5 ? codes + grow * (3 * (size_t)nb / 8) : nullptr);
}

// ------------------------------------------------------------- gate / up

struct GateUpParams {
  nslm_seed_matrix gate, up;
  const SlotPlan *plan;
  const uint16_t *x_bf16;  // [T][hidden], or null to normalise y_prev
  const float *y_prev;     // [T][hidden]
  float *h;                // [T*k][inter], indexed by pair
  int32_t T, k, hidden, inter;
  int32_t R, C, Cpad, G;   // layout over the inter rows of one expert
};

// Dot products of one (slot, row group) for exactly M tokens, then SiLU.
template <int P, int M, bool VEC, int CPAD>
__device__ __forceinline__ void gate_up_body(const GateUpParams &p, const StreamTables *tab,
                                             const float4 *xs4, const float2 *xn2, float *red,
                                             float *s_sum, const int *s_pair, const ChunkFields &fg,
                                             const ChunkFields &fu, uint32_t rowkg, uint32_t rowku,
                                             bool active, int ch, int g) {
  const int cpad = CPAD ? CPAD : p.Cpad;
  const int tid = threadIdx.x, nthr = blockDim.x, nb = p.hidden / 8;
  float ag[M], au[M];
#pragma unroll
  for (int m = 0; m < M; ++m) ag[m] = au[m] = 0.f;
  if (active) chunk_dot2<P, M, VEC, CPAD>(tab, fg, fu, nb, ch, rowkg, rowku, xs4, xn2, cpad, ag, au);
#pragma unroll
  for (int m = 0; m < M; ++m) {
    red[(2 * m) * nthr + tid] = ag[m];
    red[(2 * m + 1) * nthr + tid] = au[m];
  }
  __syncthreads();
  reduce_rows(red, 2 * M, p.R, cpad, p.C, [&](int v, int r2, float sum) { s_sum[v * p.R + r2] = sum; });
  __syncthreads();
  for (int j = tid; j < M * p.R; j += nthr) {
    const int m = j / p.R, r2 = j - m * p.R;
    const int orow = g * p.R + r2;
    if (orow < p.inter) {
      const float gs = s_sum[(2 * m) * p.R + r2], us = s_sum[(2 * m + 1) * p.R + r2];
      if (in_bounds((size_t)s_pair[m], (size_t)p.T * p.k, 10)) p.h[(size_t)s_pair[m] * p.inter + orow] = gs / (1.f + expf(-gs)) * us;
    }
  }
}

// One CTA per (slot, row group): R rows x Cpad chunk slots.  MT is the
// largest token count per slot the instantiation handles (1 or 8).
template <int P, int MT, bool VEC, int CPAD>
__global__ void __launch_bounds__(256) ffn_gate_up_kernel(const GateUpParams p) {
  extern __shared__ float4 smem4[];
  const int cpad = CPAD ? CPAD : p.Cpad;
  StreamTables *tab = reinterpret_cast<StreamTables *>(smem4);
  float4 *xs4 = smem4 + sizeof(StreamTables) / 16;
  float2 *xn2 = reinterpret_cast<float2 *>(xs4 + (size_t)MT * 16 * cpad);
  float *red = reinterpret_cast<float *>(xn2 + (size_t)MT * 8 * cpad);
  __shared__ int s_tok[kMaxPairs];
  __shared__ int s_pair[kMaxPairs];
  __shared__ float scratch[33];
  __shared__ float s_sum[2 * kMaxT * 32];

  const int s = blockIdx.x / p.G, g = blockIdx.x - (blockIdx.x / p.G) * p.G;
  const SlotPlan *pl = p.plan;
  if (s >= pl->n_slots) return;  // uniform over the CTA
  const int tid = threadIdx.x;
  const int e = pl->expert[s];
  const int p0 = pl->start[s], M = min(MT, pl->start[s + 1] - p0);
  const int rr = tid / cpad, ch = tid - rr * cpad;
  const int row = g * p.R + rr;
  const int nb = p.hidden / 8;
  const bool active = row < p.inter && ch < p.C;

  // weight loads first, so their latency overlaps the staging below
  ChunkFields fg, fu;
  uint32_t rowkg = 0, rowku = 0;
  if (active) {
    const size_t grow = (size_t)e * p.inter + row;
    load_chunk<P, VEC>(p.gate.seeds + grow * nb, p.gate.coefs + grow * nb,
                       codes_row<P>(p.gate.codes, grow, nb), nb, ch, fg, grow, (size_t)p.gate.N);
    load_chunk<P, VEC>(p.up.seeds + grow * nb, p.up.coefs + grow * nb,
                       codes_row<P>(p.up.codes, grow, nb), nb, ch, fu, grow, (size_t)p.up.N);
    rowkg = load_bias_key(p.gate, grow);
    rowku = load_bias_key(p.up, grow);
  }
  if (tid < M) {
    const int pr = pl->pair[p0 + tid];
    s_pair[tid] = pr;
    s_tok[tid] = pr / p.k;
  }
  build_stream_tables(tab);
  __syncthreads();
  stage_activations<false>(xs4, xn2, p.x_bf16, p.y_prev, s_tok, M, p.hidden, cpad, scratch);
  __syncthreads();
#define NSLM_GU(MM) gate_up_body<P, MM, VEC, CPAD>(p, tab, xs4, xn2, red, s_sum, s_pair, fg, fu, rowkg, rowku, active, ch, g)
  if (MT == 1) {
    NSLM_GU(1);
  } else {
    switch (M) {
      case 1: NSLM_GU(1); break;
      case 2: NSLM_GU((MT >= 2 ? 2 : 1)); break;
      case 3: NSLM_GU((MT >= 3 ? 3 : 1)); break;
      case 4: NSLM_GU((MT >= 4 ? 4 : 1)); break;
      case 5: NSLM_GU((MT >= 5 ? 5 : 1)); break;
      case 6: NSLM_GU((MT >= 6 ? 6 : 1)); break;
      case 7: NSLM_GU((MT >= 7 ? 7 : 1)); break;
      default: NSLM_GU((MT >= 8 ? 8 : 1)); break;
    }
  }
#undef NSLM_GU
}

// ------------------------------------------------------------------ down

struct DownParams {
  nslm_seed_matrix down;
  const SlotPlan *plan;
  const float *h;       // [T*k][inter] by pair
  float *y;             // [T][hidden]
  float *y_part;        // [NSG][T][hidden] partial sums of the slot groups
  int32_t *counters;    // [G] arrivals per row group (zero between calls)
  int32_t T, k, hidden, inter;
  int32_t R, C, Cpad, G, NSG;
  int32_t pair_cap;     // pairs whose h fit in shared memory at once
};

// acc[t] += w * <Down row chunk, h_pair> for the M pairs of one slot.
template <int P, int M, int MT, bool VEC, int CPAD>
__device__ __forceinline__ void down_slot(const StreamTables *tab, const ChunkFields &f, int nb,
                                          int ch, uint32_t rowk, const float4 *hs4,
                                          const float2 *hn2, int cpad, int v0, const int *tok,
                                          const float *w, float (&acc)[MT]) {
  float tmp[M];
#pragma unroll
  for (int m = 0; m < M; ++m) tmp[m] = 0.f;
  chunk_dot<P, M, VEC, CPAD>(tab, f, nb, ch, rowk, hs4, hn2, cpad, v0, tmp);
#pragma unroll
  for (int m = 0; m < M; ++m) {
    const float v = w[m] * tmp[m];
    if (MT == 1) {
      acc[0] += v;
    } else {
      const int t = tok[m];
#pragma unroll
      for (int u = 0; u < MT; ++u) acc[u] += (t == u) ? v : 0.f;
    }
  }
}

// One CTA per (row group g, slot group sg).  Slots are split evenly over the
// NSG groups; each CTA writes its partial y for its rows, and the last CTA of
// a row group to arrive adds the NSG partials in group order (deterministic).
template <int P, int MT, bool VEC, int CPAD>
__global__ void __launch_bounds__(512) ffn_down_kernel(const DownParams p) {
  extern __shared__ float4 smem4[];
  const int cpad = CPAD ? CPAD : p.Cpad;
  StreamTables *tab = reinterpret_cast<StreamTables *>(smem4);
  float4 *hs4 = smem4 + sizeof(StreamTables) / 16;
  float2 *hn2 = reinterpret_cast<float2 *>(hs4 + (size_t)p.pair_cap * 16 * cpad);
  float *red = reinterpret_cast<float *>(hn2 + (size_t)p.pair_cap * 8 * cpad);
  __shared__ int s_pair[kMaxPairs];
  __shared__ int s_tok[kMaxPairs];
  __shared__ float s_w[kMaxPairs];
  __shared__ int s_last;

  const SlotPlan *pl = p.plan;
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int g = blockIdx.x / p.NSG, sg = blockIdx.x - (blockIdx.x / p.NSG) * p.NSG;
  const int nslots = pl->n_slots;
  const int per = (nslots + p.NSG - 1) / p.NSG;
  const int s0 = min(nslots, sg * per), s1 = min(nslots, s0 + per);
  const int q0 = pl->start[s0], q1 = pl->start[s1];  // this group's pairs
  const int npairs = q1 - q0;
  const bool stage_all = npairs <= p.pair_cap;
  for (int i = tid; i < npairs; i += nthr) {
    const int pr = pl->pair[q0 + i];
    s_pair[i] = pr;
    s_tok[i] = pr / p.k;
    s_w[i] = pl->w[pr];
  }
  const int rr = tid / cpad, ch = tid - rr * cpad;
  const int row = g * p.R + rr;
  const int nb = p.inter / 8;
  const bool active = row < p.hidden && ch < p.C;

  ChunkFields f;
  uint32_t rowk = 0;
  if (active && s0 < s1) {
    const size_t grow = (size_t)pl->expert[s0] * p.hidden + row;
    load_chunk<P, VEC>(p.down.seeds + grow * nb, p.down.coefs + grow * nb,
                       codes_row<P>(p.down.codes, grow, nb), nb, ch, f, grow, (size_t)p.down.N);
    rowk = load_bias_key(p.down, grow);
  }
  build_stream_tables(tab);
  __syncthreads();
  if (stage_all) stage_f32(hs4, hn2, p.h, s_pair, npairs, p.inter, cpad);
  __syncthreads();

  float acc[MT];
#pragma unroll
  for (int t = 0; t < MT; ++t) acc[t] = 0.f;
  for (int s = s0; s < s1; ++s) {
    const int a0 = pl->start[s] - q0, M = min(MT, pl->start[s + 1] - pl->start[s]);
    if (!stage_all) {
      __syncthreads();
      stage_f32(hs4, hn2, p.h, s_pair + a0, M, p.inter, cpad);
      __syncthreads();
    }
    // prefetch the next slot's chunk while this one is computed
    ChunkFields fn;
    uint32_t rowkn = 0;
    if (active && s + 1 < s1) {
      const size_t grow = (size_t)pl->expert[s + 1] * p.hidden + row;
      load_chunk<P, VEC>(p.down.seeds + grow * nb, p.down.coefs + grow * nb,
                         codes_row<P>(p.down.codes, grow, nb), nb, ch, fn, grow, (size_t)p.down.N);
      rowkn = load_bias_key(p.down, grow);
    }
    if (active) {
      const int v0 = stage_all ? a0 : 0;
#define NSLM_DS(MM) down_slot<P, MM, MT, VEC, CPAD>(tab, f, nb, ch, rowk, hs4, hn2, cpad, v0, s_tok + a0, s_w + a0, acc)
      if (MT == 1) {
        NSLM_DS(1);
      } else {
        switch (M) {
          case 1: NSLM_DS(1); break;
          case 2: NSLM_DS((MT >= 2 ? 2 : 1)); break;
          case 3: NSLM_DS((MT >= 3 ? 3 : 1)); break;
          case 4: NSLM_DS((MT >= 4 ? 4 : 1)); break;
          case 5: NSLM_DS((MT >= 5 ? 5 : 1)); break;
          case 6: NSLM_DS((MT >= 6 ? 6 : 1)); break;
          case 7: NSLM_DS((MT >= 7 ? 7 : 1)); break;
          default: NSLM_DS((MT >= 8 ? 8 : 1)); break;
        }
      }
#undef NSLM_DS
    }
    f = fn;
    rowk = rowkn;
  }
  __syncthreads();
#pragma unroll
  for (int t = 0; t < MT; ++t) red[t * nthr + tid] = acc[t];
  __syncthreads();
  float *part = p.y_part + (size_t)sg * p.T * p.hidden;
  reduce_rows(red, p.T, p.R, cpad, p.C, [&](int t, int r2, float sum) {
    const int orow = g * p.R + r2;
    if (orow < p.hidden) __stcg(part + (size_t)t * p.hidden + orow, sum);
  });
  // last CTA of this row group adds the partials of all slot groups
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int old = atomicAdd(p.counters + g, 1);
    s_last = (old == p.NSG - 1);
    if (s_last) p.counters[g] = 0;  // ready for the next call
  }
  __syncthreads();
  if (s_last) {
    __threadfence();
    for (int j = tid; j < p.T * p.R; j += nthr) {
      const int t = j / p.R, r2 = j - t * p.R;
      const int orow = g * p.R + r2;
      if (orow >= p.hidden) continue;
      float sum = 0.f;
      for (int q = 0; q < p.NSG; ++q) sum += __ldcg(p.y_part + ((size_t)q * p.T + t) * p.hidden + orow);
      p.y[(size_t)t * p.hidden + orow] = sum;
    }
  }
}

// ------------------------------------------------------------------ host

constexpr int kSlotGroups = 4;

static size_t round256(size_t n) { return (n + 255) / 256 * 256; }

int32_t check_ffn_shapes(const nslm_seed_matrix *gate, const nslm_seed_matrix *up,
                         const nslm_seed_matrix *down, int32_t E, FfnDims &d) {
  int32_t st;
  if ((st = check_matrix(gate)) || (st = check_matrix(up)) || (st = check_matrix(down))) return st;
  // one format for the whole layer
  if (gate->P != up->P || gate->P != down->P) return NSLM_ERR_SHAPE;
  if (E <= 0) return NSLM_ERR_ARG;
  if (gate->N % E != 0) return NSLM_ERR_SHAPE;
  d.E = E;
  d.hidden = gate->K;
  d.inter = gate->N / E;
  d.P = gate->P;
  if (up->N != gate->N || up->K != gate->K || up->P != d.P) return NSLM_ERR_SHAPE;
  if (down->N != E * d.hidden || down->K != d.inter || down->P != d.P) return NSLM_ERR_SHAPE;
  if (d.hidden % 8 || d.inter % 8) return NSLM_ERR_SHAPE;
  return NSLM_OK;
}

FfnWorkspace ffn_workspace(char *base, int T, int k, int hidden, int inter, int L) {
  FfnWorkspace w{};
  size_t off = 0;
  w.sync = reinterpret_cast<int32_t *>(base ? base + off : nullptr);
  off += 256;
  w.rms_part = reinterpret_cast<float *>(base ? base + off : nullptr);
  off += round256((size_t)T * kMaxNormParts * sizeof(float));
  w.plans = reinterpret_cast<SlotPlan *>(base ? base + off : nullptr);
  off += round256((size_t)std::max(L, 1) * kPlanBytes);
  w.counters = reinterpret_cast<int32_t *>(base ? base + off : nullptr);
  off += round256((size_t)hidden * sizeof(int32_t));
  w.h = reinterpret_cast<float *>(base ? base + off : nullptr);
  off += round256((size_t)T * k * inter * sizeof(float));
  w.y_part = reinterpret_cast<float *>(base ? base + off : nullptr);
  off += round256((size_t)kSlotGroups * T * hidden * sizeof(float));
  w.y_mid = reinterpret_cast<float *>(base ? base + off : nullptr);
  off += round256((size_t)T * hidden * sizeof(float));
  w.ytag = reinterpret_cast<uint64_t *>(base ? base + off : nullptr);
  w.n_ytag = hidden + kMaxNormParts;
  off += round256((size_t)w.n_ytag * sizeof(uint64_t));
  w.bytes = off;
  return w;
}

template <typename Kern, typename Params>
static int32_t launch_k(Kern kern, const Params &p, int grid, int threads, size_t smem,
                        cudaStream_t s) {
  if (int32_t st = ensure_smem((const void *)kern, smem)) return st;
  ensure_stream_source(s);
  kern<<<grid, threads, smem, s>>>(p);
  return launch_status();
}

template <int P, int MT>
static int32_t launch_decode_layer_t(const FfnDims &d, const nslm_seed_matrix *gate,
                                     const nslm_seed_matrix *up, const nslm_seed_matrix *down,
                                     const SlotPlan *plan, const uint16_t *x_bf16,
                                     const float *y_prev, int T, int k, const FfnWorkspace &w,
                                     float *y, cudaStream_t s, int &launches) {
  const int sms = num_sms();
  {  // gate/up + SiLU: one CTA per (slot, row group)
    ChunkLayout L = chunk_layout(d.hidden, d.inter, 2 * sms, 128);
    GateUpParams p{};
    p.gate = *gate; p.up = *up; p.plan = plan; p.x_bf16 = x_bf16; p.y_prev = y_prev; p.h = w.h;
    p.T = T; p.k = k; p.hidden = d.hidden; p.inter = d.inter;
    p.R = L.R; p.C = L.C; p.Cpad = L.Cpad; p.G = ceil_div(d.inter, L.R);
    if (L.threads > 256 || L.R > 32) return NSLM_ERR_SHAPE;
    const size_t smem = sizeof(StreamTables) + staged_bytes(MT, L.Cpad) +
                        (size_t)2 * MT * L.threads * sizeof(float);
    if (smem > 200 * 1024) return NSLM_ERR_SHAPE;
    const bool vec = (d.hidden % 64 == 0);
    const int grid = T * k * p.G;
    int32_t st;
    if (vec && L.Cpad == 32) st = launch_k(ffn_gate_up_kernel<P, MT, true, 32>, p, grid, L.threads, smem, s);
    else if (vec) st = launch_k(ffn_gate_up_kernel<P, MT, true, 0>, p, grid, L.threads, smem, s);
    else st = launch_k(ffn_gate_up_kernel<P, MT, false, 0>, p, grid, L.threads, smem, s);
    if (st) return st;
    ++launches;
  }
  {  // down + weighted combine: one CTA per (row group, slot group)
    ChunkLayout L = chunk_layout(d.inter, d.hidden, sms, 512);
    DownParams p{};
    p.down = *down; p.plan = plan; p.h = w.h; p.y = y; p.y_part = w.y_part; p.counters = w.counters;
    p.T = T; p.k = k; p.hidden = d.hidden; p.inter = d.inter;
    p.R = L.R; p.C = L.C; p.Cpad = L.Cpad; p.G = ceil_div(d.hidden, L.R); p.NSG = kSlotGroups;
    // a slot group holds at most ceil(T*k / NSG) slots of at most T pairs
    const int group_pairs = std::min(T * k, ceil_div(T * k, kSlotGroups) * T);
    const size_t vec_bytes = staged_bytes(1, L.Cpad);
    const int fit = (int)((64 * 1024) / vec_bytes);
    p.pair_cap = std::max(MT, std::min(group_pairs, fit));
    const size_t smem = sizeof(StreamTables) + staged_bytes(p.pair_cap, L.Cpad) +
                        (size_t)MT * L.threads * sizeof(float);
    if (smem > 200 * 1024 || L.R > 32) return NSLM_ERR_SHAPE;
    const bool vec = (d.inter % 64 == 0);
    const int grid = p.G * p.NSG;
    int32_t st;
    if (vec && L.Cpad == 24) st = launch_k(ffn_down_kernel<P, MT, true, 24>, p, grid, L.threads, smem, s);
    else if (vec) st = launch_k(ffn_down_kernel<P, MT, true, 0>, p, grid, L.threads, smem, s);
    else st = launch_k(ffn_down_kernel<P, MT, false, 0>, p, grid, L.threads, smem, s);
    if (st) return st;
    ++launches;
  }
  return NSLM_OK;
}

int32_t launch_decode_layer(const FfnDims &d, const nslm_seed_matrix *gate,
                            const nslm_seed_matrix *up, const nslm_seed_matrix *down,
                            const SlotPlan *plan, const uint16_t *x_bf16, const float *y_prev,
                            int T, int k, const FfnWorkspace &w, float *y, cudaStream_t s,
                            int &launches) {
  if (d.P == 4) {
    return T == 1 ? launch_decode_layer_t<4, 1>(d, gate, up, down, plan, x_bf16, y_prev, T, k, w, y, s, launches)
                  : launch_decode_layer_t<4, 8>(d, gate, up, down, plan, x_bf16, y_prev, T, k, w, y, s, launches);
  }
  if (d.P == kP3C5) {
    return T == 1 ? launch_decode_layer_t<kP3C5, 1>(d, gate, up, down, plan, x_bf16, y_prev, T, k, w, y, s, launches)
                  : launch_decode_layer_t<kP3C5, 8>(d, gate, up, down, plan, x_bf16, y_prev, T, k, w, y, s, launches);
  }
  return T == 1 ? launch_decode_layer_t<3, 1>(d, gate, up, down, plan, x_bf16, y_prev, T, k, w, y, s, launches)
                : launch_decode_layer_t<3, 8>(d, gate, up, down, plan, x_bf16, y_prev, T, k, w, y, s, launches);
}

int32_t launch_route_plan(const float *logits, const int32_t *ids, const float *w, int T, int E,
                          int k, int L, SlotPlan *plans, int32_t *ids_out, float *w_out,
                          int32_t *counters, int n_counters, int32_t *sync, int slot_cap,
                          uint64_t *tags, int n_tags, cudaStream_t s) {
  route_plan_kernel<<<L, 256, 0, s>>>(logits, ids, w, T, E, k, plans, ids_out, w_out, counters,
                                      n_counters, sync, std::max(1, std::min(slot_cap, T)), tags,
                                      tags ? n_tags : 0);
  return launch_status();
}

NSLM_BOUNDS_ACCESSOR(moe)

}  // namespace nslm
