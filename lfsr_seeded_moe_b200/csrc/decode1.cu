// decode1.cu -- the one-token decode layer with persistent warps.
//
// "NanoSeedLM: LLM inference using pseudo-random numbers", "Why K2-Horizon-MoVA":
// for one token the layer reads 8 of the 100 experts; each is gate and up
// projections (inter x hidden), SiLU, and a down projection (hidden x inter),
// combined with the routing weights.  The weights are regenerated in
// registers ("What I changed: September 2026"), so the kernels are bound by
// the integer work of regeneration; both kernels below keep every lane on
// that work and pay the per-CTA costs (stream tables, staging) once per SM.
//
//   gate_up1_kernel  persistent warps; a warp task is one row of one routed
//                    expert: lanes take the 64-weight chunks of its gate and
//                    up rows, a shuffle tree sums them, lane 0 writes
//                    h = SiLU(g) * u.  x is staged once per CTA.
//   down1_kernel     a CTA owns a range of output rows and computes them in
//                    full over all routed experts: threads take (row, expert,
//                    chunk) tasks, partials go to shared memory, and a warp
//                    per row adds them in a fixed order (deterministic, no
//                    cross-CTA combine).  The routed h vectors are staged
//                    back to back as one long vector, so the 32 lanes of a
//                    warp read 32 consecutive chunk slots.
#include <algorithm>

#include "chunk.cuh"
#include "common.cuh"
#include "decode1.cuh"

namespace nslm {

// n / d for n < 2^22 and 0 < d < 2^16: m = ceil(2^40 / d), q = (n * m) >> 40
// (exact, since n * (m * d - 2^40) < 2^38 < 2^40 / d * d).
struct FastDiv {
  uint64_t m;
};
static FastDiv make_fastdiv(uint32_t d) { return FastDiv{((1ull << 40) + d - 1) / d}; }
__device__ __forceinline__ uint32_t fdiv(uint32_t n, FastDiv f) {
  return (uint32_t)(((uint64_t)n * f.m) >> 40);
}

// Chunk fields of a row (VEC: whole chunks; else the ragged tail is guarded).
template <int P, bool VEC>
__device__ __forceinline__ void load_row_chunk(const nslm_seed_matrix &W, size_t grow, int nb, int c,
                                               ChunkFields &f, uint32_t &rowk) {
  load_chunk<P, VEC>(W.seeds + grow * nb, W.coefs + grow * nb,
                     P == 4 ? W.codes + grow * (nb / 2) : nullptr, nb, c, f);
  rowk = row_scale_key(__ldg(W.exp_bias + grow));
}

// ------------------------------------------------------------------ gate / up

struct GateUp1Params {
  nslm_seed_matrix gate, up;
  const SlotPlan *plan;
  const uint16_t *x_bf16;  // [1][hidden], or null to normalise y_prev
  const float *y_prev;     // [1][hidden]
  float *h;                // [k][inter] by pair
  int32_t hidden, inter;
  int32_t C;               // chunks per row: ceil(hidden / 64)
  int32_t J;               // chunk rounds per lane: ceil(C / 32)
  int32_t plan_early;      // plan complete before the previous kernel started
  FastDiv div_inter, div_J;
};

template <int P, bool VEC>
__global__ void __launch_bounds__(kGateUp1Threads) gate_up1_kernel(const GateUp1Params p) {
  extern __shared__ float4 smem4[];
  const int tid = threadIdx.x, nthr = blockDim.x;
  StreamTables *tab = reinterpret_cast<StreamTables *>(smem4);
  // x in the chunk-major layout: C slots
  float4 *xs4 = smem4 + sizeof(StreamTables) / 16;
  float2 *xn2 = reinterpret_cast<float2 *>(xs4 + (size_t)kCmX4 * p.C);
  // whole chunks: [2 buffers][gate, up][threads] field slots
  const FieldSlots fs(xn2 + (size_t)kCmXn * p.C + (p.C & 1), 4 * nthr);
  __shared__ float scratch[33];
  __shared__ int s_row0, s_nslots;
  __shared__ int s_expert[kMaxK], s_pair[kMaxK];

  // The routing plan may come from the kernel just before this one; it is
  // then read only once that kernel has completed.
  if (!p.plan_early) grid_dependency_wait();
  const SlotPlan *pl = p.plan;
  if (tid == 0) {
    s_row0 = 0;
    s_nslots = min(pl->n_slots, kMaxK);
  }
  if (tid < kMaxK && tid < pl->n_slots) {
    s_expert[tid] = pl->expert[tid];
    s_pair[tid] = pl->pair[pl->start[tid]];
  }
  build_stream_tables(tab);
  __syncthreads();

  const int lane = tid & 31;
  const int gw = blockIdx.x * (nthr >> 5) + (tid >> 5);
  const int W = gridDim.x * (nthr >> 5);
  const int ntask = s_nslots * p.inter;  // one token: a slot is one pair
  const int mytasks = gw < ntask ? (ntask - 1 - gw) / W + 1 : 0;
  const int nsteps = mytasks * p.J;
  const int nb = p.hidden >> 3;

  // step -> (task, chunk round)
  auto locate = [&](int step, int &slot, int &row, int &c) {
    const int i = p.J == 1 ? step : (int)fdiv(step, p.div_J);
    const int t = gw + i * W;
    slot = (int)fdiv(t, p.div_inter);
    row = t - slot * p.inter;
    c = lane + 32 * (step - i * p.J);
  };
  // whole chunks go through the shared-memory slots one step ahead; ragged
  // rows load straight into registers
  auto fetch = [&](int step, int buf) {
    int slot, row, c;
    locate(step, slot, row, c);
    if (c < p.C) {
      const size_t grow = (size_t)s_expert[slot] * p.inter + row;
      fetch_chunk<P>(p.gate, grow, nb, c, fs, (2 * buf) * nthr + tid);
      fetch_chunk<P>(p.up, grow, nb, c, fs, (2 * buf + 1) * nthr + tid);
    }
  };
  auto load = [&](int step, ChunkFields &fg, ChunkFields &fu, uint32_t &kg, uint32_t &ku) {
    int slot, row, c;
    locate(step, slot, row, c);
    if (c < p.C) {
      const size_t grow = (size_t)s_expert[slot] * p.inter + row;
      load_row_chunk<P, VEC>(p.gate, grow, nb, c, fg, kg);
      load_row_chunk<P, VEC>(p.up, grow, nb, c, fu, ku);
    }
  };

  // the first weight fields (weights and plan are ready) overlap the wait
  ChunkFields fg, fu;
  uint32_t kg = 0, ku = 0;
  if (VEC && kAsyncFields) {
    if (nsteps > 0) fetch(0, 0);
    cp_async_commit();
  } else if (nsteps > 0) {
    load(0, fg, fu, kg, ku);
  }

  // activations (and h, which the previous kernel may still read) only after
  // the previous kernel has completed
  grid_dependency_wait();
  grid_dependents_launch();
  stage_activations<true>(xs4, xn2, p.x_bf16, p.y_prev, &s_row0, 1, p.hidden, p.C, scratch);
  __syncthreads();

  float2 ag = make_float2(0.f, 0.f), au = make_float2(0.f, 0.f);
  for (int step = 0; step < nsteps; ++step) {
    int slot, row, c;
    locate(step, slot, row, c);
    ChunkFields ng, nu;
    uint32_t nkg = 0, nku = 0;
    if (VEC && kAsyncFields) {
      if (step + 1 < nsteps) fetch(step + 1, (step + 1) & 1);
      cp_async_commit();
      cp_async_wait<1>();  // this step's slots have landed
      read_chunk<P>(fs, (2 * (step & 1)) * nthr + tid, fg, kg);
      read_chunk<P>(fs, (2 * (step & 1) + 1) * nthr + tid, fu, ku);
    } else if (step + 1 < nsteps) {
      load(step + 1, ng, nu, nkg, nku);
    }
    if (c < p.C) {
      const int nvalid = VEC ? 8 : min(8, nb - 8 * c);
      chunk_dot2_cm<P, VEC, 1>(tab->t, fg, fu, nvalid, kg, ku, xs4 + kCmX4 * c, xn2 + kCmXn * c, ag, au);
    }
    if (p.J == 1 || c + 32 >= 32 * p.J) {  // last chunk round of the task
      const float g = warp_sum(ag.x + ag.y), u = warp_sum(au.x + au.y);
      if (lane == 0) p.h[(size_t)s_pair[slot] * p.inter + row] = g / (1.f + expf(-g)) * u;
      ag = au = make_float2(0.f, 0.f);
    }
    if (!(VEC && kAsyncFields)) {
      fg = ng;
      fu = nu;
      kg = nkg;
      ku = nku;
    }
  }
}

// ---------------------------------------------------------------------- down

struct Down1Params {
  nslm_seed_matrix down;
  const SlotPlan *plan;
  const float *h;          // [k][inter] by pair
  float *y;                // [1][hidden]
  int32_t hidden, inter;
  int32_t C;               // chunks per row: ceil(inter / 64)
  int32_t rpc;             // output rows per CTA
  FastDiv div_C, div_nb;
  FastDiv div_SC[kMaxK + 1];  // by S * C for S slots
};

template <int P, bool VEC>
__global__ void __launch_bounds__(kDown1Threads) down1_kernel(const Down1Params p) {
  extern __shared__ float4 smem4[];
  // the plan was complete before the gate/up kernel ahead of this one started
  const SlotPlan *pl = p.plan;
  const int S = min(pl->n_slots, kMaxK);
  const int SC = S * p.C;
  const int tid = threadIdx.x, nthr = blockDim.x;
  StreamTables *tab = reinterpret_cast<StreamTables *>(smem4);
  // whole chunks: [2 buffers][threads] field slots
  const FieldSlots fs(smem4 + sizeof(StreamTables) / 16, 2 * nthr);
  // the S routed h vectors back to back: SC slots of the chunk-major layout
  float4 *hs4 = reinterpret_cast<float4 *>(fs.b + 2 * nthr);
  float2 *hn2 = reinterpret_cast<float2 *>(hs4 + (size_t)kCmX4 * SC);
  float *red = reinterpret_cast<float *>(hn2 + (size_t)kCmXn * SC);
  __shared__ float s_w[kMaxK];
  __shared__ int s_expert[kMaxK], s_pair[kMaxK];

  const int n0 = blockIdx.x * p.rpc;
  const int nrows = min(p.rpc, p.hidden - n0);
  const int ntask = nrows * SC;
  const int nb = p.inter >> 3;
  const FastDiv dSC = p.div_SC[S];
  if (tid < S) {
    const int pr = pl->pair[pl->start[tid]];
    s_expert[tid] = pl->expert[tid];
    s_pair[tid] = pr;
    s_w[tid] = pl->w[pr];
  }
  build_stream_tables(tab);
  __syncthreads();

  auto locate = [&](int t, int &r, int &s, int &c, int &q) {
    r = (int)fdiv(t, dSC);
    q = t - r * SC;  // chunk slot of the long vector
    s = (int)fdiv(q, p.div_C);
    c = q - s * p.C;
  };
  auto fetch = [&](int t, int buf) {
    int r, s, c, q;
    locate(t, r, s, c, q);
    fetch_chunk<P>(p.down, (size_t)s_expert[s] * p.hidden + n0 + r, nb, c, fs, buf * nthr + tid);
  };
  auto load = [&](int t, ChunkFields &f, uint32_t &k) {
    int r, s, c, q;
    locate(t, r, s, c, q);
    load_row_chunk<P, VEC>(p.down, (size_t)s_expert[s] * p.hidden + n0 + r, nb, c, f, k);
  };

  ChunkFields f;
  uint32_t rowk = 0;
  if (VEC && kAsyncFields) {
    if (tid < ntask) fetch(tid, 0);
    cp_async_commit();
  } else if (tid < ntask) {
    load(tid, f, rowk);
  }

  // h comes from the kernel just before this one
  grid_dependency_wait();
  grid_dependents_launch();
  // stage the S routed h vectors as one long vector of S * C chunk slots
  for (int i = tid; i < S * nb; i += nthr) {
    const int s = (int)fdiv(i, p.div_nb), b = i - s * nb;
    const float4 *src = reinterpret_cast<const float4 *>(p.h + (size_t)s_pair[s] * p.inter) + 2 * b;
    cm_store_block(hs4, hn2, s * p.C * 8 + b, __ldcg(src), __ldcg(src + 1));
  }
  __syncthreads();

  for (int t = tid, it = 0; t < ntask; t += nthr, ++it) {
    int r, s, c, q;
    locate(t, r, s, c, q);
    ChunkFields fn;
    uint32_t rowkn = 0;
    if (VEC && kAsyncFields) {
      if (t + nthr < ntask) fetch(t + nthr, (it + 1) & 1);
      cp_async_commit();
      cp_async_wait<1>();
      read_chunk<P>(fs, (it & 1) * nthr + tid, f, rowk);
    } else if (t + nthr < ntask) {
      load(t + nthr, fn, rowkn);
    }
    float2 acc = make_float2(0.f, 0.f);
    const int nvalid = VEC ? 8 : min(8, nb - 8 * c);
    chunk_dot_cm<P, VEC, 1>(tab->t, f, nvalid, rowk, hs4 + kCmX4 * q, hn2 + kCmXn * q, acc);
    red[t] = s_w[s] * (acc.x + acc.y);
    if (!(VEC && kAsyncFields)) {
      f = fn;
      rowk = rowkn;
    }
  }
  __syncthreads();
  // one warp per row: the row's S * C partials in a fixed order
  const int warp = tid >> 5, lane = tid & 31;
  for (int r = warp; r < nrows; r += nthr >> 5) {
    float sum = 0.f;
    for (int q = lane; q < SC; q += 32) sum += red[r * SC + q];
    sum = warp_sum(sum);
    if (lane == 0) p.y[n0 + r] = sum;
  }
}

// ---------------------------------------------------------------------- host

bool decode1_supported(const FfnDims &d, int k) {
  if (k < 1 || k > kMaxK) return false;
  // the fast divisions take divisors below 2^16 and dividends below 2^22
  if (d.inter >= (1 << 16) || d.hidden >= (1 << 16)) return false;
  if ((int64_t)k * ceil_div(d.inter / 8, 8) >= (1 << 16)) return false;
  return down1_smem(d, k) <= 200 * 1024 && gate_up1_smem(d) <= 200 * 1024;
}

size_t gate_up1_smem(const FfnDims &d) {
  return sizeof(StreamTables) + cm_bytes(ceil_div(d.hidden / 8, 8)) + 16 +
         FieldSlots::bytes(4 * kGateUp1Threads);
}

// One wave of CTAs, kDown1CtasPerSm per SM, rows split evenly.
static int down1_rows_per_cta(const FfnDims &d) {
  return std::max(1, ceil_div(d.hidden, kDown1CtasPerSm * num_sms()));
}

// Threads for a CTA's (row, expert, chunk) tasks: the fewest whole warps that
// finish them in the fewest rounds of at most kDown1Threads.
static int down1_threads(int tasks) {
  const int rounds = std::max(1, ceil_div(tasks, kDown1Threads));
  return std::min(kDown1Threads, 32 * ceil_div(ceil_div(tasks, rounds), 32));
}

size_t down1_smem(const FfnDims &d, int k) {
  const int C = ceil_div(d.inter / 8, 8);
  return sizeof(StreamTables) + FieldSlots::bytes(2 * kDown1Threads) + cm_bytes(k * C) +
         (size_t)down1_rows_per_cta(d) * k * C * sizeof(float);
}

template <int P, bool VEC>
static int32_t launch_decode1_t(const FfnDims &d, const nslm_seed_matrix *gate,
                                const nslm_seed_matrix *up, const nslm_seed_matrix *down,
                                const SlotPlan *plan, const uint16_t *x_bf16, const float *y_prev,
                                int k, float *h, float *y, bool plan_early, cudaStream_t s,
                                int &launches) {
  const int sms = num_sms();
  {
    GateUp1Params p{};
    p.gate = *gate; p.up = *up; p.plan = plan; p.x_bf16 = x_bf16; p.y_prev = y_prev; p.h = h;
    p.hidden = d.hidden; p.inter = d.inter;
    p.C = ceil_div(d.hidden / 8, 8);
    p.J = ceil_div(p.C, 32);
    p.div_inter = make_fastdiv((uint32_t)d.inter);
    p.div_J = make_fastdiv((uint32_t)p.J);
    p.plan_early = plan_early ? 1 : 0;
    const size_t smem = gate_up1_smem(d);
    auto kern = gate_up1_kernel<P, VEC>;
    int32_t st = ensure_smem((const void *)kern, smem);
    if (st) return st;
    const int per_sm = std::min(kGateUp1MaxCtasPerSm, max_active_ctas((const void *)kern, kGateUp1Threads, smem));
    if ((st = launch_after_previous(kern, sms * per_sm, kGateUp1Threads, smem, s, p))) return st;
    ++launches;
  }
  {
    Down1Params p{};
    p.down = *down; p.plan = plan; p.h = h; p.y = y;
    p.hidden = d.hidden; p.inter = d.inter;
    p.C = ceil_div(d.inter / 8, 8);
    p.rpc = down1_rows_per_cta(d);
    p.div_C = make_fastdiv((uint32_t)p.C);
    p.div_nb = make_fastdiv((uint32_t)(d.inter / 8));
    for (int S = 1; S <= kMaxK; ++S) p.div_SC[S] = make_fastdiv((uint32_t)(S * p.C));
    p.div_SC[0] = p.div_SC[1];
    const size_t smem = down1_smem(d, k);
    auto kern = down1_kernel<P, VEC>;
    int32_t st = ensure_smem((const void *)kern, smem);
    if (st) return st;
    const int threads = down1_threads(p.rpc * k * p.C);
    if ((st = launch_after_previous(kern, ceil_div(d.hidden, p.rpc), threads, smem, s, p))) return st;
    ++launches;
  }
  return NSLM_OK;
}

int32_t launch_decode1(const FfnDims &d, const nslm_seed_matrix *gate, const nslm_seed_matrix *up,
                       const nslm_seed_matrix *down, const SlotPlan *plan, const uint16_t *x_bf16,
                       const float *y_prev, int k, float *h, float *y, bool plan_early,
                       cudaStream_t s, int &launches) {
  const bool vec = d.hidden % 64 == 0 && d.inter % 64 == 0;
  if (d.P == 4)
    return vec ? launch_decode1_t<4, true>(d, gate, up, down, plan, x_bf16, y_prev, k, h, y, plan_early, s, launches)
               : launch_decode1_t<4, false>(d, gate, up, down, plan, x_bf16, y_prev, k, h, y, plan_early, s, launches);
  return vec ? launch_decode1_t<3, true>(d, gate, up, down, plan, x_bf16, y_prev, k, h, y, plan_early, s, launches)
             : launch_decode1_t<3, false>(d, gate, up, down, plan, x_bf16, y_prev, k, h, y, plan_early, s, launches);
}

}  // namespace nslm
