// stackb.cu -- the decode stack for 2..8 tokens as one persistent cooperative
// kernel.
//
// "NanoSeedLM: LLM inference using pseudo-random numbers", "Why K2-Horizon-MoVA":
// each of T tokens reads 8 of a layer's 100 experts, and tokens that pick the
// same expert share its weights.  The routing plan groups the routed
// (token, slot) pairs by expert into slots of at most kSlotTokens pairs, and
// every expert row of a slot is regenerated once for all of its pairs
// ("What I changed: September 2026": weights are rebuilt, never stored).
//
// One launch runs all layers, one CTA of 16 warps per SM, with the two phases
// of the one-token kernel (stack1.cu) per layer behind bounded grid barriers:
//
//   A (gate/up)  every CTA stages the T layer inputs (layer 0: the bf16
//                tokens; later layers: bf16(y_t / rms(y_t)) per token, the sum
//                of squares added in a fixed order from per-CTA partials);
//                warp tasks are (slot, row): the lanes take the 64-weight
//                chunks of the gate and up rows and dot every regenerated
//                block with the slot's token vectors (a one-token slot, the
//                common case, takes the one-token inner loop); lane 0 writes
//                h = SiLU(g) * u for each pair.
//   B (down)     a CTA owns a range of output rows.  The T * k routed h
//                vectors do not fit in shared memory together, so the slots
//                are taken in groups whose pairs do: the CTA stages a group's
//                h vectors, then threads take (slot, row, chunk pair) tasks
//                (chunks q and q + Cq, one per step; slot-major, so the lanes
//                of a warp nearly always share a slot) and dot every
//                regenerated down chunk with the slot's pairs.  Partial sums per (pair,
//                row, chunk pair) stay in shared memory; after the last group
//                one warp per row adds them per token, pairs in plan order
//                (deterministic, no atomics on data).
//
// Weight fields are copied with cp.async into per-thread shared-memory slots
// one step ahead, across group and phase boundaries; the first fields of a
// phase are copied between the two halves of the grid barrier before it.
#include <algorithm>

#include "chunk.cuh"
#include "common.cuh"
#include "persist.cuh"
#include "stack1.cuh"
#include "stackb.cuh"

namespace nslm {

namespace {

constexpr int MT = kSlotTokens;
// Staged blocks per thread with their loads in flight together.  Measured at
// 8 tokens per layer: 1 -> 227 us, 2 -> 256 us, 4 -> 293 us (more live
// registers push the inner loops past 128 registers and into spills).
constexpr int kStageBatch = 1;
// Blocks unrolled per loop trip in the inner loops of one-token slots
// (kRollOne) and of slots shared by several tokens (kRollMulti).  Warps of
// one SM run both kinds of slot at once; fully unrolled, the loops together
// outgrow the instruction cache (15% of warp samples stalled for
// instructions, 4% with these values).  Measured per layer at 8 tokens,
// (kRollOne, kRollMulti): (8, 8) 215.4 us, (8, 4) 205.9, (4, 4) 205.6,
// (2, 2) 208.1, (8, 2) 201.2.
constexpr int kRollOne = 8;
constexpr int kRollMulti = 2;

struct LayerMatsB {
  nslm_seed_matrix gate, up, down;
};

struct StackBParams {
  const SlotPlan *plans;  // [n] this launch's layers
  const uint16_t *x0;     // bf16 [T][hidden]: input of the first layer, or null
  const float *y_in;      // fp32 [T][hidden]: the previous layer's output when x0 is null
  float *h;               // [T*k][inter] by pair
  float *y_mid;           // [T][hidden] between layers
  float *y_out;           // [T][hidden] output of the last layer
  int32_t *sync;          // status, barrier arrivals, abort
  float *rms_part;        // [T][grid] sums of y^2 over each CTA's rows
  uint32_t barrier_base;  // arrivals recorded by earlier launches of the same call
  int32_t n, T, k, hidden, inter;
  int32_t Ch, Ci, Cq;     // 64-weight chunks per gate/up row and per down row; Cq = ceil(Ci / 2)
  int32_t J;              // chunk rounds per lane in phase A: ceil(Ch / 32)
  int32_t rpc;            // output rows per CTA in phase B
  int32_t hcap;           // h vectors the staging area holds
  int32_t stage_slots;    // chunk slots of the staging area
  FastDiv div_inter, div_J, div_Cq, div_nbi;
  LayerMatsB layer[kMaxFusedLayers];
};

template <int P>
__global__ void __launch_bounds__(kStackBThreads, 1) stackb_kernel(const __grid_constant__ StackBParams p) {
  extern __shared__ float4 smem4[];
  const int tid = threadIdx.x, nthr = blockDim.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = nthr >> 5;
  const uint32_t *tab = reinterpret_cast<const uint32_t *>(smem4);
  // staging: chunk-major slots (the T inputs in phase A, a group's h vectors in phase B)
  float4 *xs4 = smem4 + sizeof(StreamTables) / 16;
  float2 *xn2 = reinterpret_cast<float2 *>(xs4 + (size_t)kCmX4 * p.stage_slots);
  char *fbase = reinterpret_cast<char *>(xn2 + (size_t)kCmXn * p.stage_slots + (p.stage_slots & 1));
  // field slots: phase A [2 buffers][gate, up][threads]; phase B [2 buffers][threads],
  // with the down partials in the rest of phase A's area
  const FieldSlots fsA(fbase, 4 * nthr), fsB(fbase, 2 * nthr);
  float *red = reinterpret_cast<float *>(fbase + FieldSlots::bytes(2 * nthr));  // [pair][row][Cq]
  float *rowy = reinterpret_cast<float *>(fbase + FieldSlots::bytes(4 * nthr));  // [T][rpc]
  __shared__ int s_ok, s_nslots, s_npairs, s_ngroups, s_next_nslots;
  __shared__ int s_expert[kMaxPairs], s_start[kMaxPairs + 1];
  __shared__ int s_pid[kMaxPairs], s_tok[kMaxPairs];  // by plan position: pair id, token
  __shared__ float s_w[kMaxPairs];
  __shared__ int s_gslot[kMaxPairs + 1];               // group g: slots s_gslot[g] .. s_gslot[g+1]
  __shared__ int s_next_expert[kMaxPairs];
  __shared__ float s_rms[kMaxT];

  build_stream_tables(reinterpret_cast<StreamTables *>(smem4));
  const int nbh = p.hidden >> 3, nbi = p.inter >> 3;
  // phase A warp number: consecutive tasks go to different CTAs
  const int gw = warp * gridDim.x + blockIdx.x, W = gridDim.x * nwarps;
  const int n0 = blockIdx.x * p.rpc;
  const int nrows = max(0, min(p.rpc, p.hidden - n0));
  // phase B tasks per slot, padded to whole warps so that a warp never
  // straddles two slots (its token count then decides a uniform branch)
  const int RC = nrows * p.Cq, RCp = (RC + 31) & ~31;
  const FastDiv div_RCp = make_fastdiv((uint32_t)max(1, RCp));

  // one layer's plan into shared memory, and the slot groups of phase B
  // (called between block barriers)
  auto load_plan = [&](const SlotPlan *pl) {
    const int ns = pl->n_slots, np = pl->n_pairs;
    for (int i = tid; i < np; i += nthr) {
      const int pr = pl->pair[i];
      s_pid[i] = pr;
      s_tok[i] = pr / p.k;
      s_w[i] = pl->w[pr];
    }
    for (int i = tid; i < ns; i += nthr) s_expert[i] = pl->expert[i];
    for (int i = tid; i <= ns; i += nthr) s_start[i] = pl->start[i];
    if (tid == 0) {
      s_nslots = ns;
      s_npairs = np;
      // greedy groups of whole slots with at most hcap pairs each
      int g = 0, gs = 0;
      s_gslot[0] = 0;
      for (int s = 1; s < ns; ++s)
        if (pl->start[s + 1] - pl->start[gs] > p.hcap) s_gslot[++g] = gs = s;
      if (ns > 0) s_gslot[++g] = ns;
      s_ngroups = g;
    }
  };

  // ---- phase A task geometry (a step = one chunk round of one (slot, row))
  auto a_steps = [&](int nslots) {
    const int ntask = nslots * p.inter;
    return (gw < ntask ? (ntask - 1 - gw) / W + 1 : 0) * p.J;
  };
  auto a_locate = [&](int step, int &slot, int &row, int &c) {
    const int i = p.J == 1 ? step : (int)fdiv(step, p.div_J);
    const int t = gw + i * W;
    slot = (int)fdiv(t, p.div_inter);
    row = t - slot * p.inter;
    c = lane + 32 * (step - i * p.J);
  };
  // code bits of the 5-bit format: fetched into these registers with the
  // other fields of the next task, taken over at the start of its step
  uint32_t nqg = 0, nqu = 0, nqd = 0;
  auto a_fetch = [&](const LayerMatsB &Lm, const int *expert, int step, int buf) {
    int slot, row, c;
    a_locate(step, slot, row, c);
    if (c >= p.Ch) return;
    const uint32_t r32 = (uint32_t)expert[slot] * (uint32_t)p.inter + (uint32_t)row;
    const uint32_t off = r32 * (uint32_t)nbh + 8u * (uint32_t)c;
    fetch_chunk_off<P>(Lm.gate, off, r32, fsA, (2 * buf) * nthr + tid);
    fetch_chunk_off<P>(Lm.up, off, r32, fsA, (2 * buf + 1) * nthr + tid);
    if (P == kP3C5) {
      nqg = load_codes3(Lm.gate, off >> 3);
      nqu = load_codes3(Lm.up, off >> 3);
    }
  };
  // ---- phase B task geometry: task t of group g = (slot s, row r, chunk pair q);
  // its step 0 takes chunk q, step 1 chunk q + Cq
  auto b_nsteps = [&](int g) {
    const int nt = (s_gslot[g + 1] - s_gslot[g]) * RCp;
    return tid < nt ? 2 * ((nt - 1 - tid) / nthr + 1) : 0;
  };
  // r < 0 marks a padding task; c >= Ci the missing second chunk of an odd Ci
  auto b_locate = [&](int g, int step, int &r, int &s, int &q, int &c) {
    const int t = tid + (step >> 1) * nthr;
    const int sr = (int)fdiv((uint32_t)t, div_RCp);
    const int rem = t - sr * RCp;
    r = (int)fdiv((uint32_t)rem, p.div_Cq);
    q = rem - r * p.Cq;
    s = s_gslot[g] + sr;
    c = q + (step & 1) * p.Cq;
    if (rem >= RC) r = -1;
  };
  auto b_fetch = [&](const LayerMatsB &Lm, int g, int step, int buf) {
    int r, s, q, c;
    b_locate(g, step, r, s, q, c);
    if (r < 0 || c >= p.Ci) return;
    const uint32_t r32 = (uint32_t)s_expert[s] * (uint32_t)p.hidden + (uint32_t)(n0 + r);
    fetch_chunk_off<P>(Lm.down, r32 * (uint32_t)nbi + 8u * (uint32_t)c, r32, fsB, buf * nthr + tid);
    if (P == kP3C5) nqd = load_codes3(Lm.down, r32 * (uint32_t)(nbi >> 3) + (uint32_t)c);
  };

  uint32_t nbar = 0;  // grid barriers passed in this launch
  auto barrier_wait = [&]() { return grid_wait(p.sync, p.barrier_base + (++nbar) * gridDim.x, &s_ok); };

  load_plan(p.plans);
  __syncthreads();  // tables, plan
  if (a_steps(s_nslots) > 0) a_fetch(p.layer[0], s_expert, 0, 0);
  cp_async_commit();

  for (int l = 0; l < p.n; ++l) {
    const LayerMatsB &Lm = p.layer[l];
    __syncthreads();  // plan and staging reuse
    if (l > 0) load_plan(p.plans + l);
    if (l + 1 < p.n) {
      const SlotPlan *nx = p.plans + l + 1;
      for (int i = tid; i < nx->n_slots; i += nthr) s_next_expert[i] = nx->expert[i];
      if (tid == 0) s_next_nslots = nx->n_slots;
    }

    // =========================== phase A: gate/up + SiLU
    // (token t's block b is staged as block t * Ch * 8 + b; blocks are taken
    // kStageBatch per thread at a time, all loads in flight before the stores)
    const int nxb = p.T * nbh;
    if (l == 0 && p.x0) {
      for (int i0 = tid; i0 < nxb; i0 += kStageBatch * nthr) {
        uint4 v[kStageBatch];
#pragma unroll
        for (int u = 0; u < kStageBatch; ++u) {
          const int i = i0 + u * nthr;
          if (i < nxb) v[u] = __ldg(reinterpret_cast<const uint4 *>(p.x0) + i);  // [T][hidden] bf16
        }
#pragma unroll
        for (int u = 0; u < kStageBatch; ++u) {
          const int i = i0 + u * nthr;
          if (i < nxb) {
            const int t = i / nbh;
            float4 lo, hi;
            bf16x8_to_f32(v[u], lo, hi);
            cm_store_block(xs4, xn2, t * p.Ch * 8 + (i - t * nbh), lo, hi);
          }
        }
      }
    } else {
      const float4 *y4 = reinterpret_cast<const float4 *>(l == 0 ? p.y_in : p.y_mid);  // [T][hidden]
      float4 v[kStageBatch][2];
      // the first batch of loads is in flight during the sums of squares
#pragma unroll
      for (int u = 0; u < kStageBatch; ++u) {
        const int i = tid + u * nthr;
        if (i < nxb) {
          v[u][0] = __ldcg(y4 + 2 * i);
          v[u][1] = __ldcg(y4 + 2 * i + 1);
        }
      }
      if (warp < p.T) {  // rms of token `warp`: per-CTA partials in a fixed order
        float ss = 0.f;
        for (int i = lane; i < (int)gridDim.x; i += 32) ss += __ldcg(p.rms_part + warp * gridDim.x + i);
        ss = warp_sum(ss);
        if (lane == 0) s_rms[warp] = sqrtf(ss / (float)p.hidden + 1e-6f);
      }
      __syncthreads();
      for (int i0 = tid; i0 < nxb; i0 += kStageBatch * nthr) {
        if (i0 != tid) {
#pragma unroll
          for (int u = 0; u < kStageBatch; ++u) {
            const int i = i0 + u * nthr;
            if (i < nxb) {
              v[u][0] = __ldcg(y4 + 2 * i);
              v[u][1] = __ldcg(y4 + 2 * i + 1);
            }
          }
        }
#pragma unroll
        for (int u = 0; u < kStageBatch; ++u) {
          const int i = i0 + u * nthr;
          if (i < nxb) {
            const int t = i / nbh;
            const float r = s_rms[t];
            const float4 lo = v[u][0], hi = v[u][1];
#define NSLM_NORM(x) __bfloat162float(__float2bfloat16_rn(__fdiv_rn((x), r)))
            cm_store_block(xs4, xn2, t * p.Ch * 8 + (i - t * nbh),
                           make_float4(NSLM_NORM(lo.x), NSLM_NORM(lo.y), NSLM_NORM(lo.z), NSLM_NORM(lo.w)),
                           make_float4(NSLM_NORM(hi.x), NSLM_NORM(hi.y), NSLM_NORM(hi.z), NSLM_NORM(hi.w)));
#undef NSLM_NORM
          }
        }
      }
    }
    __syncthreads();
    {
      const int nsteps = a_steps(s_nslots);
      float2 ag[MT], au[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) ag[m] = au[m] = make_float2(0.f, 0.f);
      for (int step = 0; step < nsteps; ++step) {
        int slot, row, c;
        a_locate(step, slot, row, c);
        const uint32_t cqg = nqg, cqu = nqu;  // this step's 5-bit-format code bits
        if (step + 1 < nsteps) a_fetch(Lm, s_expert, step + 1, (step + 1) & 1);
        cp_async_commit();
        cp_async_wait<1>();
        ChunkFields cg, cu;
        uint32_t ckg, cku;
        read_chunk<P>(fsA, (2 * (step & 1)) * nthr + tid, cg, ckg);
        read_chunk<P>(fsA, (2 * (step & 1) + 1) * nthr + tid, cu, cku);
        if (P == kP3C5) {
          cg.codes = cqg;
          cu.codes = cqu;
        }
        const int q0 = s_start[slot], M = min(MT, s_start[slot + 1] - q0);
        int off[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) off[m] = (m < M ? s_tok[q0 + m] : 0) * p.Ch;
        if (c < p.Ch) {
          // M is warp-uniform; the literal 2 folds the token guards away
          if (M == 1)
            chunk_dot2_cm_multi<P, true, 1, MT, kRollOne>(tab, cg, cu, 8, ckg, cku, xs4 + kCmX4 * c,
                                                          xn2 + kCmXn * c, off, 1, ag, au);
          else if (M == 2)
            chunk_dot2_cm_multi<P, true, 1, MT, kRollMulti>(tab, cg, cu, 8, ckg, cku, xs4 + kCmX4 * c,
                                                            xn2 + kCmXn * c, off, 2, ag, au);
          else
            chunk_dot2_cm_multi<P, true, 1, MT, kRollMulti>(tab, cg, cu, 8, ckg, cku, xs4 + kCmX4 * c,
                                                            xn2 + kCmXn * c, off, M, ag, au);
        }
        if (p.J == 1 || c + 32 >= 32 * p.J) {
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            if (m < M) {
              const float g = warp_sum(ag[m].x + ag[m].y), u = warp_sum(au[m].x + au[m].y);
              // SiLU with the fast exp and divide (relative error ~1e-6; an
              // exp that overflows gives the limit 0)
              if (lane == 0 && in_bounds((size_t)s_pid[q0 + m], (size_t)p.T * p.k, 10))
                __stcg(p.h + (size_t)s_pid[q0 + m] * p.inter + row, __fdividef(g, 1.f + __expf(-g)) * u);
            }
            ag[m] = au[m] = make_float2(0.f, 0.f);
          }
        }
      }
    }
    // arrive; copy phase B's first fields (weights only) while the others arrive
    grid_arrive(p.sync);
    cp_async_wait<0>();
    bool pre = s_ngroups > 0 && b_nsteps(0) > 0;
    if (pre) b_fetch(Lm, 0, 0, 0);
    cp_async_commit();
    if (!barrier_wait()) break;

    // =========================== phase B: down + weighted combine
    {
      int it = 0;  // field buffer parity
      float2 acc[MT];
      for (int g = 0; g < s_ngroups; ++g) {
        // (a group holds at most hcap pairs when every slot has at most
        // kSlotTokens of them, which the plan guarantees; the clamp keeps the
        // staging in bounds regardless)
        const int qa = s_start[s_gslot[g]], np = min(p.hcap, s_start[s_gslot[g + 1]] - qa);
        // the group's h vectors, chunk-major, pair j at chunk slot j * Ci
        const int nhb = np * nbi;
        for (int i0 = tid; i0 < nhb; i0 += kStageBatch * nthr) {
          float4 v[kStageBatch][2];
#pragma unroll
          for (int u = 0; u < kStageBatch; ++u) {
            const int i = i0 + u * nthr;
            if (i < nhb) {
              const int j = (int)fdiv((uint32_t)i, p.div_nbi), b = i - j * nbi;
              const float4 *src = reinterpret_cast<const float4 *>(p.h + (size_t)s_pid[qa + j] * p.inter) + 2 * b;
              v[u][0] = __ldcg(src);
              v[u][1] = __ldcg(src + 1);
            }
          }
#pragma unroll
          for (int u = 0; u < kStageBatch; ++u) {
            const int i = i0 + u * nthr;
            if (i < nhb) {
              const int j = (int)fdiv((uint32_t)i, p.div_nbi);
              cm_store_block(xs4, xn2, j * p.Ci * 8 + (i - j * nbi), v[u][0], v[u][1]);
            }
          }
        }
        __syncthreads();
        const int n = b_nsteps(g);
        if (n > 0 && !pre) {
          b_fetch(Lm, g, 0, it & 1);
          cp_async_commit();
        }
        pre = false;
        for (int k = 0; k < n; ++k) {
          int r, s, q, c;
          b_locate(g, k, r, s, q, c);
          const uint32_t cqd = nqd;  // this task's 5-bit-format code bits
          if (k + 1 < n) {
            b_fetch(Lm, g, k + 1, (it + 1) & 1);
          } else if (g + 1 < s_ngroups && b_nsteps(g + 1) > 0) {
            b_fetch(Lm, g + 1, 0, (it + 1) & 1);
            pre = true;
          }
          cp_async_commit();
          cp_async_wait<1>();
          ChunkFields cf;
          uint32_t ck;
          read_chunk<P>(fsB, (it & 1) * nthr + tid, cf, ck);
          if (P == kP3C5) cf.codes = cqd;
          ++it;
          const int q0 = s_start[s], M = min(MT, s_start[s + 1] - q0);
          if ((k & 1) == 0) {
#pragma unroll
            for (int m = 0; m < MT; ++m) acc[m] = make_float2(0.f, 0.f);
          }
          if (r >= 0 && c < p.Ci) {
            int off[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) off[m] = (q0 - qa + m) * p.Ci;
            // M is warp-uniform (slots are padded to whole warps)
            if (M == 1)
              chunk_dot_cm_multi<P, true, 1, MT, kRollOne>(tab, cf, 8, ck, xs4 + kCmX4 * c, xn2 + kCmXn * c, off,
                                                           1, acc);
            else if (M == 2)
              chunk_dot_cm_multi<P, true, 1, MT, kRollMulti>(tab, cf, 8, ck, xs4 + kCmX4 * c, xn2 + kCmXn * c,
                                                             off, 2, acc);
            else
              chunk_dot_cm_multi<P, true, 1, MT, kRollMulti>(tab, cf, 8, ck, xs4 + kCmX4 * c, xn2 + kCmXn * c,
                                                             off, M, acc);
          }
          if ((k & 1) && r >= 0) {
#pragma unroll
            for (int m = 0; m < MT; ++m)
              if (m < M) red[((q0 + m) * p.rpc + r) * p.Cq + q] = acc[m].x + acc[m].y;
          }
        }
        __syncthreads();  // staging reuse
      }
      // y[t][row] = sum over token t's pairs (plan order) of w * sum of chunk partials
      float *yl = (l == p.n - 1) ? p.y_out : p.y_mid;
      const int np = s_npairs;
      for (int r = warp; r < nrows; r += nwarps) {
        float v0 = 0.f, v1 = 0.f;
        int t0 = -1, t1 = -1;
        if (lane < np) {
          float a = 0.f;
          for (int q = 0; q < p.Cq; ++q) a += red[(lane * p.rpc + r) * p.Cq + q];
          v0 = s_w[lane] * a;
          t0 = s_tok[lane];
        }
        if (lane + 32 < np) {
          float a = 0.f;
          for (int q = 0; q < p.Cq; ++q) a += red[((lane + 32) * p.rpc + r) * p.Cq + q];
          v1 = s_w[lane + 32] * a;
          t1 = s_tok[lane + 32];
        }
        for (int t = 0; t < p.T; ++t) {
          const float sum = warp_sum((t0 == t ? v0 : 0.f) + (t1 == t ? v1 : 0.f));
          if (lane == 0) {
            __stcg(yl + (size_t)t * p.hidden + n0 + r, sum);
            rowy[t * p.rpc + r] = sum;
          }
        }
      }
      __syncthreads();
      if (warp < p.T) {  // per-token sum of squares of this CTA's rows, fixed order
        float ss = 0.f;
        for (int r = lane; r < nrows; r += 32) ss = fmaf(rowy[warp * p.rpc + r], rowy[warp * p.rpc + r], ss);
        ss = warp_sum(ss);
        if (lane == 0) __stcg(p.rms_part + warp * gridDim.x + blockIdx.x, ss);
      }
    }
    if (l + 1 == p.n) break;
    // arrive; copy the next layer's first phase A fields while the others arrive
    grid_arrive(p.sync);
    cp_async_wait<0>();
    if (a_steps(s_next_nslots) > 0) a_fetch(p.layer[l + 1], s_next_expert, 0, 0);
    cp_async_commit();
    if (!barrier_wait()) break;
  }
  cp_async_wait<0>();
}

static_assert(sizeof(StackBParams) <= 32764, "kernel parameter space");

}  // namespace

// ---------------------------------------------------------------------- host

namespace {

struct StackBShape {
  int grid, threads, rpc, Ch, Ci, Cq, hcap, stage_slots;
  size_t smem;
};

constexpr size_t kStackBSmemMax = 224 * 1024;

// Dynamic shared memory: tables, staging, field slots (with the down partials
// inside phase A's half), per-token row sums.
size_t stackb_smem_of(int threads, int T, int rpc, int stage_slots) {
  return sizeof(StreamTables) + cm_bytes(stage_slots) + 16 + FieldSlots::bytes(4 * threads) +
         (size_t)T * rpc * sizeof(float);
}

bool stackb_shape(const FfnDims &d, int T, int k, StackBShape &sh) {
  if (T < 2 || T > kMaxT || k < 1 || k > kMaxK) return false;
  if (d.hidden % 64 || d.inter % 64) return false;
  sh.threads = kStackBThreads;
  sh.grid = num_sms();  // one CTA per SM (the shared memory allows no more)
  if (sh.grid > kMaxStack1Ctas) return false;
  sh.rpc = ceil_div(d.hidden, sh.grid);
  sh.Ch = d.hidden / 64;
  sh.Ci = d.inter / 64;
  sh.Cq = ceil_div(sh.Ci, 2);
  // down partials: all pairs x this CTA's rows x chunk pairs
  if ((size_t)T * k * sh.rpc * sh.Cq * sizeof(float) > FieldSlots::bytes(2 * sh.threads)) return false;
  // the largest group of h vectors that fits beside the T staged inputs
  const size_t fixed = stackb_smem_of(sh.threads, T, sh.rpc, 0);
  if (fixed + cm_bytes(T * sh.Ch) > kStackBSmemMax) return false;
  const int slots = (int)((kStackBSmemMax - fixed) / cm_bytes(1));
  sh.hcap = std::min(T * k, slots / sh.Ci);
  if (sh.hcap < kSlotTokens) return false;
  sh.stage_slots = std::max(T * sh.Ch, sh.hcap * sh.Ci);
  sh.smem = stackb_smem_of(sh.threads, T, sh.rpc, sh.stage_slots);
  return sh.smem <= kStackBSmemMax;
}

}  // namespace

bool stackb_supported(const FfnDims &d, int T, int k) {
  if (d.P != 3 && d.P != 4 && d.P != kP3C5) return false;
  StackBShape sh{};
  if (!stackb_shape(d, T, k, sh)) return false;
  // 32-bit element offsets into the field streams
  if ((int64_t)d.E * d.inter * (d.hidden / 8) >= (1ll << 31) || (int64_t)d.E * d.hidden * (d.inter / 8) >= (1ll << 31))
    return false;
  // fast divisions: divisors below 2^16, dividends below 2^22
  if (d.inter >= (1 << 16) || d.inter / 8 >= (1 << 16)) return false;
  if ((int64_t)kMaxPairs * sh.Cq >= (1 << 16)) return false;
  if ((int64_t)T * k * d.inter * ceil_div(sh.Ch, 32) >= (1 << 22)) return false;
  if ((int64_t)sh.rpc * T * k * sh.Cq >= (1 << 22) || (int64_t)sh.hcap * (d.inter / 8) >= (1 << 22)) return false;
  if ((int64_t)sh.rpc * sh.Cq >= (1 << 16)) return false;
  return true;
}

template <int P>
static int32_t launch_stackb_t(const FfnDims &d, const StackBShape &sh, const nslm_moe_layer *layers, int n,
                               const SlotPlan *plans, const uint16_t *x0, const float *y_in, int T, int k,
                               float *h, float *y_mid, float *y_out, int32_t *sync, float *rms_part,
                               cudaStream_t s, int &launches) {
  auto kern = stackb_kernel<P>;
  int32_t st = ensure_smem((const void *)kern, sh.smem);
  if (st) return st;
  if (max_active_ctas((const void *)kern, sh.threads, sh.smem) < 1) return NSLM_ERR_SHAPE;
  StackBParams p{};
  p.h = h;
  p.y_mid = y_mid;
  p.sync = sync;
  p.rms_part = rms_part;
  p.T = T;
  p.k = k;
  p.hidden = d.hidden;
  p.inter = d.inter;
  p.Ch = sh.Ch;
  p.Ci = sh.Ci;
  p.Cq = sh.Cq;
  p.J = ceil_div(sh.Ch, 32);
  p.rpc = sh.rpc;
  p.hcap = sh.hcap;
  p.stage_slots = sh.stage_slots;
  p.div_inter = make_fastdiv((uint32_t)d.inter);
  p.div_J = make_fastdiv((uint32_t)p.J);
  p.div_Cq = make_fastdiv((uint32_t)sh.Cq);
  p.div_nbi = make_fastdiv((uint32_t)(d.inter / 8));
  // chunks of kMaxFusedLayers layers; barrier arrivals keep counting across them
  uint32_t base = 0;
  for (int l0 = 0; l0 < n; l0 += kMaxFusedLayers) {
    const int m = std::min(kMaxFusedLayers, n - l0);
    p.plans = plans + l0;
    p.x0 = l0 == 0 ? x0 : nullptr;
    p.y_in = l0 == 0 ? y_in : y_mid;
    p.y_out = (l0 + m == n) ? y_out : y_mid;
    p.n = m;
    p.barrier_base = base;
    for (int i = 0; i < m; ++i)
      p.layer[i] = LayerMatsB{layers[l0 + i].gate, layers[l0 + i].up, layers[l0 + i].down};
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)sh.grid);
    cfg.blockDim = dim3((unsigned)sh.threads);
    cfg.dynamicSmemBytes = sh.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    ensure_stream_source(s);
    if ((st = cuda_status(cudaLaunchKernelEx(&cfg, kern, p)))) return st;
    ++launches;
    base += (uint32_t)(2 * m - 1) * (uint32_t)sh.grid;
  }
  return NSLM_OK;
}

int32_t launch_stackb(const FfnDims &d, const nslm_moe_layer *layers, int n, const SlotPlan *plans,
                      const uint16_t *x0, const float *y_in, int T, int k, float *h, float *y_mid,
                      float *y_out, int32_t *sync, float *rms_part, cudaStream_t s, int &launches) {
  StackBShape sh{};
  if (!stackb_shape(d, T, k, sh)) return NSLM_ERR_SHAPE;
  if (d.P == 4)
    return launch_stackb_t<4>(d, sh, layers, n, plans, x0, y_in, T, k, h, y_mid, y_out, sync, rms_part, s, launches);
  if (d.P == kP3C5)
    return launch_stackb_t<kP3C5>(d, sh, layers, n, plans, x0, y_in, T, k, h, y_mid, y_out, sync, rms_part, s,
                                  launches);
  return launch_stackb_t<3>(d, sh, layers, n, plans, x0, y_in, T, k, h, y_mid, y_out, sync, rms_part, s, launches);
}

NSLM_BOUNDS_ACCESSOR(stackb)

}  // namespace nslm

// ------------------------------------------------ decode dispatch, T <= 8

namespace nslm {

int decode_slot_cap(const FfnDims &d, int T, int k) {
  return (T > 1 && stackb_supported(d, T, k)) ? kSlotTokens : T;
}

int32_t launch_decode_stack(const FfnDims &d, const nslm_moe_layer *layers, int L, const uint16_t *x0,
                            int T, int k, const FfnWorkspace &fw, float *y, cudaStream_t s, int &launches) {
  if (T == 1 && stack1_supported(d, k))
    return launch_stack1(d, layers, L, fw.plans, x0, k, fw.h, fw.ytag, y, fw.sync, s, launches);
  if (T > 1 && stackb_supported(d, T, k))
    return launch_stackb(d, layers, L, fw.plans, x0, nullptr, T, k, fw.h, fw.y_mid, y, fw.sync, fw.rms_part,
                         s, launches);
  // shapes the persistent kernels do not take: two launches per layer
  for (int l = 0; l < L; ++l) {
    const uint16_t *xin = (l == 0) ? x0 : nullptr;
    const float *yprev = (l == 0) ? nullptr : fw.y_mid;
    float *yout = (l == L - 1) ? y : fw.y_mid;
    const int32_t st = launch_decode_layer(d, &layers[l].gate, &layers[l].up, &layers[l].down, fw.plans + l,
                                           xin, yprev, T, k, fw, yout, s, launches);
    if (st) return st;
  }
  return NSLM_OK;
}

}  // namespace nslm
