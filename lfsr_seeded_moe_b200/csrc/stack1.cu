// stack1.cu -- the one-token decode stack as one persistent cooperative kernel.
//
// "NanoSeedLM: LLM inference using pseudo-random numbers", "Why K2-Horizon-MoVA":
// for one token every layer reads 8 of its 100 experts: gate and up
// projections, SiLU, a down projection, and the routing-weighted sum.  The
// weights are regenerated in registers ("What I changed: September 2026").
//
// One launch runs all layers.  Each CTA (one per SM, up to 20 warps) keeps
// its stream tables and every layer's routing plan for the whole stack and
// alternates two phases (the launch is cooperative, so every CTA is
// resident):
//
//   A (gate/up)  every CTA stages the layer input x (layer 0: the bf16 token;
//                later layers: bf16(y / rms(y)) of the previous layer's fp32
//                output); warp tasks are routed rows: the lanes take the
//                64-weight chunks of the gate and up rows, a shuffle tree sums
//                them, lane 0 writes h = SiLU(g) * u.
//   B (down)     every CTA stages the routed h vectors back to back and owns
//                a range of output rows: threads take (row, expert, chunk)
//                tasks, partials go to shared memory and one warp per row adds
//                them in a fixed order (deterministic, no atomics on data).
//
// A grid barrier separates A from B: every CTA needs all of h.  From B to the
// next layer's A there is no barrier: each y row, and each CTA's sum of y^2
// over its rows, is stored as a 64-bit word tagged with the layer, and the
// next layer's staging polls exactly the words it reads until their tags
// match.  (A CTA cannot overwrite h before every CTA has read it: it starts
// the next phase A only after reading every CTA's y, which each CTA writes
// after staging h.)
//
// Phase B stages the routed h by one 256-byte bulk asynchronous copy per
// 64-value chunk (global -> shared, completing on an mbarrier; no multicast),
// then forms the block sums from shared memory.
//
// Weight fields land in per-thread shared-memory slots one task ahead: in
// phase A (hidden % 256 == 0) by bulk asynchronous copies, six lanes of each
// warp copying the step's seeds, coefficients and code words of both
// matrices in one instruction, completing on the warp's barrier of that
// buffer; otherwise, and in phase B, by cp.async.  The first task of the
// next phase is fetched before the wait, so the wait overlaps the first
// loads.  Every wait is bounded: a CTA that gives up raises the abort flag
// (all others stop at their next wait) and records status 1 in the
// workspace.
#include <algorithm>

#include "chunk.cuh"
#include "common.cuh"
#include "persist.cuh"
#include "stack1.cuh"
#include "umma.cuh"

namespace nslm {

namespace {

constexpr int kTabCopies = 1;  // interleaved stream-table copies (bank conflicts / kTabCopies)

}  // namespace

// Trace build (-DNSLM_STACK1_TRACE=1, the "trace" library variant): thread 0
// of every CTA stamps the global timer at the phase boundaries of each layer
// (stamp k of CTA c, layer l at g_stack1_trace[k][c][l]), with a block
// barrier before the stamps that mark a whole CTA's end of a phase.  The
// default build has none of it.
#ifndef NSLM_STACK1_TRACE
#define NSLM_STACK1_TRACE 0
#endif
#if NSLM_STACK1_TRACE
constexpr int kTraceStamps = 8, kTraceCtas = 256, kTraceLayers = 64;
__device__ unsigned long long g_stack1_trace[kTraceStamps][kTraceCtas][kTraceLayers];
#define NSLM_TRACE(k, sync_first)                                                              \
  do {                                                                                         \
    if (sync_first) __syncthreads();                                                           \
    if (threadIdx.x == 0 && blockIdx.x < kTraceCtas && l < kTraceLayers) {                     \
      unsigned long long t_;                                                                   \
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                                   \
      g_stack1_trace[k][blockIdx.x][l] = t_;                                                   \
    }                                                                                          \
  } while (0)
#else
#define NSLM_TRACE(k, sync_first) \
  do {                            \
  } while (0)
#endif

namespace {

struct LayerMats {
  nslm_seed_matrix gate, up, down;
};

struct Stack1Params {
  const SlotPlan *plans;  // [n] this launch's layers
  const uint16_t *x0;     // bf16 [hidden]: input of layer 0 (the first launch), else null
  float *h;               // [k][inter] by pair
  uint64_t *ytag;         // [hidden] y rows, then [grid] sums of y^2, tagged (zeroed per call)
  float *y_out;           // [hidden] output of the last layer if this launch ends the stack, else null
  int32_t *sync;          // status, barrier arrivals, abort
  uint32_t barrier_base;  // arrivals recorded by earlier launches of the same call
  uint32_t l0;            // index in the stack of this launch's first layer
  int32_t n, hidden, inter;
  int32_t h_rows;         // rows of h (the routed pairs; bounds checks)
  int32_t Ch, Ci;         // 64-weight chunks per row of gate/up (hidden) and down (inter)
  int32_t J;              // chunk rounds per lane in phase A: ceil(Ch / 32)
  int32_t rpc;            // output rows per CTA in phase B
  int32_t stage_slots;    // chunk slots of the staging area
  int32_t region_bytes;   // bytes of the staging region (chunk-major x / h, or the table form's tables)
  int32_t f3_np;          // table form: passes of 128 block positions over the hidden dimension
  FastDiv div_inter, div_J, div_Ci, div_nbi, div_W;
  FastDiv div_SC[kMaxK + 1];  // by S * Ci for S routed experts
  LayerMats layer[kMaxFusedLayers];
};

__device__ __forceinline__ bool stack_wait(const Stack1Params &p, uint32_t e, int *s_ok) {
  return grid_wait(p.sync, p.barrier_base + (e + 1) * gridDim.x, s_ok);
}

// ---------------------------------------------------------------- table form
//
// Phase A can take its dot products from tables of x instead of the staged
// x itself.  With S the 48-bit stream of a block (seed, then the next 32
// register bits; s_t = the 16 bits of S from bit t), beta_q = the byte of S
// from bit 1 + 8q, and A_r = sum_j c_j (s_{1+8j+r} - 32768) (the integer part
// of weight r), the dot product of the block with its 8 inputs x_r is exactly
//
//   sum_r x_r A_r = A0 A_0 + 32768 (A0 - X) C
//                 + sum_j c_j (T[beta_j & 127] - 65536 T[beta_{j+2} & 127]),
//
// with A0 = sum_r x_r 2^-r, X = sum_r x_r, C = sum_j c_j and the 128-entry
// table T[b] = -sum_{r=1..7} x_r 2^-r (b mod 2^r) of the block position: the
// bits 7..15 of each s_{1+8j+r} enter every r with weight 2^(m-r), i.e.
// through A0, and the low 7 bits of the two neighbouring bytes through T (the
// bits of beta_{j+2} carry the same weights as those of beta_j, times
// -65536).  Every row of a layer shares x, so one CTA builds the tables of
// 128 positions (64 KB) and all its rows use them: six table reads per block
// replace the eight per-weight dot products.  The integer A_0 comes from two
// dp2a as in the direct form; T is built and read in fp32.
//
// Layout: position o of a pass (0..127) keeps T/2 at byte (o / 64) * 32768 +
// b * 256 + w * 4, with word w = 32 (o % 2) + (o % 64) / 2: lane l, which
// takes positions 64 i + 2 l + t (one 32-bit word of seeds), reads word
// 32 t + l, in its own bank, and forms the address with one byte permute;
// constants (A0 / 2, 16384 (A0 - X)) per position follow the tables.
constexpr int kF3Positions = 128;                       // block positions per pass
constexpr int kF3TableBytes = kF3Positions * 128 * 4;   // 64 KB
constexpr int kF3MaxTasks = 4;                          // routed rows per warp it takes

// Tables and constants of the pass's 128 positions from their inputs xp
// (fp32, 8 per position).  Entry b of position o is the sum of the d_k of
// the set bits k of b, d_k = -(1/2) 2^k sum_{r>k} x_r 2^-r.
__device__ void f3_build(char *tab, float2 *cst, const float *xp, int tid, int nthr) {
  for (int job = tid; job < kF3Positions * 8; job += nthr) {
    const int o = job & (kF3Positions - 1), m = job >> 7;  // a warp: 32 positions, one entry range
    const float4 xa = *reinterpret_cast<const float4 *>(xp + 8 * o);
    const float4 xb = *reinterpret_cast<const float4 *>(xp + 8 * o + 4);
    const float x[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
    float d[7], S = 0.f;
#pragma unroll
    for (int k = 6; k >= 0; --k) {
      S = fmaf(x[k + 1], 1.f / (float)(2 << k), S);  // sum_{r>k} x_r 2^-r
      d[k] = -0.5f * (float)(1 << k) * S;
    }
    float base = 0.f;
    if (m & 1) base += d[4];
    if (m & 2) base += d[5];
    if (m & 4) base += d[6];
    float L[16];
    L[0] = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int e = 0; e < (1 << k); ++e) L[e + (1 << k)] = L[e] + d[k];
    char *dst = tab + (o >> 6) * 32768 + (32 * (o & 1) + ((o & 63) >> 1)) * 4 + 16 * m * 256;
#pragma unroll
    for (int e = 0; e < 16; ++e) *reinterpret_cast<float *>(dst + e * 256) = base + L[e];
    if (m == 0) {
      float a0 = 0.f, xs = 0.f;
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        a0 = fmaf(x[r], 1.f / (float)(1 << r), a0);
        xs += x[r];
      }
      cst[o] = make_float2(0.5f * a0, 16384.f * (a0 - xs));
    }
  }
}

// sum_r x_r A_r of one block from its seed and 16-bit coefficient word; tb:
// its table block plus 128 t (bytes), lc: 4 * lane, a0h / yh: its constants.
template <int P>
__device__ __forceinline__ float f3_block(const uint32_t *tl, uint32_t seed, uint32_t q16, uint32_t lc,
                                          const char *tb, float a0h, float yh) {
  const uint32_t nxt = tl[seed & 0xFFu] ^ tl[256u + (seed >> 8)];
  const uint32_t v = seed << 16;
  const uint32_t z1 = __funnelshift_r(v, nxt, 17), z9 = __funnelshift_r(v, nxt, 25), z17 = nxt >> 1;
  const uint32_t cp2 = coef_pairs2<P>(q16);                                 // [2c0, 2c2, 2c1, 2c3]
  const int32_t c2 = dp4a_ss(cp2, 0x01010101u, 0);                          // 2 C
  const int32_t i0 = dp2a_hi_us(z9, cp2, dp2a_lo_us(z1, cp2, -32768 * c2));  // 2 A_0
  const uint32_t m1 = z1 & 0x7F7F7F7Fu, m17 = z17 & 0x7F7F7F7Fu;
#define NSLM_T(m, k) (*reinterpret_cast<const float *>(tb + __byte_perm((m), lc, 0x5504u | ((k) << 4))))
  const float t0 = NSLM_T(m1, 0), t1 = NSLM_T(m1, 1), t2 = NSLM_T(m1, 2), t3 = NSLM_T(m1, 3);
  const float t4 = NSLM_T(m17, 2);
  float acc = fmaf(yh, (float)c2, a0h * (float)i0);
  acc = fmaf((float)(int8_t)(cp2 & 0xFFu), fmaf(-65536.f, t2, t0), acc);
  acc = fmaf((float)(int8_t)((cp2 >> 16) & 0xFFu), fmaf(-65536.f, t3, t1), acc);
  acc = fmaf((float)(int8_t)((cp2 >> 8) & 0xFFu), fmaf(-65536.f, t4, t2), acc);
  if (P == 4) acc = fmaf((float)(int8_t)(cp2 >> 24), fmaf(-65536.f, NSLM_T(m17, 3), t3), acc);
#undef NSLM_T
  return acc;
}

// This lane's share of one row's dot product over a pass: positions
// 64 i + 2 lane + t (i, t in {0, 1}) of the 128 whose fields the warp's lanes
// 0..15 copied, in order, to the slots from `slot`.
template <int P>
__device__ __forceinline__ float f3_row(const uint32_t *tl, const FieldSlots &fs, int slot, int lane,
                                        const char *tab, const float (&a0h)[2][2], const float (&yh)[2][2]) {
  const uint32_t *sw = reinterpret_cast<const uint32_t *>(fs.s + slot);
  const uint32_t *qw = reinterpret_cast<const uint32_t *>(fs.q + slot);
  const uint8_t *cb = reinterpret_cast<const uint8_t *>(fs.c + slot);
  const uint32_t rowk = row_scale_key(fs.b[slot]);
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint32_t s2 = sw[32 * i + lane], q2 = qw[32 * i + lane];
    const uint32_t cbyte = (P == 4) ? (uint32_t)cb[32 * i + lane] : 0u;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const uint32_t seed = t ? (s2 >> 16) : (s2 & 0xFFFFu), q = t ? (q2 >> 16) : (q2 & 0xFFFFu);
      const uint32_t code = (P == 4) ? ((cbyte >> (4 * t)) & 0xFu) : (q >> 12);
      const float tot = f3_block<P>(tl, seed, q, 4u * (uint32_t)lane, tab + i * 32768 + 128 * t, a0h[i][t], yh[i][t]);
      acc = fmaf(block_scale(code, rowk), tot, acc);
    }
  }
  return acc;
}

// Stage x = bf16(y / sqrt(mean(y^2) + 1e-6)) chunk-major from the tagged y
// rows and per-CTA sums of squares of layer `tag` - 1, polling each word until
// it carries `tag`.  The sum of squares is the fixed-order sum of the G
// partials.  The last warp polls the partials while the others poll their
// first block of 8 rows.  False if a wait gave up.
template <bool PLAIN>
__device__ bool stage_norm_tagged(float4 *xs4, float2 *xn2, const uint64_t *ytag, uint32_t tag, int G, int K,
                                  int32_t *sync, float *scratch) {
  const int tid = threadIdx.x, nthr = blockDim.x, nb = K >> 3;
  bool ok = true;
  uint64_t w[8];
  auto poll_block = [&](int b) {
    return poll_bounded(sync, [&] {
      const uint64_t *src = ytag + 8 * b;
#pragma unroll
      for (int j = 0; j < 8; j += 2) ld_tagged2(src + j, w[j], w[j + 1]);
      bool all = true;
#pragma unroll
      for (int j = 0; j < 8; ++j) all &= has_tag(w[j], tag);
      return all;
    });
  };
  if (tid < nb) ok &= poll_block(tid);  // the first block of this thread
  if (tid >= nthr - 32) {
    const int lane = tid & 31;
    // the first 256 partials with all loads in flight, then any others; the
    // per-lane order of the additions is that of one strided loop
    float v[8];
    ok &= poll_bounded(sync, [&] {
      bool all = true;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        v[j] = 0.f;
        if (lane + 32 * j < G) {
          const uint64_t u = ld_tagged(ytag + K + lane + 32 * j);
          all &= has_tag(u, tag);
          v[j] = tagged_value(u);
        }
      }
      return all;
    });
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) ss += v[j];
    for (int i = lane + 256; i < G; i += 32) {
      uint64_t u = 0;
      ok &= poll_bounded(sync, [&] {
        u = ld_tagged(ytag + K + i);
        return has_tag(u, tag);
      });
      ss += tagged_value(u);
    }
    ss = warp_sum(ss);
    if (lane == 0) scratch[32] = sqrtf(ss / (float)K + 1e-6f);
  }
  __syncthreads();
  const float r = scratch[32];
  for (int b = tid; b < nb; b += nthr) {
    if (b != tid) ok &= poll_block(b);
#define NSLM_NORM(u) __bfloat162float(__float2bfloat16_rn(__fdiv_rn(tagged_value(u), r)))
    const float4 a = make_float4(NSLM_NORM(w[0]), NSLM_NORM(w[1]), NSLM_NORM(w[2]), NSLM_NORM(w[3]));
    const float4 c = make_float4(NSLM_NORM(w[4]), NSLM_NORM(w[5]), NSLM_NORM(w[6]), NSLM_NORM(w[7]));
#undef NSLM_NORM
    if (PLAIN) {  // fp32 in order, for the table form's tables
      reinterpret_cast<float4 *>(xs4)[2 * b] = a;
      reinterpret_cast<float4 *>(xs4)[2 * b + 1] = c;
    } else {
      cm_store_block(xs4, xn2, b, a, c);
    }
  }
  return ok;
}

template <int P, bool VEC, bool F3, bool BA>
__global__ void __launch_bounds__(kStack1MaxThreads, 1) stack1_kernel(const __grid_constant__ Stack1Params p) {
  static_assert(!F3 || (VEC && (P == 3 || P == 4)), "the table form takes whole chunks of P = 3 or 4");
  static_assert(!BA || (VEC && !F3), "bulk phase A copies take whole chunks, direct form");
  extern __shared__ float4 smem4[];
  const int tid = threadIdx.x, nthr = blockDim.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = nthr >> 5;
  uint32_t *tab = reinterpret_cast<uint32_t *>(smem4);  // kTabCopies interleaved copies
  const uint32_t *tl = tab + (tid & (kTabCopies - 1));
  // staging: chunk-major slots (x in phase A, the routed h vectors in phase B)
  float4 *xs4 = smem4 + kTabCopies * sizeof(StreamTables) / 16;
  float2 *xn2 = reinterpret_cast<float2 *>(xs4 + (size_t)kCmX4 * p.stage_slots);
  // field slots: phase A [2 buffers][gate, up][threads], phase B [2 buffers][threads]
  const FieldSlots fs(reinterpret_cast<char *>(xs4) + p.region_bytes, 4 * nthr);
  // table form (phase A): tables, constants, per-task partial sums, x in order
  char *f3tab = reinterpret_cast<char *>(xs4);
  float2 *f3cst = reinterpret_cast<float2 *>(f3tab + kF3TableBytes);
  float2 *f3part = f3cst + kF3Positions;
  float *xplain = reinterpret_cast<float *>(f3part + nwarps * kF3MaxTasks * 32);
  float *red = reinterpret_cast<float *>(fs.b + 4 * nthr);  // phase B partials
  __shared__ float scratch[33];
  __shared__ int s_ok, s_nslots;
  __shared__ __align__(8) uint64_t s_hbar;  // completion of the bulk copies of h (one phase a layer)
  // BA: completion of each warp's bulk copies of its phase A fields, per buffer
  __shared__ __align__(8) uint64_t s_fbar[kStack1MaxThreads / 32][2];
  __shared__ int s_expert[kMaxK], s_pair[kMaxK];
  __shared__ float s_w[kMaxK];
  // every layer's routed slots (expert, pair, weight), read once at the start
  __shared__ int s_pl_n[kMaxFusedLayers], s_pl_expert[kMaxFusedLayers][kMaxK], s_pl_pair[kMaxFusedLayers][kMaxK];
  __shared__ float s_pl_w[kMaxFusedLayers][kMaxK];

  const int nbh = p.hidden >> 3, nbi = p.inter >> 3;
  // phase A warp number: consecutive tasks go to different CTAs, so every SM
  // receives the same number of routed rows (to within one)
  const int gw = warp * gridDim.x + blockIdx.x, W = gridDim.x * nwarps;
  const int n0 = blockIdx.x * p.rpc;
  const int nrows = max(0, min(p.rpc, p.hidden - n0));

  // code bits of the 5-bit format: fetched into these registers with the
  // other fields of the next task, taken over at the start of its step
  uint32_t nqg = 0, nqu = 0, nqd = 0;

  // ---- phase A task geometry (a step = one chunk round of one routed row)
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
  auto a_fetch = [&](const LayerMats &Lm, const int32_t *expert, int step, int buf, ChunkFields &fg,
                     ChunkFields &fu, uint32_t &kg, uint32_t &ku) {
    int slot, row, c;
    a_locate(step, slot, row, c);
    if (c >= p.Ch) return;
    const size_t grow = (size_t)expert[slot] * p.inter + row;
    if (VEC) {
      const uint32_t r32 = (uint32_t)grow, off = r32 * (uint32_t)nbh + 8u * (uint32_t)c;
      fetch_chunk_off<P>(Lm.gate, off, r32, fs, (2 * buf) * nthr + tid);
      fetch_chunk_off<P>(Lm.up, off, r32, fs, (2 * buf + 1) * nthr + tid);
      if (P == kP3C5) {
        nqg = load_codes3(Lm.gate, off >> 3);
        nqu = load_codes3(Lm.up, off >> 3);
      }
    } else {
      load_chunk<P, false>(Lm.gate.seeds + grow * nbh, Lm.gate.coefs + grow * nbh,
                           P == 4 ? Lm.gate.codes + grow * (nbh / 2) : nullptr, nbh, c, fg, grow,
                           (size_t)Lm.gate.N);
      load_chunk<P, false>(Lm.up.seeds + grow * nbh, Lm.up.coefs + grow * nbh,
                           P == 4 ? Lm.up.codes + grow * (nbh / 2) : nullptr, nbh, c, fu, grow,
                           (size_t)Lm.up.N);
      kg = load_bias_key(Lm.gate, grow);
      ku = load_bias_key(Lm.up, grow);
    }
  };
  // ---- BA: a warp's phase A fields by bulk asynchronous copies: per matrix
  // one copy each of the step's seeds, coefficients and code words (the
  // lanes' chunks are consecutive, so their slots and the fields in global
  // memory are both contiguous), one lane a copy, all in one instruction,
  // completing on the warp's barrier of that buffer.  The row's exponent bias
  // goes to a register as the raw word (its scale key is formed when the step
  // is read, so nothing waits for the load here).  Copy n (counted over the
  // launch) lands in buffer n % 2, phase (n / 2) % 2.
  uint32_t nfetch = 0, nread = 0, nbg = 0, nbu = 0;
  auto a_fetch_bulk = [&](const LayerMats &Lm, const int32_t *expert, int step) {
    int slot, row, c;
    a_locate(step, slot, row, c);
    const int cb = c - lane, nch = min(32, p.Ch - cb);  // this step's chunks: cb .. cb + nch - 1
    const uint32_t r32 = (uint32_t)((size_t)expert[slot] * p.inter + row);
    nbg = in_bounds(r32, (size_t)Lm.gate.N, 4) ? (uint32_t)__ldg(Lm.gate.exp_bias + r32) : 0u;
    nbu = in_bounds(r32, (size_t)Lm.up.N, 4) ? (uint32_t)__ldg(Lm.up.exp_bias + r32) : 0u;
    if (P == kP3C5 && c < p.Ch) {
      const uint32_t off = r32 * (uint32_t)nbh + 8u * (uint32_t)c;
      nqg = load_codes3(Lm.gate, off >> 3);
      nqu = load_codes3(Lm.up, off >> 3);
    }
    const uint32_t buf = nfetch++ & 1u;
    const uint32_t bar = umma::smem_u32(&s_fbar[warp][buf]);
    const uint32_t sb = 16u * (uint32_t)nch, cbytes = (P == 4) ? 4u * (uint32_t)nch : 0u;
    const size_t first = (size_t)r32 * nbh + 8u * (uint32_t)cb;
    const bool inside = in_bounds(first + 8u * (uint32_t)nch - 1, (size_t)Lm.gate.N * nbh, 1) &&
                        in_bounds(r32, (size_t)Lm.gate.N, 2);
    __syncwarp();  // every lane has read the buffer's previous fields
    if (lane == 0) {
      if (inside)
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(2u * (2u * sb + cbytes))
                     : "memory");
      else
        umma::mbar_arrive(bar);  // nothing copied: the phase completes on the arrival alone
    }
    __syncwarp();  // the expected bytes are set before any copy completes
    constexpr int kFields = (P == 4) ? 3 : 2;  // seeds, coefficients (, code words) per matrix
    if (inside && lane < 2 * kFields) {
      const int m = lane / kFields, fld = lane - m * kFields;
      const nslm_seed_matrix &W = m ? Lm.up : Lm.gate;
      const int sl = (2 * (int)buf + m) * nthr + warp * 32;
      const void *dst = fld == 0 ? (const void *)(fs.s + sl) : fld == 1 ? (const void *)(fs.q + sl) : (const void *)(fs.c + sl);
      const void *src = fld == 0 ? (const void *)(W.seeds + first)
                        : fld == 1 ? (const void *)(W.coefs + first) : (const void *)(W.codes + first / 2);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                       umma::smem_u32(dst)),
                   "l"(src), "r"(fld == 2 ? cbytes : sb), "r"(bar)
                   : "memory");
    }
  };
  // wait for copy nread and read this lane's fields of it; false on timeout
  auto a_read_bulk = [&](ChunkFields &fg_, ChunkFields &fu_) {
    const uint32_t buf = nread & 1u, par = (nread >> 1) & 1u;
    ++nread;
    if (!umma::mbar_wait_bounded(umma::smem_u32(&s_fbar[warp][buf]), par, kBarrierWaitCycles)) return false;
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      ChunkFields &f = m ? fu_ : fg_;
      const int sl = (2 * (int)buf + m) * nthr + tid;
      const uint4 sv = fs.s[sl], qv = fs.q[sl];
      f.s[0] = sv.x; f.s[1] = sv.y; f.s[2] = sv.z; f.s[3] = sv.w;
      f.q[0] = qv.x; f.q[1] = qv.y; f.q[2] = qv.z; f.q[3] = qv.w;
      f.codes = (P == 4) ? fs.c[sl] : 0u;
    }
    return true;
  };

  // ---- table form: a warp's routed rows (tasks) and, per pass, one step a task
  auto f3_tasks = [&](int nslots) {
    const int ntask = nslots * p.inter;
    return gw < ntask ? (int)fdiv((uint32_t)(ntask - 1 - gw), p.div_W) + 1 : 0;
  };
  // copy the fields of task `it`, pass `pass` (lanes 0..15: chunks 16 pass + lane)
  auto f3_fetch = [&](const LayerMats &Lm, const int32_t *expert, int it, int pass, int buf) {
    if (lane >= kF3Positions / 8) return;
    const int t = gw + it * W;
    const int slot = (int)fdiv(t, p.div_inter), row = t - slot * p.inter;
    const uint32_t r32 = (uint32_t)((size_t)expert[slot] * p.inter + row);
    const uint32_t off = r32 * (uint32_t)nbh + 8u * (uint32_t)(16 * pass + lane);
    fetch_chunk_off<P>(Lm.gate, off, r32, fs, (2 * buf) * nthr + tid);
    fetch_chunk_off<P>(Lm.up, off, r32, fs, (2 * buf + 1) * nthr + tid);
  };

  // ---- phase B task geometry (row, routed expert, chunk) of this CTA's rows
  auto b_locate = [&](int t, FastDiv dSC, int SC, int &r, int &s, int &c, int &q) {
    r = (int)fdiv(t, dSC);
    q = t - r * SC;
    s = (int)fdiv(q, p.div_Ci);
    c = q - s * p.Ci;
  };
  auto b_fetch = [&](const LayerMats &Lm, FastDiv dSC, int SC, int t, int buf, ChunkFields &f,
                     uint32_t &k) {
    int r, s, c, q;
    b_locate(t, dSC, SC, r, s, c, q);
    const size_t grow = (size_t)s_expert[s] * p.hidden + n0 + r;
    if (VEC) {
      const uint32_t r32 = (uint32_t)grow;
      fetch_chunk_off<P>(Lm.down, r32 * (uint32_t)nbi + 8u * (uint32_t)c, r32, fs, buf * nthr + tid);
      if (P == kP3C5) nqd = load_codes3(Lm.down, r32 * (uint32_t)(nbi >> 3) + (uint32_t)c);
    } else {
      load_chunk<P, false>(Lm.down.seeds + grow * nbi, Lm.down.coefs + grow * nbi,
                           P == 4 ? Lm.down.codes + grow * (nbi / 2) : nullptr, nbi, c, f, grow,
                           (size_t)Lm.down.N);
      k = load_bias_key(Lm.down, grow);
    }
  };

  // register copies of the next fields on the ragged path (unused when VEC)
  ChunkFields fg, fu, fd;
  uint32_t kg = 0, ku = 0, kd = 0;
  uint32_t nbar = 0;  // barriers passed in this launch

  // the barriers, initialised and fenced by one thread before any copy uses them
  if (tid == 0) {
    umma::mbar_init(umma::smem_u32(&s_hbar), 1);
    if (BA)
      for (int w = 0; w < nwarps; ++w)
        for (int b = 0; b < 2; ++b) umma::mbar_init(umma::smem_u32(&s_fbar[w][b]), 1);
    umma::mbar_init_fence();
  }
  __syncthreads();
  // first fields of layer 0, phase A, straight from the plan in global memory
  if (F3) {
    if (f3_tasks(min(p.plans->n_slots, kMaxK)) > 0) f3_fetch(p.layer[0], p.plans->expert, 0, 0, 0);
  } else if (a_steps(min(p.plans->n_slots, kMaxK)) > 0) {
    if (BA)
      a_fetch_bulk(p.layer[0], p.plans->expert, 0);
    else
      a_fetch(p.layer[0], p.plans->expert, 0, 0, fg, fu, kg, ku);
  }
  if (VEC) cp_async_commit();
  // the plans, by the highest threads, while the lowest stage layer 0's input
  for (int i = nthr - 1 - tid; i < p.n * kMaxK; i += nthr) {
    const int l = i / kMaxK, j = i - l * kMaxK;
    const SlotPlan *pl = p.plans + l;
    const int ns = pl->n_slots, st = pl->start[j], ex = pl->expert[j];  // j < kMaxK: in the arrays
    if (j == 0) s_pl_n[l] = min(ns, kMaxK);
    if (j < ns) {
      const int pr = pl->pair[st];
      s_pl_expert[l][j] = ex;
      s_pl_pair[l][j] = pr;
      s_pl_w[l][j] = pl->w[pr];
    }
  }
  if (p.x0) {  // layer 0's input, bf16 -> fp32 chunk-major (table form: in order)
    const uint4 *row = reinterpret_cast<const uint4 *>(p.x0);
    for (int b = tid; b < nbh; b += nthr) {
      float4 lo, hi;
      bf16x8_to_f32(__ldg(row + b), lo, hi);
      if (F3) {
        reinterpret_cast<float4 *>(xplain)[2 * b] = lo;
        reinterpret_cast<float4 *>(xplain)[2 * b + 1] = hi;
      } else {
        cm_store_block(xs4, xn2, b, lo, hi);
      }
    }
  }
  build_stream_tables_rep<kTabCopies>(tab);
  __syncthreads();  // tables, plans, layer 0's input

  for (int l = 0; l < p.n; ++l) {
    const LayerMats &Lm = p.layer[l];
    const uint32_t g = p.l0 + (uint32_t)l;  // index of this layer in the stack
    __syncthreads();  // plan and staging reuse
    if (tid < s_pl_n[l]) {
      s_expert[tid] = s_pl_expert[l][tid];
      s_pair[tid] = s_pl_pair[l][tid];
      s_w[tid] = s_pl_w[l][tid];
    }
    if (tid == 0) s_nslots = s_pl_n[l];
    NSLM_TRACE(0, false);  // layer start

    // =========================== phase A: gate/up + SiLU
    // layer 0's input was staged at the start
    const bool staged =
        g == 0 || stage_norm_tagged<F3>(F3 ? reinterpret_cast<float4 *>(xplain) : xs4, xn2, p.ytag, g,
                                        gridDim.x, p.hidden, p.sync, scratch);
    if (__syncthreads_or(!staged)) break;
    NSLM_TRACE(1, false);  // x staged
    if (F3) {
      // the table form: per pass of 128 block positions, the CTA builds their
      // tables, then every warp runs its tasks over them; lane partial sums
      // carry over passes in shared memory, so every row sums in one order
      const int ntk = f3_tasks(s_nslots);
      float2 *part = f3part + warp * kF3MaxTasks * 32 + lane;
      for (int pass = 0; pass < p.f3_np; ++pass) {
        if (pass > 0) __syncthreads();  // the previous pass's tables are read
        f3_build(f3tab, f3cst, xplain + pass * kF3Positions * 8, tid, nthr);
        __syncthreads();
        float a0h[2][2], yh[2][2];
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const float2 c = f3cst[64 * i + 2 * lane + t];
            a0h[i][t] = c.x;
            yh[i][t] = c.y;
          }
        for (int it = 0; it < ntk; ++it) {
          const int step = pass * ntk + it;
          __syncwarp();  // every lane has read the buffer the next copies refill
          if (it + 1 < ntk) f3_fetch(Lm, s_expert, it + 1, pass, (step + 1) & 1);
          else if (pass + 1 < p.f3_np) f3_fetch(Lm, s_expert, 0, pass + 1, (step + 1) & 1);
          cp_async_commit();
          cp_async_wait<1>();
          __syncwarp();  // the step's copies, made by lanes 0..15, seen by all
          const float pg = f3_row<P>(tl, fs, (2 * (step & 1)) * nthr + warp * 32, lane, f3tab, a0h, yh);
          const float pu = f3_row<P>(tl, fs, (2 * (step & 1) + 1) * nthr + warp * 32, lane, f3tab, a0h, yh);
          if (pass == 0) {
            part[it * 32] = make_float2(pg, pu);
          } else {
            const float2 o = part[it * 32];
            part[it * 32] = make_float2(o.x + pg, o.y + pu);
          }
        }
      }
      for (int it = 0; it < ntk; ++it) {
        const float2 v = part[it * 32];
        const float gs = warp_sum(v.x), us = warp_sum(v.y);
        const int t = gw + it * W;
        const int slot = (int)fdiv(t, p.div_inter), row = t - slot * p.inter;
        if (lane == 0 && in_bounds((size_t)s_pair[slot], (size_t)p.h_rows, 10))
          __stcg(p.h + (size_t)s_pair[slot] * p.inter + row, __fdividef(gs, 1.f + __expf(-gs)) * us);
      }
    } else {
      const int nsteps = a_steps(s_nslots);
      float2 ag = make_float2(0.f, 0.f), au = make_float2(0.f, 0.f);
      bool aok = true;
      for (int step = 0; step < nsteps; ++step) {
        int slot, row, c;
        a_locate(step, slot, row, c);
        ChunkFields cg = fg, cu = fu;
        uint32_t ckg = kg, cku = ku;
        if (BA) {
          ckg = row_scale_key((int32_t)nbg);
          cku = row_scale_key((int32_t)nbu);
          const uint32_t cqg = nqg, cqu = nqu;  // this step's 5-bit-format code bits
          if (!a_read_bulk(cg, cu)) {
            if (lane == 0) {
              atomicExch(p.sync + 2, 1);
              atomicCAS(p.sync, 0, 1);
            }
            aok = false;
            break;
          }
          if (P == kP3C5) {
            cg.codes = cqg;
            cu.codes = cqu;
          }
          if (step + 1 < nsteps) a_fetch_bulk(Lm, s_expert, step + 1);
        } else if (VEC) {
          const uint32_t cqg = nqg, cqu = nqu;  // this step's 5-bit-format code bits
          if (step + 1 < nsteps) a_fetch(Lm, s_expert, step + 1, (step + 1) & 1, fg, fu, kg, ku);
          cp_async_commit();
          cp_async_wait<1>();
          read_chunk<P>(fs, (2 * (step & 1)) * nthr + tid, cg, ckg);
          read_chunk<P>(fs, (2 * (step & 1) + 1) * nthr + tid, cu, cku);
          if (P == kP3C5) {
            cg.codes = cqg;
            cu.codes = cqu;
          }
        } else if (step + 1 < nsteps) {
          a_fetch(Lm, s_expert, step + 1, 0, fg, fu, kg, ku);
        }
        if (c < p.Ch) {
          const int nvalid = VEC ? 8 : min(8, nbh - 8 * c);
          chunk_dot2_cm<P, VEC, kTabCopies>(tl, cg, cu, nvalid, ckg, cku, xs4 + kCmX4 * c, xn2 + kCmXn * c, ag, au);
        }
        if (p.J == 1 || c + 32 >= 32 * p.J) {
          const float g = warp_sum(ag.x + ag.y), u = warp_sum(au.x + au.y);
          // SiLU with the fast exp and divide (relative error ~1e-6; an exp
          // that overflows gives the limit 0)
          if (lane == 0 && in_bounds((size_t)s_pair[slot], (size_t)p.h_rows, 10))
            __stcg(p.h + (size_t)s_pair[slot] * p.inter + row, __fdividef(g, 1.f + __expf(-g)) * u);
          ag = au = make_float2(0.f, 0.f);
        }
      }
      if (BA && __syncthreads_or(!aok)) break;
    }
    NSLM_TRACE(2, true);  // this CTA's phase A done
    // arrive; fetch phase B's first fields (weights only) while the others arrive
    const int SC = s_nslots * p.Ci;
    const int bt = nrows * SC;
    grid_arrive(p.sync);
    if (VEC) cp_async_wait<0>();
    if (tid < bt) b_fetch(Lm, p.div_SC[s_nslots], SC, tid, 0, fd, kd);
    if (VEC) cp_async_commit();
    if (!stack_wait(p, nbar++, &s_ok)) break;
    NSLM_TRACE(3, false);  // past the grid barrier

    // =========================== phase B: down + weighted combine
    {
      const FastDiv dSC = p.div_SC[s_nslots];
      const int nhb = s_nslots * nbi;
      if (VEC) {
        // all routed h chunks (64 values, 256 contiguous bytes each, as is
        // their chunk-major slot) by bulk asynchronous copies completing on
        // s_hbar; then the block sums from shared memory
        const int nch = s_nslots * p.Ci;
        const uint32_t hbar = umma::smem_u32(&s_hbar);
        if (tid == 0) {
          asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(hbar),
                       "r"((uint32_t)nch * 256u) : "memory");
        }
        for (int q = tid; q < nch; q += nthr) {
          const int s = (int)fdiv(q, p.div_Ci), c = q - s * p.Ci;
          const float *src = p.h + (size_t)s_pair[s] * p.inter + 64 * c;
          asm volatile("fence.proxy.async.global;" ::: "memory");
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], 256, [%2];"
                       ::"r"(umma::smem_u32(xs4 + kCmX4 * q)), "l"(src), "r"(hbar) : "memory");
        }
        const bool hok = umma::mbar_wait_bounded(hbar, (uint32_t)(l & 1), kBarrierWaitCycles);
        if (!hok && tid == 0) {
          atomicExch(p.sync + 2, 1);
          atomicCAS(p.sync, 0, 1);
        }
        if (__syncthreads_or(!hok)) break;
        for (int i = tid; i < nhb; i += nthr) {
          const int q = i >> 3, b = i & 7;  // chunk-major: blocks of a chunk consecutive
          const float4 lo = xs4[kCmX4 * q + 2 * b], hi = xs4[kCmX4 * q + 2 * b + 1];
          const float sum = ((lo.x + lo.y) + (lo.z + lo.w)) + ((hi.x + hi.y) + (hi.z + hi.w));
          xn2[kCmXn * q + b] = make_float2(-kMagic2 * sum, 0.f);
        }
      } else {
        // all routed h blocks, two per thread per round with both loads in flight
        for (int i = tid; i < nhb; i += 2 * nthr) {
          const int i2 = i + nthr;
          const int s = (int)fdiv(i, p.div_nbi), b = i - s * nbi;
          const float4 *src = reinterpret_cast<const float4 *>(p.h + (size_t)s_pair[s] * p.inter) + 2 * b;
          const float4 a0 = __ldcg(src), a1 = __ldcg(src + 1);
          float4 c0, c1;
          int s2 = 0, b2 = 0;
          if (i2 < nhb) {
            s2 = (int)fdiv(i2, p.div_nbi);
            b2 = i2 - s2 * nbi;
            const float4 *src2 = reinterpret_cast<const float4 *>(p.h + (size_t)s_pair[s2] * p.inter) + 2 * b2;
            c0 = __ldcg(src2);
            c1 = __ldcg(src2 + 1);
          }
          cm_store_block(xs4, xn2, s * p.Ci * 8 + b, a0, a1);
          if (i2 < nhb) cm_store_block(xs4, xn2, s2 * p.Ci * 8 + b2, c0, c1);
        }
      }
      __syncthreads();
      NSLM_TRACE(5, false);  // h staged
      for (int t = tid, it = 0; t < bt; t += nthr, ++it) {
        int r, s, c, q;
        b_locate(t, dSC, SC, r, s, c, q);
        ChunkFields cf = fd;
        uint32_t ck = kd;
        if (VEC) {
          const uint32_t cqd = nqd;  // this task's 5-bit-format code bits
          if (t + nthr < bt) b_fetch(Lm, dSC, SC, t + nthr, (it + 1) & 1, fd, kd);
          cp_async_commit();
          cp_async_wait<1>();
          read_chunk<P>(fs, (it & 1) * nthr + tid, cf, ck);
          if (P == kP3C5) cf.codes = cqd;
        } else if (t + nthr < bt) {
          b_fetch(Lm, dSC, SC, t + nthr, 0, fd, kd);
        }
        float2 acc = make_float2(0.f, 0.f);
        const int nvalid = VEC ? 8 : min(8, nbi - 8 * c);
        chunk_dot_cm<P, VEC, kTabCopies>(tl, cf, nvalid, ck, xs4 + kCmX4 * q, xn2 + kCmXn * q, acc);
        red[t] = s_w[s] * (acc.x + acc.y);
      }
      NSLM_TRACE(6, false);  // thread 0's phase B tasks done
      __syncthreads();
      // the stack's output in plain fp32; between layers tagged words
      const bool last = l == p.n - 1 && p.y_out;
      float *rowy = red + p.rpc * p.stage_slots;  // this CTA's outputs, for the norm partial
      for (int r = warp; r < nrows; r += nwarps) {
        float sum = 0.f;
        for (int q = lane; q < SC; q += 32) sum += red[r * SC + q];
        sum = warp_sum(sum);
        if (lane == 0) {
          if (last)
            __stcg(p.y_out + n0 + r, sum);
          else
            st_tagged(p.ytag + n0 + r, sum, g + 1);
          rowy[r] = sum;
        }
      }
      if (!last) {
        __syncthreads();
        if (warp == 0) {  // sum of squares of this CTA's rows, fixed order
          float ss = 0.f;
          for (int r = lane; r < nrows; r += 32) ss = fmaf(rowy[r], rowy[r], ss);
          ss = warp_sum(ss);
          if (lane == 0) st_tagged(p.ytag + p.hidden + blockIdx.x, ss, g + 1);
        }
      }
    }
    NSLM_TRACE(4, true);  // this CTA's phase B done (y and its sum of squares stored)
    if (l + 1 == p.n) break;
    // the next layer's first phase A fields, in flight while its input arrives
    if (VEC) cp_async_wait<0>();
    if (F3) {
      if (f3_tasks(s_pl_n[l + 1]) > 0) f3_fetch(p.layer[l + 1], s_pl_expert[l + 1], 0, 0, 0);
    } else if (a_steps(s_pl_n[l + 1]) > 0) {
      if (BA)
        a_fetch_bulk(p.layer[l + 1], s_pl_expert[l + 1], 0);
      else
        a_fetch(p.layer[l + 1], s_pl_expert[l + 1], 0, 0, fg, fu, kg, ku);
    }
    if (VEC) cp_async_commit();
  }
  if (VEC) cp_async_wait<0>();
}

}  // namespace

// ---------------------------------------------------------------------- host

static int stack1_rows_per_cta(const FfnDims &d) { return std::max(1, ceil_div(d.hidden, num_sms())); }

// Threads per CTA: whole warps in [16, kStack1MaxThreads / 32] that leave the
// fewest idle task slots in both phases (a phase A task is 16 blocks per
// lane, a phase B task 8); on a tie the most warps.  Measured on B200 for the
// 100-expert 2048/1408 layer: 20 warps 33.6 us, 16 warps 33.8, 14 warps 36.6,
// 11 warps 35.7, 26 warps (72 registers) 37.0 per layer: the unrolled block
// loop needs ~96 registers to overlap its table lookups and dot products, and
// fewer than 16 warps cannot hide the remaining latency.
static int stack1_threads(const FfnDims &d, int k) {
  const int sms = num_sms();
  const int Ch = ceil_div(d.hidden / 8, 8), Ci = ceil_div(d.inter / 8, 8);
  const int J = ceil_div(Ch, 32);
  const long long a_tasks = (long long)k * d.inter * J;
  const long long b_tasks = (long long)stack1_rows_per_cta(d) * k * Ci;
  int best = 16;
  long long best_cost = -1;
  for (int nw = kStack1MaxThreads / 32; nw >= 16; --nw) {
    const long long ra = (a_tasks + (long long)sms * nw - 1) / ((long long)sms * nw);
    const long long rb = (b_tasks + 32ll * nw - 1) / (32ll * nw);
    const long long cost = (16 * ra + 8 * rb) * nw;
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = nw;
    }
  }
  return 32 * best;
}

// The table form of phase A is an ablation build (-DNSLM_STACK1_F3=1, the
// "tableform" library variant): measured on B200 for the 100-expert
// 2048/1408 layer it executes ~85 warp instructions per phase A block against
// the direct form's ~77 (the byte permutes, int -> float conversions and
// address arithmetic of six lookups outweigh the eight dot products they
// replace), 38.1 against 36.0 us per layer.
#ifndef NSLM_STACK1_F3
#define NSLM_STACK1_F3 0
#endif
#ifndef NSLM_STACK1_BULK_A
#define NSLM_STACK1_BULK_A 1  // phase A's weight fields by bulk copies where they apply
#endif

// Bytes of the staging region: chunk-major x (phase A) and h (phase B), or
// with the table form the tables, constants, partial sums and x in order.
static size_t stack1_region_bytes(const FfnDims &d, int k, int threads, bool f3) {
  const int Ch = ceil_div(d.hidden / 8, 8), Ci = ceil_div(d.inter / 8, 8);
  const int slots = std::max(Ch, k * Ci);
  size_t r = cm_bytes(slots) + (size_t)(slots & 1) * sizeof(float2);
  if (f3)
    r = std::max(r, (size_t)kF3TableBytes + kF3Positions * sizeof(float2) +
                        (size_t)(threads / 32) * kF3MaxTasks * 32 * sizeof(float2) + (size_t)d.hidden * sizeof(float));
  return (r + 15) / 16 * 16;
}

static size_t stack1_smem(const FfnDims &d, int k, int threads, bool f3 = false) {
  const int Ch = ceil_div(d.hidden / 8, 8), Ci = ceil_div(d.inter / 8, 8);
  const int slots = std::max(Ch, k * Ci);
  return kTabCopies * sizeof(StreamTables) + stack1_region_bytes(d, k, threads, f3) +
         FieldSlots::bytes(4 * threads) + (size_t)stack1_rows_per_cta(d) * (slots + 1) * sizeof(float);
}

// Whether phase A takes the table form: whole chunks of P = 3 or 4, passes of
// 128 block positions, at most kF3MaxTasks routed rows per warp, and room.
static bool stack1_f3(const FfnDims &d, int k, int threads) {
  if (!NSLM_STACK1_F3 || (d.P != 3 && d.P != 4)) return false;
  if (d.hidden % (8 * kF3Positions) || d.inter % 64) return false;
  const long long warps = (long long)num_sms() * (threads / 32);
  if (((long long)k * d.inter + warps - 1) / warps > kF3MaxTasks) return false;
  return stack1_smem(d, k, threads, true) <= 210 * 1024;
}

bool stack1_supported(const FfnDims &d, int k) {
  if (k < 1 || k > kMaxK) return false;
  if (d.P != 3 && d.P != 4 && d.P != kP3C5) return false;
  // 32-bit element offsets into the field streams
  if ((int64_t)d.E * d.inter * (d.hidden / 8) >= (1ll << 31) || (int64_t)d.E * d.hidden * (d.inter / 8) >= (1ll << 31))
    return false;
  // fast divisions: divisors below 2^16, dividends below 2^22
  if (d.inter >= (1 << 16) || d.hidden >= (1 << 16)) return false;
  if ((int64_t)k * ceil_div(d.inter / 8, 8) >= (1 << 16)) return false;
  if ((int64_t)k * d.inter * ceil_div(d.hidden / 64, 32) >= (1 << 22)) return false;
  // dynamic shared memory plus ~7 KB of static (the per-layer plans) within 227 KB
  return stack1_smem(d, k, stack1_threads(d, k)) <= 220 * 1024;
}

template <int P, bool VEC, bool F3, bool BA>
static int32_t launch_stack1_t(const FfnDims &d, const nslm_moe_layer *layers, int n,
                               const SlotPlan *plans, const uint16_t *x0, int k, float *h,
                               uint64_t *ytag, float *y_out, int32_t *sync, cudaStream_t s,
                               int &launches) {
  const int threads = stack1_threads(d, k);
  const size_t smem = stack1_smem(d, k, threads, F3);
  auto kern = stack1_kernel<P, VEC, F3, BA>;
  int32_t st = ensure_smem((const void *)kern, smem);
  if (st) return st;
  const int per_sm = max_active_ctas((const void *)kern, threads, smem);
  const int grid = num_sms() * per_sm;
  Stack1Params p{};
  p.h = h;
  p.h_rows = k;
  p.ytag = ytag;
  p.sync = sync;
  p.hidden = d.hidden;
  p.inter = d.inter;
  p.Ch = ceil_div(d.hidden / 8, 8);
  p.Ci = ceil_div(d.inter / 8, 8);
  p.J = ceil_div(p.Ch, 32);
  p.rpc = ceil_div(d.hidden, grid);
  p.stage_slots = std::max(p.Ch, k * p.Ci);
  p.region_bytes = (int32_t)stack1_region_bytes(d, k, threads, F3);
  p.f3_np = F3 ? d.hidden / (8 * kF3Positions) : 0;
  p.div_W = make_fastdiv((uint32_t)(grid * (threads / 32)));
  if (F3 && ((long long)k * d.inter + (long long)grid * (threads / 32) - 1) / ((long long)grid * (threads / 32)) >
                kF3MaxTasks)
    return NSLM_ERR_SHAPE;
  p.div_inter = make_fastdiv((uint32_t)d.inter);
  p.div_J = make_fastdiv((uint32_t)p.J);
  p.div_Ci = make_fastdiv((uint32_t)p.Ci);
  p.div_nbi = make_fastdiv((uint32_t)(d.inter / 8));
  for (int S = 1; S <= kMaxK; ++S) p.div_SC[S] = make_fastdiv((uint32_t)(S * p.Ci));
  p.div_SC[0] = p.div_SC[1];
  if (p.rpc > stack1_rows_per_cta(d) || grid > kMaxStack1Ctas) return NSLM_ERR_SHAPE;
  // chunks of kMaxFusedLayers layers; barrier arrivals keep counting across them
  uint32_t base = 0;
  for (int l0 = 0; l0 < n; l0 += kMaxFusedLayers) {
    const int m = std::min(kMaxFusedLayers, n - l0);
    p.plans = plans + l0;
    p.x0 = l0 == 0 ? x0 : nullptr;
    p.y_out = (l0 + m == n) ? y_out : nullptr;
    p.n = m;
    p.l0 = (uint32_t)l0;
    p.barrier_base = base;
    for (int i = 0; i < m; ++i)
      p.layer[i] = LayerMats{layers[l0 + i].gate, layers[l0 + i].up, layers[l0 + i].down};
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    ensure_stream_source(s);
    if ((st = cuda_status(cudaLaunchKernelEx(&cfg, kern, p)))) return st;
    ++launches;
    base += (uint32_t)m * (uint32_t)grid;  // one grid barrier per layer
  }
  return NSLM_OK;
}

int32_t launch_stack1(const FfnDims &d, const nslm_moe_layer *layers, int n, const SlotPlan *plans,
                      const uint16_t *x0, int k, float *h, uint64_t *ytag, float *y_out, int32_t *sync,
                      cudaStream_t s, int &launches) {
  if (!x0 || !ytag) return NSLM_ERR_ARG;
  const bool vec = d.hidden % 64 == 0 && d.inter % 64 == 0;
  const bool f3 = vec && stack1_f3(d, k, stack1_threads(d, k));
  // phase A fields by bulk copies: whole chunks whose P = 4 code words make
  // 16-byte multiples (hidden % 256 == 0)
  const bool ba = vec && !f3 && NSLM_STACK1_BULK_A && d.hidden % 256 == 0;
#define NSLM_L(P_, V_, F_, B_) \
  launch_stack1_t<P_, V_, F_, B_>(d, layers, n, plans, x0, k, h, ytag, y_out, sync, s, launches)
  if (d.P == kP3C5) return ba ? NSLM_L(kP3C5, true, false, true) : NSLM_L(kP3C5, true, false, false);
  if (d.P == 4)
    return f3 ? NSLM_L(4, true, true, false) : ba ? NSLM_L(4, true, false, true)
               : vec ? NSLM_L(4, true, false, false) : NSLM_L(4, false, false, false);
  return f3 ? NSLM_L(3, true, true, false) : ba ? NSLM_L(3, true, false, true)
            : vec ? NSLM_L(3, true, false, false) : NSLM_L(3, false, false, false);
#undef NSLM_L
}

NSLM_BOUNDS_ACCESSOR(stack1)

}  // namespace nslm

// The trace build's stamps (see NSLM_STACK1_TRACE), copied to host memory.
extern "C" int32_t nslm_debug_stack_trace(uint64_t *out, size_t n_words) {
#if NSLM_STACK1_TRACE
  if (!out) return NSLM_ERR_ARG;
  if (n_words < (size_t)nslm::kTraceStamps * nslm::kTraceCtas * nslm::kTraceLayers) return NSLM_ERR_SHAPE;
  if (int32_t st = nslm::check_device()) return st;
  return nslm::cuda_status(cudaMemcpyFromSymbol(out, nslm::g_stack1_trace, sizeof(nslm::g_stack1_trace)));
#else
  (void)out;
  (void)n_words;
  return NSLM_ERR_UNSUPPORTED;
#endif
}
