// gemv.cu -- nslm_seed_gemv: the decode matrix-vector product with the
// weights regenerated from their seeds in registers ("NanoSeedLM: LLM
// inference using pseudo-random numbers", "What I changed: September 2026":
// weights are rebuilt inside the GPU kernels, in registers, every time).
//
// A CTA owns R rows x Cpad chunk slots (one thread per (row, chunk)); it
// loops over row groups (grid-stride), so the activations are staged into
// shared memory once per CTA.  Partial sums of the chunks of a row are added
// in shared memory (fixed order, so results are deterministic).
#include <type_traits>
#include <algorithm>

#include "chunk.cuh"
#include "common.cuh"
#include "persist.cuh"

namespace nslm {

struct GemvParams {
  const uint16_t *seeds;
  const uint16_t *coefs;
  const uint8_t *codes;
  const int32_t *exp_bias;
  const uint16_t *x;
  float *y;
  int32_t N, K, nb, M;
  int32_t R, C, Cpad, groups;
};

template <int P, int M, bool VEC, int CPAD>
__global__ void __launch_bounds__(512) seed_gemv_kernel(const GemvParams p) {
  extern __shared__ float4 smem4[];
  const int cpad = CPAD ? CPAD : p.Cpad;
  StreamTables *tab = reinterpret_cast<StreamTables *>(smem4);
  float4 *xs4 = smem4 + sizeof(StreamTables) / 16;
  float2 *xn2 = reinterpret_cast<float2 *>(xs4 + (size_t)M * 16 * cpad);
  float *red = reinterpret_cast<float *>(xn2 + (size_t)M * 8 * cpad);
  const int tid = threadIdx.x, nthr = blockDim.x;

  build_stream_tables(tab);
  // launched with programmatic stream serialization (as the one-vector
  // kernel): wait for the preceding kernel before the first global read
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");
  stage_bf16(xs4, xn2, p.x, nullptr, M, p.K, cpad);
  __syncthreads();

  const int rr = tid / cpad, ch = tid - rr * cpad;
  int iter = 0;
  for (int g = blockIdx.x; g < p.groups; g += gridDim.x, ++iter) {
    const int row = g * p.R + rr;
    float acc[M];
#pragma unroll
    for (int m = 0; m < M; ++m) acc[m] = 0.f;
    if (row < p.N && ch < p.C) {
      ChunkFields f;
      load_chunk<P, VEC>(p.seeds + (size_t)row * p.nb, p.coefs + (size_t)row * p.nb,
                         P == 4    ? p.codes + (size_t)row * (p.nb / 2)
                         : P == 35 ? p.codes + (size_t)row * (3 * p.nb / 8)
                                   : nullptr,
                         p.nb, ch, f, (size_t)row, (size_t)p.N);
      const uint32_t rowk = row_scale_key(__ldg(p.exp_bias + row));
      chunk_dot<P, M, VEC, CPAD>(tab, f, p.nb, ch, rowk, xs4, xn2, cpad, 0, acc);
    }
    float *rb = red + (size_t)(iter & 1) * M * nthr;
#pragma unroll
    for (int m = 0; m < M; ++m) rb[m * nthr + tid] = acc[m];
    __syncthreads();
    reduce_rows(rb, M, p.R, cpad, p.C, [&](int m, int r2, float sum) {
      const int orow = g * p.R + r2;
      if (orow < p.N) p.y[(size_t)m * p.N + orow] = sum;
    });
  }
}

static size_t gemv_smem(int M, int Cpad, int threads) {
  return sizeof(StreamTables) + staged_bytes(M, Cpad) + (size_t)2 * M * threads * sizeof(float);
}

template <int P, int M, bool VEC, int CPAD>
static int32_t launch_gemv(const GemvParams &p, int grid, int threads, size_t smem,
                           cudaStream_t s) {
  auto k = seed_gemv_kernel<P, M, VEC, CPAD>;
  if (int32_t st = ensure_smem((const void *)k, smem)) return st;
  ensure_stream_source(s);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3((unsigned)threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (int32_t st = cuda_status(cudaLaunchKernelEx(&cfg, k, p))) return st;
  return launch_status();
}

template <int P, int M>
static int32_t dispatch_cpad(const GemvParams &p, bool vec, int grid, int threads, size_t smem,
                             cudaStream_t s) {
  if (!vec) return launch_gemv<P, M, false, 0>(p, grid, threads, smem, s);
  if (M == 1) {
    switch (p.Cpad) {
      case 16: return launch_gemv<P, M, true, 16>(p, grid, threads, smem, s);
      case 24: return launch_gemv<P, M, true, 24>(p, grid, threads, smem, s);
      case 32: return launch_gemv<P, M, true, 32>(p, grid, threads, smem, s);
      case 64: return launch_gemv<P, M, true, 64>(p, grid, threads, smem, s);
      default: break;
    }
  }
  return launch_gemv<P, M, true, 0>(p, grid, threads, smem, s);
}

template <int P>
static int32_t dispatch_gemv(const GemvParams &p, bool vec, int grid, int threads, size_t smem,
                             cudaStream_t s) {
  switch (p.M) {
    case 1: return dispatch_cpad<P, 1>(p, vec, grid, threads, smem, s);
    case 2: return dispatch_cpad<P, 2>(p, vec, grid, threads, smem, s);
    case 3: return dispatch_cpad<P, 3>(p, vec, grid, threads, smem, s);
    case 4: return dispatch_cpad<P, 4>(p, vec, grid, threads, smem, s);
    case 5: return dispatch_cpad<P, 5>(p, vec, grid, threads, smem, s);
    case 6: return dispatch_cpad<P, 6>(p, vec, grid, threads, smem, s);
    case 7: return dispatch_cpad<P, 7>(p, vec, grid, threads, smem, s);
    default: return dispatch_cpad<P, 8>(p, vec, grid, threads, smem, s);
  }
}

// ------------------------------------------------------------- M = 1, whole chunks
//
// The single-vector product is latency-bound at expert sizes (1-5 MB of
// fields, a few microseconds), so this kernel issues its first weight copies
// before anything else, keeps the next task's fields in flight (cp.async into
// per-thread shared-memory slots) and has no barrier between tasks.  A CTA
// owns a range of rows; its threads take (row, chunk) tasks, partial sums go
// to shared memory and one warp per row adds them in a fixed order.
// CTAS = 2: the rows are split over two CTAs per SM of at most 14 warps (up
// to 72 registers each).  Two smaller CTAs end at different times, so the
// next GEMV's CTAs (launched early by programmatic dependent launch) take an
// SM's free slot sooner, and the unrolled block loop gets the registers to
// overlap its table lookups.  Measured on B200 in a chain of GEMVs with
// NSLM_GEMV_FIELDS_READY: 2048x4096 P=4 5.07 us with one CTA of up to 32
// warps per SM, 4.69 with two; 512x1024 3.25 -> 2.71 us.
// CTAS = 1: one CTA of up to 32 warps (48 registers) per SM, for rows so long
// that two CTAs' shared memory does not fit on an SM; there the extra warps
// pay (2048x16384 P=4: 14.9 us against 15.3 with 14 warps, P=3 with 5-bit
// coefficients 15.6 against 17.4).

template <int CTAS> struct Gemv1Shape;
template <> struct Gemv1Shape<2> { static constexpr int kThreads = 448, kMinCtas = 2; };
template <> struct Gemv1Shape<1> { static constexpr int kThreads = 1024, kMinCtas = 0; };  // 0: no minimum
constexpr size_t kSmemPerSm = 228 * 1024;     // shared memory of one B200 SM
constexpr size_t kSmemReservedPerCta = 1024;  // of which the system takes per resident CTA

struct Gemv1Params {
  nslm_seed_matrix W;
  const uint16_t *x;
  float *y;
  int32_t C;     // chunks per row (K / 64)
  int32_t rpc;   // rows per CTA
  FastDiv div_C;
};

// EARLY: the caller has declared that no kernel before this one on the stream
// writes the matrix's fields, so the first task's field copies are issued
// before griddepcontrol.wait and overlap the tail of the preceding kernel;
// the activations are read, and y written, only after the wait.
template <int P, bool EARLY, int CTAS>
__global__ void __launch_bounds__(Gemv1Shape<CTAS>::kThreads, Gemv1Shape<CTAS>::kMinCtas) gemv1_kernel(const Gemv1Params p) {
  extern __shared__ float4 smem4[];
  const int tid = threadIdx.x, nthr = blockDim.x, warp = tid >> 5, lane = tid & 31;
  StreamTables *tab = reinterpret_cast<StreamTables *>(smem4);
  const FieldSlots fs(smem4 + sizeof(StreamTables) / 16, 2 * nthr);  // [2 buffers][threads]
  float4 *xs4 = reinterpret_cast<float4 *>(fs.b + 2 * nthr);
  float2 *xn2 = reinterpret_cast<float2 *>(xs4 + (size_t)kCmX4 * p.C);
  float *red = reinterpret_cast<float *>(xn2 + (size_t)kCmXn * p.C + (p.C & 1));
  const int n0 = blockIdx.x * p.rpc;
  const int nrows = max(0, min(p.rpc, p.W.N - n0));
  const int ntask = nrows * p.C;
  const int nb = p.W.K >> 3;
  // the 5-bit format's code bits (3 bytes per chunk, not 4-byte aligned) come
  // by plain loads into one register per buffer, one task ahead like the rest
  uint32_t cq0 = 0, cq1 = 0;
  auto fetch = [&](int t, int buf) {
    const uint32_t r = fdiv((uint32_t)t, p.div_C), c = (uint32_t)t - r * (uint32_t)p.C;
    const uint32_t row = (uint32_t)n0 + r;
    fetch_chunk_off<P>(p.W, row * (uint32_t)nb + 8u * c, row, fs, buf * nthr + tid);
    if (P == kP3C5) {
      const uint8_t *cb = p.W.codes + (size_t)row * (3u * (uint32_t)nb / 8u) + 3u * c;
      const uint32_t v = (uint32_t)__ldcs(cb) | ((uint32_t)__ldcs(cb + 1) << 8) | ((uint32_t)__ldcs(cb + 2) << 16);
      if (buf) cq1 = v;
      else cq0 = v;
    }
  };
  // launched with programmatic stream serialization: wait here for the
  // preceding kernel (its writes of W or x; with EARLY only of x), then let
  // the next one launch
  if (EARLY) {  // the stream tables come from constant data: built before the wait too
    if (tid < ntask) fetch(tid, 0);
    cp_async_commit();
    for (int i = tid; i < 512; i += nthr) tab->t[i] = kStreamTab.t[i];
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");
  if (!EARLY) {
    if (tid < ntask) fetch(tid, 0);
    cp_async_commit();
  }
  // stream tables and activations: every load in flight before the first store
  {
    const uint4 *xrow = reinterpret_cast<const uint4 *>(p.x);
    uint4 xv = make_uint4(0, 0, 0, 0);
    if (tid < nb) xv = __ldg(xrow + tid);
    if (!EARLY)
      for (int i = tid; i < 512; i += nthr) tab->t[i] = kStreamTab.t[i];
    for (int b = tid; b < nb; b += nthr) {
      if (b != tid) xv = __ldg(xrow + b);
      float4 lo, hi;
      bf16x8_to_f32(xv, lo, hi);
      cm_store_block(xs4, xn2, b, lo, hi);
    }
  }
  __syncthreads();

  for (int t = tid, it = 0; t < ntask; t += nthr, ++it) {
    const uint32_t c = (uint32_t)t - fdiv((uint32_t)t, p.div_C) * (uint32_t)p.C;
    if (t + nthr < ntask) fetch(t + nthr, (it + 1) & 1);
    cp_async_commit();
    cp_async_wait<1>();
    ChunkFields f;
    uint32_t rowk;
    read_chunk<P>(fs, (it & 1) * nthr + tid, f, rowk);
    if (P == kP3C5) f.codes = (it & 1) ? cq1 : cq0;
    float2 acc = make_float2(0.f, 0.f);
    chunk_dot_cm<P, true, 1>(tab->t, f, 8, rowk, xs4 + kCmX4 * c, xn2 + kCmXn * c, acc);
    red[t] = acc.x + acc.y;
  }
  cp_async_wait<0>();
  __syncthreads();
  for (int r = warp; r < nrows; r += nthr >> 5) {
    float sum = 0.f;
    for (int q = lane; q < p.C; q += 32) sum += red[r * p.C + q];
    sum = warp_sum(sum);
    if (lane == 0) p.y[n0 + r] = sum;
  }
}

static size_t gemv1_smem(int C, int rpc, int threads) {
  return sizeof(StreamTables) + FieldSlots::bytes(2 * threads) + cm_bytes(C) + 16 +
         (size_t)rpc * C * sizeof(float);
}

NSLM_BOUNDS_ACCESSOR(gemv)

}  // namespace nslm

using namespace nslm;

static int32_t seed_gemv(const nslm_seed_matrix *W, const uint16_t *x_bf16, int32_t M, float *y,
                         bool fields_ready, nslm_stream_t stream) {
  g_launches = 0;
  int32_t st = check_matrix(W);
  if (st) return st;
  if (!x_bf16 || !y) return NSLM_ERR_ARG;
  if (M < 1 || M > 8) return NSLM_ERR_SHAPE;
  if (!aligned16(x_bf16) || !aligned16(y)) return NSLM_ERR_ALIGN;
  if ((size_t)M * W->K > 32768) return NSLM_ERR_SHAPE;  // activations must fit in shared memory
  if ((st = check_device())) return st;
  if (W->N == 0) return NSLM_OK;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // one vector, whole 64-weight chunks: the latency-oriented kernel
  if (M == 1 && W->K % 64 == 0 && (int64_t)W->N * (W->K / 8) < (1ll << 31) && W->K / 64 < (1 << 16)) {
    const int sms = num_sms();
    Gemv1Params q{};
    q.W = *W;
    q.x = x_bf16;
    q.y = y;
    q.C = W->K / 64;
    q.div_C = make_fastdiv((uint32_t)q.C);
    // two CTAs per SM where their shared memory fits on one SM together;
    // otherwise (long rows) one larger CTA per SM, so that the grid still
    // runs in one wave
    int threads = 0, per_sm = 2;
    size_t smem = 0;
    for (per_sm = 2; per_sm >= 1; --per_sm) {
      q.rpc = std::max(1, ceil_div(W->N, per_sm * sms));
      const int tasks = q.rpc * q.C;
      const int rounds = ceil_div(tasks, per_sm == 2 ? Gemv1Shape<2>::kThreads : Gemv1Shape<1>::kThreads);
      threads = std::max(64, 32 * ceil_div(ceil_div(tasks, rounds), 32));
      smem = gemv1_smem(q.C, q.rpc, threads);
      if (per_sm == 1 || 2 * (smem + kSmemReservedPerCta) <= kSmemPerSm) break;
    }
    if (smem <= 200 * 1024 && (int64_t)q.rpc * q.C < (1 << 22)) {
      auto pick = [&](auto ctas) {
        constexpr int C2 = decltype(ctas)::value;
        return fields_ready ? ((W->P == 4)       ? gemv1_kernel<4, true, C2>
                               : (W->P == kP3C5) ? gemv1_kernel<kP3C5, true, C2>
                                                 : gemv1_kernel<3, true, C2>)
                            : ((W->P == 4)       ? gemv1_kernel<4, false, C2>
                               : (W->P == kP3C5) ? gemv1_kernel<kP3C5, false, C2>
                                                 : gemv1_kernel<3, false, C2>);
      };
      auto k = per_sm == 2 ? pick(std::integral_constant<int, 2>{}) : pick(std::integral_constant<int, 1>{});
      if ((st = ensure_smem((const void *)k, smem))) return st;
      ensure_stream_source(s);
      cudaLaunchConfig_t cfg{};
      cfg.gridDim = dim3((unsigned)ceil_div(W->N, q.rpc));
      cfg.blockDim = dim3((unsigned)threads);
      cfg.dynamicSmemBytes = smem;
      cfg.stream = s;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[0].val.programmaticStreamSerializationAllowed = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      st = cuda_status(cudaLaunchKernelEx(&cfg, k, q));
      if (st == NSLM_OK) st = launch_status();
      if (st == NSLM_OK) g_launches = 1;
      return st;
    }
  }

  GemvParams p{};
  p.seeds = W->seeds; p.coefs = W->coefs; p.codes = W->codes; p.exp_bias = W->exp_bias;
  p.x = x_bf16; p.y = y; p.N = W->N; p.K = W->K; p.nb = W->K / 8; p.M = M;
  const int sms = num_sms();
  ChunkLayout L = chunk_layout(W->K, W->N, 3 * sms, 512);
  p.R = L.R; p.C = L.C; p.Cpad = L.Cpad;
  p.groups = ceil_div(W->N, L.R);
  const bool vec = (p.nb % 8 == 0);
  const size_t smem = gemv_smem(M, L.Cpad, L.threads);
  if (smem > 227 * 1024) return NSLM_ERR_SHAPE;
  const int per_sm = std::max(1, std::min(2048 / L.threads, (int)((227 * 1024) / smem)));
  const int grid = std::min(p.groups, per_sm * sms);
  st = (W->P == 4)       ? dispatch_gemv<4>(p, vec, grid, L.threads, smem, s)
       : (W->P == kP3C5) ? dispatch_gemv<kP3C5>(p, vec, grid, L.threads, smem, s)
                         : dispatch_gemv<3>(p, vec, grid, L.threads, smem, s);
  if (st == NSLM_OK) g_launches = 1;
  return st;
}

extern "C" int32_t nslm_seed_gemv(const nslm_seed_matrix *W, const uint16_t *x_bf16, int32_t M,
                                  float *y, void *ws, size_t ws_bytes, nslm_stream_t stream) {
  (void)ws;
  (void)ws_bytes;
  return seed_gemv(W, x_bf16, M, y, false, stream);
}

extern "C" int32_t nslm_seed_gemv_flags(const nslm_seed_matrix *W, const uint16_t *x_bf16, int32_t M,
                                        float *y, uint32_t flags, nslm_stream_t stream) {
  g_launches = 0;
  if (flags & ~(uint32_t)NSLM_GEMV_FIELDS_READY) return NSLM_ERR_ARG;
  return seed_gemv(W, x_bf16, M, y, (flags & NSLM_GEMV_FIELDS_READY) != 0, stream);
}
