// gemv.cu -- nslm_seed_gemv: the decode matrix-vector product with the
// weights regenerated from their seeds in registers ("NanoSeedLM: LLM
// inference using pseudo-random numbers", "What I changed: September 2026":
// weights are rebuilt inside the GPU kernels, in registers, every time).
//
// A CTA owns R rows x Cpad chunk slots (one thread per (row, chunk)); it
// loops over row groups (grid-stride), so the activations are staged into
// shared memory once per CTA.  Partial sums of the chunks of a row are added
// in shared memory (fixed order, so results are deterministic).
#include <algorithm>

#include "chunk.cuh"
#include "common.cuh"

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
                         P == 4 ? p.codes + (size_t)row * (p.nb / 2) : nullptr, p.nb, ch, f);
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
  k<<<grid, threads, smem, s>>>(p);
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

}  // namespace nslm

using namespace nslm;

extern "C" int32_t nslm_seed_gemv(const nslm_seed_matrix *W, const uint16_t *x_bf16, int32_t M,
                                  float *y, void *ws, size_t ws_bytes, nslm_stream_t stream) {
  (void)ws;
  (void)ws_bytes;
  g_launches = 0;
  int32_t st = check_matrix(W);
  if (st) return st;
  if (!x_bf16 || !y) return NSLM_ERR_ARG;
  if (M < 1 || M > 8) return NSLM_ERR_SHAPE;
  if (!aligned16(x_bf16) || !aligned16(y)) return NSLM_ERR_ALIGN;
  if ((size_t)M * W->K > 32768) return NSLM_ERR_SHAPE;  // activations must fit in shared memory
  if ((st = check_device())) return st;
  if (W->N == 0) return NSLM_OK;

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
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  st = (W->P == 4) ? dispatch_gemv<4>(p, vec, grid, L.threads, smem, s)
                   : dispatch_gemv<3>(p, vec, grid, L.threads, smem, s);
  if (st == NSLM_OK) g_launches = 1;
  return st;
}
