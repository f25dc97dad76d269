// search.cu -- the seed search (encoder) on the GPU: nslm_seed_search.
//
// "NanoSeedLM: LLM inference using pseudo-random numbers", "What I changed:
// September 2026": every block of 8 weights walks all 65,535 seeds, and the
// GPU search must give exactly the answer of the C reference (contraction
// off: "'GPU search == CPU search'").  For every seed and every code 0..15:
//   c = round_half_even(pinv(U) w / 2^(code + bias)), clamped to [-8, 7]
//   err = sum_r (w_r - 2^(code + bias) (U c)_r)^2
// with pinv(U) = (U^T U)^-1 U^T by Gauss-Jordan elimination with partial
// pivoting, in fp64.  The smallest error wins; ties go to the larger code,
// then to the lower seed.
//
// With per-column importances d ("Qwen3.8-Flash-Next-NanoSeedLM-P4", "How it
// works": the search weighted each weight's error by the mean square of its
// input activation) the error is sum_r d_r (w_r - 2^(code+bias) (U c)_r)^2 and
// the fit its least-squares minimiser, (U^T D U)^-1 U^T D w; the weighted
// pinv then differs per block and is formed for each (seed, block).
//
// A CTA takes four consecutive blocks of a row (pairs share a P = 4 codes
// byte) and forms pinv(U) once per seed for all four; its threads split the
// seed range, each keeps its best candidate per block, and a shared-memory
// tree picks the CTA's best.  The order (error, larger
// code, lower seed) is total, so the tree gives the sequential scan's answer
// whatever the split.  Every fp64 operation of the reference is issued as the
// same correctly rounded operation (__dmul_rn / __dadd_rn / __dsub_rn,
// IEEE division), so no multiply-add is ever fused; U^T U, U c and the scaled
// model are exact integers or dyadic numbers and are formed in integers.
#include <cfloat>

#include "common.cuh"
#include "regen.cuh"

namespace nslm {

namespace {

constexpr int kSearchThreads = 256;

__device__ __forceinline__ double pow2(int k) {  // 2^k, |k| < 1000
  return __longlong_as_double((long long)(1023 + k) << 52);
}

struct Cand {
  double err;
  int32_t code, seed;
  uint32_t cpack;  // c_j as nibbles
};

// a before b in the search order: smaller error, then larger code, then lower seed
__device__ __forceinline__ bool better(const Cand &a, const Cand &b) {
  if (a.err != b.err) return a.err < b.err;
  if (a.code != b.code) return a.code > b.code;
  return a.seed < b.seed;
}

// A^-1 B in place by Gauss-Jordan elimination with partial pivoting, exactly
// the reference's steps; false when A is singular.
template <int P>
__device__ __forceinline__ bool gauss_jordan(double (&A)[4][4], double (&B)[4][8]) {
#pragma unroll
  for (int col = 0; col < P; ++col) {
    int piv = col;
    double pv = fabs(A[col][col]);
#pragma unroll
    for (int r = col + 1; r < P; ++r) {
      const double ar = fabs(A[r][col]);
      if (ar > pv) { piv = r; pv = ar; }
    }
    if (pv < 1e-300) return false;
    if (piv != col) {
#pragma unroll
      for (int r = col + 1; r < P; ++r) {
        if (r != piv) continue;
#pragma unroll
        for (int q = 0; q < P; ++q) { const double t = A[col][q]; A[col][q] = A[r][q]; A[r][q] = t; }
#pragma unroll
        for (int q = 0; q < 8; ++q) { const double t = B[col][q]; B[col][q] = B[r][q]; B[r][q] = t; }
      }
    }
    const double d = A[col][col];
#pragma unroll
    for (int q = 0; q < P; ++q) A[col][q] = __ddiv_rn(A[col][q], d);
#pragma unroll
    for (int q = 0; q < 8; ++q) B[col][q] = __ddiv_rn(B[col][q], d);
#pragma unroll
    for (int r = 0; r < P; ++r) {
      if (r == col) continue;
      const double f = A[r][col];
      if (f == 0.0) continue;
#pragma unroll
      for (int q = 0; q < P; ++q) A[r][q] = __dsub_rn(A[r][q], __dmul_rn(f, A[col][q]));
#pragma unroll
      for (int q = 0; q < 8; ++q) B[r][q] = __dsub_rn(B[r][q], __dmul_rn(f, B[col][q]));
    }
  }
  return true;
}

// pinv(U) for one seed: returns false when U^T U is singular (the seed is
// skipped).  u[r][j] = s_{1+8j+r} - 32768, so U = u / 32768.
template <int P>
__device__ bool pinv_of(const int32_t (&u)[8][4], double (&B)[4][8]) {
  double A[4][4];
#pragma unroll
  for (int a = 0; a < P; ++a)
#pragma unroll
    for (int b = 0; b < P; ++b) {
      long long s = 0;
#pragma unroll
      for (int r = 0; r < 8; ++r) s += (long long)u[r][a] * u[r][b];
      A[a][b] = (double)s * pow2(-30);  // exact: |s| < 2^33
    }
#pragma unroll
  for (int a = 0; a < P; ++a)
#pragma unroll
    for (int r = 0; r < 8; ++r) B[a][r] = (double)u[r][a] * pow2(-15);
  return gauss_jordan<P>(A, B);
}

// The weighted pinv (U^T D U)^-1 U^T D, in the reference's operation order:
// A[a][b] = sum_r ((U_ra U_rb) d_r), B[a][r] = U_ra d_r (U_ra U_rb is exact).
template <int P>
__device__ bool pinv_weighted(const int32_t (&u)[8][4], const double *d, double (&B)[4][8]) {
  double A[4][4];
#pragma unroll
  for (int a = 0; a < P; ++a)
#pragma unroll
    for (int b = 0; b < P; ++b) {
      double s = 0.0;
#pragma unroll
      for (int r = 0; r < 8; ++r)
        s = __dadd_rn(s, __dmul_rn((double)((long long)u[r][a] * u[r][b]) * pow2(-30), d[r]));
      A[a][b] = s;
    }
#pragma unroll
  for (int a = 0; a < P; ++a)
#pragma unroll
    for (int r = 0; r < 8; ++r) B[a][r] = __dmul_rn((double)u[r][a] * pow2(-15), d[r]);
  return gauss_jordan<P>(A, B);
}

struct SearchParams {
  const float *w;            // [N][K]
  const float *imp;          // [K] importances, or null (unweighted)
  nslm_seed_matrix out;      // seeds, coefs, codes written; exp_bias read
  double *err;               // [N][K/8] or null
  int32_t seed_lo, seed_hi;
  int32_t nb;                // blocks per row
};

// Blocks searched together by one CTA: pinv(U) depends only on the seed, so
// it is formed once per seed for all of them (an even count keeps the P = 4
// code bytes inside one CTA).
constexpr int kSearchGroup = 4;

template <int P, bool WEIGHTED>
__global__ void __launch_bounds__(kSearchThreads) seed_search_kernel(const SearchParams p) {
  __shared__ StreamTables tab;
  __shared__ Cand s_c[kSearchThreads];
  __shared__ double s_w[kSearchGroup][8];
  __shared__ double s_d[kSearchGroup][8];
  build_stream_tables(&tab);
  const int tid = threadIdx.x;
  const int groups_row = (p.nb + kSearchGroup - 1) / kSearchGroup;
  const int64_t row = blockIdx.x / groups_row;
  const int b0 = (int)(blockIdx.x - row * groups_row) * kSearchGroup;
  const int nblk = min(kSearchGroup, p.nb - b0);
  const int32_t bias = p.out.exp_bias[row];
  if (tid < 8 * nblk) {
    s_w[tid >> 3][tid & 7] = (double)p.w[row * (int64_t)p.nb * 8 + 8 * b0 + tid];
    s_d[tid >> 3][tid & 7] = WEIGHTED ? (double)p.imp[8 * b0 + tid] : 1.0;
  }
  __syncthreads();

  Cand best[kSearchGroup];
#pragma unroll
  for (int g = 0; g < kSearchGroup; ++g) best[g] = Cand{INFINITY, -1, -1, 0u};
  for (int seed = p.seed_lo + tid; seed <= p.seed_hi; seed += kSearchThreads) {
    // states s_1 .. s_{8P} as windows of the stream word (offsets up to 32:
    // the clamping funnel shift, which gives hi itself at 32)
    uint32_t lo, hi;
    stream_word(&tab, (uint32_t)seed, lo, hi);
    int32_t u[8][4];
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        u[r][j] = (j < P) ? (int32_t)(__funnelshift_rc(lo, hi, 1 + 8 * j + r) & 0xFFFFu) - 32768 : 0;
    double B[4][8];
    if (!WEIGHTED && !pinv_of<P>(u, B)) continue;
#pragma unroll
    for (int g = 0; g < kSearchGroup; ++g) {
      if (g >= nblk) break;
      if (WEIGHTED && !pinv_weighted<P>(u, s_d[g], B)) continue;
      double w[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) w[r] = s_w[g][r];
      double proj[4];
#pragma unroll
      for (int a = 0; a < P; ++a) {
        double s = 0.0;
#pragma unroll
        for (int r = 0; r < 8; ++r) s = __dadd_rn(s, __dmul_rn(B[a][r], w[r]));
        proj[a] = s;
      }
      bool zero_seen = false;
      for (int code = 15; code >= 0; --code) {
        const double inv = pow2(-(code + bias));  // proj / 2^(code+bias), exact
        int32_t c[4];
        uint32_t cp = 0;
#pragma unroll
        for (int a = 0; a < P; ++a) {
          double v = rint(__dmul_rn(proj[a], inv));
          v = fmin(fmax(v, -8.0), 7.0);
          c[a] = (int32_t)v;
          cp |= ((uint32_t)c[a] & 0xFu) << (4 * a);
        }
        // all-zero coefficients give the same error for every code; the
        // first (largest) such code is the only one that can win
        if (cp == 0u) {
          if (zero_seen) continue;
          zero_seen = true;
        }
        // 2^(code+bias) (U c)_r = A_r 2^(code+bias-15), A_r = sum_j u_rj c_j (exact)
        const double sc = pow2(code + bias - 15);
        double err = 0.0;
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          int32_t A = 0;
#pragma unroll
          for (int a = 0; a < P; ++a) A += u[r][a] * c[a];
          const double e = __dsub_rn(w[r], (double)A * sc);
          err = WEIGHTED ? __dadd_rn(err, __dmul_rn(s_d[g][r], __dmul_rn(e, e))) : __dadd_rn(err, __dmul_rn(e, e));
        }
        const Cand cand{err, code, seed, cp};
        if (better(cand, best[g])) best[g] = cand;
      }
    }
  }

  uint32_t code_byte = 0;
#pragma unroll
  for (int g = 0; g < kSearchGroup; ++g) {
    if (g >= nblk) break;
    __syncthreads();  // s_c of the previous block is consumed
    s_c[tid] = best[g];
    __syncthreads();
    for (int off = kSearchThreads / 2; off > 0; off >>= 1) {
      if (tid < off && better(s_c[tid + off], s_c[tid])) s_c[tid] = s_c[tid + off];
      __syncthreads();
    }
    if (tid == 0) {
      const Cand c = s_c[0];
      const int64_t idx = row * (int64_t)p.nb + b0 + g;
      const bool found = c.seed > 0;
      const uint32_t code = found ? (uint32_t)c.code : 0u;
      const_cast<uint16_t *>(p.out.seeds)[idx] = found ? (uint16_t)c.seed : (uint16_t)0;
      const uint32_t q = (found ? c.cpack : 0u) | (P == 3 ? code << 12 : 0u);
      const_cast<uint16_t *>(p.out.coefs)[idx] = (uint16_t)q;
      code_byte |= code << (4 * (g & 1));
      if (p.err) p.err[idx] = found ? c.err : INFINITY;
      if (P == 4 && (g & 1))
        const_cast<uint8_t *>(p.out.codes)[row * (int64_t)(p.nb / 2) + (b0 + g) / 2] = (uint8_t)code_byte;
      if (g & 1) code_byte = 0;
    }
  }
}

}  // namespace

}  // namespace nslm

using namespace nslm;

extern "C" int32_t nslm_seed_search(const float *w, const float *imp, const nslm_seed_matrix *out,
                                    int32_t seed_lo, int32_t seed_hi, double *err, nslm_stream_t stream) {
  g_launches = 0;
  int32_t st = check_matrix(out);
  if (st) return st;
  if (out->P == kP3C5) return NSLM_ERR_SHAPE;  // the search encodes P = 3 and P = 4
  if (!w) return NSLM_ERR_ARG;
  if (seed_lo < 1 || seed_hi > 65535 || seed_lo > seed_hi) return NSLM_ERR_ARG;
  if (out->N == 0) return NSLM_OK;
  if ((st = check_device())) return st;
  SearchParams p{};
  p.w = w;
  p.imp = imp;
  p.out = *out;
  p.err = err;
  p.seed_lo = seed_lo;
  p.seed_hi = seed_hi;
  p.nb = out->K / 8;
  const int64_t grid = (int64_t)out->N * ((p.nb + kSearchGroup - 1) / kSearchGroup);
  if (grid > 0x7FFFFFFF) return NSLM_ERR_SHAPE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (out->P == 4) {
    if (imp) seed_search_kernel<4, true><<<(unsigned)grid, kSearchThreads, 0, s>>>(p);
    else seed_search_kernel<4, false><<<(unsigned)grid, kSearchThreads, 0, s>>>(p);
  } else {
    if (imp) seed_search_kernel<3, true><<<(unsigned)grid, kSearchThreads, 0, s>>>(p);
    else seed_search_kernel<3, false><<<(unsigned)grid, kSearchThreads, 0, s>>>(p);
  }
  st = launch_status();
  if (st == NSLM_OK) g_launches = 1;
  return st;
}
