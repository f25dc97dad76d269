// grouped.cu -- the batched (prefill / batch-decode) seed matmul on the
// tcgen05 tensor cores: nslm_seed_grouped_gemm, and the T > 8 path of
// nslm_moe_seed_ffn.
//
// The pages run prompts through grouped expert GEMMs (NanoSeedLM documentation
// index, Results: "the grouped expert GEMMs") and rebuild weights inside the
// kernels ("NanoSeedLM: LLM inference using pseudo-random numbers", "What I
// changed: September 2026").  Here a CTA owns a tile of 128 weight rows of one
// expert and up to `bn` of that expert's token rows.  For every 64-wide K
// slice, all threads regenerate the 128 x 64 weight tile from its seeds as
// bf16 (round to nearest even of the exact fp32 weight) straight into shared
// memory, copy the matching token rows, and one thread issues tcgen05.mma
// (bf16 x bf16 -> fp32 in tensor memory).  Two shared-memory stages let the
// tensor core work on one slice while the threads regenerate the next.  The
// weights are never written to global memory.
//
// Shared-memory layout of both operands is the K-major, no-swizzle canonical
// layout: one 8-weight block of a row is one 16-byte row of an 8 x 16-byte
// core matrix, so each regenerated block is a single 16-byte store.
#include <algorithm>

#include "chunk.cuh"
#include "common.cuh"
#include "grouped.cuh"
#include "umma.cuh"

namespace nslm {

constexpr int kBM = 128;        // weight rows per tile (MMA M)
constexpr int kBK = 64;         // K per stage: 8 blocks, 128 bytes of bf16 per row
constexpr int kGThreads = 512;
constexpr int kStages = 2;
constexpr long long kWaitCycles = 4000000000LL;  // ~2 s: a wait longer than this is an error

enum GMode { GMODE_GEMM = 0, GMODE_GATEUP = 1, GMODE_DOWN = 2 };

struct GroupedParams {
  nslm_seed_matrix A0, A1;  // A1: up projection (GATEUP only)
  int32_t E, rows, K, nb;
  int32_t R;                // B rows available
  const uint16_t *x;        // bf16 B rows [R][K]
  const int32_t *row_of;    // sorted row -> B row (null: identity)
  const int32_t *offsets;   // [E + 1] sorted-row offsets per expert
  const int32_t *tile_start;// [E + 1] tiles before expert e
  int32_t mtiles, bn, tmem_cols;
  int32_t *status;          // set to 1 if a wait timed out
  float *y;                 // GEMM: fp32 [R][rows]
  uint16_t *h;              // GATEUP: bf16 [R][rows]
  float *part;              // DOWN: fp32 [pairs][rows]
  const int32_t *pair_of;   // DOWN: sorted row -> pair
  const float *pair_w;      // DOWN: pair -> routing weight
};

// Regenerate blocks (b, b+1) of one row as bf16 and store them as two 16-byte
// core-matrix rows.  seeds2/coefs2 hold the two blocks' 16-bit fields, code2
// their two exponent nibbles.
template <int P>
__device__ __forceinline__ void regen_pair_bf16(const StreamTables *tab, uint32_t seeds2, uint32_t coefs2,
                                                uint32_t code2, uint32_t rowk, uint4 *dst0, uint4 *dst1) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t seed = h ? (seeds2 >> 16) : (seeds2 & 0xFFFFu);
    const uint32_t q = h ? (coefs2 >> 16) : (coefs2 & 0xFFFFu);
    uint32_t lo, hi;
    stream_word(tab, seed, lo, hi);
    const uint32_t cb2 = coef_bytes2<P>(q);
    const int32_t base = (int32_t)kMagic2Bits - 32768 * dp4a_ss(cb2, 0x01010101u, 0);
    const uint32_t code = (P == 4) ? ((code2 >> (4 * h)) & 0xFu) : (q >> 12);
    const float s = block_scale(code, rowk);
    const float2 s2 = make_float2(s, s), off2 = make_float2(-kMagic2 * s, -kMagic2 * s);
    uint32_t packed[4];
#pragma unroll
    for (int r = 0; r < 8; r += 2) {
      const int32_t a0 = dp4a_us(__funnelshift_r(lo, hi, 1 + r), cb2, base) +
                         256 * dp4a_us(__funnelshift_r(lo, hi, 9 + r), cb2, 0);
      const int32_t a1 = dp4a_us(__funnelshift_r(lo, hi, 2 + r), cb2, base) +
                         256 * dp4a_us(__funnelshift_r(lo, hi, 10 + r), cb2, 0);
      // (Mg + A) * s - Mg * s = A * s exactly (power-of-two scale)
      const float2 w = __ffma2_rn(make_float2(__int_as_float(a0), __int_as_float(a1)), s2, off2);
      const __nv_bfloat162 b = __floats2bfloat162_rn(w.x, w.y);
      packed[r >> 1] = *reinterpret_cast<const uint32_t *>(&b);
    }
    *(h ? dst1 : dst0) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  }
}

template <int P, int MODE>
__global__ void __launch_bounds__(kGThreads, 1) grouped_seed_gemm_kernel(const GroupedParams p) {
  constexpr int NA = (MODE == GMODE_GATEUP) ? 2 : 1;
  extern __shared__ __align__(1024) uint8_t gsm[];
  StreamTables *tab = reinterpret_cast<StreamTables *>(gsm);
  uint8_t *a_base = gsm + 2048;                                   // [stage][NA][128 rows x 128 B]
  uint8_t *b_base = a_base + (size_t)kStages * NA * kBM * 128;    // [stage][bn rows x 128 B]
  __shared__ __align__(8) uint64_t mbar[kStages];
  __shared__ uint32_t tmem_base_s;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  build_stream_tables(tab);
  if (warp == 0) umma::tmem_alloc(umma::smem_u32(&tmem_base_s), (uint32_t)p.tmem_cols);
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) umma::mbar_init(umma::smem_u32(&mbar[s]), 1);
    umma::mbar_init_fence();
  }
  umma::fence_before_sync();
  __syncthreads();
  umma::fence_after_sync();
  const uint32_t tmem = tmem_base_s;

  const int total_tiles = p.tile_start[p.E];
  const int ksteps = p.K / kBK;
  uint32_t it = 0;  // stage iterations issued by this CTA
  bool abort = false;
  for (int t = blockIdx.x; t < total_tiles && !abort; t += gridDim.x) {
    // the expert owning tile t: the last e with tile_start[e] <= t
    int lo_e = 0, hi_e = p.E - 1;
    while (lo_e < hi_e) {
      const int mid = (lo_e + hi_e + 1) >> 1;
      if (p.tile_start[mid] <= t) lo_e = mid; else hi_e = mid - 1;
    }
    const int e = lo_e;
    const int local = t - p.tile_start[e];
    const int mt = local % p.mtiles, nt = local / p.mtiles;
    const int seg_begin = max(0, p.offsets[e]), seg_end = min(p.R, p.offsets[e + 1]);
    const int r_begin = seg_begin + nt * p.bn;
    const int n_valid = max(0, min(p.bn, seg_end - r_begin));
    const int N = max(16, (n_valid + 15) & ~15);
    const int m0 = mt * kBM;
    const uint32_t idesc = umma::idesc_bf16_f32(kBM, N);

    for (int kt = 0; kt < ksteps; ++kt, ++it) {
      const int stage = it & 1;
      bool ok = true;
      if (it >= 2) ok = umma::mbar_wait_bounded(umma::smem_u32(&mbar[stage]), ((it >> 1) - 1) & 1, kWaitCycles);
      if (__syncthreads_or(!ok)) { abort = true; break; }

      // ---- A: NA x 128 rows x 8 blocks, two blocks per task
      for (int u = tid; u < NA * kBM * 4; u += kGThreads) {
        const int a = u / (kBM * 4), rem = u - a * (kBM * 4);
        const int row = rem & (kBM - 1), bp = rem >> 7;  // block pair 0..3
        const nslm_seed_matrix &W = a ? p.A1 : p.A0;
        uint8_t *tile = a_base + (size_t)(stage * NA + a) * kBM * 128;
        uint4 *dst0 = reinterpret_cast<uint4 *>(tile + ((row >> 3) * 8 + 2 * bp) * 128 + (row & 7) * 16);
        uint4 *dst1 = reinterpret_cast<uint4 *>(tile + ((row >> 3) * 8 + 2 * bp + 1) * 128 + (row & 7) * 16);
        const int grow = m0 + row;
        if (grow < p.rows) {
          const size_t r = (size_t)e * p.rows + grow;
          const int b = kt * 8 + 2 * bp;
          const uint32_t s2 = __ldcs(reinterpret_cast<const uint32_t *>(W.seeds + r * p.nb + b));
          const uint32_t q2 = __ldcs(reinterpret_cast<const uint32_t *>(W.coefs + r * p.nb + b));
          const uint32_t c2 = (P == 4) ? (uint32_t)__ldcs(W.codes + r * (p.nb / 2) + b / 2) : 0u;
          regen_pair_bf16<P>(tab, s2, q2, c2, row_scale_key(__ldg(W.exp_bias + r)), dst0, dst1);
        } else {
          *dst0 = make_uint4(0, 0, 0, 0);
          *dst1 = make_uint4(0, 0, 0, 0);
        }
      }
      // ---- B: N token rows x 8 chunks of 16 bytes (zeros past n_valid)
      uint8_t *btile = b_base + (size_t)stage * p.bn * 128;
      for (int u = tid; u < N * 8; u += kGThreads) {
        const int n = u % N, kc = u / N;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (n < n_valid) {
          const int sr = r_begin + n;
          const int xr = p.row_of ? p.row_of[sr] : sr;
          v = __ldg(reinterpret_cast<const uint4 *>(p.x + (size_t)xr * p.K + kt * kBK + kc * 8));
        }
        *reinterpret_cast<uint4 *>(btile + ((n >> 3) * 8 + kc) * 128 + (n & 7) * 16) = v;
      }
      umma::fence_proxy_async();
      __syncthreads();
      if (tid == 0) {
        umma::fence_after_sync();
        const uint32_t bsa = umma::smem_u32(btile);
#pragma unroll
        for (int s = 0; s < kBK / 16; ++s) {
          const uint64_t bd = umma::smem_desc_kmajor(bsa + s * 256, 128, 1024);
#pragma unroll
          for (int a = 0; a < NA; ++a) {
            const uint32_t asa = umma::smem_u32(a_base + (size_t)(stage * NA + a) * kBM * 128);
            const uint64_t ad = umma::smem_desc_kmajor(asa + s * 256, 128, 1024);
            umma::mma_bf16(tmem + (uint32_t)(a * p.bn), ad, bd, idesc, (kt | s) != 0);
          }
        }
        umma::commit(umma::smem_u32(&mbar[stage]));
      }
    }
    if (abort) break;

    // ---- epilogue: wait for the tile's last MMAs, read D from tensor memory
    const uint32_t last = it - 1;
    const bool ok = umma::mbar_wait_bounded(umma::smem_u32(&mbar[last & 1]), (last >> 1) & 1, kWaitCycles);
    if (__syncthreads_or(!ok)) { abort = true; break; }
    umma::fence_after_sync();
    const int q = warp & 3;                     // lane quarter this warp may read
    const int row = m0 + 32 * q + lane;
    const bool row_ok = row < p.rows;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * q) << 16);
    for (int c = warp >> 2; c * 8 < N; c += kGThreads / 128) {
      float v[8], v2[8];
      umma::tmem_ld8(lane_addr + (uint32_t)(c * 8), v);
      if (MODE == GMODE_GATEUP) umma::tmem_ld8(lane_addr + (uint32_t)(p.bn + c * 8), v2);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int n = c * 8 + j;
        if (!row_ok || n >= n_valid) continue;
        const size_t sr = (size_t)(r_begin + n);
        if (MODE == GMODE_GEMM) {
          p.y[sr * p.rows + row] = v[j];
        } else if (MODE == GMODE_GATEUP) {
          const float g = v[j], up = v2[j];
          p.h[sr * p.rows + row] = __bfloat16_as_ushort(__float2bfloat16_rn(g / (1.f + expf(-g)) * up));
        } else {
          const int pr = p.pair_of[sr];
          p.part[(size_t)pr * p.rows + row] = p.pair_w[pr] * v[j];
        }
      }
    }
    umma::fence_before_sync();
    __syncthreads();
  }

  if (abort) {
    if (tid == 0) atomicExch(p.status, 1);
    // let MMAs still in flight finish (bounded) before the tensor memory is freed
    if (it > 0) {
      const uint32_t last = it - 1;
      umma::mbar_wait_bounded(umma::smem_u32(&mbar[last & 1]), (last >> 1) & 1, kWaitCycles);
    }
  }
  umma::fence_before_sync();
  __syncthreads();
  if (warp == 0) umma::tmem_dealloc(tmem, (uint32_t)p.tmem_cols);
}

// ---------------------------------------------------------------- planning

// Tiles per expert (prefix sum) from the sorted-row offsets, one CTA.
__global__ void __launch_bounds__(1024) tile_prefix_kernel(const int32_t *__restrict__ offsets, int E,
                                                           int mtiles, int bn, int R,
                                                           int32_t *__restrict__ tile_start,
                                                           int32_t *__restrict__ status) {
  __shared__ int32_t s[1025];
  const int tid = threadIdx.x;
  if (tid == 0 && status) *status = 0;
  for (int e = tid; e < E; e += blockDim.x) {
    const int b = max(0, offsets[e]), en = min(R, offsets[e + 1]);
    const int n = max(0, en - b);
    s[e] = mtiles * ((n + bn - 1) / bn);
  }
  __syncthreads();
  if (tid == 0) {  // E <= 1024: a serial scan is a few microseconds at most
    int acc = 0;
    for (int e = 0; e < E; ++e) { const int v = s[e]; tile_start[e] = acc; acc += v; }
    tile_start[E] = acc;
  }
}

// The batched FFN's routing plan, one CTA: expert histogram, offsets, a
// stable counting sort of the (token, slot) pairs by expert (ties in pair
// order), and the tile prefix sums of both grouped GEMMs.  Pairs whose expert
// id is outside [0, E) are dropped.
__global__ void __launch_bounds__(1024) batched_plan_kernel(const int32_t *__restrict__ ids, int T, int E,
                                                            int k, int bn, int mt_gu, int mt_dn,
                                                            BatchedPlan bp) {
  __shared__ int32_t cnt[1024];
  __shared__ int32_t base[1024];
  const int tid = threadIdx.x, TK = T * k;
  for (int e = tid; e < E; e += blockDim.x) cnt[e] = 0;
  if (tid == 0) *bp.status = 0;
  __syncthreads();
  for (int i = tid; i < TK; i += blockDim.x) {
    const int e = ids[i];
    if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  if (tid == 0) {
    int acc = 0, tg = 0, td = 0;
    for (int e = 0; e < E; ++e) {
      bp.offsets[e] = acc;
      base[e] = acc;
      bp.tiles_gu[e] = tg;
      bp.tiles_dn[e] = td;
      const int n = cnt[e];
      acc += n;
      tg += mt_gu * ((n + bn - 1) / bn);
      td += mt_dn * ((n + bn - 1) / bn);
    }
    bp.offsets[E] = acc;
    bp.tiles_gu[E] = tg;
    bp.tiles_dn[E] = td;
  }
  __syncthreads();
  if (tid < 32) {  // one warp walks the pairs in order: stable positions
    const unsigned lt = (1u << tid) - 1u;
    for (int c = 0; c < TK; c += 32) {
      const int i = c + tid;
      int e = (i < TK) ? ids[i] : -1;
      if (e < 0 || e >= E) e = -1;
      const unsigned grp = __match_any_sync(0xffffffffu, e);
      const int rank = __popc(grp & lt);
      if (e >= 0) {
        const int pos = base[e] + rank;
        bp.row_of[pos] = i / k;
        bp.pair_of[pos] = i;
      }
      __syncwarp();
      if (e >= 0 && rank == 0) base[e] += __popc(grp);
      __syncwarp();
    }
  }
}

// y[t][c] = sum over the token's valid slots q of part[t*k + q][c].
__global__ void batched_reduce_kernel(const float *__restrict__ part, const int32_t *__restrict__ ids,
                                      int T, int k, int E, int hidden, float *__restrict__ y) {
  const size_t n = (size_t)T * hidden;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const int t = (int)(i / hidden), c = (int)(i - (size_t)t * hidden);
    float s = 0.f;
    for (int q = 0; q < k; ++q) {
      const int e = ids[t * k + q];
      if (e >= 0 && e < E) s += __ldcg(part + ((size_t)t * k + q) * hidden + c);
    }
    y[i] = s;
  }
}

// ---------------------------------------------------------------- host

static int tmem_cols_for(int ncols) {
  int c = 32;
  while (c < ncols) c <<= 1;
  return c;
}

static size_t grouped_smem(int NA, int bn) {
  return 2048 + (size_t)kStages * NA * kBM * 128 + (size_t)kStages * bn * 128;
}

template <int P, int MODE>
static int32_t launch_grouped_t(const GroupedParams &p, cudaStream_t s) {
  constexpr int NA = (MODE == GMODE_GATEUP) ? 2 : 1;
  const size_t smem = grouped_smem(NA, p.bn);
  auto kern = grouped_seed_gemm_kernel<P, MODE>;
  if (int32_t st = ensure_smem((const void *)kern, smem)) return st;
  kern<<<num_sms(), kGThreads, smem, s>>>(p);
  return launch_status();
}

int32_t launch_grouped(const GroupedParams &p, int P, int mode, cudaStream_t s) {
  if (P == 4) {
    if (mode == GMODE_GEMM) return launch_grouped_t<4, GMODE_GEMM>(p, s);
    if (mode == GMODE_GATEUP) return launch_grouped_t<4, GMODE_GATEUP>(p, s);
    return launch_grouped_t<4, GMODE_DOWN>(p, s);
  }
  if (mode == GMODE_GEMM) return launch_grouped_t<3, GMODE_GEMM>(p, s);
  if (mode == GMODE_GATEUP) return launch_grouped_t<3, GMODE_GATEUP>(p, s);
  return launch_grouped_t<3, GMODE_DOWN>(p, s);
}

static int choose_bn(int max_rows_per_expert) {
  const int r = std::max(16, (std::min(max_rows_per_expert, 256) + 15) & ~15);
  return r;
}

BatchedPlan batched_workspace(char *base, int T, int k, int E, int hidden, int inter) {
  BatchedPlan b{};
  auto r256 = [](size_t n) { return (n + 255) / 256 * 256; };
  size_t off = 0;
  const int TK = T * k;
  auto take = [&](size_t n) { char *q = base ? base + off : nullptr; off += r256(n); return q; };
  b.status = reinterpret_cast<int32_t *>(take(sizeof(int32_t)));
  b.offsets = reinterpret_cast<int32_t *>(take((size_t)(E + 1) * sizeof(int32_t)));
  b.tiles_gu = reinterpret_cast<int32_t *>(take((size_t)(E + 1) * sizeof(int32_t)));
  b.tiles_dn = reinterpret_cast<int32_t *>(take((size_t)(E + 1) * sizeof(int32_t)));
  b.row_of = reinterpret_cast<int32_t *>(take((size_t)TK * sizeof(int32_t)));
  b.pair_of = reinterpret_cast<int32_t *>(take((size_t)TK * sizeof(int32_t)));
  b.h = reinterpret_cast<uint16_t *>(take((size_t)TK * inter * sizeof(uint16_t)));
  b.part = reinterpret_cast<float *>(take((size_t)TK * hidden * sizeof(float)));
  b.bytes = off;
  return b;
}

int32_t launch_batched_ffn(const FfnDims &d, const nslm_seed_matrix *gate, const nslm_seed_matrix *up,
                           const nslm_seed_matrix *down, const uint16_t *x_bf16, const int32_t *ids,
                           const float *w, int T, int k, float *y, void *ws, cudaStream_t s,
                           int &launches) {
  if (d.hidden % kBK || d.inter % kBK || d.E > 1024) return NSLM_ERR_SHAPE;
  const BatchedPlan bp = batched_workspace(reinterpret_cast<char *>(ws), T, k, d.E, d.hidden, d.inter);
  const int bn = choose_bn(T);  // an expert gets at most T pairs (one per token)
  const int mt_gu = ceil_div(d.inter, kBM), mt_dn = ceil_div(d.hidden, kBM);
  batched_plan_kernel<<<1, 1024, 0, s>>>(ids, T, d.E, k, bn, mt_gu, mt_dn, bp);
  if (int32_t st = launch_status()) return st;
  ++launches;
  const int TK = T * k;
  {
    GroupedParams p{};
    p.A0 = *gate; p.A1 = *up; p.E = d.E; p.rows = d.inter; p.K = d.hidden; p.nb = d.hidden / 8;
    p.R = TK; p.x = x_bf16; p.row_of = bp.row_of; p.offsets = bp.offsets; p.tile_start = bp.tiles_gu;
    p.mtiles = mt_gu; p.bn = bn; p.tmem_cols = tmem_cols_for(2 * bn); p.status = bp.status; p.h = bp.h;
    // the gathered rows index x (T rows), not the sorted rows: bound by T via row_of
    if (int32_t st = launch_grouped(p, d.P, GMODE_GATEUP, s)) return st;
    ++launches;
  }
  {
    GroupedParams p{};
    p.A0 = *down; p.E = d.E; p.rows = d.hidden; p.K = d.inter; p.nb = d.inter / 8;
    p.R = TK; p.x = bp.h; p.row_of = nullptr; p.offsets = bp.offsets; p.tile_start = bp.tiles_dn;
    p.mtiles = mt_dn; p.bn = bn; p.tmem_cols = tmem_cols_for(bn); p.status = bp.status;
    p.part = bp.part; p.pair_of = bp.pair_of; p.pair_w = w;
    if (int32_t st = launch_grouped(p, d.P, GMODE_DOWN, s)) return st;
    ++launches;
  }
  const size_t n = (size_t)T * d.hidden;
  const int grid = (int)std::min<size_t>((n + 255) / 256, (size_t)num_sms() * 8);
  batched_reduce_kernel<<<grid, 256, 0, s>>>(bp.part, ids, T, k, d.E, d.hidden, y);
  if (int32_t st = launch_status()) return st;
  ++launches;
  return NSLM_OK;
}

size_t grouped_ws_bytes(int E) {
  return ((size_t)(E + 2) * sizeof(int32_t) + 255) / 256 * 256;
}

}  // namespace nslm

using namespace nslm;

extern "C" int32_t nslm_seed_grouped_gemm(const nslm_seed_matrix *W, int32_t E,
                                          const uint16_t *x_bf16, const int32_t *offsets,
                                          int32_t R, float *y, void *ws, size_t ws_bytes,
                                          nslm_stream_t stream) {
  g_launches = 0;
  int32_t st = check_matrix(W);
  if (st) return st;
  if (!x_bf16 || !offsets || !y) return NSLM_ERR_ARG;
  if (E < 1 || E > 1024 || R < 0) return NSLM_ERR_SHAPE;
  if (W->N % E != 0) return NSLM_ERR_SHAPE;
  if (W->K % kBK != 0) return NSLM_ERR_SHAPE;  // the tensor-core path takes 64-wide K slices
  if (!aligned16(x_bf16) || !aligned16(y)) return NSLM_ERR_ALIGN;
  const size_t need = grouped_ws_bytes(E);
  if (!ws || ws_bytes < need) return NSLM_ERR_WORKSPACE;
  if (!aligned16(ws)) return NSLM_ERR_ALIGN;
  if ((st = check_device())) return st;
  if (R == 0 || W->N == 0) return NSLM_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int32_t *status = reinterpret_cast<int32_t *>(ws);
  int32_t *tile_start = status + 1;
  const int rows = W->N / E;
  const int bn = choose_bn(R);
  const int mtiles = ceil_div(rows, kBM);
  tile_prefix_kernel<<<1, 1024, 0, s>>>(offsets, E, mtiles, bn, R, tile_start, status);
  if ((st = launch_status())) return st;
  GroupedParams p{};
  p.A0 = *W; p.E = E; p.rows = rows; p.K = W->K; p.nb = W->K / 8; p.R = R; p.x = x_bf16;
  p.row_of = nullptr; p.offsets = offsets; p.tile_start = tile_start; p.mtiles = mtiles; p.bn = bn;
  p.tmem_cols = tmem_cols_for(bn); p.status = status; p.y = y;
  st = launch_grouped(p, W->P, GMODE_GEMM, s);
  if (st == NSLM_OK) g_launches = 2;
  return st;
}
