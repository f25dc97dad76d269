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
// memory (512 threads, each owning two blocks of two rows per slice), copy the
// matching token rows, and one thread issues tcgen05.mma
// (bf16 x bf16 -> fp32 in tensor memory).  Three shared-memory stages let the
// tensor core work on one slice while the threads regenerate the next and
// the token rows of the one after are in flight.  The weights are never
// written to global memory.
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
constexpr int kMaxBn = 256;     // token rows per tile at most (2 x bn tensor-memory columns)
constexpr int kGThreads = 512;                  // producer threads (warps 0-15)
constexpr int kEpiWarp0 = kGThreads / 32;       // warps 16-19: the epilogue warpgroup
constexpr int kMmaWarp = kEpiWarp0 + 4;         // warp 20: issues the MMAs
constexpr int kCtaThreads = 32 * (kMmaWarp + 1);
constexpr int kStages = 3;  // slice i uses stage i % 3: the token rows of slice i+1 are
                             // copied while slice i is regenerated, into the stage that
                             // the MMAs of slice i-2 have released
constexpr long long kWaitCycles = 4000000000LL;  // ~2 s: a wait longer than this is an error

enum GMode { GMODE_GEMM = 0, GMODE_GATEUP = 1, GMODE_DOWN = 2 };

struct GroupedParams {
  nslm_seed_matrix A0, A1;  // A1: up projection (GATEUP only)
  int32_t E, rows, K, nb;
  int32_t R;                // sorted rows (GEMM: rows of x and y; FFN: routed pairs)
  int32_t x_rows;           // rows of x (bounds checks)
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

// Stream tables: kTabCopies interleaved copies (entry e of copy c at word
// kTabCopies * e + c), lane l reading copy l % kTabCopies.  Measured on B200
// (100-expert batched layer, P=3): one copy 727 / 890 us at T = 64 / 512,
// eight copies 727 / 1252 us -- the larger shared footprint costs more than
// the bank conflicts it removes.
constexpr int kTabCopies = 1;

// Tile shapes: every thread owns two tasks per K slice -- two consecutive
// blocks (16 weights) of the same row of both 128-row sub-tiles.  GATEUP tiles are
// 128 rows of gate and the same 128 rows of up (two accumulators); the other
// modes use 256-row tiles (two M=128 halves, two accumulators).
template <int MODE> struct TileShape {
  static constexpr int kRows = (MODE == GMODE_GATEUP) ? kBM : 2 * kBM;
};

// Pipeline (no CTA-wide barrier in the main loop; slice i uses stage i % 3),
// three roles:
//   producers (warps 0-15), per K slice i: start the async copies of their
//     token-row chunks of slice i+1 (after waiting empty[(i+1) % 3], i.e. for
//     the MMAs of slice i-2) -> regenerate their two tasks' blocks of slice i
//     (weight fields were loaded three slices earlier) -> wait for their
//     copies of slice i -> proxy fence -> arrive full[i % 3]
//   the MMA warp (warp 20, lane 0), per K slice: wait full[stage] -> (first
//     slice of a tile: wait acc_empty) -> issue the MMAs -> commit
//     empty[stage] (and acc_full after the tile's last slice)
//   the epilogue warpgroup (warps 16-19), per tile: wait acc_full -> read D
//     from tensor memory -> store -> arrive acc_empty; the producers never
//     stop for it
// Every wait is bounded; a thread that gives up raises a shared abort flag
// that all threads check before each slice.
struct SliceFields {  // packed fields of one thread's two tasks for one K slice
  uint32_t s2[2], q2[2], c2[2];
};

// (bp: the thread's block pair, nw: 32-bit words per row of seeds, for the
// bounds-check build)
template <int P>
__device__ __forceinline__ void load_slice(const uint32_t *const (&sp)[2], const uint32_t *const (&qp)[2],
                                           const uint8_t *const (&cp)[2], const bool (&ok)[2], int kt,
                                           SliceFields &f, int bp, int nw) {
  if (!in_bounds((size_t)(4 * kt + bp), (size_t)nw, 5)) {
    f = SliceFields{};
    return;
  }
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    f.s2[j] = ok[j] ? __ldcs(sp[j] + 4 * kt) : 0u;
    f.q2[j] = ok[j] ? __ldcs(qp[j] + 4 * kt) : 0u;
    f.c2[j] = (P == 4 && ok[j]) ? (uint32_t)__ldcs(cp[j] + 4 * kt) : 0u;
    if (P == kP3C5 && ok[j]) {
      // the pair's 6 code bits (bits 1..3 of two codes) at bit 6 bp of the
      // slice's 3 bytes: one byte for bp = 0, 3, two for bp = 1, 2; cp is the
      // row's codes; bit 0 of each code is bit 15 of its coefs half
      const uint8_t *cb = cp[j] + 3 * kt + ((6 * bp) >> 3);
      uint32_t t = __ldcs(cb);
      if (bp == 1 || bp == 2) t |= (uint32_t)__ldcs(cb + 1) << 8;
      const uint32_t c6 = (t >> ((6 * bp) & 7)) & 0x3Fu, q = f.q2[j];
      f.c2[j] = (((q >> 15) & 1u) | ((c6 & 7u) << 1)) | ((((q >> 31) & 1u) | ((c6 >> 3) << 1)) << 4);
    }
  }
}


// The tile the CTA's n-th tile index t covers.
struct TileInfo {
  int e, m0, r_begin, n_valid, N;
};
template <int MODE>
__device__ __forceinline__ TileInfo tile_info(const GroupedParams &p, int t) {
  int lo_e = 0, hi_e = p.E - 1;  // the last e with tile_start[e] <= t
  while (lo_e < hi_e) {
    const int mid = (lo_e + hi_e + 1) >> 1;
    if (p.tile_start[mid] <= t) lo_e = mid; else hi_e = mid - 1;
  }
  TileInfo ti;
  ti.e = lo_e;
  const int local = t - p.tile_start[ti.e];
  const int mt = local % p.mtiles, nt = local / p.mtiles;
  const int seg_begin = max(0, p.offsets[ti.e]), seg_end = min(p.R, p.offsets[ti.e + 1]);
  ti.r_begin = seg_begin + nt * p.bn;
  ti.n_valid = max(0, min(p.bn, seg_end - ti.r_begin));
  ti.N = max(16, (ti.n_valid + 15) & ~15);
  ti.m0 = mt * TileShape<MODE>::kRows;
  return ti;
}

template <int P, int MODE>
__global__ void __launch_bounds__(kCtaThreads, 1) grouped_seed_gemm_kernel(const GroupedParams p) {
  extern __shared__ __align__(1024) uint8_t gsm[];
  uint32_t *tab = reinterpret_cast<uint32_t *>(gsm);             // kTabCopies interleaved copies
  uint8_t *a_base = gsm + kTabCopies * 2048;                     // [stage][sub 0..1][128 rows x 128 B]
  uint8_t *b_base = a_base + (size_t)kStages * 2 * kBM * 128;    // [stage][bn rows x 128 B]
  __shared__ __align__(8) uint64_t full_bar[kStages];
  __shared__ __align__(8) uint64_t empty_bar[kStages];
  __shared__ __align__(8) uint64_t acc_full_bar, acc_empty_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ volatile int s_abort;
  // DOWN epilogue: each epilogue warp's copy of the tile's pair ids and weights
  __shared__ int s_epr[MODE == GMODE_DOWN ? 4 : 1][MODE == GMODE_DOWN ? kMaxBn : 1];
  __shared__ float s_epw[MODE == GMODE_DOWN ? 4 : 1][MODE == GMODE_DOWN ? kMaxBn : 1];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // a producer's tasks: row trow, block pair bp, of sub-tiles 0 and 1.  A
  // warp covers 8 rows x the 4 block pairs: a field load touches 8 sectors
  // (4 lanes per 16-byte row piece), and each 8-lane wavefront of the tile
  // stores writes 8 consecutive rows (128 contiguous bytes)
  const int trow = ((tid >> 5) << 3) | (tid & 7), bp = (tid >> 3) & 3;
  build_stream_tables_rep<kTabCopies>(tab);
  const uint32_t *tl = tab + (lane & (kTabCopies - 1));
  if (warp == 0) umma::tmem_alloc(umma::smem_u32(&tmem_base_s), (uint32_t)p.tmem_cols);
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      umma::mbar_init(umma::smem_u32(&full_bar[s]), kGThreads);
      umma::mbar_init(umma::smem_u32(&empty_bar[s]), 1);
    }
    umma::mbar_init(umma::smem_u32(&acc_full_bar), 1);
    umma::mbar_init(umma::smem_u32(&acc_empty_bar), 128);
    umma::mbar_init_fence();
    s_abort = 0;
  }
  umma::fence_before_sync();
  __syncthreads();
  umma::fence_after_sync();
  const uint32_t tmem = tmem_base_s;

  const int total_tiles = p.tile_start[p.E];
  const int ksteps = p.K / kBK;
  uint32_t it = 0;      // K slices produced (or consumed) by this thread's role
  uint32_t ntile = 0;   // tiles finished

  if (warp == kMmaWarp) {  // ---- lane 0 waits for each slice and issues its MMAs
    if (lane == 0) {
      for (int t = blockIdx.x; t < total_tiles && !s_abort; t += gridDim.x, ++ntile) {
        const TileInfo ti = tile_info<MODE>(p, t);
        const uint32_t idesc = umma::idesc_bf16_f32(kBM, max(16, (ti.n_valid + 15) & ~15));
        for (int kt = 0; kt < ksteps; ++kt, ++it) {
          const int stage = it % kStages;
          bool go = umma::mbar_wait_bounded(umma::smem_u32(&full_bar[stage]), (it / kStages) & 1, kWaitCycles);
          if (go && kt == 0 && ntile > 0)  // the epilogue has drained the last tile's accumulators
            go = umma::mbar_wait_bounded(umma::smem_u32(&acc_empty_bar), (ntile - 1) & 1, kWaitCycles);
          if (!go) { s_abort = 1; break; }
          umma::fence_after_sync();
          const uint32_t asa = umma::smem_u32(a_base + (size_t)stage * 2 * kBM * 128);
          const uint32_t bsa = umma::smem_u32(b_base + (size_t)stage * p.bn * 128);
#pragma unroll
          for (int s = 0; s < kBK / 16; ++s) {
            const uint64_t bd = umma::smem_desc_kmajor(bsa + s * 256, 128, 1024);
#pragma unroll
            for (int a = 0; a < 2; ++a) {
              const uint64_t ad = umma::smem_desc_kmajor(asa + a * kBM * 128 + s * 256, 128, 1024);
              umma::mma_bf16(tmem + (uint32_t)(a * p.bn), ad, bd, idesc, (kt | s) != 0);
            }
          }
          umma::commit(umma::smem_u32(&empty_bar[stage]));
          if (kt == ksteps - 1) umma::commit(umma::smem_u32(&acc_full_bar));
        }
      }
    }
    __syncwarp();
  } else if (warp >= kEpiWarp0) {  // ---- epilogue warpgroup: tensor memory -> outputs
    const int ew = warp - kEpiWarp0;  // tensor-memory lanes 32 ew .. 32 ew + 31
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++ntile) {
      if (s_abort) break;
      const TileInfo ti = tile_info<MODE>(p, t);
      __syncwarp();
      if (MODE == GMODE_DOWN) {
        // the tile's pair ids and routing weights, loaded once per tile and
        // warp before the accumulators are ready (loaded per element they
        // were two dependent global loads on the tile's critical path)
#pragma unroll 4
        for (int n = lane; n < ti.N; n += 32) {
          const bool v = n < ti.n_valid;
          const int pr = v ? p.pair_of[ti.r_begin + n] : 0;
          s_epr[ew][n] = pr;
          s_epw[ew][n] = v ? p.pair_w[pr] : 0.f;
        }
        __syncwarp();
      }
      const bool acc_ok = umma::mbar_wait_bounded(umma::smem_u32(&acc_full_bar), ntile & 1, kWaitCycles);
      if (!acc_ok) s_abort = 1;
      // tcgen05.ld is warp-collective: the whole warp takes one decision
      if (!__all_sync(0xffffffffu, acc_ok && !s_abort)) break;
      umma::fence_after_sync();
      const uint32_t lane_addr = tmem + ((uint32_t)(32 * ew) << 16);
      if (MODE == GMODE_GATEUP) {
        const int row = ti.m0 + 32 * ew + lane;
        const bool rok = row < p.rows;
        for (int c = 0; c * 8 < ti.N; ++c) {
          float g[8], up[8];
          umma::tmem_ld8(lane_addr + (uint32_t)(c * 8), g);
          umma::tmem_ld8(lane_addr + (uint32_t)(p.bn + c * 8), up);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int n = c * 8 + j;
            if (!rok || n >= ti.n_valid) continue;
            const size_t sr = (size_t)(ti.r_begin + n);
            const float hv = __fdividef(g[j], 1.f + __expf(-g[j])) * up[j];
            if (in_bounds(sr, (size_t)p.R, 7)) p.h[sr * p.rows + row] = __bfloat16_as_ushort(__float2bfloat16_rn(hv));
          }
        }
      } else {
#pragma unroll
        for (int mh = 0; mh < 2; ++mh) {
          const int row = ti.m0 + mh * kBM + 32 * ew + lane;
          const bool rok = row < p.rows;
          for (int c = 0; c * 8 < ti.N; ++c) {
            float v[8];
            umma::tmem_ld8(lane_addr + (uint32_t)(mh * p.bn + c * 8), v);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int n = c * 8 + j;
              if (!rok || n >= ti.n_valid) continue;
              const size_t sr = (size_t)(ti.r_begin + n);
              if (MODE == GMODE_GEMM) {
                if (in_bounds(sr, (size_t)p.R, 8)) p.y[sr * p.rows + row] = v[j];
              } else {
                const size_t pr = (size_t)s_epr[MODE == GMODE_DOWN ? ew : 0][MODE == GMODE_DOWN ? n : 0];
                if (in_bounds(pr, (size_t)p.R, 9))
                  p.part[pr * p.rows + row] = s_epw[MODE == GMODE_DOWN ? ew : 0][MODE == GMODE_DOWN ? n : 0] * v[j];
              }
            }
          }
        }
      }
      umma::fence_before_sync();
      umma::mbar_arrive(umma::smem_u32(&acc_empty_bar));
    }
  } else {  // ---- producers (warps 0-15)
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
      if (s_abort) break;
      const TileInfo ti = tile_info<MODE>(p, t);
      const int N = ti.N;
      // the two tasks' weight rows for the whole tile
      const uint32_t *sp[2];
      const uint32_t *qp[2];
      const uint8_t *cpp[2];
      bool ok[2];
      uint32_t rowk[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const nslm_seed_matrix &W = (MODE == GMODE_GATEUP && j) ? p.A1 : p.A0;
        const int grow = ti.m0 + (MODE == GMODE_GATEUP ? 0 : j * kBM) + trow;
        ok[j] = grow < p.rows;
        size_t wr = (size_t)ti.e * p.rows + (ok[j] ? grow : 0);
        if (!in_bounds(wr, (size_t)W.N, 5)) {
          ok[j] = false;
          wr = 0;
        }
        sp[j] = reinterpret_cast<const uint32_t *>(W.seeds + wr * p.nb) + bp;
        qp[j] = reinterpret_cast<const uint32_t *>(W.coefs + wr * p.nb) + bp;
        cpp[j] = (P == 4) ? W.codes + wr * (p.nb / 2) + bp
                 : (P == kP3C5) ? W.codes + wr * (size_t)(3 * p.nb / 8) : nullptr;
        rowk[j] = load_bias_key(W, wr);
      }
      const size_t a_off = ((trow >> 3) * 8 + 2 * bp) * 128 + (trow & 7) * 16;
      // token rows this thread copies: chunks (n, kc) for n = trow, trow + 128 and kc = bp, bp + 4
      const uint16_t *brow[2];
      uint32_t bbytes[2], bdst[2][2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int n = trow + 128 * i;
#pragma unroll
        for (int h = 0; h < 2; ++h) bdst[i][h] = ((n >> 3) * 8 + bp + 4 * h) * 128 + (n & 7) * 16;
        bool v = n < ti.n_valid;
        int xr = v ? (p.row_of ? p.row_of[ti.r_begin + n] : ti.r_begin + n) : 0;
        if (v && !in_bounds((size_t)xr, (size_t)p.x_rows, 6)) {
          v = false;
          xr = 0;
        }
        brow[i] = p.x + (size_t)xr * p.K;
        bbytes[i] = v ? 16u : 0u;  // zero-fill rows past n_valid
      }

      // Token rows of slice kt+1 are copied while slice kt is regenerated; the
      // stage they land in is free once the MMAs of slice (it+1) - kStages are done.
      const uint32_t b_stage0 = umma::smem_u32(b_base);
      auto copy_b = [&](int kt_b, uint32_t it_b) -> bool {
        if (it_b >= (uint32_t)kStages &&
            !umma::mbar_wait_bounded(umma::smem_u32(&empty_bar[it_b % kStages]), (it_b / kStages - 1) & 1,
                                     kWaitCycles))
          return false;
        const uint32_t bsa = b_stage0 + (uint32_t)((it_b % kStages) * p.bn * 128);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          if (trow + 128 * i < N) {
#pragma unroll
            for (int h = 0; h < 2; ++h)
              cp_async16(bsa + bdst[i][h], brow[i] + kt_b * kBK + (bp + 4 * h) * 8, bbytes[i]);
          }
        }
        return true;
      };
      if (!copy_b(0, it)) s_abort = 1;
      cp_async_commit();

      // weight fields three slices ahead, in three register sets: slice kt
      // uses set kt % 3 and reloads it for slice kt + 3 (the loop is unrolled
      // by three, so no set is ever copied while its loads are in flight)
      SliceFields f0, f1, f2;
      const int nw = p.nb / 2;
      load_slice<P>(sp, qp, cpp, ok, 0, f0, bp, nw);
      if (ksteps > 1) load_slice<P>(sp, qp, cpp, ok, 1, f1, bp, nw);
      if (ksteps > 2) load_slice<P>(sp, qp, cpp, ok, 2, f2, bp, nw);
      auto slice = [&](SliceFields &f, int kt) {
        const int stage = it % kStages;
        // the stage of slice it was claimed when its token rows were copied
        if (kt + 1 < ksteps && !copy_b(kt + 1, it + 1)) s_abort = 1;
        cp_async_commit();
        uint8_t *atile = a_base + (size_t)stage * 2 * kBM * 128;
        // rows past the matrix carry zero coefficient fields, which regenerate
        // to exactly zero weights: no branch
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          uint4 *dst0 = reinterpret_cast<uint4 *>(atile + j * kBM * 128 + a_off);
          uint4 *dst1 = reinterpret_cast<uint4 *>(atile + j * kBM * 128 + a_off + 128);
          regen_pair_bf16<P, kTabCopies>(tl, f.s2[j], f.q2[j], f.c2[j], rowk[j], dst0, dst1);
        }
        if (kt + 3 < ksteps) load_slice<P>(sp, qp, cpp, ok, kt + 3, f, bp, nw);
        cp_async_wait<1>();  // this slice's token rows (the next slice's may still be in flight)
        umma::fence_proxy_async();
        umma::mbar_arrive(umma::smem_u32(&full_bar[stage]));
        ++it;
      };
      for (int kt = 0; kt < ksteps; kt += 3) {
        if (s_abort) break;
        slice(f0, kt);
        if (kt + 1 >= ksteps || s_abort) break;
        slice(f1, kt + 1);
        if (kt + 2 >= ksteps || s_abort) break;
        slice(f2, kt + 2);
      }
      cp_async_wait_all();
    }
  }

  cp_async_wait_all();
  __syncthreads();
  if (s_abort) {
    if (tid == 0) atomicExch(p.status, 1);
    // let MMAs still in flight finish (bounded) before the tensor memory is freed
    if (warp == kMmaWarp && lane == 0 && it > 0) {
      const uint32_t last = it - 1;
      umma::mbar_wait_bounded(umma::smem_u32(&empty_bar[last % kStages]), (last / kStages) & 1, kWaitCycles);
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

// Test export: the bf16 hidden activations a batched FFN call left in its
// workspace, moved from sorted order to pair order (h_out[t*k + q][inter]).
__global__ void batched_hidden_kernel(const BatchedPlan bp, int E, int inter, uint16_t *__restrict__ h_out) {
  const int n = bp.offsets[E];  // valid pairs
  const int per = inter / 8;    // 16-byte pieces per row
  const size_t total = (size_t)n * per;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int pos = (int)(i / per), c = (int)(i - (size_t)pos * per);
    const int pair = bp.pair_of[pos];
    reinterpret_cast<uint4 *>(h_out + (size_t)pair * inter)[c] =
        reinterpret_cast<const uint4 *>(bp.h + (size_t)pos * inter)[c];
  }
}

// ---------------------------------------------------------------- host

static int tmem_cols_for(int ncols) {
  int c = 32;
  while (c < ncols) c <<= 1;
  return c;
}

static size_t grouped_smem(int bn) {
  return kTabCopies * 2048 + (size_t)kStages * 2 * kBM * 128 + (size_t)kStages * bn * 128;
}

template <int P, int MODE>
static int32_t launch_grouped_t(const GroupedParams &p, cudaStream_t s) {
  const size_t smem = grouped_smem(p.bn);
  auto kern = grouped_seed_gemm_kernel<P, MODE>;
  if (int32_t st = ensure_smem((const void *)kern, smem)) return st;
  kern<<<num_sms(), kCtaThreads, smem, s>>>(p);
  return launch_status();
}

int32_t launch_grouped(const GroupedParams &p, int P, int mode, cudaStream_t s) {
  if (P == kP3C5) {
    if (mode == GMODE_GEMM) return launch_grouped_t<kP3C5, GMODE_GEMM>(p, s);
    if (mode == GMODE_GATEUP) return launch_grouped_t<kP3C5, GMODE_GATEUP>(p, s);
    return launch_grouped_t<kP3C5, GMODE_DOWN>(p, s);
  }
  if (P == 4) {
    if (mode == GMODE_GEMM) return launch_grouped_t<4, GMODE_GEMM>(p, s);
    if (mode == GMODE_GATEUP) return launch_grouped_t<4, GMODE_GATEUP>(p, s);
    return launch_grouped_t<4, GMODE_DOWN>(p, s);
  }
  if (mode == GMODE_GEMM) return launch_grouped_t<3, GMODE_GEMM>(p, s);
  if (mode == GMODE_GATEUP) return launch_grouped_t<3, GMODE_GATEUP>(p, s);
  return launch_grouped_t<3, GMODE_DOWN>(p, s);
}

// Token rows per tile (up to 256: two accumulators of 256 fp32 columns fill the
// 512 tensor-memory columns); experts with more rows take several tiles.
static int choose_bn(int max_rows_per_expert) {
  return std::max(16, (std::min(max_rows_per_expert, kMaxBn) + 15) & ~15);
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
  const int mt_gu = ceil_div(d.inter, TileShape<GMODE_GATEUP>::kRows);
  const int mt_dn = ceil_div(d.hidden, TileShape<GMODE_DOWN>::kRows);
  batched_plan_kernel<<<1, 1024, 0, s>>>(ids, T, d.E, k, bn, mt_gu, mt_dn, bp);
  if (int32_t st = launch_status()) return st;
  ++launches;
  const int TK = T * k;
  {
    GroupedParams p{};
    p.A0 = *gate; p.A1 = *up; p.E = d.E; p.rows = d.inter; p.K = d.hidden; p.nb = d.hidden / 8;
    p.R = TK; p.x_rows = T; p.x = x_bf16; p.row_of = bp.row_of; p.offsets = bp.offsets; p.tile_start = bp.tiles_gu;
    p.mtiles = mt_gu; p.bn = bn; p.tmem_cols = tmem_cols_for(2 * bn); p.status = bp.status; p.h = bp.h;
    // the gathered rows index x (T rows), not the sorted rows: bound by T via row_of
    if (int32_t st = launch_grouped(p, d.P, GMODE_GATEUP, s)) return st;
    ++launches;
  }
  {
    GroupedParams p{};
    p.A0 = *down; p.E = d.E; p.rows = d.hidden; p.K = d.inter; p.nb = d.inter / 8;
    p.R = TK; p.x_rows = TK; p.x = bp.h; p.row_of = nullptr; p.offsets = bp.offsets; p.tile_start = bp.tiles_dn;
    p.mtiles = mt_dn; p.bn = bn; p.tmem_cols = tmem_cols_for(2 * bn); p.status = bp.status;
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

NSLM_BOUNDS_ACCESSOR(grouped)

}  // namespace nslm

using namespace nslm;

extern "C" int32_t nslm_debug_batched_hidden(const void *ws, size_t ws_bytes, int32_t T, int32_t E,
                                             int32_t hidden, int32_t inter, int32_t k, uint16_t *h_out,
                                             nslm_stream_t stream) {
  g_launches = 0;
  if (!ws || !h_out) return NSLM_ERR_ARG;
  if (T <= kMaxT || k < 1 || k > kMaxK || E < 1 || E > 1024 || hidden % kBK || inter % kBK || hidden <= 0 ||
      inter <= 0)
    return NSLM_ERR_SHAPE;
  const BatchedPlan bp = batched_workspace(static_cast<char *>(const_cast<void *>(ws)), T, k, E, hidden, inter);
  if (ws_bytes < bp.bytes) return NSLM_ERR_WORKSPACE;
  if (!aligned16(ws) || !aligned16(h_out)) return NSLM_ERR_ALIGN;
  int32_t st = check_device();
  if (st) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  batched_hidden_kernel<<<num_sms() * 4, 256, 0, s>>>(bp, E, inter, h_out);
  st = launch_status();
  if (st == NSLM_OK) g_launches = 1;
  return st;
}

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
  const int mtiles = ceil_div(rows, TileShape<GMODE_GEMM>::kRows);
  tile_prefix_kernel<<<1, 1024, 0, s>>>(offsets, E, mtiles, bn, R, tile_start, status);
  if ((st = launch_status())) return st;
  GroupedParams p{};
  p.A0 = *W; p.E = E; p.rows = rows; p.K = W->K; p.nb = W->K / 8; p.R = R; p.x_rows = R; p.x = x_bf16;
  p.row_of = nullptr; p.offsets = offsets; p.tile_start = tile_start; p.mtiles = mtiles; p.bn = bn;
  p.tmem_cols = tmem_cols_for(2 * bn); p.status = status; p.y = y;
  st = launch_grouped(p, W->P, GMODE_GEMM, s);
  if (st == NSLM_OK) g_launches = 2;
  return st;
}
