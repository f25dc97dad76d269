// regen.cuh -- device-side SeedLM block regeneration for sm_100a.
//
// A block of 8 weights is a 16-bit LFSR seed, P int4 coefficients and a 4-bit
// exponent code ("NanoSeedLM: LLM inference using pseudo-random numbers",
// "Where this started").  With s_t the register state t steps after the seed
// (the seed is s_0: "What I changed: September 2026"), the weights are
//
//   w_r = 2^(code + bias) * sum_j c_j * (s_{1+8j+r} - 32768) / 32768
//       = 2^(code + bias - 15) * A_r,   A_r = sum_j c_j * (s_{1+8j+r} - 32768),
//
// an integer A_r with |A_r| < 2^21 (at most 4 * 8 * 32768, or 3 * 16 * 32768 for
// 5-bit coefficients) times a power of two, so fp32 holds w_r
// exactly.  This file rebuilds A_r without stepping the register:
//
// 1. Stream word.  The register is a Fibonacci LFSR (x^16 + x^14 + x^13 +
//    x^11 + 1), so the states are 16-bit windows of one bit stream:
//    s_t = (W >> t) & 0xFFFF, where W holds the seed in bits 0..15 and the
//    new bit 16+k = W_k ^ W_{k+2} ^ W_{k+3} ^ W_{k+5} ("'LFSR is free'": the
//    24 or 32 bits that follow a seed are a linear function of it, so states
//    become shifts of a 64-bit word).  The 8P new bits are linear over GF(2)
//    in the seed, so they are the XOR of two 256-entry table rows, one per
//    seed byte (computed at compile time; each CTA copies the 2 KB into
//    shared memory).
//
// 2. Two-way dot products.  The decode kernels and the tensor-core tile
//    producer turn the stream and the coefficients into the 8 integers A_r
//    with 15 funnel shifts and 16 dp2a per block (chunk.cuh, block_magic).
//
// Measured on this B200 (warp instructions per clock per SM): LOP3/SHF/PRMT
// share one pipe at 2.0, DP4A/IMAD another at 2.0, and a mix of the two
// reaches 3.4; the inner loop is written to alternate the two pipes.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace nslm {

// ---------------------------------------------------------------- stream

// Smem tables: for a seed s, the 32 bits that follow it in the stream are
// tab[s & 0xFF] ^ tab[256 + (s >> 8)].
struct StreamTables {
  uint32_t t[512];
};

// The table contents, computed at compile time from the bit recurrence
// (bit 16+k = bit k ^ bit k+2 ^ bit k+3 ^ bit k+5): entry v < 256 holds the 32
// bits that follow start value v, entry 256 + v those that follow v << 8.
struct StreamTableInit {
  uint32_t t[512];
  constexpr StreamTableInit() : t() {
    for (int i = 0; i < 512; ++i) {
      uint64_t w = i < 256 ? (uint64_t)i : (uint64_t)(i - 256) << 8;
      for (int k = 0; k < 32; ++k) {
        uint64_t b = ((w >> k) ^ (w >> (k + 2)) ^ (w >> (k + 3)) ^ (w >> (k + 5))) & 1u;
        w |= b << (16 + k);
      }
      t[i] = (uint32_t)(w >> 16);
    }
  }
};
static __device__ const StreamTableInit kStreamTab{};

// ------------------------------------------------- stream source (ablation)
//
// NSLM_STREAM_SOURCE selects where the chunk regenerators of the decode
// kernels take a block's stream bits from:
//   0 (the library): the two 256-entry GF(2) tables above, in shared memory;
//   1: one 32-bit word per seed, the bits that follow it (65,536 entries,
//      256 KB, L2-resident), one 4-byte global load per block -- the table
//      of "NanoSeedLM: LLM inference using pseudo-random numbers", "'LFSR is
//      free'";
//   2: a 65,536-entry basis table holding per seed the 16 words W >> t,
//      t = 1..16, that the two-way dot products consume (64 B per seed, 4 MB,
//      L2-resident): four 16-byte global loads per block and no shifts.
// 1 and 2 are built only as separate libraries, to measure those designs
// against the tables kept here; results are identical in all three.
#ifndef NSLM_STREAM_SOURCE
#define NSLM_STREAM_SOURCE 0
#endif

#if NSLM_STREAM_SOURCE != 0
static __device__ uint4 g_stream_src[NSLM_STREAM_SOURCE == 1 ? 65536 / 4 : 65536 * 4];

static __global__ void fill_stream_src_kernel() {
  const uint32_t s = blockIdx.x * blockDim.x + threadIdx.x;  // seed 0..65535
  const uint32_t nxt = kStreamTab.t[s & 0xFFu] ^ kStreamTab.t[256u + (s >> 8)];
  if (NSLM_STREAM_SOURCE == 1) {
    reinterpret_cast<uint32_t *>(g_stream_src)[s] = nxt;
  } else {
    uint32_t z[16];
    for (int t = 1; t < 16; ++t) z[t - 1] = __funnelshift_r(s << 16, nxt, 16 + t);
    z[15] = nxt;
    for (int k = 0; k < 4; ++k) g_stream_src[4 * s + k] = make_uint4(z[4 * k], z[4 * k + 1], z[4 * k + 2], z[4 * k + 3]);
  }
}

// Fill this translation unit's table before its first launch.
static inline void ensure_stream_source(cudaStream_t s) {
  static bool done = false;
  if (!done) {
    fill_stream_src_kernel<<<256, 256, 0, s>>>();
    done = true;
  }
}
#else
static inline void ensure_stream_source(cudaStream_t) {}
#endif

// Copy the tables into shared memory with all threads of the CTA (the caller
// synchronises afterwards).
__device__ __forceinline__ void build_stream_tables(StreamTables *tab) {
  for (int i = threadIdx.x; i < 512; i += blockDim.x) tab->t[i] = kStreamTab.t[i];
}

// R interleaved copies of the tables: entry e of copy c at word R * e + c.
template <int R>
__device__ __forceinline__ void build_stream_tables_rep(uint32_t *t) {
  for (int i = threadIdx.x; i < 512 * R; i += blockDim.x) t[i] = kStreamTab.t[i / R];
}

// The stream of seed `HALF` (0: bits 0..15, 1: bits 16..31) of a packed word
// of two seeds, as v = seed << 16 and nxt = the 32 bits that follow the seed:
// then W >> t = funnelshift_r(v, nxt, 16 + t) for 1 <= t < 16, and
// W >> 16 = nxt.
template <int HALF>
__device__ __forceinline__ void stream_pair_of(const StreamTables *tab, uint32_t sw, uint32_t &v,
                                               uint32_t &nxt) {
  const uint32_t b0 = HALF ? ((sw >> 16) & 0xFFu) : (sw & 0xFFu);
  const uint32_t b1 = HALF ? (sw >> 24) : ((sw >> 8) & 0xFFu);
  nxt = tab->t[b0] ^ tab->t[256u + b1];
  v = HALF ? (sw & 0xFFFF0000u) : (sw << 16);
}

// W = seed | next32 << 16, returned as (lo = bits 0..31, hi = bits 32..47).
__device__ __forceinline__ void stream_word(const StreamTables *tab, uint32_t seed,
                                            uint32_t &lo, uint32_t &hi) {
  uint32_t nxt = tab->t[seed & 0xFFu] ^ tab->t[256u + ((seed >> 8) & 0xFFu)];
  lo = __byte_perm(seed, nxt, 0x5410);  // seed bytes 0,1 then next bytes 0,1
  hi = nxt >> 16;
}

// ------------------------------------------------------- dot-product ops

__device__ __forceinline__ int32_t dp4a_us(uint32_t a_u8x4, uint32_t b_s8x4, int32_t acc) {
  int32_t d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a_u8x4), "r"(b_s8x4), "r"(acc));
  return d;
}

__device__ __forceinline__ int32_t dp4a_ss(uint32_t a_s8x4, uint32_t b_s8x4, int32_t acc) {
  int32_t d;
  asm("dp4a.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a_s8x4), "r"(b_s8x4), "r"(acc));
  return d;
}

// Two-way dot products of two unsigned 16-bit halves of a with the signed
// bytes 0,1 (lo) or 2,3 (hi) of b, accumulated into acc.
__device__ __forceinline__ int32_t dp2a_lo_us(uint32_t a_u16x2, uint32_t b_s8x4, int32_t acc) {
  int32_t d;
  asm("dp2a.lo.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a_u16x2), "r"(b_s8x4), "r"(acc));
  return d;
}
__device__ __forceinline__ int32_t dp2a_hi_us(uint32_t a_u16x2, uint32_t b_s8x4, int32_t acc) {
  int32_t d;
  asm("dp2a.hi.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a_u16x2), "r"(b_s8x4), "r"(acc));
  return d;
}

// ----------------------------------------------------------------- block

// Scale 2^(code + bias - 15) as an fp32 bit pattern: rowk = (bias + 112) << 23.
__device__ __forceinline__ float block_scale(uint32_t code, uint32_t rowk) {
  return __uint_as_float(rowk + (code << 23));
}

__device__ __forceinline__ uint32_t row_scale_key(int32_t bias) {
  return (uint32_t)(bias + 112) << 23;
}

}  // namespace nslm
