// chunk.cuh -- the inner loop shared by the decode kernels: one thread takes
// one chunk (8 consecutive blocks = 64 weights) of one row, regenerates its
// weights in registers and dots them with M activation vectors held in
// shared memory.
//
// Dot-product form.  For block b with weights w_r = scale * A_r (A_r an
// integer, |A_r| <= 2^20) the regeneration yields G_r = Mg + A_r exactly as an
// fp32 value (Mg = 1.5 * 2^22, so G_r lies in [2^22, 2^23) where the fp32 step
// is 0.5).  Then
//     sum_r x_r A_r = sum_r x_r G_r - Mg * sum_r x_r,
// and the staged activations carry, per block, the pair (-Mg * sum_r x_r, 0)
// that seeds the packed fp32x2 accumulation, so no per-weight subtraction is
// needed.  The rounding of the Mg-sized terms costs about 2^-24 * 2^22.6 |x|
// per product, against a block sum of order 2^17 |x|.
#pragma once
#include <cuda_bf16.h>

#include "regen.cuh"

namespace nslm {

constexpr uint32_t kMagic2Bits = 0x4AC00000u;  // 1.5 * 2^22 as fp32
constexpr float kMagic2 = 6291456.0f;

// Shared-memory layout of activation vectors, chosen so that the threads of
// a warp, which hold consecutive chunk positions, read consecutive words:
//   xs4[((m * 8 + i) * 2 + h) * cpad + ch] = x[m][64 ch + 8 i + 4 h .. +3]
//   xn2[(m * 8 + i) * cpad + ch]           = (-Mg * sum of block 8ch+i, 0)
__device__ __forceinline__ int xs_index(int m, int i, int h, int ch, int cpad) {
  return ((m * 8 + i) * 2 + h) * cpad + ch;
}
__device__ __forceinline__ int xn_index(int m, int i, int ch, int cpad) {
  return (m * 8 + i) * cpad + ch;
}

// Bytes of shared memory for V staged vectors of a layout with cpad chunk slots.
__host__ __device__ inline size_t staged_bytes(int V, int cpad) {
  return (size_t)V * 8 * cpad * (2 * sizeof(float4) + sizeof(float2));
}

// Store the 8 values of block b of vector m (and its offset pair).
__device__ __forceinline__ void xs_store_block(float4 *xs4, float2 *xn2, int m, int b, int cpad,
                                               float4 lo, float4 hi) {
  xs4[xs_index(m, b & 7, 0, b >> 3, cpad)] = lo;
  xs4[xs_index(m, b & 7, 1, b >> 3, cpad)] = hi;
  const float sum = ((lo.x + lo.y) + (lo.z + lo.w)) + ((hi.x + hi.y) + (hi.z + hi.w));
  xn2[xn_index(m, b & 7, b >> 3, cpad)] = make_float2(-kMagic2 * sum, 0.f);
}

// 8 bf16 values (one 16-byte word) -> two float4.
__device__ __forceinline__ void bf16x8_to_f32(uint4 raw, float4 &lo, float4 &hi) {
  lo = make_float4(__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xFFFF0000u),
                   __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xFFFF0000u));
  hi = make_float4(__uint_as_float(raw.z << 16), __uint_as_float(raw.z & 0xFFFF0000u),
                   __uint_as_float(raw.w << 16), __uint_as_float(raw.w & 0xFFFF0000u));
}

// Stage bf16 rows src[row(m)][K] (16-byte aligned rows, K % 8 == 0) as
// vectors m < M of the layout; row(m) = rows ? rows[m] : m.  Blocks past K are
// never read by the dot loops, so nothing is zero-filled.
__device__ __forceinline__ void stage_bf16(float4 *xs4, float2 *xn2, const uint16_t *__restrict__ src,
                                           const int *rows, int M, int K, int cpad) {
  const int nb = K >> 3;
  for (int m = 0; m < M; ++m) {
    const uint4 *row = reinterpret_cast<const uint4 *>(src + (size_t)(rows ? rows[m] : m) * K);
    for (int b = threadIdx.x; b < nb; b += blockDim.x) {
      float4 lo, hi;
      bf16x8_to_f32(__ldg(row + b), lo, hi);
      xs_store_block(xs4, xn2, m, b, cpad, lo, hi);
    }
  }
}

// Stage fp32 rows src[row(m)][K] (16-byte aligned rows, K % 8 == 0).
__device__ __forceinline__ void stage_f32(float4 *xs4, float2 *xn2, const float *__restrict__ src,
                                          const int *rows, int M, int K, int cpad) {
  const int nb = K >> 3;
  for (int m = 0; m < M; ++m) {
    const float4 *row = reinterpret_cast<const float4 *>(src + (size_t)(rows ? rows[m] : m) * K);
    for (int b = threadIdx.x; b < nb; b += blockDim.x)
      xs_store_block(xs4, xn2, m, b, cpad, __ldcg(row + 2 * b), __ldcg(row + 2 * b + 1));
  }
}

// Fields of the 8 blocks of a chunk: seeds and coefs as 4 words of two
// 16-bit values, codes as 8 nibbles (P = 4; unused for P = 3).
struct ChunkFields {
  uint32_t s[4];
  uint32_t q[4];
  uint32_t codes;
};

// Loads with an evict-first hint: every packed byte is read once per call.
template <int P, bool VEC>
__device__ __forceinline__ void load_chunk(const uint16_t *__restrict__ seeds_row,
                                           const uint16_t *__restrict__ coefs_row,
                                           const uint8_t *__restrict__ codes_row, int nb,
                                           int ch, ChunkFields &f) {
  const int b0 = ch * 8;
  if (VEC) {
    uint4 s = __ldcs(reinterpret_cast<const uint4 *>(seeds_row + b0));
    uint4 q = __ldcs(reinterpret_cast<const uint4 *>(coefs_row + b0));
    f.s[0] = s.x; f.s[1] = s.y; f.s[2] = s.z; f.s[3] = s.w;
    f.q[0] = q.x; f.q[1] = q.y; f.q[2] = q.z; f.q[3] = q.w;
    f.codes = (P == 4) ? __ldcs(reinterpret_cast<const uint32_t *>(codes_row + b0 / 2)) : 0u;
  } else {
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint32_t sv = 0, qv = 0;
      int b = b0 + 2 * w;
      if (b < nb) { sv = __ldcs(seeds_row + b); qv = __ldcs(coefs_row + b); }
      if (b + 1 < nb) { sv |= (uint32_t)__ldcs(seeds_row + b + 1) << 16; qv |= (uint32_t)__ldcs(coefs_row + b + 1) << 16; }
      f.s[w] = sv; f.q[w] = qv;
    }
    uint32_t cd = 0;
    if (P == 4) {
#pragma unroll
      for (int w = 0; w < 4; ++w)
        if (b0 + 2 * w < nb) cd |= (uint32_t)__ldcs(codes_row + b0 / 2 + w) << (8 * w);
    }
    f.codes = cd;
  }
}

// Two's-complement nibbles -> doubled signed bytes [2c0, 2c1, 2c2, 2c3]
// (P = 3: byte 3 is 0; the top nibble there is the exponent code).
template <int P>
__device__ __forceinline__ uint32_t coef_bytes2(uint32_t q16) {
  uint32_t v = (q16 | (q16 << 12)) & 0x0F0F0F0Fu;       // [c0, c2, c1, c3] as nibbles
  v = __byte_perm(v, 0u, P == 4 ? 0x3120 : 0x4120);     // [c0, c1, c2, c3|0]
  // 2c mod 256 per byte: 2q, plus 224 where bit 3 is set (no carry out)
  return (v << 1) + (v & 0x08080808u) * 28u;
}

// Regenerate block i (0..7) of a loaded chunk: G[r] = Mg + A_r (exact fp32);
// returns the block's power-of-two scale 2^(code + bias - 15).
template <int P>
__device__ __forceinline__ float regen_chunk_block(const StreamTables *tab, const ChunkFields &f,
                                                   int i, uint32_t rowk, float (&G)[8]) {
  const uint32_t sw = f.s[i >> 1], qw = f.q[i >> 1];
  const uint32_t seed = (i & 1) ? (sw >> 16) : (sw & 0xFFFFu);
  const uint32_t q = (i & 1) ? (qw >> 16) : (qw & 0xFFFFu);
  uint32_t lo, hi;
  stream_word(tab, seed, lo, hi);
  const uint32_t cb2 = coef_bytes2<P>(q);
  const int32_t base = (int32_t)kMagic2Bits - 32768 * dp4a_ss(cb2, 0x01010101u, 0);
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    // bytes of W >> (9+r) weigh 256, bytes of W >> (1+r) weigh 1; the sum is
    // the bit pattern of Mg + 2 A_r ulps = Mg + A_r
    const int32_t d1 = dp4a_us(__funnelshift_r(lo, hi, 9 + r), cb2, 0);
    G[r] = __int_as_float(dp4a_us(__funnelshift_r(lo, hi, 1 + r), cb2, imad(d1, 256, base)));
  }
  const uint32_t code = (P == 4) ? ((f.codes >> (4 * i)) & 0xFu) : (q >> 12);
  return block_scale(code, rowk);
}

// <G, x> - Mg * sum(x) for one staged vector, as a packed pair sum.
__device__ __forceinline__ float block_dot(const float (&G)[8], const float4 &xa, const float4 &xb,
                                           const float2 &xn) {
  float2 p = __ffma2_rn(make_float2(G[0], G[1]), make_float2(xa.x, xa.y), xn);
  p = __ffma2_rn(make_float2(G[2], G[3]), make_float2(xa.z, xa.w), p);
  p = __ffma2_rn(make_float2(G[4], G[5]), make_float2(xb.x, xb.y), p);
  p = __ffma2_rn(make_float2(G[6], G[7]), make_float2(xb.z, xb.w), p);
  return p.x + p.y;
}

// acc[m] += sum over the chunk's blocks of scale_b * <w_b, x_{v0+m}[b]>, for
// exactly M vectors (M a compile-time constant: no per-block branches).
// CPAD is the layout's chunk-slot count when known at compile time, else 0.
template <int P, int M, bool VEC, int CPAD>
__device__ __forceinline__ void chunk_dot(const StreamTables *tab, const ChunkFields &f, int nb,
                                          int ch, uint32_t rowk, const float4 *xs4,
                                          const float2 *xn2, int cpad_rt, int v0,
                                          float (&acc)[M]) {
  const int cpad = CPAD ? CPAD : cpad_rt;
  const float4 *xa_base = xs4 + (v0 * 16) * cpad + ch;
  const float2 *xn_base = xn2 + (v0 * 8) * cpad + ch;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (!VEC && ch * 8 + i >= nb) break;
    float G[8];
    const float scale = regen_chunk_block<P>(tab, f, i, rowk, G);
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const float4 xa = xa_base[((m * 8 + i) * 2 + 0) * cpad];
      const float4 xb = xa_base[((m * 8 + i) * 2 + 1) * cpad];
      const float2 xn = xn_base[(m * 8 + i) * cpad];
      acc[m] = fmaf(scale, block_dot(G, xa, xb, xn), acc[m]);
    }
  }
}

// Two chunks (e.g. the gate and up rows of one expert) against the same
// activations, interleaved block by block for instruction-level parallelism.
template <int P, int M, bool VEC, int CPAD>
__device__ __forceinline__ void chunk_dot2(const StreamTables *tab, const ChunkFields &fa,
                                           const ChunkFields &fb, int nb, int ch, uint32_t rowka,
                                           uint32_t rowkb, const float4 *xs4, const float2 *xn2,
                                           int cpad_rt, float (&acca)[M], float (&accb)[M]) {
  const int cpad = CPAD ? CPAD : cpad_rt;
  const float4 *xa_base = xs4 + ch;
  const float2 *xn_base = xn2 + ch;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (!VEC && ch * 8 + i >= nb) break;
    float Ga[8], Gb[8];
    const float sa = regen_chunk_block<P>(tab, fa, i, rowka, Ga);
    const float sb = regen_chunk_block<P>(tab, fb, i, rowkb, Gb);
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const float4 xa = xa_base[((m * 8 + i) * 2 + 0) * cpad];
      const float4 xb = xa_base[((m * 8 + i) * 2 + 1) * cpad];
      const float2 xn = xn_base[(m * 8 + i) * cpad];
      acca[m] = fmaf(sa, block_dot(Ga, xa, xb, xn), acca[m]);
      accb[m] = fmaf(sb, block_dot(Gb, xa, xb, xn), accb[m]);
    }
  }
}

// Sum of a float over the 32 lanes of a warp (fixed order: deterministic).
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// Row sums of per-thread partials: red[v * nthr + r * cpad + c] holds value v of
// chunk c of row r.  One warp per (v, r), lanes over chunks, then a shuffle
// tree; emit(v, r, sum) runs on lane 0.
template <typename Emit>
__device__ __forceinline__ void reduce_rows(const float *red, int V, int R, int cpad, int C,
                                            Emit emit) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  for (int j = warp; j < V * R; j += nw) {
    const int v = j / R, r = j - v * R;
    const float *src = red + v * blockDim.x + r * cpad;
    float s = 0.f;
    for (int c = lane; c < C; c += 32) s += src[c];
    s = warp_sum(s);
    if (lane == 0) emit(v, r, s);
  }
}

}  // namespace nslm
