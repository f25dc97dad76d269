// chunk.cuh -- the inner loop shared by the decode kernels: one thread takes
// one chunk (8 consecutive blocks = 64 weights) of one row, regenerates its
// weights in registers and dots them with M activation vectors held in
// shared memory.
//
// Dot-product form.  For block b with weights w_r = scale * A_r (A_r an
// integer, |A_r| < 2^21 (4 * 8 * 32768 for int4, 3 * 16 * 32768 for the 5-bit
// format)) the regeneration yields G_r = Mg + A_r exactly as an
// fp32 value (Mg = 1.5 * 2^22, so G_r lies in [2^22, 2^23) where the fp32 step
// is 0.5).  Then
//     sum_r x_r A_r = sum_r x_r G_r - Mg * sum_r x_r,
// and the staged activations carry, per block, the pair (-Mg * sum_r x_r, 0)
// that seeds the packed fp32x2 accumulation, so no per-weight subtraction is
// needed.  The rounding of the Mg-sized terms costs about 2^-24 * 2^22.6 |x|
// per product, against a block sum of order 2^17 |x|.
#pragma once
#include <cuda_bf16.h>

#include "../../include/nslm.h"
#include "common.cuh"
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

// Chunk-major layout, for kernels in which every lane reads one chunk slot:
//   xs4[17 q + 2 i + h] = x[64 q + 8 i + 4 h .. +3]
//   xn2[9 q + i]        = (-Mg * sum of block 8 q + i, 0)
// A lane's 24 reads are then immediate offsets from two base addresses, and
// the odd strides (17 x 16 bytes, 9 x 8 bytes) put consecutive slots in
// distinct banks.
constexpr int kCmX4 = 17, kCmXn = 9;
__host__ __device__ inline size_t cm_bytes(int slots) {
  return (size_t)slots * (kCmX4 * sizeof(float4) + kCmXn * sizeof(float2));
}
__device__ __forceinline__ void cm_store_block(float4 *xs4, float2 *xn2, int b, float4 lo, float4 hi) {
  const int q = b >> 3, i = b & 7;
  xs4[kCmX4 * q + 2 * i] = lo;
  xs4[kCmX4 * q + 2 * i + 1] = hi;
  const float sum = ((lo.x + lo.y) + (lo.z + lo.w)) + ((hi.x + hi.y) + (hi.z + hi.w));
  xn2[kCmXn * q + i] = make_float2(-kMagic2 * sum, 0.f);
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

// Asynchronous global -> shared copies (cp.async): 16 bytes with zero fill
// past src_bytes, 16 bytes, 4 bytes; commit / wait on this thread's groups.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// Fields of the 8 blocks of a chunk: seeds and coefs as 4 words of two
// 16-bit values, codes as 8 nibbles (P = 4; unused for P = 3).
struct ChunkFields {
  uint32_t s[4];
  uint32_t q[4];
  uint32_t codes;
};

// Loads with an evict-first hint: every packed byte is read once per call.
// row / nrows: the row's index in its matrix and the matrix's row count (for
// the bounds-check build; a chunk outside the matrix loads as zero fields).
template <int P, bool VEC>
__device__ __forceinline__ void load_chunk(const uint16_t *__restrict__ seeds_row,
                                           const uint16_t *__restrict__ coefs_row,
                                           const uint8_t *__restrict__ codes_row, int nb,
                                           int ch, ChunkFields &f, size_t row = 0, size_t nrows = 1) {
  const int b0 = ch * 8;
  if (!in_bounds(row, nrows, 4) || !in_bounds((size_t)b0 + (VEC ? 7 : 0), (size_t)nb, 3)) {
    f = ChunkFields{};
    return;
  }
  if (VEC) {
    uint4 s = __ldcs(reinterpret_cast<const uint4 *>(seeds_row + b0));
    uint4 q = __ldcs(reinterpret_cast<const uint4 *>(coefs_row + b0));
    f.s[0] = s.x; f.s[1] = s.y; f.s[2] = s.z; f.s[3] = s.w;
    f.q[0] = q.x; f.q[1] = q.y; f.q[2] = q.z; f.q[3] = q.w;
    f.codes = (P == 4) ? __ldcs(reinterpret_cast<const uint32_t *>(codes_row + b0 / 2)) : 0u;
    if (P == 35)  // code bits 1..3 of the chunk's 8 blocks: bytes 3ch .. 3ch+2
      f.codes = (uint32_t)__ldcs(codes_row + 3 * ch) | ((uint32_t)__ldcs(codes_row + 3 * ch + 1) << 8) |
                ((uint32_t)__ldcs(codes_row + 3 * ch + 2) << 16);
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

// The 5-bit format's 24 code bits (bits 1..3 of 8 blocks' codes) of chunk
// `chunk` of a matrix (counted over all rows): 3 bytes at 3 * chunk, which are
// not 4-byte aligned, so they come by plain loads into a register, not into
// the cp.async field slots.
__device__ __forceinline__ uint32_t load_codes3(const nslm_seed_matrix &W, size_t chunk) {
  if (!in_bounds(chunk, (size_t)W.N * (size_t)(W.K >> 6), 1)) return 0u;
  const uint8_t *q = W.codes + 3 * chunk;
  return (uint32_t)__ldcs(q) | ((uint32_t)__ldcs(q + 1) << 8) | ((uint32_t)__ldcs(q + 2) << 16);
}

// The scale key of a row's exponent bias (bounds-checked like the fields).
__device__ __forceinline__ uint32_t load_bias_key(const nslm_seed_matrix &W, size_t row) {
  return row_scale_key(in_bounds(row, (size_t)W.N, 4) ? __ldg(W.exp_bias + row) : 0);
}

// Shared-memory landing slots for the fields of one whole chunk per thread
// (structure of arrays over the n threads of a CTA, so that a warp's 16-byte
// reads are contiguous): seeds, coefs, codes word, exponent bias.
struct FieldSlots {
  uint4 *s, *q;
  uint32_t *c;
  int32_t *b;
  __host__ __device__ static size_t bytes(int n) { return (size_t)n * 40; }
  __device__ __forceinline__ FieldSlots(void *base, int n) {
    s = reinterpret_cast<uint4 *>(base);
    q = s + n;
    c = reinterpret_cast<uint32_t *>(q + n);
    b = reinterpret_cast<int32_t *>(c + n);
  }
};

// Start the copies of chunk ch of row `grow` (whole chunks) into slot i.
template <int P>
__device__ __forceinline__ void fetch_chunk(const nslm_seed_matrix &W, size_t grow, int nb, int ch,
                                            const FieldSlots &fs, int i) {
  if (!in_bounds(grow, (size_t)W.N, 2) || !in_bounds((size_t)ch * 8 + 7, (size_t)nb, 1)) return;
  cp_async16(fs.s + i, W.seeds + grow * nb + ch * 8);
  cp_async16(fs.q + i, W.coefs + grow * nb + ch * 8);
  if (P == 4) cp_async4(fs.c + i, W.codes + grow * (nb / 2) + ch * 4);
  cp_async4(fs.b + i, W.exp_bias + grow);
}

// The same for a row whose chunk starts at element `off` of the seeds/coefs
// streams (off = row * nb + 8 * chunk, 32-bit: a matrix holds < 2^31 blocks).
template <int P>
__device__ __forceinline__ void fetch_chunk_off(const nslm_seed_matrix &W, uint32_t off, uint32_t row,
                                                const FieldSlots &fs, int i) {
  if (!in_bounds((size_t)off + 7, (size_t)W.N * (size_t)(W.K >> 3), 1) || !in_bounds(row, (size_t)W.N, 2))
    return;
  cp_async16(fs.s + i, W.seeds + off);
  cp_async16(fs.q + i, W.coefs + off);
  if (P == 4) cp_async4(fs.c + i, W.codes + (off >> 1));
  cp_async4(fs.b + i, W.exp_bias + row);
}

// Read slot i back (after the copies have completed).
template <int P>
__device__ __forceinline__ void read_chunk(const FieldSlots &fs, int i, ChunkFields &f, uint32_t &rowk) {
  const uint4 s = fs.s[i], q = fs.q[i];
  f.s[0] = s.x; f.s[1] = s.y; f.s[2] = s.z; f.s[3] = s.w;
  f.q[0] = q.x; f.q[1] = q.y; f.q[2] = q.z; f.q[3] = q.w;
  f.codes = (P == 4) ? fs.c[i] : 0u;
  rowk = row_scale_key(fs.b[i]);
}

// Two's-complement nibbles -> doubled signed bytes in the order dp2a pairs
// them with the 16-bit halves of a funnel shift: [2c0, 2c2, 2c1, 2c3]
// (P = 3: byte 3 is 0; the top nibble there is the exponent code).
template <int P>
__device__ __forceinline__ uint32_t coef_pairs2(uint32_t q16) {
  if (P == 35) {  // [2c0, 2c2, 2c1, 0] from three 5-bit fields: 2c mod 256
    const uint32_t v = (q16 & 0x1Fu) | ((q16 >> 2) & 0x1F00u) | ((q16 << 11) & 0x1F0000u);
    return (v << 1) + (v & 0x101010u) * 12u;
  }
  const uint32_t v = (q16 | (q16 << 12)) & (P == 4 ? 0x0F0F0F0Fu : 0x000F0F0Fu);
  // 2c mod 256 per byte: 2q, plus 224 where bit 3 is set (no carry out)
  return (v << 1) + (v & 0x08080808u) * 28u;
}

// G[r] = Mg + A_r (exact fp32) from the stream (v, nxt) of a block and its
// coefficient pairs.  W >> (1+r) holds the states s_{1+r} and s_{17+r} in its
// two 16-bit halves (j = 0, 2) and W >> (9+r) holds s_{9+r} and s_{25+r}
// (j = 1, 3), so two dp2a give sum_j 2 c_j s_{1+8j+r}; the accumulator starts
// at the bits of Mg minus 2 * 32768 * sum_j c_j, and the fp32 step at Mg is 0.5.
__device__ __forceinline__ void block_magic(uint32_t v, uint32_t nxt, uint32_t cp2, float (&G)[8]) {
  const int32_t base = (int32_t)kMagic2Bits - 32768 * dp4a_ss(cp2, 0x01010101u, 0);
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const uint32_t z = (r == 7) ? nxt : __funnelshift_r(v, nxt, 25 + r);  // W >> (9+r)
    G[r] = __int_as_float(dp2a_hi_us(z, cp2, dp2a_lo_us(__funnelshift_r(v, nxt, 17 + r), cp2, base)));
  }
}

#if NSLM_STREAM_SOURCE != 0
// block_magic from the L2-resident table of the ablation builds.
__device__ __forceinline__ void block_magic_src(uint32_t seed, uint32_t cp2, float (&G)[8]) {
  const int32_t base = (int32_t)kMagic2Bits - 32768 * dp4a_ss(cp2, 0x01010101u, 0);
#if NSLM_STREAM_SOURCE == 1
  const uint32_t nxt = __ldg(reinterpret_cast<const uint32_t *>(g_stream_src) + seed);
  const uint32_t v = seed << 16;
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const uint32_t z = (r == 7) ? nxt : __funnelshift_r(v, nxt, 25 + r);
    G[r] = __int_as_float(dp2a_hi_us(z, cp2, dp2a_lo_us(__funnelshift_r(v, nxt, 17 + r), cp2, base)));
  }
#else
  const uint4 *e = g_stream_src + 4 * seed;  // W >> 1 .. W >> 16
  const uint4 a = __ldg(e), b = __ldg(e + 1), c = __ldg(e + 2), d = __ldg(e + 3);
  const uint32_t z[16] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w, c.x, c.y, c.z, c.w, d.x, d.y, d.z, d.w};
#pragma unroll
  for (int r = 0; r < 8; ++r) G[r] = __int_as_float(dp2a_hi_us(z[8 + r], cp2, dp2a_lo_us(z[r], cp2, base)));
#endif
}
#endif

// Regenerate block i (0..7) of a loaded chunk: G[r] = Mg + A_r (exact fp32);
// returns the block's power-of-two scale 2^(code + bias - 15).
template <int P>
__device__ __forceinline__ float regen_chunk_block(const StreamTables *tab, const ChunkFields &f,
                                                   int i, uint32_t rowk, float (&G)[8]) {
  const uint32_t sw = f.s[i >> 1], qw = f.q[i >> 1];
  const uint32_t q = (i & 1) ? (qw >> 16) : (qw & 0xFFFFu);
#if NSLM_STREAM_SOURCE == 0
  uint32_t v, nxt;
  if (i & 1) stream_pair_of<1>(tab, sw, v, nxt);
  else stream_pair_of<0>(tab, sw, v, nxt);
  block_magic(v, nxt, coef_pairs2<P>(q), G);
#else
  block_magic_src((i & 1) ? (sw >> 16) : (sw & 0xFFFFu), coef_pairs2<P>(q), G);
#endif
  const uint32_t code = (P == 4) ? ((f.codes >> (4 * i)) & 0xFu)
                      : (P == 35) ? (((q >> 15) & 1u) | (((f.codes >> (3 * i)) & 7u) << 1))
                                  : (q >> 12);
  return block_scale(code, rowk);
}

// The same from R interleaved copies of the stream tables (entry e of copy c
// at word R * e + c); tl points at this lane's copy (lane mod R), so lanes
// that share a copy are R-fold fewer and bank conflicts fall accordingly.
template <int P, int R>
__device__ __forceinline__ float regen_chunk_block_r(const uint32_t *tl, const ChunkFields &f, int i,
                                                     uint32_t rowk, float (&G)[8]) {
  const uint32_t sw = f.s[i >> 1], qw = f.q[i >> 1];
  const uint32_t q = (i & 1) ? (qw >> 16) : (qw & 0xFFFFu);
#if NSLM_STREAM_SOURCE == 0
  const uint32_t b0 = (i & 1) ? ((sw >> 16) & 0xFFu) : (sw & 0xFFu);
  const uint32_t b1 = (i & 1) ? (sw >> 24) : ((sw >> 8) & 0xFFu);
  const uint32_t nxt = tl[R * b0] ^ tl[R * (256u + b1)];
  const uint32_t v = (i & 1) ? (sw & 0xFFFF0000u) : (sw << 16);
  block_magic(v, nxt, coef_pairs2<P>(q), G);
#else
  block_magic_src((i & 1) ? (sw >> 16) : (sw & 0xFFFFu), coef_pairs2<P>(q), G);
#endif
  const uint32_t code = (P == 4) ? ((f.codes >> (4 * i)) & 0xFu)
                      : (P == 35) ? (((q >> 15) & 1u) | (((f.codes >> (3 * i)) & 7u) << 1))
                                  : (q >> 12);
  return block_scale(code, rowk);
}

// Regenerate blocks (b, b+1) of one row as bf16 (round to nearest even of
// the exact weight) and store them as two 16-byte rows: the tile producer of
// the tensor-core path.  seeds2/coefs2 hold the two blocks' 16-bit fields;
// code2 their two exponent nibbles (low nibble: block b) for P = 4 and the
// 5-bit format, unused for P = 3 (the code is the top nibble of coefs); tl is
// this lane's copy of R interleaved stream tables.
template <int P, int R>
__device__ __forceinline__ void regen_pair_bf16(const uint32_t *tl, uint32_t seeds2, uint32_t coefs2,
                                                uint32_t code2, uint32_t rowk, uint4 *dst0, uint4 *dst1) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t q = h ? (coefs2 >> 16) : (coefs2 & 0xFFFFu);
    const uint32_t b0 = h ? ((seeds2 >> 16) & 0xFFu) : (seeds2 & 0xFFu);
    const uint32_t b1 = h ? (seeds2 >> 24) : ((seeds2 >> 8) & 0xFFu);
    const uint32_t nxt = tl[R * b0] ^ tl[R * (256u + b1)];
    const uint32_t v = h ? (seeds2 & 0xFFFF0000u) : (seeds2 << 16);
    float G[8];
    block_magic(v, nxt, coef_pairs2<P>(q), G);
    const uint32_t code = (P == 3) ? (q >> 12) : ((code2 >> (4 * h)) & 0xFu);
    const float s = block_scale(code, rowk);
    const float off = -kMagic2 * s;
    uint32_t packed[4];
#pragma unroll
    for (int r = 0; r < 8; r += 2) {
      // (Mg + A) * s - Mg * s = A * s exactly (power-of-two scale)
      const __nv_bfloat162 bb = __floats2bfloat162_rn(fmaf(G[r], s, off), fmaf(G[r + 1], s, off));
      packed[r >> 1] = *reinterpret_cast<const uint32_t *>(&bb);
    }
    *(h ? dst1 : dst0) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  }
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

// <G, x> - Mg * sum(x) for one staged block, as a packed pair of partial sums.
__device__ __forceinline__ float2 block_dot2(const float (&G)[8], const float4 &xa, const float4 &xb,
                                             const float2 &xn) {
  float2 p = __ffma2_rn(make_float2(G[0], G[1]), make_float2(xa.x, xa.y), xn);
  p = __ffma2_rn(make_float2(G[2], G[3]), make_float2(xa.z, xa.w), p);
  p = __ffma2_rn(make_float2(G[4], G[5]), make_float2(xb.x, xb.y), p);
  return __ffma2_rn(make_float2(G[6], G[7]), make_float2(xb.z, xb.w), p);
}

// scale * (<G, x> - Mg * sum(x)) added to acc, for one staged block.
__device__ __forceinline__ void block_fma(const float (&G)[8], float s, const float4 &xa, const float4 &xb,
                                          const float2 &xn, float2 &acc) {
  acc = __ffma2_rn(make_float2(s, s), block_dot2(G, xa, xb, xn), acc);
}

// One chunk against the staged slot at xa (16 float4) / xn (8 float2) of the
// chunk-major layout: acc += sum_b scale_b * <w_b, x_b>.  tl: this lane's
// copy of R interleaved stream tables.
template <int P, bool VEC, int R>
__device__ __forceinline__ void chunk_dot_cm(const uint32_t *tl, const ChunkFields &f, int nvalid,
                                             uint32_t rowk, const float4 *xa, const float2 *xn, float2 &acc) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (!VEC && i >= nvalid) break;
    float G[8];
    const float s = regen_chunk_block_r<P, R>(tl, f, i, rowk, G);
    block_fma(G, s, xa[2 * i], xa[2 * i + 1], xn[i], acc);
  }
}

// The gate and up chunks of one row against the same staged slot.
template <int P, bool VEC, int R>
__device__ __forceinline__ void chunk_dot2_cm(const uint32_t *tl, const ChunkFields &fa,
                                              const ChunkFields &fb, int nvalid, uint32_t rowka,
                                              uint32_t rowkb, const float4 *xa, const float2 *xn,
                                              float2 &acca, float2 &accb) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (!VEC && i >= nvalid) break;
    float Ga[8], Gb[8];
    const float sa = regen_chunk_block_r<P, R>(tl, fa, i, rowka, Ga);
    const float sb = regen_chunk_block_r<P, R>(tl, fb, i, rowkb, Gb);
    const float4 x0 = xa[2 * i], x1 = xa[2 * i + 1];
    const float2 x2 = xn[i];
    block_fma(Ga, sa, x0, x1, x2, acca);
    block_fma(Gb, sb, x0, x1, x2, accb);
  }
}

// Moves a chunk's fields down by N2 words (2 * N2 blocks): block 2 * N2
// becomes block 0.  Lets a loop over the chunk run rolled, N2 words a trip,
// with every field index still a compile-time constant (so in registers).
template <int P, int N2>
__device__ __forceinline__ void shift_chunk(ChunkFields &f) {
  static_assert(N2 == 1 || N2 == 2, "a shift of one or two words");
#pragma unroll
  for (int w = 0; w + N2 < 4; ++w) {
    f.s[w] = f.s[w + N2];
    f.q[w] = f.q[w + N2];
  }
  // codes: 4 bits a block at P = 4, 3 at the 5-bit P = 3 format, none at P = 3
  f.codes = (P == 4) ? (f.codes >> (8 * N2)) : (P == 35) ? (f.codes >> (6 * N2)) : 0u;
}

// The same for up to MT vectors that share the regenerated weights: vector m
// (m < M) has its chunk slot at xa + kCmX4 * off[m], xn + kCmXn * off[m].
// A vector past M is skipped (M is the same for all lanes of a warp in the
// gate/up phase, and nearly always so in the down phase).  BPI blocks are
// unrolled per loop trip (8: the whole chunk); a smaller BPI keeps the code
// small when several of these loops are live on one SM at once, at the cost
// of a few register moves per block.  The arithmetic, and its order, is the
// same for every BPI.
template <int P, bool VEC, int R, int MT, int BPI = 8>
__device__ __forceinline__ void chunk_dot_cm_multi(const uint32_t *tl, const ChunkFields &f, int nvalid,
                                                   uint32_t rowk, const float4 *xa, const float2 *xn,
                                                   const int (&off)[MT], int M, float2 (&acc)[MT]) {
  static_assert(BPI == 2 || BPI == 4 || BPI == 8, "blocks per trip");
  ChunkFields g = f;
#pragma unroll 1
  for (int i0 = 0; i0 < 8; i0 += BPI) {
#pragma unroll
    for (int j = 0; j < BPI; ++j) {
      const int i = i0 + j;
      if (!VEC && i >= nvalid) break;
      float G[8];
      const float s = regen_chunk_block_r<P, R>(tl, g, j, rowk, G);
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        if (m < M) {
          const float4 *x = xa + kCmX4 * off[m];
          block_fma(G, s, x[2 * i], x[2 * i + 1], xn[kCmXn * off[m] + i], acc[m]);
        }
      }
    }
    if constexpr (BPI < 8) shift_chunk<P, BPI / 2>(g);
  }
}

template <int P, bool VEC, int R, int MT, int BPI = 8>
__device__ __forceinline__ void chunk_dot2_cm_multi(const uint32_t *tl, const ChunkFields &fa,
                                                    const ChunkFields &fb, int nvalid, uint32_t rowka,
                                                    uint32_t rowkb, const float4 *xa, const float2 *xn,
                                                    const int (&off)[MT], int M, float2 (&acca)[MT],
                                                    float2 (&accb)[MT]) {
  static_assert(BPI == 2 || BPI == 4 || BPI == 8, "blocks per trip");
  ChunkFields ga = fa, gb = fb;
#pragma unroll 1
  for (int i0 = 0; i0 < 8; i0 += BPI) {
#pragma unroll
    for (int j = 0; j < BPI; ++j) {
      const int i = i0 + j;
      if (!VEC && i >= nvalid) break;
      float Ga[8], Gb[8];
      const float sa = regen_chunk_block_r<P, R>(tl, ga, j, rowka, Ga);
      const float sb = regen_chunk_block_r<P, R>(tl, gb, j, rowkb, Gb);
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        if (m < M) {
          const float4 *x = xa + kCmX4 * off[m];
          const float4 x0 = x[2 * i], x1 = x[2 * i + 1];
          const float2 x2 = xn[kCmXn * off[m] + i];
          block_fma(Ga, sa, x0, x1, x2, acca[m]);
          block_fma(Gb, sb, x0, x1, x2, accb[m]);
        }
      }
    }
    if constexpr (BPI < 8) {
      shift_chunk<P, BPI / 2>(ga);
      shift_chunk<P, BPI / 2>(gb);
    }
  }
}

// Sum of a float over the 32 lanes of a warp (fixed order: deterministic).
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// ------------------------------------------------------- activation staging

// Stage the activations of M tokens (rows[m]) into vectors m of the chunk
// layout.  Source is either bf16 x [T][K], or fp32 y [T][K] normalised per
// token to bf16(y / sqrt(mean(y^2) + 1e-6)).
template <bool CM>
static __device__ __noinline__ void stage_activations(float4 *xs4, float2 *xn2, const uint16_t *__restrict__ x_bf16,
                                  const float *__restrict__ y_prev, const int *rows, int M, int K,
                                  int cpad, float *scratch /* >= 33 floats */) {
  const int tid = threadIdx.x, nthr = blockDim.x, nb = K >> 3;
  if (x_bf16) {
    if (!CM) {
      stage_bf16(xs4, xn2, x_bf16, rows, M, K, cpad);
      return;
    }
    // chunk-major: one vector
    const uint4 *row = reinterpret_cast<const uint4 *>(x_bf16 + (size_t)rows[0] * K);
    for (int b = tid; b < nb; b += nthr) {
      float4 lo, hi;
      bf16x8_to_f32(__ldg(row + b), lo, hi);
      cm_store_block(xs4, xn2, b, lo, hi);
    }
    return;
  }
  for (int m = 0; m < M; ++m) {
    const float4 *row = reinterpret_cast<const float4 *>(y_prev + (size_t)rows[m] * K);
    float ss = 0.f;
    for (int i = tid; i < 2 * nb; i += nthr) {
      const float4 v = __ldcg(row + i);
      ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss))));
    }
    ss = warp_sum(ss);
    if ((tid & 31) == 0) scratch[tid >> 5] = ss;
    __syncthreads();
    if (tid == 0) {
      float t = 0.f;
      for (int w = 0; w < (nthr + 31) / 32; ++w) t += scratch[w];
      scratch[32] = sqrtf(t / (float)K + 1e-6f);
    }
    __syncthreads();
    const float r = scratch[32];
    for (int b = tid; b < nb; b += nthr) {
      float4 lo = __ldcg(row + 2 * b), hi = __ldcg(row + 2 * b + 1);
#define NSLM_NORM(v) __bfloat162float(__float2bfloat16_rn(__fdiv_rn((v), r)))
      lo = make_float4(NSLM_NORM(lo.x), NSLM_NORM(lo.y), NSLM_NORM(lo.z), NSLM_NORM(lo.w));
      hi = make_float4(NSLM_NORM(hi.x), NSLM_NORM(hi.y), NSLM_NORM(hi.z), NSLM_NORM(hi.w));
#undef NSLM_NORM
      if (CM) cm_store_block(xs4, xn2, b, lo, hi);
      else xs_store_block(xs4, xn2, m, b, cpad, lo, hi);
    }
    __syncthreads();  // scratch is reused by the next token
  }
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
