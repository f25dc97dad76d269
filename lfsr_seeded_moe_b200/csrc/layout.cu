// layout.cu -- conversion between this library's field streams and the
// "nibbles" layout of seed packs ("Qwen3.8-Flash-Next-NanoSeedLM-P4",
// "Files": the routed experts are NAME.seeds, NAME.nibbles, NAME.exp_bias).
//
// In the nibbles stream, block b of a row holds nibbles (P+1)b .. (P+1)b+P:
// c_0 .. c_{P-1} (two's complement) and then the exponent code; nibble n of a
// row is in byte n / 2, the low half for even n.  Seeds and biases are the
// same streams in both layouts.  The decode and tensor-core kernels read
// 16-byte-aligned per-field streams, so a nibbles pack is converted once at
// load time: for P = 4 a pair of blocks is 5 nibbles-bytes <-> two coefs words
// and one codes byte; for P = 3 the two layouts are the same bytes.
#include "common.cuh"

namespace nslm {
namespace {

// One thread per pair of blocks (P = 4) or per block (P = 3).
template <int P, bool TO_NIBBLES>
__global__ void __launch_bounds__(256) nibbles_kernel(uint8_t *nib, nslm_seed_matrix m, int64_t units) {
  const int64_t u = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (u >= units) return;
  uint16_t *coefs = const_cast<uint16_t *>(m.coefs);
  if (P == 3) {  // 4 nibbles per block, the coefs word's bytes
    uint8_t *nb = nib + 2 * u;
    if (TO_NIBBLES) {
      const uint16_t q = coefs[u];
      nb[0] = (uint8_t)(q & 0xFFu);
      nb[1] = (uint8_t)(q >> 8);
    } else {
      coefs[u] = (uint16_t)(nb[0] | (nb[1] << 8));
    }
    return;
  }
  // P = 4: blocks 2u, 2u+1 of the matrix (rows hold an even number of
  // blocks, so a pair never straddles rows) are nibbles-bytes 5u .. 5u+4
  uint8_t *codes = const_cast<uint8_t *>(m.codes);
  uint8_t *nb = nib + 5 * u;
  if (TO_NIBBLES) {
    const uint64_t q0 = coefs[2 * u], q1 = coefs[2 * u + 1], cb = codes[u];
    const uint64_t v = q0 | ((cb & 0xFu) << 16) | (q1 << 20) | ((cb >> 4) << 36);
#pragma unroll
    for (int i = 0; i < 5; ++i) nb[i] = (uint8_t)(v >> (8 * i));
  } else {
    uint64_t v = 0;
#pragma unroll
    for (int i = 0; i < 5; ++i) v |= (uint64_t)nb[i] << (8 * i);
    coefs[2 * u] = (uint16_t)(v & 0xFFFFu);
    coefs[2 * u + 1] = (uint16_t)((v >> 20) & 0xFFFFu);
    codes[u] = (uint8_t)(((v >> 16) & 0xFu) | (((v >> 36) & 0xFu) << 4));
  }
}

int32_t convert_nibbles(uint8_t *nib, const nslm_seed_matrix *m, bool to_nibbles, nslm_stream_t stream) {
  g_launches = 0;
  if (!m || !nib || !m->coefs) return NSLM_ERR_ARG;
  if ((m->P != 3 && m->P != 4) || m->N < 0 || m->K < 0 || m->K % 8) return NSLM_ERR_SHAPE;
  if (m->P == 4 && (m->K % 16 || !m->codes)) return m->codes ? NSLM_ERR_SHAPE : NSLM_ERR_ARG;
  const int64_t blocks = (int64_t)m->N * (m->K / 8);
  if (blocks == 0) return NSLM_OK;
  int32_t st = check_device();
  if (st) return st;
  const int64_t units = m->P == 4 ? blocks / 2 : blocks;
  const int64_t grid = (units + 255) / 256;
  if (grid > 0x7FFFFFFF) return NSLM_ERR_SHAPE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (m->P == 4) {
    if (to_nibbles) nibbles_kernel<4, true><<<(unsigned)grid, 256, 0, s>>>(nib, *m, units);
    else nibbles_kernel<4, false><<<(unsigned)grid, 256, 0, s>>>(nib, *m, units);
  } else {
    if (to_nibbles) nibbles_kernel<3, true><<<(unsigned)grid, 256, 0, s>>>(nib, *m, units);
    else nibbles_kernel<3, false><<<(unsigned)grid, 256, 0, s>>>(nib, *m, units);
  }
  st = launch_status();
  if (st == NSLM_OK) g_launches = 1;
  return st;
}

}  // namespace
}  // namespace nslm

using namespace nslm;

extern "C" int32_t nslm_unpack_nibbles(const uint8_t *nibbles, const nslm_seed_matrix *out, nslm_stream_t stream) {
  return convert_nibbles(const_cast<uint8_t *>(nibbles), out, false, stream);
}

extern "C" int32_t nslm_pack_nibbles(const nslm_seed_matrix *in, uint8_t *nibbles, nslm_stream_t stream) {
  return convert_nibbles(nibbles, in, true, stream);
}
