// abi.cu -- host-side validation, workspace sizing and the remaining C entry
// points of libnslm (routing, expert FFN, layer stack, debug decompression).
#include <algorithm>
#include <mutex>
#include <numeric>

#include "chunk.cuh"
#include "common.cuh"
#include "grouped.cuh"
#include "moe.cuh"
#include "stack1.cuh"
#include "stackb.cuh"

namespace nslm {

thread_local int32_t g_launches = 0;

namespace {
constexpr int kMaxDevices = 64;
int g_cc_major[kMaxDevices];  // 0 = not queried yet
int g_sms[kMaxDevices];
struct SmemEntry {
  const void *kernel;
  int device;
  size_t bytes;
};
SmemEntry g_smem[256];
int g_smem_n = 0;
std::mutex g_mu;

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}
}  // namespace

int32_t check_device() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return cuda_status(cudaErrorNoDevice);
  if (g_cc_major[dev] == 0) {
    int major = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return cuda_status(cudaErrorNoDevice);
    g_sms[dev] = sms;
    g_cc_major[dev] = major;
  }
  return g_cc_major[dev] == 10 ? NSLM_OK : NSLM_ERR_UNSUPPORTED;
}

int32_t num_sms() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 148;
  if (g_cc_major[dev] == 0) check_device();
  return g_sms[dev] > 0 ? g_sms[dev] : 148;
}

int32_t ensure_smem(const void *kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return NSLM_OK;
  const int dev = current_device();
  std::lock_guard<std::mutex> lock(g_mu);
  for (int i = 0; i < g_smem_n; ++i)
    if (g_smem[i].kernel == kernel && g_smem[i].device == dev && g_smem[i].bytes >= bytes) return NSLM_OK;
  const int32_t st = cuda_status(
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes));
  if (st) return st;
  for (int i = 0; i < g_smem_n; ++i)
    if (g_smem[i].kernel == kernel && g_smem[i].device == dev) {
      g_smem[i].bytes = bytes;
      return NSLM_OK;
    }
  if (g_smem_n < 256) g_smem[g_smem_n++] = SmemEntry{kernel, dev, bytes};
  return NSLM_OK;
}

struct OccEntry {
  const void *kernel;
  int device, threads;
  size_t smem;
  int ctas;
};
static OccEntry g_occ[256];
static int g_occ_n = 0;

int32_t max_active_ctas(const void *kernel, int threads, size_t smem) {
  const int dev = current_device();
  std::lock_guard<std::mutex> lock(g_mu);
  for (int i = 0; i < g_occ_n; ++i)
    if (g_occ[i].kernel == kernel && g_occ[i].device == dev && g_occ[i].threads == threads && g_occ[i].smem == smem)
      return g_occ[i].ctas;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem) != cudaSuccess) {
    (void)cudaGetLastError();
    n = 1;
  }
  n = n < 1 ? 1 : n;
  if (g_occ_n < 256) g_occ[g_occ_n++] = OccEntry{kernel, dev, threads, smem, n};
  return n;
}

int32_t check_matrix(const nslm_seed_matrix *W) {
  if (!W) return NSLM_ERR_ARG;
  if (W->P != 3 && W->P != 4 && W->P != kP3C5) return NSLM_ERR_SHAPE;
  if (W->N < 0 || W->K <= 0) return NSLM_ERR_SHAPE;
  if (W->K % (W->P == 4 ? 16 : (W->P == kP3C5 ? 64 : 8)) != 0) return NSLM_ERR_SHAPE;
  if (W->N > 0) {
    if (!W->seeds || !W->coefs || !W->exp_bias) return NSLM_ERR_ARG;
    if (W->P != 3 && !W->codes) return NSLM_ERR_ARG;
    if (!aligned16(W->seeds) || !aligned16(W->coefs) || !aligned16(W->exp_bias)) return NSLM_ERR_ALIGN;
    if (W->P != 3 && !aligned16(W->codes)) return NSLM_ERR_ALIGN;
  }
  return NSLM_OK;
}

ChunkLayout chunk_layout(int32_t K, int32_t N, int32_t target_ctas, int32_t max_threads) {
  ChunkLayout L{};
  const int nb = K / 8;
  L.C = ceil_div(nb, 8);
  // candidates: Cpad = C (rows a multiple of 32/gcd), or C rounded up to a
  // multiple of 8 or of 32; pick the least idle lanes that still gives at
  // least target_ctas row groups, else the most row groups
  int best_cpad = -1, best_r = 0;
  double best_score = -1e30;
  const int cands[3] = {L.C, ceil_div(L.C, 8) * 8, ceil_div(L.C, 32) * 32};
  for (int cpad : cands) {
    int rmin = 32 / std::gcd(cpad, 32);
    if (rmin * cpad > 1024) continue;
    int r = rmin;
    while (r * 2 * cpad <= max_threads && ceil_div(N, r * 2) >= target_ctas) r *= 2;
    const double idle = double(cpad - L.C) / cpad;
    const int groups = ceil_div(std::max(N, 1), r);
    const double fill = std::min(1.0, double(groups) / target_ctas);
    const double score = fill * (1.0 - idle);
    if (score > best_score + 1e-9) { best_score = score; best_cpad = cpad; best_r = r; }
  }
  if (best_cpad < 0) { best_cpad = ceil_div(L.C, 32) * 32; best_r = 1; }
  L.Cpad = best_cpad;
  L.R = best_r;
  L.threads = L.R * L.Cpad;
  return L;
}

// --------------------------------------------------------- debug kernels

// The debug dumps run the hot kernels' own regenerators, so that their
// bit-exact comparison with the oracle covers the code that computes products.

// The 5-bit format's exponent code of block `col` of a row: bit 0 in bit 15 of
// the coefs word, bits 1..3 at bits 3 col .. 3 col + 2 of the row's codes bytes.
__device__ __forceinline__ uint32_t p3c5_code(const uint8_t *codes_row, uint32_t q, int col) {
  const int bit = 3 * col;
  uint32_t two = codes_row[bit >> 3];
  if ((bit & 7) > 5) two |= (uint32_t)codes_row[(bit >> 3) + 1] << 8;
  return ((q >> 15) & 1u) | (((two >> (bit & 7)) & 7u) << 1);
}

__device__ __forceinline__ const uint8_t *codes_row_of(const nslm_seed_matrix &W, int P, size_t row, int nb) {
  if (P == 4) return W.codes + row * (size_t)(nb / 2);
  if (P == kP3C5) return W.codes + row * (size_t)(3 * nb / 8);
  return nullptr;
}

// fp32: the decode kernels' chunk regenerator (regen_chunk_block_r, i.e.
// block_magic on the shared-memory stream tables) gives G[r] = Mg + A_r and the
// block's scale; the weight is (G[r] - Mg) * scale, both steps exact.  One
// thread per 64-weight chunk of a row, loaded as the decode kernels load it.
template <int P>
__global__ void decompress_f32_kernel(const nslm_seed_matrix W, float *w32) {
  __shared__ StreamTables tab;
  build_stream_tables(&tab);
  __syncthreads();
  const int nb = W.K / 8, C = (nb + 7) / 8;
  const size_t nchunk = (size_t)W.N * C;
  for (size_t t = (size_t)blockIdx.x * blockDim.x + threadIdx.x; t < nchunk;
       t += (size_t)gridDim.x * blockDim.x) {
    const size_t row = t / C;
    const int ch = (int)(t - row * C);
    const uint16_t *sr = W.seeds + row * nb, *qr = W.coefs + row * nb;
    const uint8_t *cr = codes_row_of(W, P, row, nb);
    ChunkFields f;
    if (nb % 8 == 0) load_chunk<P, true>(sr, qr, cr, nb, ch, f, row, (size_t)W.N);
    else load_chunk<P, false>(sr, qr, cr, nb, ch, f, row, (size_t)W.N);
    const uint32_t rowk = row_scale_key(W.exp_bias[row]);
    const int nvalid = min(8, nb - 8 * ch);
    float *dst = w32 + row * (size_t)W.K + (size_t)ch * 64;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i >= nvalid) break;
      float G[8];
      const float scale = regen_chunk_block_r<P, 1>(tab.t, f, i, rowk, G);
#pragma unroll
      for (int r = 0; r < 8; ++r) dst[8 * i + r] = (G[r] - kMagic2) * scale;
    }
  }
}

// bf16: the tensor-core tile producer's routine (regen_pair_bf16), one
// thread per pair of blocks (b, b + 1) of a row, each written as the 16-byte
// row the producer stores into shared memory.  A row with an odd block count
// pairs its last block with an empty one whose output is discarded.
template <int P>
__global__ void decompress_bf16_kernel(const nslm_seed_matrix W, uint16_t *wbf) {
  __shared__ StreamTables tab;
  build_stream_tables(&tab);
  __syncthreads();
  const int nb = W.K / 8, npair = (nb + 1) / 2;
  const size_t ntask = (size_t)W.N * npair;
  for (size_t t = (size_t)blockIdx.x * blockDim.x + threadIdx.x; t < ntask;
       t += (size_t)gridDim.x * blockDim.x) {
    const size_t row = t / npair;
    const int b = 2 * (int)(t - row * npair);
    const bool two = b + 1 < nb;
    const uint16_t *sr = W.seeds + row * nb, *qr = W.coefs + row * nb;
    const uint32_t s2 = (uint32_t)sr[b] | (two ? (uint32_t)sr[b + 1] << 16 : 0u);
    const uint32_t q2 = (uint32_t)qr[b] | (two ? (uint32_t)qr[b + 1] << 16 : 0u);
    const uint8_t *cr = codes_row_of(W, P, row, nb);
    uint32_t c2 = 0;
    if (P == 4) c2 = cr[b / 2];
    if (P == kP3C5) c2 = p3c5_code(cr, q2 & 0xFFFFu, b) | (two ? p3c5_code(cr, q2 >> 16, b + 1) << 4 : 0u);
    uint4 *dst0 = reinterpret_cast<uint4 *>(wbf + row * (size_t)W.K + (size_t)b * 8);
    uint4 spare;
    regen_pair_bf16<P, 1>(tab.t, s2, q2, c2, row_scale_key(W.exp_bias[row]), dst0, two ? dst0 + 1 : &spare);
  }
}

static int32_t decompress(const nslm_seed_matrix *W, float *w32, uint16_t *wbf, nslm_stream_t stream) {
  g_launches = 0;
  int32_t st = check_matrix(W);
  if (st) return st;
  if (!w32 && !wbf) return NSLM_ERR_ARG;
  if ((st = check_device())) return st;
  if (W->N == 0) return NSLM_OK;
  if (!aligned16(w32 ? (const void *)w32 : (const void *)wbf)) return NSLM_ERR_ALIGN;
  const int nb = W->K / 8;
  const size_t ntask = (size_t)W->N * (w32 ? (nb + 7) / 8 : (nb + 1) / 2);
  const int threads = 256;
  const int grid = (int)std::min<size_t>((ntask + threads - 1) / threads, (size_t)num_sms() * 8);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (w32) {
    if (W->P == 4) decompress_f32_kernel<4><<<grid, threads, 0, s>>>(*W, w32);
    else if (W->P == kP3C5) decompress_f32_kernel<kP3C5><<<grid, threads, 0, s>>>(*W, w32);
    else decompress_f32_kernel<3><<<grid, threads, 0, s>>>(*W, w32);
  } else {
    if (W->P == 4) decompress_bf16_kernel<4><<<grid, threads, 0, s>>>(*W, wbf);
    else if (W->P == kP3C5) decompress_bf16_kernel<kP3C5><<<grid, threads, 0, s>>>(*W, wbf);
    else decompress_bf16_kernel<3><<<grid, threads, 0, s>>>(*W, wbf);
  }
  st = launch_status();
  if (st == NSLM_OK) g_launches = 1;
  return st;
}

NSLM_BOUNDS_ACCESSOR(abi)

#if NSLM_BOUNDS_CHECK
int32_t bounds_error_gemv();
int32_t bounds_error_grouped();
int32_t bounds_error_moe();
int32_t bounds_error_stack1();
int32_t bounds_error_stackb();
int32_t bounds_error_probe();
int32_t bounds_error_all() {
  int32_t (*const fns[])() = {bounds_error_abi, bounds_error_gemv, bounds_error_grouped, bounds_error_moe,
                              bounds_error_stack1, bounds_error_stackb, bounds_error_probe};
  int32_t first = 0;
  for (auto f : fns) {
    const int32_t v = f();
    if (v < 0) return NSLM_ERR_CUDA;
    if (first == 0) first = v;
  }
  return first;
}
#else
int32_t bounds_error_all() { return NSLM_ERR_UNSUPPORTED; }
#endif

}  // namespace nslm

using namespace nslm;

extern "C" {

const char *nslm_status_string(int32_t status) {
  switch (status) {
    case NSLM_OK: return "ok";
    case NSLM_ERR_ARG: return "invalid argument";
    case NSLM_ERR_ALIGN: return "device pointer not 16-byte aligned";
    case NSLM_ERR_SHAPE: return "unsupported shape";
    case NSLM_ERR_WORKSPACE: return "workspace missing or too small";
    case NSLM_ERR_CUDA: return "CUDA error";
    case NSLM_ERR_TIMEOUT: return "a device-side wait gave up";
    case NSLM_ERR_UNSUPPORTED: return "device is not sm_100";
    default: return "unknown status";
  }
}

int32_t nslm_last_launch_count(void) { return g_launches; }

int32_t nslm_debug_bounds_status(void) {
  int32_t st = check_device();
  if (st) return st;
  if ((st = cuda_status(cudaDeviceSynchronize()))) return st;
  return bounds_error_all();
}

int32_t nslm_device_status(const void *ws, nslm_stream_t stream) {
  int32_t st = check_device();
  if (st) return st;
  const int32_t *word = static_cast<const int32_t *>(ws);
  if (!word && (st = static_scratch_status_word(&word))) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = cuda_status(cudaStreamSynchronize(s)))) return st;
  int32_t v = 0;
  if ((st = cuda_status(cudaMemcpyAsync(&v, word, sizeof(v), cudaMemcpyDeviceToHost, s)))) return st;
  if ((st = cuda_status(cudaStreamSynchronize(s)))) return st;
  return v == 0 ? NSLM_OK : NSLM_ERR_TIMEOUT;
}

size_t nslm_workspace_bytes(int32_t op, int32_t T, int32_t E, int32_t hidden, int32_t inter,
                            int32_t k, int32_t L) {
  (void)E;
  (void)hidden;
  switch (op) {
    case NSLM_OP_GEMV: return 0;
    case NSLM_OP_GROUPED_GEMM: return grouped_ws_bytes(std::max(E, 1));
    case NSLM_OP_MOE_FFN:
      if (T <= kMaxT)
        return ffn_workspace(nullptr, std::max(T, 1), std::max(k, 1), std::max(hidden, 0),
                             std::max(inter, 0), 1).bytes;
      return batched_workspace(nullptr, T, std::max(k, 1), std::max(E, 1), std::max(hidden, 0),
                               std::max(inter, 0)).bytes;
    case NSLM_OP_MOE_FFN_HYBRID:
      return nslm_workspace_bytes(NSLM_OP_MOE_FFN, T, E, hidden, inter, k, 0) +
             hybrid_extra_bytes(std::max(T, 1), std::max(k, 1), std::max(hidden, 0));
    case NSLM_OP_MOE_STACK:
      return ffn_workspace(nullptr, std::max(T, 1), std::max(k, 1), std::max(hidden, 0),
                           std::max(inter, 0), std::max(L, 1)).bytes;
    default: return 0;
  }
}

int32_t nslm_debug_decompress(const nslm_seed_matrix *W, float *w_out, nslm_stream_t stream) {
  if (!w_out) return NSLM_ERR_ARG;
  return decompress(W, w_out, nullptr, stream);
}

int32_t nslm_debug_decompress_bf16(const nslm_seed_matrix *W, uint16_t *w_out, nslm_stream_t stream) {
  if (!w_out) return NSLM_ERR_ARG;
  return decompress(W, nullptr, w_out, stream);
}

int32_t nslm_moe_route_topk(const float *logits, int32_t T, int32_t E, int32_t k, int32_t *ids,
                            float *w, nslm_stream_t stream) {
  g_launches = 0;
  if (!logits || !ids || !w) return NSLM_ERR_ARG;
  if (T < 0 || k < 1 || k > kMaxK || E < k || E > 1024) return NSLM_ERR_SHAPE;
  int32_t st = check_device();
  if (st) return st;
  if (T == 0) return NSLM_OK;
  // routes chunks of up to 8 tokens per CTA; plans are not needed here, so
  // each chunk writes only ids and w
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  for (int t0 = 0; t0 < T; t0 += kMaxT) {
    const int tn = std::min(kMaxT, T - t0);
    st = launch_route_plan(logits + (size_t)t0 * E, nullptr, nullptr, tn, E, k, 1, nullptr,
                           ids + (size_t)t0 * k, w + (size_t)t0 * k, nullptr, 0, nullptr, tn, nullptr, 0,
                           s);
    if (st) return st;
    ++g_launches;
  }
  return NSLM_OK;
}

int32_t nslm_moe_seed_ffn(const nslm_seed_matrix *gate, const nslm_seed_matrix *up,
                          const nslm_seed_matrix *down, int32_t E, const uint16_t *x_bf16,
                          const int32_t *ids, const float *w, int32_t T, int32_t k, float *y,
                          void *ws, size_t ws_bytes, nslm_stream_t stream) {
  g_launches = 0;
  FfnDims d{};
  int32_t st = check_ffn_shapes(gate, up, down, E, d);
  if (st) return st;
  if (!x_bf16 || !ids || !w || !y) return NSLM_ERR_ARG;
  if (k < 1 || k > kMaxK || T < 0) return NSLM_ERR_SHAPE;
  if (!aligned16(x_bf16) || !aligned16(y)) return NSLM_ERR_ALIGN;
  if (T == 0) return NSLM_OK;
  if (T > kMaxT && (d.hidden % 64 || d.inter % 64 || E > 1024)) return NSLM_ERR_SHAPE;
  const size_t need = nslm_workspace_bytes(NSLM_OP_MOE_FFN, T, E, d.hidden, d.inter, k, 0);
  if (!ws || ws_bytes < need) return NSLM_ERR_WORKSPACE;
  if (!aligned16(ws)) return NSLM_ERR_ALIGN;
  if ((st = check_device())) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (T > kMaxT) {  // tensor-core path: bf16 weights, bf16 hidden activation
    int launches = 0;
    st = launch_batched_ffn(d, gate, up, down, x_bf16, ids, w, T, k, y, ws, s, launches);
    if (st == NSLM_OK) g_launches = launches;
    return st;
  }
  const FfnWorkspace fw = ffn_workspace(reinterpret_cast<char *>(ws), T, k, d.hidden, d.inter, 1);
  if ((st = launch_route_plan(nullptr, ids, w, T, E, k, 1, fw.plans, nullptr, nullptr, fw.counters,
                              d.hidden, fw.sync, decode_slot_cap(d, T, k), nullptr, 0, s)))
    return st;
  int launches = 1;
  const nslm_moe_layer layer{*gate, *up, *down};
  st = launch_decode_stack(d, &layer, 1, x_bf16, T, k, fw, y, s, launches);
  if (st == NSLM_OK) g_launches = launches;
  return st;
}

int32_t nslm_moe_stack_decode(const nslm_moe_layer *layers, int32_t L, int32_t E, int32_t k,
                              const float *logits, const uint16_t *x0_bf16, int32_t T, float *y,
                              void *ws, size_t ws_bytes, nslm_stream_t stream) {
  g_launches = 0;
  if (!layers || !logits || !x0_bf16 || !y) return NSLM_ERR_ARG;
  if (L < 1 || T < 1 || T > kMaxT || k < 1 || k > kMaxK || E < k || E > 1024) return NSLM_ERR_SHAPE;
  FfnDims d{};
  int32_t st = check_ffn_shapes(&layers[0].gate, &layers[0].up, &layers[0].down, E, d);
  if (st) return st;
  for (int l = 1; l < L; ++l) {
    FfnDims dl{};
    if ((st = check_ffn_shapes(&layers[l].gate, &layers[l].up, &layers[l].down, E, dl))) return st;
    if (dl.hidden != d.hidden || dl.inter != d.inter || dl.P != d.P) return NSLM_ERR_SHAPE;
  }
  if (!aligned16(x0_bf16) || !aligned16(y) || !aligned16(logits)) return NSLM_ERR_ALIGN;
  const size_t need = nslm_workspace_bytes(NSLM_OP_MOE_STACK, T, E, d.hidden, d.inter, k, L);
  if (!ws || ws_bytes < need) return NSLM_ERR_WORKSPACE;
  if (!aligned16(ws)) return NSLM_ERR_ALIGN;
  if ((st = check_device())) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const FfnWorkspace fw = ffn_workspace(reinterpret_cast<char *>(ws), T, k, d.hidden, d.inter, L);
  if ((st = launch_route_plan(logits, nullptr, nullptr, T, E, k, L, fw.plans, nullptr, nullptr,
                              fw.counters, d.hidden, fw.sync, decode_slot_cap(d, T, k),
                              T == 1 && L > 1 ? fw.ytag : nullptr, fw.n_ytag, s)))
    return st;
  int launches = 1;
  st = launch_decode_stack(d, layers, L, x0_bf16, T, k, fw, y, s, launches);
  if (st == NSLM_OK) g_launches = launches;
  return st;
}

}  // extern "C"
