// probe.cu -- test export: the bounded device waits of the persistent decode
// kernels (grid barrier) and of the tensor-core pipeline (mbarrier) give up
// after their limit and report it, instead of hanging.  One CTA waits for an
// event that nothing produces (or, for the positive case, one that already
// happened) with the kernels' own wait routines and a caller-chosen limit.
#include "chunk.cuh"
#include "common.cuh"
#include "persist.cuh"
#include "umma.cuh"

namespace nslm {
namespace {

// out[0..3]: the sync words the grid barrier uses (status, arrivals, abort),
// initialised by the caller; out[4] = 1 if the wait succeeded, 0 if it gave up.
__global__ void grid_wait_probe_kernel(int32_t *out, long long cycles) {
  __shared__ int s_ok;
  const bool ok = grid_wait(out, 1u, &s_ok, cycles);  // one arrival, which no CTA makes unless preset
  if (threadIdx.x == 0) out[4] = ok ? 1 : 0;
}

// The tagged-word wait of the one-token stack on the 64-bit word at out[6..7]
// (value bits, tag), waiting for tag 1 with out[0..3] as the sync words;
// out[4] = 1 if the wait succeeded, 0 if it gave up; out[5] = the value bits
// it saw.
__global__ void tag_wait_probe_kernel(int32_t *out, long long cycles) {
  if (threadIdx.x != 0) return;
  const uint64_t *word = reinterpret_cast<const uint64_t *>(out + 6);
  uint64_t w = 0;
  const bool ok = poll_bounded(
      out,
      [&] {
        w = ld_tagged(word);
        return has_tag(w, 1u);
      },
      cycles);
  out[4] = ok ? 1 : 0;
  out[5] = (int32_t)(uint32_t)w;
}

// out[0] = 1 if the mbarrier wait succeeded, 0 if it gave up; `arrive` = 1
// completes the barrier's phase before the wait.
__global__ void mbar_wait_probe_kernel(int32_t *out, long long cycles, int arrive) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    umma::mbar_init(umma::smem_u32(&bar), 1);
    umma::mbar_init_fence();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (arrive) umma::mbar_arrive(umma::smem_u32(&bar));
    out[0] = umma::mbar_wait_bounded(umma::smem_u32(&bar), 0, cycles) ? 1 : 0;
  }
}

}  // namespace
// The bounds-check build's self-test: a field copy one chunk past the end of
// W, which the copy's own check refuses (site 1) before any address is formed.
__global__ void bounds_probe_kernel(const nslm_seed_matrix W) {
#if NSLM_BOUNDS_CHECK
  __shared__ __align__(16) unsigned char slots[64];
  const FieldSlots fs(slots, 1);
  const uint32_t nb = (uint32_t)(W.K >> 3);
  if (threadIdx.x == 0) fetch_chunk_off<4>(W, (uint32_t)W.N * nb, 0u, fs, 0);
  cp_async_wait_all();
#else
  (void)W;
#endif
}

NSLM_BOUNDS_ACCESSOR(probe)

}  // namespace nslm

using namespace nslm;

extern "C" int32_t nslm_debug_wait_probe(int32_t kind, int32_t *out, int64_t cycles, nslm_stream_t stream) {
  g_launches = 0;
  if (!out || cycles <= 0 || kind < 0 || kind > 3) return NSLM_ERR_ARG;
  if (kind == 3 && reinterpret_cast<uintptr_t>(out) % 8) return NSLM_ERR_ALIGN;
  int32_t st = check_device();
  if (st) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (kind == 0) grid_wait_probe_kernel<<<1, 32, 0, s>>>(out, (long long)cycles);
  else if (kind == 3) tag_wait_probe_kernel<<<1, 32, 0, s>>>(out, (long long)cycles);
  else mbar_wait_probe_kernel<<<1, 32, 0, s>>>(out, (long long)cycles, kind == 2 ? 1 : 0);
  st = launch_status();
  if (st == NSLM_OK) g_launches = 1;
  return st;
}

extern "C" int32_t nslm_debug_bounds_probe(const nslm_seed_matrix *W, nslm_stream_t stream) {
  g_launches = 0;
#if NSLM_BOUNDS_CHECK
  int32_t st = check_matrix(W);
  if (st) return st;
  if (W->P != 4 || W->N < 1 || W->K % 64) return NSLM_ERR_SHAPE;
  if ((st = check_device())) return st;
  bounds_probe_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(*W);
  st = launch_status();
  if (st == NSLM_OK) g_launches = 1;
  return st;
#else
  (void)W;
  (void)stream;
  return NSLM_ERR_UNSUPPORTED;
#endif
}
