// common.cuh -- shared host/device helpers of libnslm (not part of the ABI).
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/nslm.h"

namespace nslm {

// P value of the P = 3, 5-bit-coefficient format (NSLM_P3C5 in the header).
constexpr int kP3C5 = 35;

// Launch accounting for benchmarks: kernels enqueued by the last call made on
// this host thread.
extern thread_local int32_t g_launches;

inline bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

inline int32_t cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return NSLM_OK;
  (void)cudaGetLastError();
  return NSLM_ERR_CUDA;
}

// Status of the launches just enqueued (consumes a pending launch error).
inline int32_t launch_status() { return cuda_status(cudaGetLastError()); }

int32_t check_device();  // NSLM_ERR_UNSUPPORTED unless the current device is sm_100
int32_t num_sms();       // of the current device (cached per device)

// Raise a kernel's dynamic shared-memory limit to at least `bytes` on the
// current device; the attribute call is made once per (kernel, device, size).
int32_t ensure_smem(const void *kernel, size_t bytes);

// Resident CTAs per SM of a kernel at this block size and dynamic shared
// memory (cached per kernel, device and configuration; at least 1).
int32_t max_active_ctas(const void *kernel, int threads, size_t smem);

int32_t check_matrix(const nslm_seed_matrix *W);

// Device address of the status word (offset 0) of the built-in scratch array
// of nslm_moe_seed_ffn_static on the current device.
int32_t static_scratch_status_word(const int32_t **out);

// Work layout of one seed matrix product: a CTA covers R rows x C chunks of
// 8 blocks (64 weights); C = ceil(nb / 8).
struct ChunkLayout {
  int32_t C;        // chunks per row
  int32_t Cpad;     // chunk slots per row in the CTA (>= C)
  int32_t R;        // rows per CTA
  int32_t threads;  // R * Cpad, a multiple of 32
};
ChunkLayout chunk_layout(int32_t K, int32_t N, int32_t target_ctas, int32_t max_threads);

__host__ __device__ inline int32_t ceil_div(int32_t a, int32_t b) { return (a + b - 1) / b; }

// ------------------------------------------------------------ bounds checks
//
// A build with -DNSLM_BOUNDS_CHECK=1 (python -m lfsr_seeded_moe_b200.build
// --bounds-check) compares the index of every checked global access with the
// extent its kernel was given.  An index outside records the site's number in
// a device word (the first site wins) and the access is skipped: nothing traps
// and no address outside a buffer is formed.  nslm_debug_bounds_status reads
// and clears the word.  In the normal build the checks compile to nothing.
// Site numbers: 1-2 field copies by offset, 3-4 field loads by row, 5-6 the
// tensor-core producer's field and token-row loads, 7-9 the tensor-core
// epilogue's stores, 10-11 the decode kernels' h and y stores, 12 the GEMV's
// y store, 99 the self-test probe.
#ifndef NSLM_BOUNDS_CHECK
#define NSLM_BOUNDS_CHECK 0
#endif
#if NSLM_BOUNDS_CHECK
static __device__ int32_t g_bounds_error;  // one per translation unit
// Host accessor of this translation unit's word: returns it, then clears it.
#define NSLM_BOUNDS_ACCESSOR(tu)                                                  \
  int32_t bounds_error_##tu() {                                                   \
    int32_t v = 0, z = 0;                                                         \
    if (cudaMemcpyFromSymbol(&v, g_bounds_error, sizeof(v)) != cudaSuccess) return -1; \
    if (cudaMemcpyToSymbol(g_bounds_error, &z, sizeof(z)) != cudaSuccess) return -1;   \
    return v;                                                                     \
  }
#else
#define NSLM_BOUNDS_ACCESSOR(tu)
#endif

// True when idx < n; otherwise (bounds-check build) records `site` and
// returns false so that the caller skips the access.
__device__ __forceinline__ bool in_bounds(size_t idx, size_t n, int site) {
#if NSLM_BOUNDS_CHECK
  if (idx >= n) {
    atomicCAS(&g_bounds_error, 0, site);
    return false;
  }
#else
  (void)idx;
  (void)n;
  (void)site;
#endif
  return true;
}

int32_t bounds_error_all();  // the first recorded site over all translation units (and clears them)

}  // namespace nslm
