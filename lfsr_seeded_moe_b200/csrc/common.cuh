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

}  // namespace nslm
