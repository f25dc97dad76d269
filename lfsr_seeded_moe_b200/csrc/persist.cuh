// persist.cuh -- pieces shared by the persistent cooperative decode kernels
// (one token: stack1.cu; 2..8 tokens: stackb.cu) and the one-vector GEMV:
// exact division by a run-time constant and the bounded grid barrier.
#pragma once
#include <cstdint>

#include "common.cuh"

namespace nslm {

// n / d for n < 2^22 and 0 < d < 2^16: m = ceil(2^40 / d), q = (n * m) >> 40
// (exact, since n * (m * d - 2^40) < 2^38 < 2^40).
struct FastDiv {
  uint64_t m;
};
__host__ __device__ inline FastDiv make_fastdiv(uint32_t d) { return FastDiv{((1ull << 40) + d - 1) / d}; }
__device__ __forceinline__ uint32_t fdiv(uint32_t n, FastDiv f) {
  return (uint32_t)(((uint64_t)n * f.m) >> 40);
}

// Status words at the head of the decode workspace: sync[0] status (0 ok,
// 1 a wait gave up), sync[1] barrier arrivals, sync[2] abort flag.
constexpr long long kBarrierWaitCycles = 2000000000ll;  // ~1 s at 1.9 GHz

__device__ __forceinline__ uint32_t ld_acquire(const int32_t *p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// A grid-wide barrier in two halves, so that work which does not depend on
// other CTAs (the next phase's weight prefetch) runs between them.
// Arrival: block barrier, then a release reduction by thread 0 (it orders the
// CTA's writes, gathered by the block barrier, before it).
__device__ __forceinline__ void grid_arrive(int32_t *sync) {
  __syncthreads();
  if (threadIdx.x == 0) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(sync + 1) : "memory");
}

// Wait until `target` arrivals: thread 0 polls with acquire loads, bounded by
// kBarrierWaitCycles; a CTA that gives up raises the abort flag and records
// status 1, and every CTA stops at its next wait.  False when aborting.
static __device__ bool grid_wait(int32_t *sync, uint32_t target, int *s_ok,
                                 long long max_cycles = kBarrierWaitCycles) {
  if (threadIdx.x == 0) {
    int ok = 1;
    if (ld_acquire(sync + 1) < target) {
      const long long t0 = clock64();
      for (uint32_t it = 1; ld_acquire(sync + 1) < target; ++it) {
        if ((it & 63) == 0) {
          if (ld_acquire(sync + 2) != 0) {
            ok = 0;
            break;
          }
          if (clock64() - t0 > max_cycles) {
            atomicExch(sync + 2, 1);
            atomicCAS(sync, 0, 1);
            ok = 0;
            break;
          }
        }
      }
    }
    *s_ok = ok;
  }
  __syncthreads();
  return *s_ok != 0;
}

// Values handed from one layer to the next as 64-bit words: the fp32 bits in
// the low half, the tag of the layer that wrote them in the high half.  An
// aligned 64-bit access is single-copy atomic, so a reader that sees the tag
// it expects also sees the value stored with it: no fence, flag or barrier
// is needed between the writer and the reader of one word.
__device__ __forceinline__ void st_tagged(uint64_t *p, float v, uint32_t tag) {
  const uint64_t w = ((uint64_t)tag << 32) | __float_as_uint(v);
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}
__device__ __forceinline__ uint64_t ld_tagged(const uint64_t *p) {
  uint64_t w;
  asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(w) : "l"(p) : "memory");
  return w;
}
__device__ __forceinline__ void ld_tagged2(const uint64_t *p, uint64_t &a, uint64_t &b) {
  asm volatile("ld.relaxed.gpu.global.v2.b64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "l"(p) : "memory");
}
__device__ __forceinline__ bool has_tag(uint64_t w, uint32_t tag) { return (uint32_t)(w >> 32) == tag; }
__device__ __forceinline__ float tagged_value(uint64_t w) { return __uint_as_float((uint32_t)w); }

// Call `ready()` (which reloads what it checks) until it returns true.  Gives
// up, returning false, when another CTA has raised the abort flag or after
// max_cycles, raising the flag and recording status 1 itself, as grid_wait.
template <class F>
__device__ bool poll_bounded(int32_t *sync, F &&ready, long long max_cycles = kBarrierWaitCycles) {
  if (ready()) return true;
  const long long t0 = clock64();
  for (uint32_t it = 1;; ++it) {
    if (ready()) return true;
    if ((it & 63) == 0) {
      if (ld_acquire(sync + 2) != 0) return false;
      if (clock64() - t0 > max_cycles) {
        atomicExch(sync + 2, 1);
        atomicCAS(sync, 0, 1);
        return false;
      }
    }
  }
}

}  // namespace nslm
