// cache.cu -- routed experts kept in host memory behind a VRAM cache of
// recently used experts ("NanoSeedLM" README, "Highlights": the CUDA engine
// can keep the routed experts in RAM, and a VRAM cache holds the recently used
// ones; the news list: LRU beat LFU and a hot set as the cache policy).
//
// The cache is three stacked seed matrices of S expert slots in device memory.
// One step for one layer, all on the caller's stream and without a host round
// trip (so it can live in a CUDA graph):
//   1. cache_lru_kernel (one CTA): for the routed (token, slot) pairs in
//      order, a hit refreshes the slot's tick; a miss takes the least recently
//      used slot not yet used in this step (empty slots first, then the
//      lowest tick, ties to the lowest slot), records a copy job and writes
//      the slot id in place of the expert id.
//   2. cache_copy_kernel: every CTA copies 16-byte words of the jobs' field
//      ranges (seeds, coefs, codes, exp_bias of gate, up and down) from the
//      source stacks, which may be host memory the device can address
//      (pinned host memory under unified addressing), into the slots.
// The caller then runs nslm_moe_seed_ffn on the cache stacks with the slot
// ids.  State (device, int32): [0] clock, [1] jobs of the last step, [2] hits,
// [3] misses, [4, 4+64) job experts, [68, 68+64) job slots, then key+1 per
// slot (0 = empty) and the slot's last-use tick.
#include <climits>

#include "common.cuh"
#include "moe.cuh"

namespace nslm {
namespace {

constexpr int kCacheThreads = 256;
constexpr int kCacheMaxSlots = 4096;   // the LRU keeps keys and ticks in shared memory (32 KB)
constexpr int kStateHead = 4 + 2 * kMaxPairs;

struct CacheMats {
  nslm_seed_matrix gate, up, down;
};

// (value, index) minimum over the CTA, ties to the lower index.
__device__ __forceinline__ void cta_argmin(uint64_t &v, uint64_t *s_red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const uint64_t o = __shfl_xor_sync(0xffffffffu, v, off);
    v = o < v ? o : v;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();  // s_red of the previous reduction is consumed
  if (lane == 0) s_red[warp] = v;
  __syncthreads();
  v = ~0ull;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) v = s_red[w] < v ? s_red[w] : v;
}

__global__ void __launch_bounds__(kCacheThreads) cache_lru_kernel(int32_t *state, int S, int E, int layer,
                                                                  const int32_t *ids, int n, int32_t *slot_ids) {
  __shared__ int32_t s_key[kCacheMaxSlots];
  __shared__ uint32_t s_tick[kCacheMaxSlots];
  __shared__ uint64_t s_red[kCacheThreads / 32];
  __shared__ int32_t s_jobs, s_hits, s_miss;
  const int tid = threadIdx.x;
  int32_t *key = state + kStateHead;
  uint32_t *tick = reinterpret_cast<uint32_t *>(key + S);
  for (int s = tid; s < S; s += blockDim.x) {
    s_key[s] = key[s];
    s_tick[s] = tick[s];
  }
  const uint32_t clock = (uint32_t)state[0] + 1u;
  if (tid == 0) s_jobs = s_hits = s_miss = 0;
  __syncthreads();
  for (int i = 0; i < n; ++i) {
    const int e = ids[i];
    if (e < 0 || e >= E) {  // dropped pair: no slot
      if (tid == 0) slot_ids[i] = -1;
      continue;
    }
    const int32_t k1 = layer * E + e + 1;
    uint64_t hit = ~0ull;
    for (int s = tid; s < S; s += blockDim.x)
      if (s_key[s] == k1) hit = (uint64_t)s;
    cta_argmin(hit, s_red);
    int slot;
    if (hit != ~0ull) {
      slot = (int)hit;
      if (tid == 0) ++s_hits;
    } else {
      // least recently used among the slots not touched in this step
      uint64_t best = ~0ull;
      for (int s = tid; s < S; s += blockDim.x)
        if (s_tick[s] != clock) {
          const uint64_t v = ((uint64_t)(s_key[s] == 0 ? 0u : s_tick[s]) << 32) | (uint32_t)s;
          best = v < best ? v : best;
        }
      cta_argmin(best, s_red);
      slot = (int)(best & 0xFFFFFFFFu);  // the host guarantees S >= n, so one exists
      if (tid == 0) {
        state[4 + s_jobs] = e;
        state[4 + kMaxPairs + s_jobs] = slot;
        ++s_jobs;
        ++s_miss;
        s_key[slot] = k1;
      }
    }
    if (tid == 0) {
      s_tick[slot] = clock;
      slot_ids[i] = slot;
    }
    __syncthreads();
  }
  for (int s = tid; s < S; s += blockDim.x) {
    key[s] = s_key[s];
    tick[s] = s_tick[s];
  }
  if (tid == 0) {
    state[0] = (int32_t)clock;
    state[1] = s_jobs;
    state[2] += s_hits;
    state[3] += s_miss;
  }
}

// The 12 byte ranges of one expert (gate, up, down x seeds, coefs, codes,
// exp_bias), each a multiple of 16 bytes (checked on the host).
struct Range {
  const char *src;
  char *dst;
  int64_t bytes;
};

__device__ __forceinline__ Range expert_range(const CacheMats &src, const CacheMats &dst, int m, int f, int e, int v,
                                              int R_gu, int R_d) {
  const nslm_seed_matrix &a = m == 0 ? src.gate : (m == 1 ? src.up : src.down);
  const nslm_seed_matrix &b = m == 0 ? dst.gate : (m == 1 ? dst.up : dst.down);
  const int64_t R = m == 2 ? R_d : R_gu, nb = a.K / 8;
  Range r{nullptr, nullptr, 0};
  if (f == 0) {
    r.src = reinterpret_cast<const char *>(a.seeds + e * R * nb);
    r.dst = reinterpret_cast<char *>(const_cast<uint16_t *>(b.seeds) + v * R * nb);
    r.bytes = R * nb * 2;
  } else if (f == 1) {
    r.src = reinterpret_cast<const char *>(a.coefs + e * R * nb);
    r.dst = reinterpret_cast<char *>(const_cast<uint16_t *>(b.coefs) + v * R * nb);
    r.bytes = R * nb * 2;
  } else if (f == 2) {
    if (a.P == 4) {
      r.src = reinterpret_cast<const char *>(a.codes + e * R * (nb / 2));
      r.dst = reinterpret_cast<char *>(const_cast<uint8_t *>(b.codes) + v * R * (nb / 2));
      r.bytes = R * (nb / 2);
    }
  } else {
    r.src = reinterpret_cast<const char *>(a.exp_bias + e * R);
    r.dst = reinterpret_cast<char *>(const_cast<int32_t *>(b.exp_bias) + v * R);
    r.bytes = R * 4;
  }
  return r;
}

__global__ void __launch_bounds__(kCacheThreads) cache_copy_kernel(const int32_t *state, CacheMats src, CacheMats dst,
                                                                   int R_gu, int R_d) {
  const int jobs = state[1];
  for (int j = 0; j < jobs; ++j) {
    const int e = state[4 + j], v = state[4 + kMaxPairs + j];
    for (int m = 0; m < 3; ++m)
      for (int f = 0; f < 4; ++f) {
        const Range r = expert_range(src, dst, m, f, e, v, R_gu, R_d);
        const int64_t words = r.bytes / 16;
        const uint4 *s4 = reinterpret_cast<const uint4 *>(r.src);
        uint4 *d4 = reinterpret_cast<uint4 *>(r.dst);
        for (int64_t w = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; w < words;
             w += (int64_t)gridDim.x * blockDim.x)
          d4[w] = s4[w];
      }
  }
}

bool aligned16p(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace nslm

using namespace nslm;

extern "C" size_t nslm_expert_cache_state_bytes(int32_t slots) {
  if (slots < 1) return 0;
  return (size_t)(kStateHead + 2 * (size_t)slots) * sizeof(int32_t);
}

extern "C" int32_t nslm_expert_cache_fetch(const nslm_seed_matrix *gate_src, const nslm_seed_matrix *up_src,
                                           const nslm_seed_matrix *down_src, int32_t E, int32_t layer,
                                           const nslm_seed_matrix *gate_cache, const nslm_seed_matrix *up_cache,
                                           const nslm_seed_matrix *down_cache, int32_t S, void *state,
                                           const int32_t *ids, int32_t T, int32_t k, int32_t *slot_ids,
                                           nslm_stream_t stream) {
  g_launches = 0;
  if (!gate_src || !up_src || !down_src || !gate_cache || !up_cache || !down_cache || !state || !ids || !slot_ids)
    return NSLM_ERR_ARG;
  FfnDims d{}, dc{};
  int32_t st = check_ffn_shapes(gate_src, up_src, down_src, E, d);
  if (st) return st;
  if (S < 1 || S > kCacheMaxSlots || T < 1 || k < 1 || k > kMaxK || T * k > kMaxPairs || S < T * k || layer < 0)
    return NSLM_ERR_SHAPE;
  if ((int64_t)layer * E + E >= INT_MAX) return NSLM_ERR_SHAPE;
  if ((st = check_ffn_shapes(gate_cache, up_cache, down_cache, S, dc))) return st;
  if (dc.hidden != d.hidden || dc.inter != d.inter || dc.P != d.P) return NSLM_ERR_SHAPE;
  if (d.P == kP3C5) return NSLM_ERR_SHAPE;  // the copies know the P = 3 and P = 4 streams
  // whole 16-byte words per range: rows a multiple of 4 (biases), K a multiple of 64
  if (d.hidden % 64 || d.inter % 64) return NSLM_ERR_SHAPE;
  const nslm_seed_matrix *all[6] = {gate_src, up_src, down_src, gate_cache, up_cache, down_cache};
  for (const nslm_seed_matrix *m : all)
    if (!aligned16p(m->seeds) || !aligned16p(m->coefs) || !aligned16p(m->exp_bias) ||
        (m->P == 4 && !aligned16p(m->codes)))
      return NSLM_ERR_ALIGN;
  if (!aligned16p(state)) return NSLM_ERR_ALIGN;
  if ((st = check_device())) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cache_lru_kernel<<<1, kCacheThreads, 0, s>>>(static_cast<int32_t *>(state), S, E, layer, ids, T * k, slot_ids);
  if ((st = launch_status())) return st;
  const CacheMats src{*gate_src, *up_src, *down_src}, dst{*gate_cache, *up_cache, *down_cache};
  cache_copy_kernel<<<num_sms() * 4, kCacheThreads, 0, s>>>(static_cast<const int32_t *>(state), src, dst,
                                                            d.inter, d.hidden);
  if ((st = launch_status())) return st;
  g_launches = 2;
  return NSLM_OK;
}
